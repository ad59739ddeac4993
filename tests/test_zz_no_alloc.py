"""The no-allocation decode entry point, through the C ABI.

pa_paged_attn_decode_noalloc serves callers that cannot allocate device
memory: it keeps its scratch in a static array inside the library instead of
taking a workspace.  This file is collected last on purpose: if it fails, a
run that stops at the first failure has already run every other test.  It
passes alone in a fresh process (the first call on the device then does the
set-up) and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_326_b200 import workloads as W
from tests.gpu_helpers import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from paged_kv_cache_326_b200 import build
    build.build()
    import paged_kv_cache_326_b200 as P
    P.lib()
    return P


def _noalloc_raw(P, out, w, status):
    """Direct C-ABI call (ctypes), no binding logic in between."""
    S, H, D = w.q.shape
    return P.lib().pa_paged_attn_decode_noalloc(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(w.q.data_ptr()),
        ctypes.c_void_p(w.k_cache.data_ptr()), ctypes.c_void_p(w.v_cache.data_ptr()),
        ctypes.c_void_p(w.block_tables.data_ptr()), ctypes.c_void_p(w.context_lens.data_ptr()),
        ctypes.c_float(w.scale), S, H, D, w.block_size, w.max_blocks_per_seq, w.num_blocks,
        P.binding.PA_F16 if w.q.dtype == torch.float16 else P.binding.PA_BF16,
        ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("make", [lambda: W.opt13b_batch64(device="cuda"),
                                  lambda: W.skewed(block_size=16, device="cuda"),
                                  lambda: W.tiny(device="cuda")],
                         ids=["opt13b_batch64", "skewed_bf16", "tiny"])
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(P, make):
    w = make()
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping)
    ref = torch.empty_like(w.q)
    ws = torch.empty(P.pa_paged_attn_decode_workspace_size(
        w.num_seqs, w.num_heads, w.head_dim, w.block_size, w.max_blocks_per_seq),
        dtype=torch.uint8, device="cuda")
    P.pa_paged_attn_decode(ref, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                           w.scale, workspace=ws)
    torch.cuda.synchronize()
    ref64 = ref.double().cpu().numpy()
    for call in range(2):
        out = torch.full_like(w.q, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _noalloc_raw(P, out, w, status)
        torch.cuda.synchronize()
        assert rc == 0, P.pa_status_string(rc)
        assert status.item() == 0, P.pa_status_string(status.item())
        c = compare(out, ref64, w.q.dtype)
        assert c.ok, f"call {call + 1}: {c}"


def test_noalloc_rejects_sizes_beyond_its_scratch(P):
    """Sizes whose workspace exceeds the static 16 MiB come back as
    PA_ERR_TOO_LARGE before any launch (null data pointers are never
    touched)."""
    lib = P.lib()
    S, H, D, B, MB = 4096, 64, 128, 16, 128
    assert P.pa_paged_attn_decode_workspace_size(S, H, D, B, MB) > (16 << 20)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.pa_paged_attn_decode_noalloc(None, None, None, None, None, None, ctypes.c_float(1.0),
                                          S, H, D, B, MB, 1 << 20, P.binding.PA_F16,
                                          ctypes.c_void_p(status.data_ptr()), None)
    assert rc == P.binding.PA_ERR_TOO_LARGE
    assert "scratch" in P.pa_status_string(rc)


def test_noalloc_limit_is_the_16bit_kernels_need(P):
    """The 16 MiB limit applies to what the 16-bit kernels, the only ones
    this call runs, need.  At 256 texts x 40 heads x 128 (blocks of 16, 128
    per text) the general workspace query, which also sizes for the 8-bit
    kernel's larger grid, asks for more than 16 MiB; the call still accepts
    the size and matches the workspace entry point."""
    w = W.skewed(block_size=16, device="cuda")
    assert (w.num_seqs, w.num_heads, w.head_dim, w.max_blocks_per_seq) == (256, 40, 128, 128)
    assert P.pa_paged_attn_decode_workspace_size(256, 40, 128, 16, 128) > (16 << 20)
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping)
    ref = torch.empty_like(w.q)
    P.pa_paged_attn_decode(ref, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                           w.scale)
    out = torch.full_like(w.q, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = _noalloc_raw(P, out, w, status)
    torch.cuda.synchronize()
    assert rc == 0, P.pa_status_string(rc)
    assert status.item() == 0
    c = compare(out, ref.double().cpu().numpy(), w.q.dtype)
    assert c.ok, str(c)
