"""The prompt phase on the GPU (pa_prefill) against the oracle: causal
attention within each packed prompt, within the fp16/bf16 tolerance, and the
prompts' keys and values stored bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_326_b200 import workloads as W
from tests.gpu_helpers import compare, host_f32, new_status

pytestmark = pytest.mark.gpu

LENS = [1, 7, 63, 64, 65, 130, 0, 300, 1000]


@pytest.fixture(scope="module", autouse=True)
def lib():
    from paged_kv_cache_326_b200 import build
    build.build()
    import paged_kv_cache_326_b200 as P
    return P.lib()


# PA_OPT_PREFILL_KERNEL values: 5th-generation tensor cores, warp-level MMA
PREFILL_KERNELS = {"tcgen05": 2, "mma": 1}


@pytest.fixture(params=list(PREFILL_KERNELS))
def prefill_kernel(request):
    """Run the test once on each prefill kernel."""
    import paged_kv_cache_326_b200 as P
    P.pa_set_option(P.PA_OPT_PREFILL_KERNEL, PREFILL_KERNELS[request.param])
    yield request.param
    P.pa_set_option(P.PA_OPT_PREFILL_KERNEL, 0)


def run_prefill(w, status=None, store=True):
    import paged_kv_cache_326_b200 as P
    out = torch.empty_like(w.q)
    if store:
        P.pa_prefill(out, w.q, w.k, w.v, w.cu_seqlens, w.max_seqlen, w.scale, w.k_cache,
                     w.v_cache, w.slot_mapping, status=status)
    else:
        P.pa_prefill(out, w.q, w.k, w.v, w.cu_seqlens, w.max_seqlen, w.scale, status=status)
    return out


def check(w, rows=None):
    kb = w.k_cache.view(torch.int16).cpu().numpy()
    vb = w.v_cache.view(torch.int16).cpu().numpy()
    st = new_status()
    out = run_prefill(w, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    ek, ev = oracle.cache_write(kb, vb, w.k.view(torch.int16).cpu().numpy(),
                                w.v.view(torch.int16).cpu().numpy(),
                                w.slot_mapping.cpu().numpy(), w.block_size)
    assert np.array_equal(w.k_cache.view(torch.int16).cpu().numpy(), ek), "k pool"
    assert np.array_equal(w.v_cache.view(torch.int16).cpu().numpy(), ev), "v pool"
    ref = oracle.prefill(host_f32(w.q), host_f32(w.k), host_f32(w.v), w.cu_seqlens.cpu().numpy(),
                         w.scale)
    got = out
    if rows is not None:
        ref, got = ref[rows], out[torch.as_tensor(rows, device=out.device)]
    c = compare(got, ref, w.q.dtype)
    assert c.ok, f"{w.name}: {c}"
    return c


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("heads", [(4, 4), (8, 2), (6, 1)], ids=lambda hk: f"q{hk[0]}kv{hk[1]}")
def test_prefill_ragged_prompts(dtype, head_dim, heads, prefill_kernel):
    Hq, Hkv = heads
    w = W.make_prefill("prefill", LENS, Hq, Hkv, head_dim, dtype, seed=head_dim + Hq,
                       device="cuda")
    c = check(w)
    print(f"prefill {prefill_kernel} {dtype} D{head_dim} q{Hq}kv{Hkv}", c)


def test_prefill_opt13b_sampled_rows(prefill_kernel):
    """16 prompts of 2,048 tokens x 40 heads: a sample of rows spread over
    every tile, the diagonal ones and each prompt's last."""
    w = W.opt13b_prefill(device="cuda", num_prompts=4)
    rng = np.random.default_rng(7)
    rows = sorted(set(rng.choice(w.q.shape[0], 64, replace=False).tolist()) |
                  {int(x) - 1 for x in w.cu_seqlens[1:].tolist()} | {0, 63, 64, 2047, 2048})
    c = check(w, rows)
    print(f"prefill {prefill_kernel} opt13b", c)


def test_prefill_first_position_returns_its_value(prefill_kernel):
    for dtype in (torch.float16, torch.bfloat16):
        w = W.make_prefill("first", [5, 1, 70], 4, 2, 128, dtype, seed=3, device="cuda")
        out = run_prefill(w, store=False)
        torch.cuda.synchronize()
        for s in range(3):
            a = int(w.cu_seqlens[s])
            assert torch.equal(out[a], w.v[a].repeat_interleave(2, dim=0)), dtype


def test_prefill_bad_offsets_and_short_max_seqlen_are_reported(prefill_kernel):
    import paged_kv_cache_326_b200 as P
    w = W.make_prefill("bad", [10, 20], 2, 2, 64, torch.float16, seed=4, device="cuda")
    st = new_status()
    bad = torch.tensor([0, 25, 20], dtype=torch.int32, device="cuda")   # decreasing
    P.pa_prefill(torch.empty_like(w.q), w.q, w.k, w.v, bad, 25, w.scale, status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_LEN
    st = new_status()
    P.pa_prefill(torch.empty_like(w.q), w.q, w.k, w.v, w.cu_seqlens, 8, w.scale, status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_LEN
    check(W.make_prefill("after", [10, 20], 2, 2, 64, torch.float16, seed=4, device="cuda"))


def test_prefill_then_decode_continues_the_prompt():
    """The stored prompt feeds the decode step: after pa_prefill, one decode
    step (write the next token, attend) agrees with the oracle's decode over
    the prompt plus that token."""
    import paged_kv_cache_326_b200 as P
    lens = [37, 100, 5]
    w = W.make_prefill("cont", lens, 8, 8, 128, torch.float16, seed=5, device="cuda",
                       spare_blocks=16)
    run_prefill(w)
    g = torch.Generator(device="cuda").manual_seed(6)
    S, H, D, B = 3, 8, 128, w.block_size
    q = torch.randn(S, H, D, generator=g, device="cuda").half()
    k = torch.randn(S, H, D, generator=g, device="cuda").half()
    v = torch.randn(S, H, D, generator=g, device="cuda").half()
    tables = w.block_tables.clone()
    # room for the next token: prompts ending on a block boundary get a spare block
    used = set(tables[tables >= 0].tolist())
    spare = [b for b in range(w.k_cache.shape[0]) if b not in used]
    mb = tables.shape[1] + 1
    t2 = torch.full((S, mb), -1, dtype=torch.int32, device="cuda")
    t2[:, :tables.shape[1]] = tables
    slots = []
    for s, L in enumerate(lens):
        if L % B == 0:
            t2[s, L // B] = spare.pop()
        slots.append(int(t2[s, L // B]) * B + L % B)
    slots = torch.tensor(slots, device="cuda")
    ctx = torch.tensor([L + 1 for L in lens], dtype=torch.int32, device="cuda")
    kc0 = host_f32(w.k_cache)
    vc0 = host_f32(w.v_cache)
    P.pa_kv_cache_write(k, v, w.k_cache, w.v_cache, slots)
    out = torch.empty_like(q)
    P.pa_paged_attn_decode(out, q, w.k_cache, w.v_cache, t2, ctx, w.scale)
    torch.cuda.synchronize()
    kc, vc = oracle.cache_write(kc0, vc0, host_f32(k), host_f32(v), slots.cpu().numpy(), B)
    ref = oracle.paged_decode(host_f32(q), kc, vc, t2.cpu().numpy(), ctx.cpu().numpy(), w.scale, B)
    c = compare(out, ref, torch.float16)
    assert c.ok, c


def test_prefill_kernels_agree_and_are_deterministic():
    """Both prefill kernels compute the same function: equal within the
    tolerance; each bitwise reproducible run to run."""
    import paged_kv_cache_326_b200 as P
    w = W.make_prefill("agree", [700, 129, 1, 64], 8, 2, 128, torch.bfloat16, seed=8,
                       device="cuda")
    res = {}
    try:
        for name, mode in PREFILL_KERNELS.items():
            P.pa_set_option(P.PA_OPT_PREFILL_KERNEL, mode)
            a = run_prefill(w, store=False)
            b = run_prefill(w, store=False)
            torch.cuda.synchronize()
            assert torch.equal(a, b), name
            res[name] = a
    finally:
        P.pa_set_option(P.PA_OPT_PREFILL_KERNEL, 0)
    diff = (res["tcgen05"].float() - res["mma"].float()).abs().max().item()
    assert diff <= 2e-2, diff


def test_prefill_tcgen05_wait_limit_gives_up_cleanly():
    """A wait limit below zero makes every barrier wait give up at once: the
    kernel records PA_ERR_TIMEOUT, drains what it issued, frees its tensor
    memory and returns; the next call is correct."""
    import paged_kv_cache_326_b200 as P
    w = W.make_prefill("timeout", [200, 70], 4, 4, 128, torch.float16, seed=9, device="cuda")
    st = new_status()
    P.pa_set_option(P.PA_OPT_PREFILL_KERNEL, 2)
    P.pa_set_option(P.binding.PA_OPT_WAIT_LIMIT_NS, -1)
    try:
        run_prefill(w, st, store=False)
        torch.cuda.synchronize()
    finally:
        P.pa_set_option(P.binding.PA_OPT_WAIT_LIMIT_NS, 1_000_000_000)
        P.pa_set_option(P.PA_OPT_PREFILL_KERNEL, 0)
    assert st.item() == P.binding.PA_ERR_TIMEOUT
    check(W.make_prefill("after", [200, 70], 4, 4, 128, torch.float16, seed=9, device="cuda"))
