"""The 8-bit (E4M3) KV cache on the GPU against the oracle: the quantizing
write bit for bit over whole pools, decode attention within the fp16/bf16
tolerance (the oracle attends over the same codes, widened exactly)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_326_b200 import workloads as W
from tests.gpu_helpers import (compare, gpu_step_fp8, new_status, oracle_inputs, run_oracle_fp8)

pytestmark = pytest.mark.gpu

SHAPE_LENS = [0, 1, 3, 16, 17, 33, 64, 100, 129, 160]


@pytest.fixture(scope="module", autouse=True)
def lib():
    from paged_kv_cache_326_b200 import build
    build.build()
    import paged_kv_cache_326_b200 as P
    return P.lib()


@pytest.fixture(params=[1, 0], ids=["cuda_cores", "auto"])
def fp8_kernel(request):
    """PA_OPT_FP8_KERNEL: 1 the CUDA-core kernel everywhere; 0 the default
    (tensor cores for fp16 queries, head_dim 128, blocks of 8-32)."""
    import paged_kv_cache_326_b200 as P
    P.pa_set_option(P.PA_OPT_FP8_KERNEL, request.param)
    yield request.param
    P.pa_set_option(P.PA_OPT_FP8_KERNEL, 0)


def gpu_step_fp8_fused(w, status=None, out=None):
    """The 8-bit step through the one-launch entry point pa_decode_step_fp8."""
    import paged_kv_cache_326_b200 as P
    if out is None:
        out = torch.empty_like(w.q)
    P.pa_decode_step_fp8(out, w.q, w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping,
                         w.block_tables, w.context_lens, w.scale, w.meta["k_scale"],
                         w.meta["v_scale"], status=status)
    return out


def parity_fp8(w, seqs=None, heads_per_seq=None, seed=0, step=gpu_step_fp8):
    S, H, D = w.q.shape
    seqs = np.arange(S) if seqs is None else np.asarray(seqs)
    pairs = None
    if heads_per_seq is not None and heads_per_seq < H:
        rng = np.random.default_rng(seed)
        pairs = [(int(s), int(h)) for s in seqs for h in rng.choice(H, heads_per_seq, replace=False)]
    oi = oracle_inputs(w.q, w.k, w.v, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                       w.slot_mapping, w.block_size, seqs)
    kb, vb = w.k_cache.cpu().numpy(), w.v_cache.cpu().numpy()
    st = new_status()
    out = step(w, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    ks, vs = w.meta["k_scale"], w.meta["v_scale"]
    ek, ev = oracle.cache_write_fp8(kb, vb, w.k.float().cpu().numpy(), w.v.float().cpu().numpy(),
                                    w.slot_mapping.cpu().numpy(), w.block_size, ks, vs)
    assert np.array_equal(w.k_cache.cpu().numpy(), ek), "8-bit k pool differs"
    assert np.array_equal(w.v_cache.cpu().numpy(), ev), "8-bit v pool differs"
    ref = run_oracle_fp8(oi, w.scale, w.block_size, ks, vs, pairs)
    got = out.index_select(0, torch.as_tensor(seqs, device=out.device))
    mask = None
    if pairs is not None:
        pos = {int(s): i for i, s in enumerate(seqs)}
        mask = np.zeros((len(seqs), H, D), dtype=bool)
        for s, h in pairs:
            mask[pos[s], h] = True
    c = compare(got, ref, w.q.dtype, mask)
    assert c.ok, f"{w.name}: {c}"
    return c


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("block_size", [4, 8, 16, 32])
def test_fp8_every_shape_ragged(dtype, head_dim, block_size, fp8_kernel):
    w = W.make_decode_fp8("fp8_shape", SHAPE_LENS, num_heads=3, head_dim=head_dim,
                          block_size=block_size,
                          num_blocks=3 * sum(W.blocks_needed(L, block_size) for L in SHAPE_LENS),
                          dtype=dtype, seed=head_dim + block_size, device="cuda",
                          max_blocks_per_seq=160 // block_size)
    parity_fp8(w)


def test_fp8_opt13b_batch64(fp8_kernel):
    w = W.opt13b_batch64_fp8(device="cuda")
    c = parity_fp8(w, heads_per_seq=6, seed=3)
    print("fp8 opt13b", fp8_kernel, c)


def test_fp8_tensor_cores_all_outputs_of_a_large_batch():
    """The tensor-core kernel forced on 24 texts of the batch-64 shapes
    (lengths 128..2048), every head against the oracle."""
    import paged_kv_cache_326_b200 as P
    lens = W.opt13b_batch64_lens()[:24]
    need = sum(W.blocks_needed(L, 16) for L in lens)
    w = W.make_decode_fp8("fp8_first24", lens, num_heads=40, head_dim=128, block_size=16,
                          num_blocks=(3 * need + 1) // 2, dtype=torch.float16, seed=12,
                          device="cuda", max_blocks_per_seq=128)
    P.pa_set_option(P.PA_OPT_FP8_KERNEL, 2)
    try:
        c = parity_fp8(w)
    finally:
        P.pa_set_option(P.PA_OPT_FP8_KERNEL, 0)
    print("fp8 tensor cores, 24 texts", c)


def test_fp8_tensor_cores_refuse_what_they_do_not_cover():
    """Forcing the tensor-core kernel where it does not apply (bf16 queries,
    head_dim 64, blocks of 4) is an argument error, not a silent fallback."""
    import paged_kv_cache_326_b200 as P
    P.pa_set_option(P.PA_OPT_FP8_KERNEL, 2)
    try:
        for dtype, D, B in ((torch.bfloat16, 128, 16), (torch.float16, 64, 16),
                            (torch.float16, 128, 4)):
            w = W.make_decode_fp8("fp8_refuse", [5, 40], num_heads=2, head_dim=D, block_size=B,
                                  num_blocks=32, dtype=dtype, seed=1, device="cuda",
                                  max_blocks_per_seq=64 // B)
            with pytest.raises(P.PagedAttnError):
                P.pa_paged_attn_decode_fp8(torch.empty_like(w.q), w.q, w.k_cache, w.v_cache,
                                           w.block_tables, w.context_lens, w.scale,
                                           w.meta["k_scale"], w.meta["v_scale"])
    finally:
        P.pa_set_option(P.PA_OPT_FP8_KERNEL, 0)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("group", [2, 4, 5, 8])
@pytest.mark.parametrize("head_dim,block_size", [(64, 8), (128, 16), (128, 4), (64, 32)],
                         ids=["d64b8", "d128b16", "d128b4", "d64b32"])
def test_fp8_grouped_query_every_shape(dtype, group, head_dim, block_size):
    """Grouped-query pools of 8-bit codes (pa_paged_attn_decode_fp8_gqa):
    2 key/value heads, each shared by `group` query heads, ragged lengths
    from 0 to 160; the quantizing write bit for bit, every output against
    the oracle."""
    w = W.make_decode_fp8("fp8_gqa", SHAPE_LENS, num_heads=2 * group, head_dim=head_dim,
                          block_size=block_size,
                          num_blocks=3 * sum(W.blocks_needed(L, block_size) for L in SHAPE_LENS),
                          dtype=dtype, seed=group * 7 + head_dim + block_size, device="cuda",
                          max_blocks_per_seq=160 // block_size, num_kv_heads=2)
    parity_fp8(w)


def test_fp8_grouped_query_llama2_70b(fp8_kernel):
    """The Llama-2-70B-shaped layer (64 query heads over 8 key/value heads,
    lengths 128..4096) over 8-bit caches: 12 texts x 8 sampled heads each."""
    w = W.llama2_70b_gqa_fp8(device="cuda", num_seqs=24, num_blocks=6144)
    c = parity_fp8(w, seqs=range(0, 24, 2), heads_per_seq=8, seed=5)
    print("fp8 grouped-query llama2-70b", fp8_kernel, c)


@pytest.mark.parametrize("group", [2, 3, 8, 12, 16])
@pytest.mark.parametrize("block_size", [8, 16, 32])
def test_fp8_grouped_query_tensor_cores(group, block_size):
    """The tensor-core kernel forced on grouped-query 8-bit pools: a key/value
    head's query heads are the tile's columns (groups above 8 in equal
    subsets of at most 8: 12 as 2 x 6, 16 as 2 x 8; 3 leaves columns that
    repeat a head); ragged lengths 0..300 spanning several chunks and a
    partial last one; every output against the oracle."""
    import paged_kv_cache_326_b200 as P
    lens = [0, 1, 7, 31, 32, 33, 95, 160, 300, 257, 64, 5]
    w = W.make_decode_fp8("fp8_gqa_tc", lens, num_heads=3 * group, head_dim=128,
                          block_size=block_size,
                          num_blocks=3 * sum(W.blocks_needed(L, block_size) for L in lens),
                          dtype=torch.float16, seed=group * 11 + block_size, device="cuda",
                          max_blocks_per_seq=320 // block_size, num_kv_heads=3)
    P.pa_set_option(P.PA_OPT_FP8_KERNEL, 2)
    try:
        parity_fp8(w)
    finally:
        P.pa_set_option(P.PA_OPT_FP8_KERNEL, 0)


def test_fp8_grouped_query_tensor_cores_all_outputs_of_a_large_batch():
    """The tensor-core kernel forced on 16 texts of the Llama-2-70B shape
    (64 query heads over 8 key/value heads, lengths up to 4096): every head
    of every text against the oracle, so texts split across many warps and
    merged are covered."""
    import paged_kv_cache_326_b200 as P
    w = W.llama2_70b_gqa_fp8(device="cuda", num_seqs=16, num_blocks=4096)
    P.pa_set_option(P.PA_OPT_FP8_KERNEL, 2)
    try:
        c = parity_fp8(w)
    finally:
        P.pa_set_option(P.PA_OPT_FP8_KERNEL, 0)
    print("fp8 grouped-query tensor cores, 16 texts", c)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("block_size", [4, 8, 16, 32])
def test_fp8_one_launch_step_every_shape_ragged(dtype, head_dim, block_size, fp8_kernel):
    """pa_decode_step_fp8: the new tokens' codes in the pool bit for bit, every
    output against the oracle (which writes, then attends)."""
    w = W.make_decode_fp8("fp8_step", SHAPE_LENS, num_heads=3, head_dim=head_dim,
                          block_size=block_size,
                          num_blocks=3 * sum(W.blocks_needed(L, block_size) for L in SHAPE_LENS),
                          dtype=dtype, seed=head_dim * 3 + block_size, device="cuda",
                          max_blocks_per_seq=160 // block_size)
    parity_fp8(w, step=gpu_step_fp8_fused)


def test_fp8_one_launch_step_opt13b_batch64():
    w = W.opt13b_batch64_fp8(device="cuda")
    c = parity_fp8(w, heads_per_seq=6, seed=4, step=gpu_step_fp8_fused)
    print("fp8 one-launch step opt13b", c)


def test_fp8_one_launch_step_equals_two_calls_bitwise(fp8_kernel):
    """Same inputs, same kernel (CUDA cores, or the default: tensor cores):
    the one-launch 8-bit step and the quantizing write followed by the 8-bit
    decode give the same output and the same pools, bit for bit (the new
    row's codes come from the same quantizer)."""
    a = W.opt13b_batch64_fp8(device="cuda")
    b = W.opt13b_batch64_fp8(device="cuda")
    out_a = gpu_step_fp8(a)
    out_b = gpu_step_fp8_fused(b)
    torch.cuda.synchronize()
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.v_cache, b.v_cache)
    assert torch.equal(out_a, out_b)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
def test_fp8_one_launch_step_single_token_returns_its_value(dtype):
    """One token per text, the new one: out = value(code(v / v_scale)) *
    v_scale rounded to the output type, bit for bit (fp16: the tensor-core
    kernel, whose stage row is the new token's codes; bf16: CUDA cores)."""
    w = W.make_decode_fp8("fp8_step_one", [1] * 6, num_heads=5, head_dim=128, block_size=16,
                          num_blocks=16, dtype=dtype, seed=8, device="cuda")
    out = gpu_step_fp8_fused(w)
    torch.cuda.synchronize()
    vs = np.float32(w.meta["v_scale"])
    codes = oracle.quantize(w.v.float().cpu().numpy(), vs)
    vals = torch.from_numpy(oracle.e4m3_decode(codes).astype(np.float32))
    want = (vals * torch.tensor(vs)).to(out.dtype)
    assert torch.equal(out.cpu(), want)


def test_fp8_write_rounds_saturates_and_keeps_signs():
    """Inputs at ties, past the largest code (saturating), subnormal and
    signed zero, through both scales: codes equal the oracle's."""
    import paged_kv_cache_326_b200 as P
    H, D, B, N = 2, 64, 8, 4
    ks, vs = 0.5, 2.0
    base = torch.tensor([0.0, -0.0, 1.0625, 1.1875, 600.0, -1e4, 2.0 ** -11, 0.3, -2.5, 447.9],
                        dtype=torch.float32)
    row = torch.cat([base, torch.linspace(-300, 300, D - base.numel())])
    k = torch.stack([row * ks, -row * ks]).view(1, 2, D).repeat(3, 1, 1).to(torch.float16)
    v = torch.stack([row * vs, row * vs * 0.5]).view(1, 2, D).repeat(3, 1, 1).to(torch.float16)
    kc = torch.full((N, H, B, D), 0x55, dtype=torch.uint8)
    vc = kc.clone()
    slots = torch.tensor([3, -1, 17])
    ek, ev = oracle.cache_write_fp8(kc.numpy(), vc.numpy(), k.float().numpy(), v.float().numpy(),
                                    slots.numpy(), B, ks, vs)
    kd, vd = kc.cuda(), vc.cuda()
    st = new_status()
    P.pa_kv_cache_write_fp8(k.cuda(), v.cuda(), kd, vd, slots.cuda(), ks, vs, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert np.array_equal(kd.cpu().numpy(), ek) and np.array_equal(vd.cpu().numpy(), ev)


def test_fp8_single_token_returns_its_value(fp8_kernel):
    """One stored token: the output is value(code) * v_scale rounded to the
    output type, bit for bit."""
    w = W.make_decode_fp8("fp8_one", [1] * 6, num_heads=5, head_dim=128, block_size=16,
                          num_blocks=16, dtype=torch.float16, seed=3, device="cuda")
    out = gpu_step_fp8(w)
    torch.cuda.synchronize()
    vs = np.float32(w.meta["v_scale"])
    codes = oracle.quantize(w.v.float().cpu().numpy(), vs)          # IEEE fp32 quotient
    vals = torch.from_numpy(oracle.e4m3_decode(codes).astype(np.float32))
    want = (vals * torch.tensor(vs)).to(out.dtype)                   # fp32 product, then RN
    assert torch.equal(out.cpu(), want)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
def test_fp8_split_and_single_pass_agree(dtype, fp8_kernel):
    import paged_kv_cache_326_b200 as P
    for warps in (1, 4096):
        P.pa_set_option(P.binding.PA_OPT_DECODE_WARPS, warps)
        try:
            parity_fp8(W.make_decode_fp8("fp8_split", [300, 17, 1, 1000, 64, 0, 511, 129],
                                         num_heads=4, head_dim=128, block_size=16,
                                         num_blocks=256, dtype=dtype, seed=9,
                                         device="cuda", max_blocks_per_seq=64))
        finally:
            P.pa_set_option(P.binding.PA_OPT_DECODE_WARPS, 0)


def test_fp8_pools_copy_bit_exact():
    import paged_kv_cache_326_b200 as P
    g = torch.Generator().manual_seed(5)
    kc = torch.randint(0, 256, (40, 3, 16, 128), generator=g, dtype=torch.uint8).cuda()
    vc = torch.randint(0, 256, (40, 3, 16, 128), generator=g, dtype=torch.uint8).cuda()
    pairs = [(1, 30), (2, 31), (2, 32), (39, 0)]
    ek, ev = oracle.copy_blocks(kc.cpu().numpy(), vc.cpu().numpy(), kc.cpu().numpy(),
                                vc.cpu().numpy(), pairs)
    P.pa_copy_blocks(kc, vc, kc, vc, torch.tensor(pairs, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(kc.cpu().numpy(), ek) and np.array_equal(vc.cpu().numpy(), ev)


@pytest.mark.parametrize("bad", [0.0, -1.0, float("inf"), float("nan")])
def test_fp8_scales_must_be_finite_and_positive(bad):
    import paged_kv_cache_326_b200 as P
    w = W.make_decode_fp8("fp8_bad", [5, 9], num_heads=2, head_dim=64, block_size=8,
                          num_blocks=8, dtype=torch.float16, seed=1, device="cuda")
    with pytest.raises(P.PagedAttnError):
        P.pa_kv_cache_write_fp8(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, bad, 1.0)
    with pytest.raises(P.PagedAttnError):
        P.pa_paged_attn_decode_fp8(torch.empty_like(w.q), w.q, w.k_cache, w.v_cache,
                                   w.block_tables, w.context_lens, w.scale, 1.0, bad)
