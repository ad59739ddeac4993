"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Cache writes: bit-exact over the whole pool, untouched slots included.
Attention: the fp16 / bf16 tolerance in tests/gpu_helpers.py.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_326_b200 import workloads as W
from tests.gpu_helpers import (compare, gpu_step, gpu_step_fused, new_status, oracle_inputs,
                               run_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from paged_kv_cache_326_b200 import build
    build.build()
    import paged_kv_cache_326_b200 as P
    return P.lib()


def _pairs_mask(pairs, S_sel, seqs, H, D):
    pos = {int(s): i for i, s in enumerate(seqs)}
    m = np.zeros((S_sel, H, D), dtype=bool)
    for s, h in pairs:
        m[pos[int(s)], int(h)] = True
    return m


def parity(w, seqs=None, heads_per_seq=None, seed=0, check_pool=False, step=gpu_step):
    """GPU decode step (two calls, or the fused one) vs the oracle."""
    S, H, D = w.q.shape
    seqs = np.arange(S) if seqs is None else np.asarray(seqs)
    pairs = None
    if heads_per_seq is not None and heads_per_seq < H:
        rng = np.random.default_rng(seed)
        pairs = [(int(s), int(h)) for s in seqs for h in rng.choice(H, heads_per_seq, replace=False)]
    oi = oracle_inputs(w.q, w.k, w.v, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                       w.slot_mapping, w.block_size, seqs)
    if check_pool:
        kb = w.k_cache.view(torch.int16).cpu().numpy()
        vb = w.v_cache.view(torch.int16).cpu().numpy()
    st = new_status()
    out = step(w, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    if check_pool:
        ek, ev = oracle.cache_write(kb, vb, w.k.view(torch.int16).cpu().numpy(),
                                    w.v.view(torch.int16).cpu().numpy(),
                                    w.slot_mapping.cpu().numpy(), w.block_size)
        assert np.array_equal(w.k_cache.view(torch.int16).cpu().numpy(), ek), "k pool differs"
        assert np.array_equal(w.v_cache.view(torch.int16).cpu().numpy(), ev), "v pool differs"
        del kb, vb, ek, ev
    ref = run_oracle(oi, w.scale, w.block_size, pairs)
    got = out.index_select(0, torch.as_tensor(seqs, device=out.device))
    mask = None if pairs is None else _pairs_mask(pairs, len(seqs), seqs, H, D)
    c = compare(got, ref, w.q.dtype, mask)
    assert c.ok, f"{w.name}: {c}"
    return c


# ---------------------------------------------------------------------------
# the five named workloads
# ---------------------------------------------------------------------------

def test_tiny():
    parity(W.tiny(device="cuda"), check_pool=True)


def test_opt13b_batch64_full_parity_and_write():
    w = W.opt13b_batch64(device="cuda")
    c = parity(w, check_pool=True)
    print("opt13b_batch64", c)


@pytest.mark.parametrize("block_size", [8, 16, 32])
def test_skewed_bf16(block_size):
    w = W.skewed(block_size=block_size, device="cuda")
    c = parity(w, heads_per_seq=4, seed=block_size)
    print(f"skewed B={block_size}", c)


def test_shared_prefix_through_block_manager():
    import paged_kv_cache_326_b200 as P
    bm = P.BlockManager(8192, 16)

    class Adapter:
        add_seq = staticmethod(bm.add_seq)
        fork = staticmethod(bm.fork)
        append_slot = staticmethod(bm.append_slot)

        @staticmethod
        def export(ids, mb):
            t, l = bm.export(ids, mb)
            return t.numpy(), l.numpy()

    w = W.shared_prefix(Adapter(), num_blocks=8192, device="cuda")
    assert len(w.meta["cow"]) > 0
    # samples of one prompt share their prompt's full blocks
    t = w.block_tables.cpu()
    assert (t[0, :8] == t[7, :8]).all()
    c = parity(w, heads_per_seq=3, seed=4)
    print("shared_prefix", c)


@pytest.mark.slow
def test_full_step_40_layers():
    """40 layers x (write + attend) over one shared pool (blocks alias across
    layers); the oracle replays every layer's writes and checks every head of
    6 sampled texts on 5 layers."""
    import paged_kv_cache_326_b200 as P
    fs = W.full_step(device="cuda")
    B = fs.block_size
    check_layers = [0, 9, 21, 30, 39]
    rng = np.random.default_rng(5)
    seqs = np.sort(rng.choice(fs.context_lens.numel(), 6, replace=False))
    sel = torch.as_tensor(seqs, device="cuda")
    need = torch.unique(torch.cat([fs.block_tables[l].index_select(0, sel).flatten()
                                   for l in check_layers]))
    need = need[need >= 0]
    N = fs.k_cache.shape[0]
    remap = torch.full((N,), -1, dtype=torch.int64, device="cuda")
    remap[need] = torch.arange(need.numel(), device="cuda")
    kc = fs.k_cache.index_select(0, need).float().cpu().numpy()
    vc = fs.v_cache.index_select(0, need).float().cpu().numpy()

    st = new_status()
    outs = {}
    for layer in range(fs.num_layers):
        P.pa_kv_cache_write(fs.k[layer], fs.v[layer], fs.k_cache, fs.v_cache,
                            fs.slot_mapping[layer], status=st)
        out = torch.empty_like(fs.q[layer])
        P.pa_paged_attn_decode(out, fs.q[layer], fs.k_cache, fs.v_cache, fs.block_tables[layer],
                               fs.context_lens, fs.scale, status=st)
        if layer in check_layers:
            outs[layer] = out
    torch.cuda.synchronize()
    assert st.item() == 0

    H = fs.q[0].shape[1]
    done = 0
    for layer in check_layers:
        ks, vs, slots = [], [], []
        for l2 in range(done, layer + 1):
            s = fs.slot_mapping[l2]
            nb = remap[(s // B).clamp(min=0)]
            hit = (s >= 0) & (nb >= 0)
            idx = torch.nonzero(hit).flatten()
            ks.append(fs.k[l2].index_select(0, idx).float().cpu().numpy())
            vs.append(fs.v[l2].index_select(0, idx).float().cpu().numpy())
            slots.append((nb[idx] * B + s[idx] % B).cpu().numpy())
        done = layer + 1
        kc, vc = oracle.cache_write(kc, vc, np.concatenate(ks), np.concatenate(vs),
                                    np.concatenate(slots), B)
        t = fs.block_tables[layer].index_select(0, sel).to(torch.int64)
        t = torch.where(t >= 0, remap[t.clamp(min=0)], torch.full_like(t, -1)).cpu().numpy()
        assert (t[t >= 0] >= 0).all()
        q = fs.q[layer].index_select(0, sel).float().cpu().numpy()
        pairs = [(i, h) for i in range(len(seqs)) for h in range(H)]
        ref = oracle.paged_decode(q, kc, vc, t, fs.context_lens.index_select(0, sel).cpu().numpy(),
                                  fs.scale, B, pairs)
        mask = np.zeros(ref.shape, dtype=bool)
        for i, h in pairs:
            mask[i, h] = True
        c = compare(outs[layer].index_select(0, sel), ref, torch.float16, mask)
        assert c.ok, f"layer {layer}: {c}"
        print(f"full_step layer {layer}", c)


# ---------------------------------------------------------------------------
# every compiled shape, ragged lengths, edge cases
# ---------------------------------------------------------------------------

SHAPE_LENS = [0, 1, 3, 16, 17, 33, 64, 100, 129, 160]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("block_size", [4, 8, 16, 32])
def test_every_shape_ragged(dtype, head_dim, block_size):
    w = W.make_decode("shape", SHAPE_LENS, num_heads=3, head_dim=head_dim, block_size=block_size,
                      num_blocks=3 * sum(W.blocks_needed(L, block_size) for L in SHAPE_LENS),
                      dtype=dtype, seed=head_dim + block_size, device="cuda",
                      max_blocks_per_seq=160 // block_size)
    parity(w, check_pool=True)


def test_single_token_returns_its_value_exactly():
    w = W.make_decode("one", [1] * 7, num_heads=5, head_dim=128, block_size=16, num_blocks=16,
                      dtype=torch.float16, seed=3, device="cuda")
    out = gpu_step(w)
    torch.cuda.synchronize()
    assert torch.equal(out, w.v), "one token: output must be its value, bit for bit"


def test_empty_texts_give_zeros():
    w = W.make_decode("empty", [0, 5, 0, 40], num_heads=2, head_dim=64, block_size=8,
                      num_blocks=16, dtype=torch.float16, seed=4, device="cuda")
    out = gpu_step(w)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0
    assert torch.isfinite(out).all()


def test_run_to_run_bitwise_determinism():
    w = W.opt13b_batch64(device="cuda")
    import paged_kv_cache_326_b200 as P
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping)
    outs = []
    for _ in range(3):
        out = torch.empty_like(w.q)
        P.pa_paged_attn_decode(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                               w.scale)
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


@pytest.mark.parametrize("warps", [1, 7, 4096])
def test_split_and_single_pass_agree(warps):
    """1 warp: no text is split (single pass).  Many warps: every text is cut
    into many partials merged by the log-sum-exp reduce.  Both match the
    oracle and each other."""
    import paged_kv_cache_326_b200 as P
    lens = [300, 17, 1, 1000, 64, 0, 511, 129]
    w = W.make_decode("split", lens, num_heads=4, head_dim=128, block_size=16, num_blocks=256,
                      dtype=torch.float16, seed=9, device="cuda", max_blocks_per_seq=64)
    P.pa_set_option(P.binding.PA_OPT_DECODE_WARPS, warps)
    try:
        c = parity(w)
    finally:
        P.pa_set_option(P.binding.PA_OPT_DECODE_WARPS, 0)
    print(f"warps={warps}", c)


# ---------------------------------------------------------------------------
# bad data is reported through the status word, never faults
# ---------------------------------------------------------------------------

def test_block_id_outside_pool_is_reported_and_skipped():
    import paged_kv_cache_326_b200 as P
    w = W.tiny(device="cuda")
    w.block_tables[2, 1] = w.num_blocks + 7
    st = new_status()
    gpu_step(w, st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_BLOCK
    parity(W.tiny(device="cuda"))          # the context is still healthy


def test_context_length_past_table_is_reported():
    import paged_kv_cache_326_b200 as P
    w = W.tiny(device="cuda")
    w.context_lens[1] = w.max_blocks_per_seq * w.block_size + 5
    out = torch.empty_like(w.q)
    st = new_status()
    P.pa_paged_attn_decode(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                           w.scale, status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_LEN


def test_slot_outside_pool_is_reported_and_skipped():
    import paged_kv_cache_326_b200 as P
    w = W.tiny(device="cuda")
    before = w.k_cache.clone()
    w.slot_mapping[0] = w.num_blocks * w.block_size + 3
    w.slot_mapping[1] = -1
    st = new_status()
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_SLOT
    expect, _ = oracle.cache_write(before.view(torch.int16).cpu().numpy(),
                                   before.view(torch.int16).cpu().numpy(),
                                   w.k.view(torch.int16).cpu().numpy(),
                                   w.k.view(torch.int16).cpu().numpy(),
                                   [-1, -1] + w.slot_mapping[2:].tolist(), w.block_size)
    assert np.array_equal(w.k_cache.view(torch.int16).cpu().numpy(), expect)


def test_bounded_wait_gives_up_with_status_and_context_survives():
    """A wait limit below zero makes every barrier wait give up at once: the
    kernel records PA_ERR_TIMEOUT, drains its copies and returns; the next
    call, with the default limit, is correct."""
    import paged_kv_cache_326_b200 as P
    w = W.tiny(device="cuda")
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping)
    out = torch.empty_like(w.q)
    st = new_status()
    P.pa_set_option(P.binding.PA_OPT_WAIT_LIMIT_NS, -1)
    try:
        P.pa_paged_attn_decode(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                               w.scale, status=st)
        torch.cuda.synchronize()
    finally:
        P.pa_set_option(P.binding.PA_OPT_WAIT_LIMIT_NS, 1_000_000_000)
    assert st.item() == P.binding.PA_ERR_TIMEOUT
    parity(W.tiny(device="cuda"))


# ---------------------------------------------------------------------------
# the one-launch step (pa_decode_step)
# ---------------------------------------------------------------------------

def test_fused_step_tiny():
    parity(W.tiny(device="cuda"), check_pool=True, step=gpu_step_fused)


def test_fused_step_opt13b_batch64():
    c = parity(W.opt13b_batch64(device="cuda"), check_pool=True, step=gpu_step_fused)
    print("fused opt13b_batch64", c)


def test_fused_step_skewed_bf16():
    c = parity(W.skewed(block_size=16, device="cuda"), heads_per_seq=4, seed=7,
               step=gpu_step_fused)
    print("fused skewed", c)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("block_size", [4, 8, 16, 32])
def test_fused_step_every_shape_ragged(dtype, head_dim, block_size):
    w = W.make_decode("shape", SHAPE_LENS, num_heads=3, head_dim=head_dim, block_size=block_size,
                      num_blocks=3 * sum(W.blocks_needed(L, block_size) for L in SHAPE_LENS),
                      dtype=dtype, seed=head_dim + block_size, device="cuda",
                      max_blocks_per_seq=160 // block_size)
    parity(w, check_pool=True, step=gpu_step_fused)


def test_fused_step_equals_two_calls_bitwise():
    """Same inputs, same split: the one-launch step and write-then-decode give
    the same output and the same pool, bit for bit."""
    a = W.opt13b_batch64(device="cuda")
    b = W.opt13b_batch64(device="cuda")
    out_a = gpu_step(a)
    out_b = gpu_step_fused(b)
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    assert torch.equal(a.v_cache.view(torch.int16), b.v_cache.view(torch.int16))


def test_fused_step_single_token_returns_its_value():
    w = W.make_decode("one", [1] * 7, num_heads=5, head_dim=128, block_size=16, num_blocks=16,
                      dtype=torch.float16, seed=3, device="cuda")
    out = gpu_step_fused(w)
    torch.cuda.synchronize()
    assert torch.equal(out, w.v)


# ---------------------------------------------------------------------------
# grouped-query attention (pa_paged_attn_decode_gqa)
# ---------------------------------------------------------------------------

def gpu_step_gqa(w, status=None, out=None):
    import paged_kv_cache_326_b200 as P
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=status)
    if out is None:
        out = torch.empty_like(w.q)
    P.pa_paged_attn_decode_gqa(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                               w.scale, status=status)
    return out


GQA_LENS = [0, 1, 17, 100, 300, 1000, 2048, 33]
# PA_OPT_GQA_KERNEL values: the tensor-core kernel, the CUDA-core kernel.
GQA_KERNELS = {"tensor": 2, "cores": 1}


@pytest.fixture(params=list(GQA_KERNELS))
def gqa_kernel(request):
    """Run the test once on each grouped-query kernel."""
    import paged_kv_cache_326_b200 as P
    P.pa_set_option(P.PA_OPT_GQA_KERNEL, GQA_KERNELS[request.param])
    yield request.param
    P.pa_set_option(P.PA_OPT_GQA_KERNEL, 0)


def _tensor_applies(Hq, Hkv, block_size):
    return Hq != Hkv and block_size >= 8


@pytest.mark.parametrize("heads", [(16, 8), (12, 4), (6, 2), (40, 8), (32, 8), (64, 8),
                                   (48, 2), (16, 1), (64, 1), (8, 8)],
                         ids=lambda hk: f"q{hk[0]}kv{hk[1]}")
def test_gqa_group_sizes(heads, gqa_kernel):
    """Group sizes 2 to 64: whole column tiles (8, 16), padded ones (3, 5, 6),
    groups split into subsets (24, 32, 64), and plain multi-head (8, 8)."""
    Hq, Hkv = heads
    if gqa_kernel == "tensor" and not _tensor_applies(Hq, Hkv, 16):
        pytest.skip("multi-head attention runs on the CUDA-core kernel")
    w = W.make_decode("gqa", GQA_LENS, num_heads=Hq, head_dim=128, block_size=16,
                      num_blocks=2 * sum(W.blocks_needed(L, 16) for L in GQA_LENS),
                      dtype=torch.float16, seed=Hq + Hkv, device="cuda",
                      max_blocks_per_seq=2048 // 16, num_kv_heads=Hkv)
    c = parity(w, check_pool=True, step=gpu_step_gqa)
    print(f"gqa {gqa_kernel} q{Hq} kv{Hkv}", c)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("block_size", [4, 8, 16, 32])
def test_gqa_every_shape_ragged(dtype, head_dim, block_size, gqa_kernel):
    """Every head_dim x block size x dtype, ragged lengths (partial chunks and
    partial blocks, whose unwritten rows hold NaN), 16 query heads on 4
    key/value heads."""
    if gqa_kernel == "tensor" and not _tensor_applies(16, 4, block_size):
        pytest.skip("blocks of 4 run on the CUDA-core kernel")
    w = W.make_decode("gqa_shape", SHAPE_LENS, num_heads=16, head_dim=head_dim,
                      block_size=block_size,
                      num_blocks=3 * sum(W.blocks_needed(L, block_size) for L in SHAPE_LENS),
                      dtype=dtype, seed=head_dim + block_size, device="cuda",
                      max_blocks_per_seq=160 // block_size, num_kv_heads=4)
    parity(w, check_pool=True, step=gpu_step_gqa)


def test_gqa_llama2_70b_shape(gqa_kernel):
    w = W.llama2_70b_gqa(device="cuda")
    c = parity(w, heads_per_seq=8, seed=6, step=gpu_step_gqa)
    print(f"gqa {gqa_kernel} llama2_70b", c)


@pytest.mark.parametrize("warps", [1, 4096])
def test_gqa_split_and_single_pass(warps, gqa_kernel):
    import paged_kv_cache_326_b200 as P
    w = W.make_decode("gqa_split", [300, 17, 1, 1000, 0, 511], num_heads=32, head_dim=128,
                      block_size=16, num_blocks=256, dtype=torch.bfloat16, seed=11, device="cuda",
                      max_blocks_per_seq=64, num_kv_heads=8)
    P.pa_set_option(P.binding.PA_OPT_DECODE_WARPS, warps)
    try:
        parity(w, step=gpu_step_gqa)
    finally:
        P.pa_set_option(P.binding.PA_OPT_DECODE_WARPS, 0)


def test_gqa_single_token_returns_its_value(gqa_kernel):
    """One stored token: softmax weight 1, so every query head of a group gets
    its key/value head's value (the tensor-core kernel rounds the weight 1.0
    to fp16 exactly, so this stays bit-exact)."""
    w = W.make_decode("gqa_one", [1] * 5, num_heads=16, head_dim=128, block_size=16,
                      num_blocks=8, dtype=torch.float16, seed=13, device="cuda", num_kv_heads=2)
    out = gpu_step_gqa(w)
    torch.cuda.synchronize()
    assert torch.equal(out, w.v.repeat_interleave(8, dim=1))


def test_gqa_kernels_agree_and_are_deterministic():
    """Both kernels compute the same function: equal within the tolerance;
    each is bitwise reproducible run to run."""
    import paged_kv_cache_326_b200 as P
    w = W.llama2_70b_gqa(device="cuda", num_seqs=16)
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping)
    res = {}
    try:
        for name, mode in GQA_KERNELS.items():
            P.pa_set_option(P.PA_OPT_GQA_KERNEL, mode)
            outs = []
            for _ in range(2):
                out = torch.empty_like(w.q)
                P.pa_paged_attn_decode_gqa(out, w.q, w.k_cache, w.v_cache, w.block_tables,
                                           w.context_lens, w.scale)
                outs.append(out)
            torch.cuda.synchronize()
            assert torch.equal(outs[0], outs[1]), name
            res[name] = outs[0]
    finally:
        P.pa_set_option(P.PA_OPT_GQA_KERNEL, 0)
    diff = (res["tensor"].float() - res["cores"].float()).abs()
    assert diff.max().item() <= 4e-3, diff.max().item()


def test_gqa_tensor_kernel_refuses_shapes_it_does_not_cover():
    import paged_kv_cache_326_b200 as P
    w = W.make_decode("gqa_b4", [5, 9], num_heads=8, head_dim=64, block_size=4, num_blocks=16,
                      dtype=torch.float16, seed=3, device="cuda", num_kv_heads=2)
    out = torch.empty_like(w.q)
    P.pa_set_option(P.PA_OPT_GQA_KERNEL, 2)
    try:
        with pytest.raises(P.PagedAttnError):
            P.pa_paged_attn_decode_gqa(out, w.q, w.k_cache, w.v_cache, w.block_tables,
                                       w.context_lens, w.scale)
    finally:
        P.pa_set_option(P.PA_OPT_GQA_KERNEL, 0)


def test_gqa_bad_block_and_timeout_are_reported(gqa_kernel):
    """A table entry outside the pool and a wait that gives up are recorded
    in the status word; the kernel skips the block / returns, and the next
    call is correct."""
    import paged_kv_cache_326_b200 as P
    mk = lambda: W.make_decode("gqa_err", [40, 17, 100], num_heads=16, head_dim=128,
                               block_size=16, num_blocks=32, dtype=torch.float16, seed=5,
                               device="cuda", num_kv_heads=2)
    w = mk()
    w.block_tables[2, 1] = w.num_blocks + 3
    st = new_status()
    gpu_step_gqa(w, st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_BLOCK
    w = mk()
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping)
    st = new_status()
    P.pa_set_option(P.binding.PA_OPT_WAIT_LIMIT_NS, -1)
    try:
        out = torch.empty_like(w.q)
        P.pa_paged_attn_decode_gqa(out, w.q, w.k_cache, w.v_cache, w.block_tables,
                                   w.context_lens, w.scale, status=st)
        torch.cuda.synchronize()
    finally:
        P.pa_set_option(P.binding.PA_OPT_WAIT_LIMIT_NS, 1_000_000_000)
    assert st.item() == P.binding.PA_ERR_TIMEOUT
    parity(mk(), step=gpu_step_gqa)
