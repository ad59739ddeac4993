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


# ---- the store of the prompt's keys and values -------------------------------

@pytest.mark.parametrize("block_size", [4, 8, 32])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
def test_prefill_stores_at_every_block_size(block_size, dtype, prefill_kernel):
    """Blocks of 8 and 32 are stored by the tcgen05 kernel from its tiles,
    blocks of 4 by the separate cache write: the pool is bit-exact either
    way."""
    w = W.make_prefill("blocks", LENS, 4, 2, 128, dtype, seed=20 + block_size, device="cuda",
                       block_size=block_size)
    check(w)


def _rescatter(w, seed, negative=0):
    """Every token gets a random distinct slot anywhere in the pool (so no
    block of tokens fills a physical block in order), and `negative` random
    tokens get -1 (not stored)."""
    g = torch.Generator().manual_seed(seed)
    T = w.slot_mapping.numel()
    N, B = w.k_cache.shape[0], w.block_size
    slots = torch.randperm(N * B, generator=g)[:T].to(torch.int64)
    if negative:
        slots[torch.randperm(T, generator=g)[:negative]] = -1
    w.slot_mapping = slots.to(w.slot_mapping.device)
    return w


@pytest.mark.parametrize("head_dim", [64, 128])
def test_prefill_scattered_and_skipped_slots_are_stored_row_by_row(head_dim, prefill_kernel):
    w = _rescatter(W.make_prefill("scatter", LENS, 4, 4, head_dim, torch.float16, seed=31,
                                  device="cuda", spare_blocks=64), 32, negative=100)
    check(w)


def test_prefill_aligned_blocks_and_stragglers_mixed():
    """Prompts whose slots fill whole blocks in order, except a few tokens
    moved to free slots and a few skipped: both store paths in one call."""
    w = W.make_prefill("mixed", [300, 130, 77], 4, 2, 128, torch.bfloat16, seed=33,
                       device="cuda", spare_blocks=16)
    sl = w.slot_mapping.clone()
    used = set((sl // w.block_size).tolist())
    free = [b for b in range(w.k_cache.shape[0]) if b not in used]
    for i, t in enumerate([5, 17, 200, 301, 431]):
        sl[t] = free[i] * w.block_size + 3
    sl[[40, 41, 290]] = -1
    w.slot_mapping = sl
    check(w)


def test_prefill_slot_outside_the_pool_is_reported(prefill_kernel):
    import paged_kv_cache_326_b200 as P
    w = W.make_prefill("badslot", [70, 20], 2, 2, 128, torch.float16, seed=34, device="cuda")
    N, B = w.k_cache.shape[0], w.block_size
    w.slot_mapping[3] = N * B + 5
    st = new_status()
    run_prefill(w, st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_SLOT


# ---- the prompt phase over a stored prefix -----------------------------------

def _with_prefix(prefix, new, Hq, Hkv, D, dtype, B, seed):
    """Whole prompts (prefix + new tokens) made as one packed prompt set; the
    prefixes' keys and values stored in the pool by the cache write; the new
    tokens packed as their own rows."""
    import paged_kv_cache_326_b200 as P
    lens = [c + n for c, n in zip(prefix, new)]
    w = W.make_prefill("whole", lens, Hq, Hkv, D, dtype, seed=seed, device="cuda",
                       block_size=B, spare_blocks=4)
    cu = w.cu_seqlens.tolist()
    pre_rows = torch.tensor([cu[s] + i for s, c in enumerate(prefix) for i in range(c)],
                            dtype=torch.long, device="cuda")
    new_rows = torch.tensor([cu[s] + c + i for s, (c, n) in enumerate(zip(prefix, new))
                             for i in range(n)], dtype=torch.long, device="cuda")
    if pre_rows.numel():
        P.pa_kv_cache_write(w.k[pre_rows].contiguous(), w.v[pre_rows].contiguous(), w.k_cache,
                            w.v_cache, w.slot_mapping[pre_rows].contiguous())
    torch.cuda.synchronize()
    x = dict(q=w.q[new_rows].contiguous(), k=w.k[new_rows].contiguous(),
             v=w.v[new_rows].contiguous(),
             cu=torch.tensor([0] + list(np.cumsum(new)), dtype=torch.int32, device="cuda"),
             slots=w.slot_mapping[new_rows].contiguous(),
             cached=torch.tensor(prefix, dtype=torch.int32, device="cuda"),
             new_rows=new_rows)
    return w, x


@pytest.mark.parametrize("B", [8, 16, 32])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("heads,D", [((4, 4), 128), ((8, 2), 64)], ids=["mha128", "gqa64"])
def test_prefill_with_prefix_matches_oracle(B, dtype, heads, D):
    import paged_kv_cache_326_b200 as P
    Hq, Hkv = heads
    prefix = [0, B, 64, 3 * B, 160, 96]
    new = [37, 1, 200, 64, 0, 129]
    w, x = _with_prefix(prefix, new, Hq, Hkv, D, dtype, B, seed=40 + B + D)
    kc0 = w.k_cache.view(torch.int16).cpu().numpy()
    vc0 = w.v_cache.view(torch.int16).cpu().numpy()
    out = torch.empty_like(x["q"])
    st = new_status()
    P.pa_prefill_with_prefix(out, x["q"], x["k"], x["v"], x["cu"], max(new), w.scale, w.k_cache,
                             w.v_cache, w.block_tables, x["cached"], x["slots"], status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    # the new tokens' keys and values joined the pool, nothing else changed
    ek, ev = oracle.cache_write(kc0, vc0, x["k"].view(torch.int16).cpu().numpy(),
                                x["v"].view(torch.int16).cpu().numpy(), x["slots"].cpu().numpy(), B)
    assert np.array_equal(w.k_cache.view(torch.int16).cpu().numpy(), ek)
    assert np.array_equal(w.v_cache.view(torch.int16).cpu().numpy(), ev)
    ref = oracle.prefill_with_prefix(host_f32(x["q"]), host_f32(x["k"]), host_f32(x["v"]),
                                     x["cu"].cpu().numpy(), host_f32(w.k_cache),
                                     host_f32(w.v_cache), w.block_tables.cpu().numpy(),
                                     prefix, w.scale, B)
    c = compare(out, ref, dtype)
    assert c.ok, f"prefix prefill: {c}"
    # the same rows of the ordinary prompt phase over the whole prompts
    whole = oracle.prefill(host_f32(w.q), host_f32(w.k), host_f32(w.v), w.cu_seqlens.cpu().numpy(),
                           w.scale)[x["new_rows"].cpu().numpy()]
    c2 = compare(out, whole, dtype)
    assert c2.ok, f"vs whole prompts: {c2}"
    print(f"prefix prefill B{B} {dtype} q{Hq}kv{Hkv} D{D}", c)


def test_prefill_with_prefix_bad_lengths_and_blocks_are_reported():
    import paged_kv_cache_326_b200 as P
    w, x = _with_prefix([32, 16], [10, 5], 2, 2, 128, torch.float16, 16, seed=50)
    out = torch.empty_like(x["q"])
    st = new_status()
    bad = torch.tensor([32, 7], dtype=torch.int32, device="cuda")   # not a whole block
    P.pa_prefill_with_prefix(out, x["q"], x["k"], x["v"], x["cu"], 10, w.scale, w.k_cache,
                             w.v_cache, w.block_tables, bad, status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_LEN
    st = new_status()
    tables = w.block_tables.clone()
    tables[0, 1] = w.k_cache.shape[0] + 3
    P.pa_prefill_with_prefix(out, x["q"], x["k"], x["v"], x["cu"], 10, w.scale, w.k_cache,
                             w.v_cache, tables, x["cached"], status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_BLOCK


def test_reused_prefix_then_decode_through_the_block_manager():
    """Two requests share a 48-token system prompt (blocks of 16).  The first
    is prefilled whole; the second, added by token ids, takes over the three
    full blocks and prefills only its own tokens over them.  One decode step
    of both then agrees with the oracle's decode over the whole texts."""
    import paged_kv_cache_326_b200 as P
    B, H, D, N = 16, 4, 128, 64
    g = torch.Generator().manual_seed(61)
    system = list(range(100, 148))
    prompts = [system + list(range(7)), system + list(range(200, 230))]
    # token t at position p has fixed key and value rows (as a model would)
    table_q = torch.randn(256, 96, H, D, generator=g).half()
    table_k = torch.randn(256, 96, H, D, generator=g).half()
    table_v = torch.randn(256, 96, H, D, generator=g).half()
    rows = lambda tab, toks, lo: torch.stack([tab[t, p] for p, t in enumerate(toks)])[lo:].cuda()
    bm = P.BlockManager(N, B)
    kc = torch.full((N, H, B, D), float("nan"), dtype=torch.float16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    scale = W.fp32_scale(D)
    outs = []
    for sid, toks in enumerate(prompts):
        cached = bm.add_seq_tokens(sid, toks)
        tables, lens = bm.export([sid], 8)
        tables = tables.cuda()
        slots = torch.tensor([int(tables[0, p // B]) * B + p % B for p in range(cached, len(toks))],
                             dtype=torch.int64, device="cuda")
        q, k, v = (rows(t, toks, cached) for t in (table_q, table_k, table_v))
        out = torch.empty_like(q)
        cu = torch.tensor([0, len(toks) - cached], dtype=torch.int32, device="cuda")
        P.pa_prefill_with_prefix(out, q, k, v, cu, len(toks) - cached, scale, kc, vc, tables,
                                 torch.tensor([cached], dtype=torch.int32, device="cuda"), slots)
        outs.append((cached, out))
    assert [c for c, _ in outs] == [0, 48]
    torch.cuda.synchronize()
    # the second prompt's new rows against the prompt phase over its whole text
    toks = prompts[1]
    whole = oracle.prefill(host_f32(rows(table_q, toks, 0)), host_f32(rows(table_k, toks, 0)),
                           host_f32(rows(table_v, toks, 0)), [0, len(toks)], scale)[48:]
    c = compare(outs[1][1], whole, torch.float16)
    assert c.ok, c
    # one decode step of both texts
    qd = torch.randn(2, H, D, generator=g).half().cuda()
    kd = torch.randn(2, H, D, generator=g).half().cuda()
    vd = torch.randn(2, H, D, generator=g).half().cuda()
    slots = torch.tensor([bm.append_slot(s)[0] for s in (0, 1)], dtype=torch.int64, device="cuda")
    tables, lens = bm.export([0, 1], 8)
    kc0, vc0 = host_f32(kc), host_f32(vc)
    P.pa_kv_cache_write(kd, vd, kc, vc, slots)
    dout = torch.empty_like(qd)
    P.pa_paged_attn_decode(dout, qd, kc, vc, tables.cuda(), lens.cuda(), scale)
    torch.cuda.synchronize()
    kc1, vc1 = oracle.cache_write(kc0, vc0, host_f32(kd), host_f32(vd), slots.cpu().numpy(), B)
    ref = oracle.paged_decode(host_f32(qd), kc1, vc1, tables.numpy(), lens.numpy(), scale, B)
    c = compare(dout, ref, torch.float16)
    assert c.ok, c
