"""Checks that pin the oracle to something other than itself.

Each ``pin_*`` takes the decode function under test, with the oracle's
signature ``fn(q, k_cache, v_cache, block_tables, context_lens, scale,
block_size) -> out``, and raises AssertionError when it disagrees with what
the pages and the mathematics fix.  tests/test_oracle.py runs them on the
oracle; tests/test_oracle_mutants.py runs them on copies of the oracle with
planted mistakes and requires each copy to fail at least one.

The ground truth here is built in the opposite direction to the oracle: texts
are drawn as contiguous [L][H][D] tensors first, then scattered into a paged
pool through a random block table, so a wrong gather cannot agree with it.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f64(t):
    return t.to(torch.float64).numpy() if isinstance(t, torch.Tensor) else np.asarray(t, np.float64)


# ---------------------------------------------------------------------------
# contiguous texts -> paged pool (independent of the oracle's gather)
# ---------------------------------------------------------------------------

def random_texts(lens, H, D, seed, dtype=torch.float16):
    g = torch.Generator().manual_seed(seed)
    K = [torch.randn(L, H, D, generator=g).to(dtype) for L in lens]
    V = [torch.randn(L, H, D, generator=g).to(dtype) for L in lens]
    q = torch.randn(len(lens), H, D, generator=g).to(dtype)
    return q, K, V


def scatter_to_pool(K, V, block_size, num_blocks, seed, dtype=torch.float16):
    """Place token t of text s at (table[s][t // B], t % B), blocks drawn from
    a seeded permutation; unused rows are NaN."""
    H, D = K[0].shape[1], K[0].shape[2]
    g = torch.Generator().manual_seed(seed + 77)
    perm = torch.randperm(num_blocks, generator=g).tolist()
    kc = torch.full((num_blocks, H, block_size, D), float("nan"), dtype=dtype)
    vc = torch.full((num_blocks, H, block_size, D), float("nan"), dtype=dtype)
    nblk = [-(-k.shape[0] // block_size) for k in K]
    tables = np.full((len(K), max([1] + nblk)), -1, dtype=np.int64)
    at = 0
    for s, (k, v) in enumerate(zip(K, V)):
        for j in range(nblk[s]):
            phys = perm[at]
            at += 1
            tables[s, j] = phys
            lo, hi = j * block_size, min(k.shape[0], (j + 1) * block_size)
            kc[phys, :, : hi - lo, :] = k[lo:hi].permute(1, 0, 2)
            vc[phys, :, : hi - lo, :] = v[lo:hi].permute(1, 0, 2)
    return kc, vc, tables


def sdpa_contiguous(q, K, V, scale):
    """torch's attention in fp64 on the unpaged texts (a library routine,
    written independently of the oracle)."""
    outs = []
    for s in range(len(K)):
        if K[s].shape[0] == 0:
            outs.append(torch.zeros(q.shape[1], q.shape[2], dtype=torch.float64))
            continue
        qs = q[s].to(torch.float64)[:, None, :]             # [H][1][D]
        ks = K[s].to(torch.float64).permute(1, 0, 2)         # [H][L][D]
        vs = V[s].to(torch.float64).permute(1, 0, 2)
        o = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, scale=scale)
        outs.append(o[:, 0, :])
    return torch.stack(outs).numpy()


def brute_force(q, K, V, scale):
    """Scalar loops with math.exp / math.fsum."""
    S, H, D = q.shape
    out = np.zeros((S, H, D))
    qn = f64(q)
    for s in range(S):
        Ks, Vs = f64(K[s]), f64(V[s])
        L = Ks.shape[0]
        if L == 0:
            continue
        for h in range(H):
            z = [scale * math.fsum(qn[s, h, d] * Ks[t, h, d] for d in range(D)) for t in range(L)]
            zmax = max(z)
            e = [math.exp(x - zmax) for x in z]
            tot = math.fsum(e)
            for d in range(D):
                out[s, h, d] = math.fsum(e[t] * Vs[t, h, d] for t in range(L)) / tot
    return out


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

LENS_SMALL = [5, 9, 16, 23, 1, 31]


def pin_unpaged_sdpa(fn):
    for B, dtype, seed in ((4, torch.float16, 11), (8, torch.bfloat16, 12), (16, torch.float16, 13)):
        H, D = 3, 16
        q, K, V = random_texts(LENS_SMALL, H, D, seed, dtype)
        kc, vc, tables = scatter_to_pool(K, V, B, 40, seed, dtype)
        scale = 1.0 / math.sqrt(D)
        got = fn(f64(q), f64(kc), f64(vc), tables, LENS_SMALL, scale, B)
        ref = sdpa_contiguous(q, K, V, scale)
        err = np.abs(got - ref).max()
        assert err <= 1e-12, f"unpaged sdpa B={B}: max err {err}"


def pin_brute_force(fn):
    lens = [5, 9, 16, 23]
    H, D, B = 2, 8, 4
    q, K, V = random_texts(lens, H, D, 21)
    kc, vc, tables = scatter_to_pool(K, V, B, 16, 21)
    scale = 0.3535
    got = fn(f64(q), f64(kc), f64(vc), tables, lens, scale, B)
    ref = brute_force(q, K, V, scale)
    err = np.abs(got - ref).max()
    assert err <= 1e-12, f"brute force: max err {err}"


def pin_golden_closed_form(fn):
    g = load_golden("attention_closed_form.json")
    got = fn(np.array(g["q"]), np.array(g["k_cache"]), np.array(g["v_cache"]),
             np.array(g["block_tables"]), g["context_lens"], g["scale"], g["block_size"])
    err = np.abs(got - np.array(g["expected_out"])).max()
    assert err <= g["tol"], f"closed form: {got.ravel()} vs {g['expected_out']}"


def pin_single_token(fn):
    """One token: its weight is exactly 1, so the output is its value, exactly."""
    H, D, B = 4, 32, 4
    q, K, V = random_texts([1, 1, 1], H, D, 31)
    kc, vc, tables = scatter_to_pool(K, V, B, 8, 31)
    got = fn(f64(q), f64(kc), f64(vc), tables, [1, 1, 1], 0.17677669, B)
    for s in range(3):
        assert np.array_equal(got[s], f64(V[s])[0]), "single token output != its value"


def pin_uniform_scores(fn):
    """q = 0 (and, separately, all keys equal): every weight is 1/L, so the
    output is the mean of the values."""
    H, D, B = 2, 16, 4
    lens = [7, 12]
    q, K, V = random_texts(lens, H, D, 41)
    kc, vc, tables = scatter_to_pool(K, V, B, 8, 41)
    zero_q = np.zeros_like(f64(q))
    got = fn(zero_q, f64(kc), f64(vc), tables, lens, 0.25, B)
    for s, L in enumerate(lens):
        mean = f64(V[s]).mean(axis=0)
        assert np.abs(got[s] - mean).max() <= 1e-12, "q=0 is not the mean of V"
    Keq = [torch.ones_like(k) * 0.5 for k in K]
    kc2, vc2, tables2 = scatter_to_pool(Keq, V, B, 8, 42)
    got2 = fn(f64(q), f64(kc2), f64(vc2), tables2, lens, 0.25, B)
    for s, L in enumerate(lens):
        mean = f64(V[s]).mean(axis=0)
        assert np.abs(got2[s] - mean).max() <= 1e-12, "equal keys are not the mean of V"


def pin_dominant_key(fn):
    """One key far ahead of the others (score gap > 800): the others' weights
    underflow, so the output is that key's value."""
    H, D, B = 1, 4, 4
    L = 10
    rng = np.random.default_rng(5)
    K = rng.normal(size=(L, H, D))
    V = rng.normal(size=(L, H, D))
    q = np.zeros((1, H, D))
    q[0, 0, 0] = 1.0
    K[:, 0, 0] = 0.0
    K[6, 0, 0] = 1000.0
    Kt, Vt = [torch.tensor(K)], [torch.tensor(V)]
    kc, vc, tables = scatter_to_pool(Kt, Vt, B, 6, 51, torch.float64)
    got = fn(q, f64(kc), f64(vc), tables, [L], 1.0, B)
    assert np.abs(got[0, 0] - V[6, 0]).max() <= 1e-12, "dominant key's value not returned"


def pin_relabel_invariance(fn):
    """Renumbering the physical blocks (pool and tables together) changes
    nothing, bit for bit."""
    H, D, B, N = 3, 16, 4, 40
    q, K, V = random_texts(LENS_SMALL, H, D, 61)
    kc, vc, tables = scatter_to_pool(K, V, B, N, 61)
    base = fn(f64(q), f64(kc), f64(vc), tables, LENS_SMALL, 0.25, B)
    perm = np.random.default_rng(7).permutation(N)
    kc2 = np.empty_like(f64(kc))
    vc2 = np.empty_like(f64(vc))
    kc2[perm] = f64(kc)
    vc2[perm] = f64(vc)
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
    got = fn(f64(q), kc2, vc2, t2, LENS_SMALL, 0.25, B)
    assert np.array_equal(base, got), "not invariant under block relabelling"


def pin_block_size_invariance(fn):
    """The same texts stored with blocks of 4, 8, 16 or 32 give the same
    output, bit for bit."""
    H, D = 2, 16
    q, K, V = random_texts(LENS_SMALL, H, D, 71)
    outs = []
    for B in (4, 8, 16, 32):
        kc, vc, tables = scatter_to_pool(K, V, B, 64, 71 + B)
        outs.append(fn(f64(q), f64(kc), f64(vc), tables, LENS_SMALL, 0.25, B))
    for o in outs[1:]:
        assert np.array_equal(outs[0], o), "output depends on block size"


def pin_shared_prefix(fn):
    """A text reading shared prefix blocks gives the same output as a copy of
    it whose blocks are private; two texts with the same table, length and
    query give the same output."""
    H, D, B = 2, 8, 4
    q, K, V = random_texts([10, 10], H, D, 81)
    K[1][:8] = K[0][:8]
    V[1][:8] = V[0][:8]
    kc, vc, tables = scatter_to_pool(K, V, B, 12, 81)
    private = fn(f64(q), f64(kc), f64(vc), tables, [10, 10], 0.3, B)
    shared_tables = tables.copy()
    shared_tables[1, :2] = tables[0, :2]
    shared = fn(f64(q), f64(kc), f64(vc), shared_tables, [10, 10], 0.3, B)
    assert np.array_equal(private, shared), "shared prefix blocks change the output"
    q2 = q.clone()
    q2[1] = q2[0]
    same = fn(f64(q2), f64(kc), f64(vc), np.stack([tables[0], tables[0]]), [10, 10], 0.3, B)
    assert np.array_equal(same[0], same[1]), "identical texts differ"


def pin_nan_tail_and_unused_entries(fn):
    """Rows past the context (NaN) and table entries past the last block
    (garbage) never reach the output; an empty text gives zeros."""
    H, D, B = 2, 8, 4
    q, K, V = random_texts([6, 3, 0], H, D, 91)
    kc, vc, tables = scatter_to_pool(K, V, B, 8, 91)
    t = np.concatenate([tables, np.full((3, 2), 10**6)], axis=1)
    got = fn(f64(q), f64(kc), f64(vc), t, [6, 3, 0], 0.3, B)
    assert np.isfinite(got).all(), "NaN padding leaked"
    assert np.array_equal(got[2], np.zeros((H, D))), "empty text is not zero"


ATTENTION_PINS = [pin_unpaged_sdpa, pin_brute_force, pin_golden_closed_form, pin_single_token,
                  pin_uniform_scores, pin_dominant_key, pin_relabel_invariance,
                  pin_block_size_invariance, pin_shared_prefix, pin_nan_tail_and_unused_entries]


def pin_cache_write_golden(write_fn):
    g = load_golden("cache_write_tiny.json")
    shape = (g["num_blocks"], g["num_heads"], g["block_size"], g["head_dim"])
    kc = np.zeros(shape, dtype=np.uint16)
    vc = np.zeros(shape, dtype=np.uint16)
    k = np.array(g["k"], dtype=np.uint16)
    v = np.array(g["v"], dtype=np.uint16)
    kc2, vc2 = write_fn(kc, vc, k, v, g["slot_mapping"], g["block_size"])
    assert np.array_equal(kc2, np.array(g["expected_k_cache"], dtype=np.uint16)), "k cache write"
    assert np.array_equal(vc2, np.array(g["expected_v_cache"], dtype=np.uint16)), "v cache write"
    assert not kc.any() and not vc.any(), "write modified its input"


def pin_cache_write_then_read(write_fn):
    """Writing every token of contiguous texts through their slots rebuilds
    the pool that the independent scatter builds."""
    H, D, B = 2, 8, 4
    lens = [5, 9, 3]
    q, K, V = random_texts(lens, H, D, 101)
    kc_ref, vc_ref, tables = scatter_to_pool(K, V, B, 10, 101)
    kc = torch.full_like(kc_ref, float("nan")).view(torch.int16).numpy()
    vc = torch.full_like(vc_ref, float("nan")).view(torch.int16).numpy()
    ks, vs, slots = [], [], []
    for s, L in enumerate(lens):
        for t in range(L):
            ks.append(K[s][t].view(torch.int16).numpy())
            vs.append(V[s][t].view(torch.int16).numpy())
            slots.append(int(tables[s, t // B]) * B + t % B)
    kc2, vc2 = write_fn(kc, vc, np.stack(ks), np.stack(vs), slots, B)
    assert np.array_equal(kc2, kc_ref.view(torch.int16).numpy()), "rebuilt k pool differs"
    assert np.array_equal(vc2, vc_ref.view(torch.int16).numpy()), "rebuilt v pool differs"


WRITE_PINS = [pin_cache_write_golden, pin_cache_write_then_read]


# ---------------------------------------------------------------------------
# grouped-query attention (several query heads share one key/value head)
# ---------------------------------------------------------------------------

def pin_gqa_equals_replicated_mha(fn):
    """Sharing a key/value head between G query heads is the same as giving
    each query head its own copy: a pool with the heads repeated (np.repeat,
    built independently) gives the same output bit for bit."""
    Hq, Hkv, D, B = 8, 2, 16, 4
    lens = [5, 9, 16, 1]
    q, _, _ = random_texts(lens, Hq, D, 201)
    _, K, V = random_texts(lens, Hkv, D, 202)
    kc, vc, tables = scatter_to_pool(K, V, B, 24, 203)
    got = fn(f64(q), f64(kc), f64(vc), tables, lens, 0.25, B)
    rep = np.repeat
    ref = fn(f64(q), rep(f64(kc), Hq // Hkv, axis=1), rep(f64(vc), Hq // Hkv, axis=1), tables,
             lens, 0.25, B)
    assert np.array_equal(got, ref), "GQA differs from replicated MHA"


def pin_gqa_unpaged_sdpa(fn):
    """GQA against torch's fp64 attention on unpaged texts whose key/value
    heads are repeated for each query head."""
    Hq, Hkv, D, B = 6, 3, 16, 8
    lens = [7, 23, 2]
    q, _, _ = random_texts(lens, Hq, D, 211)
    _, K, V = random_texts(lens, Hkv, D, 212)
    kc, vc, tables = scatter_to_pool(K, V, B, 12, 213)
    got = fn(f64(q), f64(kc), f64(vc), tables, lens, 0.3, B)
    Kr = [k.repeat_interleave(Hq // Hkv, dim=1) for k in K]
    Vr = [v.repeat_interleave(Hq // Hkv, dim=1) for v in V]
    ref = sdpa_contiguous(q, Kr, Vr, 0.3)
    assert np.abs(got - ref).max() <= 1e-12, "GQA vs sdpa"


def pin_mqa_single_head(fn):
    """One key/value head for all query heads (multi-query): head h's output
    is attention of q_h over the one shared head."""
    Hq, D, B = 4, 8, 4
    lens = [6, 11]
    q, _, _ = random_texts(lens, Hq, D, 221)
    _, K, V = random_texts(lens, 1, D, 222)
    kc, vc, tables = scatter_to_pool(K, V, B, 8, 223)
    got = fn(f64(q), f64(kc), f64(vc), tables, lens, 0.5, B)
    ref = brute_force(q, [k.expand(-1, Hq, -1) for k in K], [v.expand(-1, Hq, -1) for v in V], 0.5)
    assert np.abs(got - ref).max() <= 1e-12, "MQA vs brute force"


GQA_PINS = [pin_gqa_equals_replicated_mha, pin_gqa_unpaged_sdpa, pin_mqa_single_head]


# ---------------------------------------------------------------------------
# block copies (copy-on-write, moving blocks between pools)
# ---------------------------------------------------------------------------

def pin_copy_on_write_worked_example(copy_fn):
    """The pages' worked example ("The KV Cache and PagedAttention", Shared,
    Copied on Write; golden cow_two_answers.json): two answers share a
    6-token prompt in blocks 0 and 1 of 4 places; the first answer's write
    copies block 1 to block 2 and lands at slot 10, the second writes in
    place at slot 6.  Afterwards each answer reads the prompt followed by its
    own token, and neither sees the other's."""
    g = load_golden("cow_two_answers.json")
    B, N, P = g["block_size"], g["num_blocks"], g["prompt_tokens"]
    H, D = 2, 8
    rng = np.random.default_rng(301)
    prompt = rng.standard_normal((P, H, D))
    tok = rng.standard_normal((2, H, D))          # each answer's new key (values alike)
    kc = np.full((N, H, B, D), np.nan)
    for t in range(P):                            # the prompt in blocks 0, 1 (in order)
        kc[t // B, :, t % B] = prompt[t]
    vc = kc.copy()
    a1 = g["answer1_append"]
    kc, vc = copy_fn(kc, vc, kc, vc, [(a1["cow_src"], a1["cow_dst"])])
    kc, vc = cache_write_plain(kc, vc, tok[0:1], tok[0:1], [a1["slot"]], B)
    a2 = g["answer2_append"]
    assert a2["cow_src"] < 0
    kc, vc = cache_write_plain(kc, vc, tok[1:2], tok[1:2], [a2["slot"]], B)
    for i, name in enumerate(["answer1", "answer2"]):
        table = g["after_answer2"]["tables"][name]
        got = np.stack([kc[table[t // B], :, t % B] for t in range(P + 1)])
        want = np.concatenate([prompt, tok[i:i + 1]])
        assert np.array_equal(got, want), f"{name} does not read the prompt plus its own token"


def cache_write_plain(kc, vc, k, v, slots, B):
    """A write done here, by plain indexing (the pin must not lean on the
    oracle's own cache_write)."""
    kc, vc = kc.copy(), vc.copy()
    for t, slot in enumerate(slots):
        kc[slot // B, :, slot % B] = k[t]
        vc[slot // B, :, slot % B] = v[t]
    return kc, vc


def pin_copy_blocks_bits_vs_index_copy(copy_fn):
    """Raw 16-bit patterns (NaN payloads and signed zeros included) land
    unchanged: the result equals torch's index_copy_ of the chosen source
    blocks into the destination pool."""
    rng = np.random.default_rng(311)
    shape_s, shape_d = (12, 3, 4, 8), (9, 3, 4, 8)
    src_k = rng.integers(0, 1 << 16, size=shape_s, dtype=np.uint16)
    src_v = rng.integers(0, 1 << 16, size=shape_s, dtype=np.uint16)
    src_k[0, 0, 0, :3] = [0x7E01, 0x8000, 0xFC00]
    dst_k = rng.integers(0, 1 << 16, size=shape_d, dtype=np.uint16)
    dst_v = rng.integers(0, 1 << 16, size=shape_d, dtype=np.uint16)
    pairs = [(0, 4), (11, 0), (5, 8), (5, 2)]
    before = dst_k.copy()
    kd, vd = copy_fn(src_k, src_v, dst_k, dst_v, pairs)
    idx_s = torch.tensor([p[0] for p in pairs])
    idx_d = torch.tensor([p[1] for p in pairs])
    for got, src, dst in ((kd, src_k, dst_k), (vd, src_v, dst_v)):
        s16, d16 = torch.from_numpy(src.view(np.int16)), torch.from_numpy(dst.view(np.int16))
        ref = d16.clone().index_copy_(0, idx_d, s16.index_select(0, idx_s)).numpy()
        assert np.array_equal(got.view(np.int16), ref), "block copy differs from index_copy_"
    assert np.array_equal(dst_k, before), "copy modified its input"


def pin_copy_out_and_back(copy_fn):
    """Moving blocks out to another pool and back into new places (a swap
    out and in) restores every value, and blocks not named stay as they were."""
    rng = np.random.default_rng(321)
    kc = rng.standard_normal((10, 2, 4, 8))
    vc = rng.standard_normal((10, 2, 4, 8))
    host_k = np.zeros((3, 2, 4, 8))
    host_v = np.zeros((3, 2, 4, 8))
    out_pairs = [(7, 0), (2, 1), (9, 2)]
    hk, hv = copy_fn(kc, vc, host_k, host_v, out_pairs)
    back_pairs = [(0, 3), (1, 5), (2, 6)]
    kc2, vc2 = copy_fn(hk, hv, kc, vc, back_pairs)
    for (src, _), (_, dst) in zip(out_pairs, back_pairs):
        assert np.array_equal(kc2[dst], kc[src]) and np.array_equal(vc2[dst], vc[src])
    untouched = [b for b in range(10) if b not in (3, 5, 6)]
    assert np.array_equal(kc2[untouched], kc[untouched]) and np.array_equal(vc2[untouched], vc[untouched])


COPY_PINS = [pin_copy_on_write_worked_example, pin_copy_blocks_bits_vs_index_copy,
             pin_copy_out_and_back]


# ---------------------------------------------------------------------------
# 8-bit (E4M3) KV cache
# ---------------------------------------------------------------------------

def _torch_e4m3(x32: np.ndarray) -> np.ndarray:
    """torch's float32 -> float8_e4m3fn cast (round to nearest even), as codes."""
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_e4m3_every_fp16_vs_torch(encode):
    """Every finite fp16 value below the first magnitude that rounds past 448
    (464), subnormals and both zeros included: the codes equal torch's cast."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = bits.view(np.float16).astype(np.float32)
    keep = np.isfinite(x) & (np.abs(x) < 464.0)
    got = encode(x[keep])
    assert np.array_equal(got, _torch_e4m3(x[keep])), "E4M3 codes differ from torch's cast"


def pin_e4m3_random_fp32_vs_torch(encode):
    """Random fp32 magnitudes spread over 2^-12 .. 2^8.8 (exponents drawn
    uniformly), both signs."""
    rng = np.random.default_rng(401)
    mag = np.exp2(rng.uniform(-12, 8.8, size=200000)).astype(np.float32)
    x = np.where(rng.random(200000) < 0.5, -mag, mag).astype(np.float32)
    assert np.array_equal(encode(x), _torch_e4m3(x)), "E4M3 codes differ from torch (fp32)"


def pin_e4m3_closed_forms(encode, decode):
    """The format's constants: largest finite 1.75 * 2^8 = 448 (code 0x7E),
    smallest normal 2^-6 (0x08), smallest subnormal 2^-9 (0x01), NaN at
    S.1111.111 only, 254 finite codes increasing with the code; saturation of
    large magnitudes and infinities to +-448; signed zero; ties to even
    worked by hand: with scale 0.5, 1.0 -> 2.0 = 0x40, -2.5 -> -5.0 = 0xCA,
    0.3 -> 0.6 (nearer 0.625 = 0x32 than 0.5625), 500 -> 448 = 0x7E."""
    v = decode(np.arange(256, dtype=np.uint8))
    assert v[0x7E] == 448.0 and v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.isnan(v).sum() == 2
    assert np.all(np.diff(v[:0x7F]) > 0) and np.array_equal(v[0x80:0xFF], -v[:0x7F])
    big = np.array([1e6, -1e6, np.inf, -np.inf, 470.0], dtype=np.float32)
    assert encode(big).tolist() == [0x7E, 0xFE, 0x7E, 0xFE, 0x7E]
    assert encode(np.array([0.0, -0.0], dtype=np.float32)).tolist() == [0x00, 0x80]
    assert encode(np.array([np.nan], dtype=np.float32)).tolist() == [0x7F]
    x = np.array([1.0, -2.5, 0.3, 500.0], dtype=np.float32) / np.float32(0.5)
    assert encode(x).tolist() == [0x40, 0xCA, 0x32, 0x7E]


def pin_fp8_attention_on_representable_values(decode_fp8, quantize):
    """Keys and values that E4M3 holds exactly (small multiples of powers of
    two) times a power-of-two scale: quantizing them loses nothing, so
    attention over the 8-bit cache equals attention over the same pool in
    fp16, computed here with torch (fp64) on the unpaged texts."""
    H, D, B = 2, 8, 4
    lens = [6, 11, 1]
    rng = np.random.default_rng(411)
    mant = rng.integers(-15, 16, size=(64, H, B, D)).astype(np.float32) / 8.0
    k_scale, v_scale = 0.25, 4.0
    kc = mant * np.float32(k_scale)
    vc = np.roll(mant, 1, axis=3) * np.float32(v_scale)
    kq = quantize(kc, k_scale)
    vq = quantize(vc, v_scale)
    tables = rng.permutation(64)[:12].reshape(3, 4)
    q = rng.standard_normal((3, H, D))
    got = decode_fp8(q, kq, vq, tables, lens, 0.3, B, k_scale, v_scale)
    Ks = [torch.from_numpy(np.stack([kc[tables[s, t // B], :, t % B] for t in range(L)]).astype(np.float64))
          for s, L in enumerate(lens)]
    Vs = [torch.from_numpy(np.stack([vc[tables[s, t // B], :, t % B] for t in range(L)]).astype(np.float64))
          for s, L in enumerate(lens)]
    ref = sdpa_contiguous(torch.from_numpy(q), Ks, Vs, 0.3)
    assert np.abs(got - ref).max() <= 1e-12, "8-bit cache attention vs exact values"


# ---------------------------------------------------------------------------
# prompt phase (prefill)
# ---------------------------------------------------------------------------

def _packed_prompts(lens, H, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    T = sum(lens)
    q = torch.randn(T, H, D, generator=g).to(torch.float16)
    k = torch.randn(T, Hkv, D, generator=g).to(torch.float16)
    v = torch.randn(T, Hkv, D, generator=g).to(torch.float16)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, k, v, cu


def pin_prefill_vs_torch_causal(prefill_fn):
    """torch's fp64 attention with is_causal=True on each prompt (key/value
    heads repeated for grouped-query prompts)."""
    lens, H, Hkv, D = [1, 7, 20, 3], 4, 2, 16
    q, k, v, cu = _packed_prompts(lens, H, Hkv, D, 501)
    got = prefill_fn(f64(q), f64(k), f64(v), cu, 0.3)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        qs = q[a:b].double().permute(1, 0, 2)
        ks = k[a:b].double().repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)
        vs = v[a:b].double().repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, is_causal=True,
                                                               scale=0.3)
        assert np.abs(got[a:b] - ref.permute(1, 0, 2).numpy()).max() <= 1e-12, "prefill vs sdpa"


def pin_prefill_last_row_is_decode(prefill_fn):
    """The prompt's last position sees the whole prompt: its output equals the
    decode-phase attention of that token over the prompt stored in a paged
    pool (the decode oracle, pinned on its own)."""
    from oracle import paged_decode
    lens, H, D, B = [9, 4, 13], 2, 8, 4
    q, k, v, cu = _packed_prompts(lens, H, H, D, 511)
    got = prefill_fn(f64(q), f64(k), f64(v), cu, 0.25)
    Ks = [k[cu[s]:cu[s + 1]] for s in range(3)]
    Vs = [v[cu[s]:cu[s + 1]] for s in range(3)]
    kc, vc, tables = scatter_to_pool(Ks, Vs, B, 16, 512)
    last = np.stack([f64(q[cu[s + 1] - 1]) for s in range(3)])
    ref = paged_decode(last, f64(kc), f64(vc), tables, lens, 0.25, B)
    for s in range(3):
        assert np.abs(got[cu[s + 1] - 1] - ref[s]).max() <= 1e-12, "last row vs decode"


def pin_prefill_first_row_and_brute_force(prefill_fn):
    """Position 0 sees only itself: its output is its value, exactly.  Every
    row of a tiny prompt against scalar brute force with math.fsum."""
    lens, H, D = [5], 1, 4
    q, k, v, cu = _packed_prompts(lens, H, H, D, 521)
    got = prefill_fn(f64(q), f64(k), f64(v), cu, 0.5)
    assert np.array_equal(got[0], f64(v[0])), "first row is not its value"
    Q, K, V = f64(q)[:, 0], f64(k)[:, 0], f64(v)[:, 0]
    for t in range(5):
        z = [0.5 * math.fsum(Q[t, d] * K[u, d] for d in range(D)) for u in range(t + 1)]
        m = max(z)
        e = [math.exp(x - m) for x in z]
        den = math.fsum(e)
        want = [math.fsum(e[u] * V[u, d] for u in range(t + 1)) / den for d in range(D)]
        assert np.abs(got[t, 0] - np.array(want)).max() <= 1e-12, f"row {t} vs brute force"


PREFILL_PINS = [pin_prefill_vs_torch_causal, pin_prefill_last_row_is_decode,
                pin_prefill_first_row_and_brute_force]


# ---------------------------------------------------------------------------
# prompt phase over a stored prefix (fn(q, k, v, cu, k_cache, v_cache,
# tables, cached_lens, scale, block_size) -> out)
# ---------------------------------------------------------------------------

def _prefixed_prompts(prefix_lens, new_lens, H, Hkv, D, B, seed, num_blocks=64):
    """Whole prompts drawn as contiguous tensors; each prompt's first
    prefix_lens[s] tokens' keys and values scattered into a paged pool (the
    pin's own scatter), the rest packed as the new rows."""
    g = torch.Generator().manual_seed(seed)
    whole = [(torch.randn(c + n, H, D, generator=g).to(torch.float16),
              torch.randn(c + n, Hkv, D, generator=g).to(torch.float16),
              torch.randn(c + n, Hkv, D, generator=g).to(torch.float16))
             for c, n in zip(prefix_lens, new_lens)]
    kc, vc, tables = scatter_to_pool([w[1][:c] for w, c in zip(whole, prefix_lens)],
                                     [w[2][:c] for w, c in zip(whole, prefix_lens)], B,
                                     num_blocks, seed)
    q = torch.cat([w[0][c:] for w, c in zip(whole, prefix_lens)])
    k = torch.cat([w[1][c:] for w, c in zip(whole, prefix_lens)])
    v = torch.cat([w[2][c:] for w, c in zip(whole, prefix_lens)])
    cu = np.concatenate([[0], np.cumsum(new_lens)]).astype(np.int64)
    return whole, q, k, v, cu, kc, vc, tables


def pin_prefix_rows_of_the_whole_prompt(fn):
    """The new rows equal torch's fp64 causal attention over the whole prompt
    (prefix and new tokens contiguous, key/value heads repeated), restricted
    to the new rows; a zero-length prefix is the ordinary prompt phase."""
    pre, new, H, Hkv, D, B = [8, 0, 24, 4, 16], [5, 9, 1, 12, 0], 4, 2, 8, 4
    whole, q, k, v, cu, kc, vc, tables = _prefixed_prompts(pre, new, H, Hkv, D, B, 531)
    got = fn(f64(q), f64(k), f64(v), cu, f64(kc), f64(vc), tables, pre, 0.35, B)
    for s, (c, n) in enumerate(zip(pre, new)):
        if n == 0:
            continue
        qw, kw, vw = (t.double().permute(1, 0, 2) for t in whole[s])
        kw = kw.repeat_interleave(H // Hkv, dim=0)
        vw = vw.repeat_interleave(H // Hkv, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qw, kw, vw, is_causal=True,
                                                               scale=0.35)
        ref = ref.permute(1, 0, 2)[c:].numpy()
        assert np.abs(got[cu[s]:cu[s + 1]] - ref).max() <= 1e-12, f"prompt {s} vs whole"


def pin_prefix_brute_force(fn):
    """Every new row of a tiny prompt (6 stored tokens in blocks of 2, 3 new)
    against scalar brute force with math.fsum over the contiguous prompt."""
    pre, new, D, B = [6], [3], 4, 2
    whole, q, k, v, cu, kc, vc, tables = _prefixed_prompts(pre, new, 1, 1, D, B, 541)
    got = fn(f64(q), f64(k), f64(v), cu, f64(kc), f64(vc), tables, pre, 0.5, B)
    Q, K, V = (f64(t)[:, 0] for t in whole[0])
    for i in range(3):
        P = 6 + i
        z = [0.5 * math.fsum(Q[P, d] * K[u, d] for d in range(D)) for u in range(P + 1)]
        m = max(z)
        e = [math.exp(x - m) for x in z]
        den = math.fsum(e)
        want = [math.fsum(e[u] * V[u, d] for u in range(P + 1)) / den for d in range(D)]
        assert np.abs(got[i, 0] - np.array(want)).max() <= 1e-12, f"new row {i}"


def pin_prefix_blocks_can_sit_anywhere(fn):
    """The same stored prefixes under another seeded placement of their
    blocks in the pool give bit-identical rows."""
    pre, new, H, D, B = [12, 20], [7, 3], 2, 8, 4
    _, q, k, v, cu, kc, vc, tables = _prefixed_prompts(pre, new, H, H, D, B, 551)
    _, q2, k2, v2, cu2, kc2, vc2, tables2 = _prefixed_prompts(pre, new, H, H, D, B, 551,
                                                              num_blocks=97)
    assert not np.array_equal(tables, tables2)
    a = fn(f64(q), f64(k), f64(v), cu, f64(kc), f64(vc), tables, pre, 0.3, B)
    b = fn(f64(q2), f64(k2), f64(v2), cu2, f64(kc2), f64(vc2), tables2, pre, 0.3, B)
    assert np.array_equal(a, b), "placement changed the result"


PREFIX_PINS = [pin_prefix_rows_of_the_whole_prompt, pin_prefix_brute_force,
               pin_prefix_blocks_can_sit_anywhere]


# ---------------------------------------------------------------------------
# shared prefixes
# ---------------------------------------------------------------------------

def _forked_groups(prompt_lens, tail_lens, group_size, H, D, B, seed, dtype=torch.float16,
                   Hq=None):
    """Groups of texts built as the block manager builds them, written out by
    hand: the prompt's full blocks are stored once and listed first in every
    member's table; a partial last prompt block is copied into each member's
    first private block (copy on write), followed by the member's own tokens.
    Returns q, the contiguous K and V of every text, the pool, and the prefix
    and tail tables and lengths.  H is the pool's head count; Hq (default H)
    the query heads."""
    Hq = H if Hq is None else Hq
    g = torch.Generator().manual_seed(seed)
    G = len(prompt_lens)
    S = G * group_size
    prompts = [(torch.randn(L, H, D, generator=g).to(dtype), torch.randn(L, H, D, generator=g).to(dtype))
               for L in prompt_lens]
    tails = [(torch.randn(L, H, D, generator=g).to(dtype), torch.randn(L, H, D, generator=g).to(dtype))
             for L in tail_lens]
    q = torch.randn(S, Hq, D, generator=g).to(dtype)
    nb = sum(L // B for L in prompt_lens) + 8
    nb += sum(-(-(prompt_lens[s // group_size] % B + tail_lens[s]) // B) for s in range(S))
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(seed + 5)).tolist()
    kc = torch.full((nb, H, B, D), float("nan"), dtype=dtype)
    vc = torch.full((nb, H, B, D), float("nan"), dtype=dtype)
    at = 0
    prefix_tables, prefix_lens, tail_tables, K, V = [], [], [], [], []
    for gi, L in enumerate(prompt_lens):
        pk, pv = prompts[gi]
        full = L // B
        row = []
        for j in range(full):
            phys = perm[at]
            at += 1
            kc[phys] = pk[j * B:(j + 1) * B].permute(1, 0, 2)
            vc[phys] = pv[j * B:(j + 1) * B].permute(1, 0, 2)
            row.append(phys)
        prefix_tables.append(row)
        prefix_lens.append(full * B)
        for m in range(group_size):
            s = gi * group_size + m
            tk, tv = tails[s]
            own_k = torch.cat([pk[full * B:], tk])
            own_v = torch.cat([pv[full * B:], tv])
            trow = []
            for j in range(-(-own_k.shape[0] // B)):
                phys = perm[at]
                at += 1
                lo, hi = j * B, min(own_k.shape[0], (j + 1) * B)
                kc[phys, :, :hi - lo] = own_k[lo:hi].permute(1, 0, 2)
                vc[phys, :, :hi - lo] = own_v[lo:hi].permute(1, 0, 2)
                trow.append(phys)
            tail_tables.append(trow)
            K.append(torch.cat([pk, tk]))
            V.append(torch.cat([pv, tv]))
    t_lens = [K[s].shape[0] - prefix_lens[s // group_size] for s in range(S)]
    return q, K, V, kc, vc, prefix_tables, prefix_lens, tail_tables, t_lens


def pin_shared_vs_unpaged_sdpa(shared_fn):
    """Two groups of three forked texts (prompts of 13 and 8 tokens, B = 4)
    against torch's fp64 attention on each text's contiguous tokens."""
    H, D, B, gs = 2, 8, 4, 3
    q, K, V, kc, vc, pt, pl, tt, tl = _forked_groups([13, 8], [1, 5, 3, 2, 0, 7], gs, H, D, B, 601)
    got = shared_fn(f64(q), f64(kc), f64(vc), pt, pl, tt, tl, gs, 0.35, B)
    ref = sdpa_contiguous(q, K, V, 0.35)
    err = np.abs(got - ref).max()
    assert err <= 1e-12, f"shared prefix vs unpaged sdpa: max err {err}"


def pin_shared_brute_force_and_empty(shared_fn):
    """Scalar brute force on a tiny group; a group with no shared block (a
    prompt shorter than a block) and a text with no tokens at all."""
    H, D, B, gs = 1, 4, 4, 2
    q, K, V, kc, vc, pt, pl, tt, tl = _forked_groups([9, 3], [2, 1, 0, 4], gs, H, D, B, 611)
    assert pl[1] == 0, "the second prompt has no full block"
    got = shared_fn(f64(q), f64(kc), f64(vc), pt, pl, tt, tl, gs, 0.5, B)
    ref = brute_force(q, K, V, 0.5)
    assert np.abs(got - ref).max() <= 1e-12, "shared prefix vs brute force"
    q2, K2, V2, kc2, vc2, pt2, pl2, tt2, tl2 = _forked_groups([0], [0, 2], 2, H, D, B, 612)
    got2 = shared_fn(f64(q2), f64(kc2), f64(vc2), pt2, pl2, tt2, tl2, 2, 0.5, B)
    assert np.array_equal(got2[0], np.zeros((H, D))), "a text with no tokens is not zero"
    assert np.abs(got2[1] - brute_force(q2[1:], K2[1:], V2[1:], 0.5)[0]).max() <= 1e-12


def pin_split_worked_example(split_fn):
    """Hand-worked splits (B = 16): two pairs whose first two blocks agree,
    then diverge; a pair right after a fork, whose shared second block is
    only partly filled (so it stays out of the prefix); a trio whose third
    member differs at block 1; a pair with nothing in common."""
    bt = [[5, 6, 7, -1], [5, 6, 8, -1], [5, 9, 10, 11], [5, 9, 12, -1]]
    got = split_fn(np.array(bt), [40, 36, 64, 48], 16, 2)
    want = ([[5, 6], [5, 9]], [32, 32], [[7], [8], [10, 11], [12]], [8, 4, 32, 16])
    assert [list(map(list, got[0])), list(got[1]), list(map(list, got[2])), list(got[3])] == \
        [want[0], want[1], want[2], want[3]], f"worked split: {got}"
    got = split_fn(np.array([[3, 4], [3, 4]]), [20, 20], 16, 2)
    assert list(map(list, got[0])) == [[3]] and list(got[1]) == [16], "partial shared block"
    assert list(map(list, got[2])) == [[4], [4]] and list(got[3]) == [4, 4]
    got = split_fn(np.array([[1, 2, 3], [1, 2, 4], [1, 7, 8]]), [48, 48, 48], 16, 3)
    assert list(map(list, got[0])) == [[1]] and list(got[1]) == [16], "trio"
    assert list(map(list, got[2])) == [[2, 3], [2, 4], [7, 8]] and list(got[3]) == [32, 32, 32]
    got = split_fn(np.array([[1, 2], [3, 2]]), [32, 32], 16, 2)
    assert list(map(list, got[0])) == [[]] and list(got[1]) == [0], "nothing shared"
    assert list(map(list, got[2])) == [[1, 2], [3, 2]] and list(got[3]) == [32, 32]


def pin_split_then_shared_is_decode(split_fn, shared_fn):
    """Splitting forked tables and attending over prefix then tail reads the
    same tokens in the same order as the joined table: the output equals
    plain paged decode bit for bit."""
    from oracle import paged_decode
    H, D, B, gs = 2, 8, 4, 4
    q, K, V, kc, vc, pt, pl, tt, tl = _forked_groups([14, 4, 17], [3, 1, 6, 2, 5, 0, 4, 4, 1, 2, 3, 9],
                                                     gs, H, D, B, 621)
    S = q.shape[0]
    width = max(len(pt[s // gs]) + len(tt[s]) for s in range(S))
    joined = np.full((S, width), -1, dtype=np.int64)
    lens = []
    for s in range(S):
        row = pt[s // gs] + tt[s]
        joined[s, :len(row)] = row
        lens.append(pl[s // gs] + tl[s])
    ref = paged_decode(f64(q), f64(kc), f64(vc), joined, lens, 0.3, B)
    spt, spl, stt, stl = split_fn(joined, lens, B, gs)
    got = shared_fn(f64(q), f64(kc), f64(vc), spt, spl, stt, stl, gs, 0.3, B)
    assert np.array_equal(got, ref), "split + shared decode differs from paged decode"


def pin_shared_grouped_query_vs_unpaged_sdpa(shared_fn):
    """Grouped-query pools: two groups of three forked texts, 6 query heads
    over 2 key/value heads (query head h reads key/value head h // 3),
    against torch's fp64 attention on each text's contiguous tokens with the
    key/value heads repeated for their query heads; a mistake in the head
    map (h for h // 3, or h % 2) fails it."""
    H, Hq, D, B, gs = 2, 6, 8, 4, 3
    q, K, V, kc, vc, pt, pl, tt, tl = _forked_groups([13, 8], [1, 5, 3, 2, 0, 7], gs, H, D, B,
                                                     613, Hq=Hq)
    got = shared_fn(f64(q), f64(kc), f64(vc), pt, pl, tt, tl, gs, 0.35, B)
    rep = Hq // H
    ref = sdpa_contiguous(q, [k.repeat_interleave(rep, dim=1) for k in K],
                          [v.repeat_interleave(rep, dim=1) for v in V], 0.35)
    err = np.abs(got - ref).max()
    assert err <= 1e-12, f"grouped-query shared prefix vs unpaged sdpa: max err {err}"


SHARED_PINS = [pin_shared_vs_unpaged_sdpa, pin_shared_brute_force_and_empty,
               pin_shared_grouped_query_vs_unpaged_sdpa]
SPLIT_PINS = [pin_split_worked_example]
