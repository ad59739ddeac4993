"""Block copies on the GPU (pa_copy_blocks) against the oracle: bit-exact over
whole pools, within a pool (copy-on-write) and between pools (blocks moved
out to pinned host memory and back), plus a parallel-sampling session run
through the C++ block manager with every copy made on the device."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import compare, new_status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from paged_kv_cache_326_b200 import build
    build.build()
    import paged_kv_cache_326_b200 as P
    return P.lib()


def _bits_pool(N, H, B, D, dtype, seed, device="cuda", pin=False):
    """A pool of random 16-bit patterns (NaN and infinity payloads included)."""
    g = torch.Generator().manual_seed(seed)
    t = torch.randint(-(1 << 15), 1 << 15, (N, H, B, D), generator=g, dtype=torch.int32)
    t = t.to(torch.int16).view(dtype)
    if device == "cpu":
        return t.pin_memory() if pin else t
    return t.to(device)


def _pairs(n_src, n_dst, count, seed, same_pool):
    """count pairs with distinct destinations; within one pool no block is
    both a source and a destination."""
    rng = np.random.default_rng(seed)
    if same_pool:
        perm = rng.permutation(n_src)
        dst = perm[:count]
        src = rng.choice(perm[count:], size=count, replace=True)
    else:
        dst = rng.permutation(n_dst)[:count]
        src = rng.integers(0, n_src, size=count)
    return [(int(s), int(d)) for s, d in zip(src, dst)]


def _i16(t):
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("shape", [(40, 128, 16), (3, 64, 4), (8, 128, 32), (1, 64, 8)],
                         ids=lambda s: f"h{s[0]}d{s[1]}b{s[2]}")
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
def test_copy_within_pool_bit_exact(shape, dtype):
    import paged_kv_cache_326_b200 as P
    H, D, B = shape
    N = 96
    kc, vc = _bits_pool(N, H, B, D, dtype, 1), _bits_pool(N, H, B, D, dtype, 2)
    pairs = _pairs(N, N, 37, H + D + B, same_pool=True)
    ek, ev = oracle.copy_blocks(_i16(kc), _i16(vc), _i16(kc), _i16(vc), pairs)
    st = new_status()
    P.pa_copy_blocks(kc, vc, kc, vc, torch.tensor(pairs, dtype=torch.int32, device="cuda"),
                     status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert np.array_equal(_i16(kc), ek) and np.array_equal(_i16(vc), ev)


def test_copy_between_device_pools():
    import paged_kv_cache_326_b200 as P
    H, D, B = 5, 128, 16
    sk, sv = _bits_pool(50, H, B, D, torch.float16, 3), _bits_pool(50, H, B, D, torch.float16, 4)
    dk, dv = _bits_pool(30, H, B, D, torch.float16, 5), _bits_pool(30, H, B, D, torch.float16, 6)
    pairs = _pairs(50, 30, 30, 7, same_pool=False)
    ek, ev = oracle.copy_blocks(_i16(sk), _i16(sv), _i16(dk), _i16(dv), pairs)
    P.pa_copy_blocks(sk, sv, dk, dv, torch.tensor(pairs, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(_i16(dk), ek) and np.array_equal(_i16(dv), ev)


def test_blocks_moved_out_to_pinned_host_and_back():
    """"When Memory Runs Out": blocks go out to CPU memory and come back,
    later, into other free blocks of the pool."""
    import paged_kv_cache_326_b200 as P
    H, D, B, N = 4, 64, 16, 64
    kc, vc = _bits_pool(N, H, B, D, torch.bfloat16, 8), _bits_pool(N, H, B, D, torch.bfloat16, 9)
    hk = _bits_pool(10, H, B, D, torch.bfloat16, 10, device="cpu", pin=True)
    hv = _bits_pool(10, H, B, D, torch.bfloat16, 11, device="cpu", pin=True)
    out_pairs = [(b, i) for i, b in enumerate([3, 17, 40, 41, 63, 0, 9, 22, 30, 5])]
    ek, ev = oracle.copy_blocks(_i16(kc), _i16(vc), _i16(hk), _i16(hv), out_pairs)
    P.pa_copy_blocks(kc, vc, hk, hv, torch.tensor(out_pairs, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(_i16(hk), ek) and np.array_equal(_i16(hv), ev)
    back_pairs = [(i, b) for i, b in enumerate([50, 51, 52, 1, 2, 4, 6, 7, 8, 10])]
    ek2, ev2 = oracle.copy_blocks(_i16(hk), _i16(hv), _i16(kc), _i16(vc), back_pairs)
    P.pa_copy_blocks(hk, hv, kc, vc, torch.tensor(back_pairs, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(_i16(kc), ek2) and np.array_equal(_i16(vc), ev2)


def test_block_ids_outside_a_pool_are_reported_and_skipped():
    import paged_kv_cache_326_b200 as P
    H, D, B, N = 2, 64, 8, 20
    kc, vc = _bits_pool(N, H, B, D, torch.float16, 12), _bits_pool(N, H, B, D, torch.float16, 13)
    pairs = [(1, 2), (-1, 3), (4, N), (5, 6)]
    ek, ev = oracle.copy_blocks(_i16(kc), _i16(vc), _i16(kc), _i16(vc), [(1, 2), (5, 6)])
    st = new_status()
    P.pa_copy_blocks(kc, vc, kc, vc, torch.tensor(pairs, dtype=torch.int32, device="cuda"),
                     status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_BLOCK
    assert np.array_equal(_i16(kc), ek) and np.array_equal(_i16(vc), ev)


def test_unmapped_host_memory_is_refused_before_launch():
    """Pageable host memory is not addressable by the GPU: the library
    refuses it on the host (nothing is launched)."""
    import paged_kv_cache_326_b200 as P
    H, D, B = 2, 64, 8
    kc = _bits_pool(8, H, B, D, torch.float16, 14)
    host = torch.zeros((8, H, B, D), dtype=torch.float16)   # pageable
    assert not host.is_pinned()
    pairs = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    code = P.lib().pa_copy_blocks(
        ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(kc.data_ptr()), 8,
        ctypes.c_void_p(host.data_ptr()), ctypes.c_void_p(host.data_ptr()), 8,
        ctypes.c_void_p(pairs.data_ptr()), 1, H, D, B, 0, None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == P.binding.PA_ERR_INVALID
    with pytest.raises(TypeError):
        P.pa_copy_blocks(kc, kc, host, host, pairs)
    assert not host.any()


def test_parallel_sampling_session_with_device_copies():
    """Prompts forked into samples that then generate, one token per sample
    per round, through the C++ block manager: each copy-on-write pair is
    made by pa_copy_blocks, each token stored by pa_kv_cache_write; the
    oracle replays the same session (its block-manager model, copy_blocks,
    cache_write).  Pools agree bit for bit after every round; attention at
    the end agrees within the tolerance."""
    import paged_kv_cache_326_b200 as P
    H, D, B, N = 4, 64, 8, 256
    dt = torch.float16
    rng = np.random.default_rng(21)
    bm = P.BlockManager(N, B)
    model = oracle.BlockManagerModel(N, B)
    kc = torch.full((N, H, B, D), float("nan"), dtype=dt, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    okc, ovc = _i16(kc), _i16(vc)
    st = new_status()
    g = torch.Generator(device="cuda").manual_seed(22)
    seqs = []
    for p in range(4):
        L = int(rng.integers(5, 41))
        base = 10 * p
        bm.add_seq(base, L)
        model.add_seq(base, L)
        # the prompt's tokens: slots block*B + place through the table
        tables, _ = bm.export([base], (L + B - 1) // B)
        slots = torch.tensor([int(tables[0, t // B]) * B + t % B for t in range(L)],
                             dtype=torch.int64, device="cuda")
        k = torch.randn((L, H, D), generator=g, device="cuda").to(dt)
        v = torch.randn((L, H, D), generator=g, device="cuda").to(dt)
        P.pa_kv_cache_write(k, v, kc, vc, slots, status=st)
        okc, ovc = oracle.cache_write(okc, ovc, _i16(k), _i16(v), slots.cpu().numpy(), B)
        for s in range(1, 4):
            bm.fork(base, base + s)
            model.fork(base, base + s)
        seqs += [base + s for s in range(4)]
    for _ in range(12):
        for sid in seqs:
            slot, src, dst = bm.append_slot(sid)
            assert (slot, src, dst) == tuple(model.append_slot(sid))
            if src >= 0:
                pair = torch.tensor([[src, dst]], dtype=torch.int32, device="cuda")
                P.pa_copy_blocks(kc, vc, kc, vc, pair, status=st)
                okc, ovc = oracle.copy_blocks(okc, ovc, okc, ovc, [(src, dst)])
            k = torch.randn((1, H, D), generator=g, device="cuda").to(dt)
            v = torch.randn((1, H, D), generator=g, device="cuda").to(dt)
            P.pa_kv_cache_write(k, v, kc, vc, torch.tensor([slot], device="cuda"), status=st)
            okc, ovc = oracle.cache_write(okc, ovc, _i16(k), _i16(v), [slot], B)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert np.array_equal(_i16(kc), okc) and np.array_equal(_i16(vc), ovc)
    mb = max(model.tokens[s] for s in seqs) // B + 1
    tables, lens = bm.export(seqs, mb)
    q = torch.randn((len(seqs), H, D), generator=g, device="cuda").to(dt)
    out = torch.empty_like(q)
    P.pa_paged_attn_decode(out, q, kc, vc, tables.to("cuda"), lens.to("cuda"), D ** -0.5,
                           status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    f16 = lambda a: a.view(np.float16).astype(np.float64)
    ref = oracle.paged_decode(q.double().cpu().numpy(), f16(okc), f16(ovc), tables.numpy(),
                              lens.numpy(), float(np.float32(D ** -0.5)), B)
    c = compare(out, ref, dt)
    assert c.ok, c


@pytest.mark.parametrize("count", [1, 7, 700])
def test_copy_small_blocks_many_pairs(count):
    """Blocks of 512 bytes (1 head x 4 x 64, 32 vectors): one CTA per copy
    with most of its threads idle, one pair or 700 of them.  Bit-exact in
    every case."""
    import paged_kv_cache_326_b200 as P
    H, D, B, N = 1, 64, 4, 1600
    kc, vc = (_bits_pool(N, H, B, D, torch.float16, 11 + i) for i in range(2))
    pairs = _pairs(N, N, count, 12 + count, same_pool=True)
    ek, ev = oracle.copy_blocks(_i16(kc), _i16(vc), _i16(kc), _i16(vc), pairs)
    st = new_status()
    P.pa_copy_blocks(kc, vc, kc, vc, torch.tensor(pairs, dtype=torch.int32, device="cuda"),
                     status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert np.array_equal(_i16(kc), ek) and np.array_equal(_i16(vc), ev)


def test_copy_bad_pair_in_the_middle_is_reported_and_skipped():
    """A pair naming a block outside the pool, between good ones: the status
    word says PA_ERR_BAD_BLOCK, that pair copies nothing, every other pair
    is exact."""
    import paged_kv_cache_326_b200 as P
    H, D, B, N = 8, 128, 16, 64
    kc, vc = (_bits_pool(N, H, B, D, torch.bfloat16, 21 + i) for i in range(2))
    good = _pairs(N, N, 20, 23, same_pool=True)
    pairs = good[:10] + [(N + 5, good[10][1])] + good[11:]
    ek, ev = oracle.copy_blocks(_i16(kc), _i16(vc), _i16(kc), _i16(vc),
                                good[:10] + good[11:])
    st = new_status()
    P.pa_copy_blocks(kc, vc, kc, vc, torch.tensor(pairs, dtype=torch.int32, device="cuda"),
                     status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_BLOCK
    assert np.array_equal(_i16(kc), ek) and np.array_equal(_i16(vc), ev)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
def test_copy_runs_of_one_source(dtype):
    """Runs of consecutive pairs with one source (a prompt's block copied for
    each of its samples): runs of 1, 3, 8, 9 and 17 pairs, a run whose source
    is outside the pool, and a run with a bad destination inside it.  The
    bad pairs are reported and copy nothing; every other pair is exact."""
    import paged_kv_cache_326_b200 as P
    H, D, B, N = 4, 128, 16, 200
    kc, vc = (_bits_pool(N, H, B, D, dtype, 31 + i) for i in range(2))
    rng = np.random.default_rng(33)
    perm = [int(x) for x in rng.permutation(N)]
    srcs, dsts = perm[:10], iter(perm[10:])
    pairs, good = [], []
    for k, n in enumerate([1, 3, 8, 9, 17, 2, 5, 4]):
        for i in range(n):
            p = (srcs[k], next(dsts))
            if k == 5:
                p = (N + 3, p[1])            # source outside the pool
            if k == 4 and i == 11:
                p = (p[0], -2)               # destination outside the pool
            pairs.append(p)
            if 0 <= p[0] < N and 0 <= p[1] < N:
                good.append(p)
    ek, ev = oracle.copy_blocks(_i16(kc), _i16(vc), _i16(kc), _i16(vc), good)
    st = new_status()
    P.pa_copy_blocks(kc, vc, kc, vc, torch.tensor(pairs, dtype=torch.int32, device="cuda"),
                     status=st)
    torch.cuda.synchronize()
    assert st.item() == P.binding.PA_ERR_BAD_BLOCK
    assert np.array_equal(_i16(kc), ek) and np.array_equal(_i16(vc), ev)


def test_write_probe_writes_the_whole_buffer():
    import paged_kv_cache_326_b200 as P
    buf = torch.zeros(3 << 20, dtype=torch.uint8, device="cuda")
    P.binding.pa_write_probe(buf)
    torch.cuda.synchronize()
    w = buf.view(torch.int32).view(-1, 4).cpu()
    idx = torch.arange(w.shape[0], dtype=torch.int64)
    assert torch.equal(w[:, 0].to(torch.int64) & 0xFFFFFFFF, idx & 0xFFFFFFFF)
    assert torch.equal(w[:, 2], ~w[:, 0])
