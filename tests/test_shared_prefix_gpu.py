"""The shared-prefix decode (prefix pass on the tensor cores, tail pass,
log-sum-exp merge) on the GPU against the oracle, on workloads built by the
C++ block manager: parallel sampling from forked prompts with copy-on-write
of the partial last prompt block."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_326_b200 import workloads as W
from tests.gpu_helpers import compare, new_status, oracle_inputs, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from paged_kv_cache_326_b200 import build
    build.build()
    import paged_kv_cache_326_b200 as P
    return P.lib()


def build_case(dtype, D, B, prompts, samples, prompt_range, gen_range, H, seed, num_blocks=None,
               Hkv=None):
    import paged_kv_cache_326_b200 as P
    mb = -(-(prompt_range[1] + gen_range[1]) // B) + 1
    if num_blocks is None:
        num_blocks = prompts * samples * mb + 64
    bm = P.BlockManager(num_blocks, B, shuffle_seed=seed + 1)

    class Adapter:
        add_seq = staticmethod(bm.add_seq)
        fork = staticmethod(bm.fork)
        append_slot = staticmethod(bm.append_slot)

        @staticmethod
        def export(ids, m):
            t, l = bm.export(ids, m)
            return t.numpy(), l.numpy()

    return W.shared_prefix(Adapter(), num_blocks=num_blocks, seed=seed, device="cuda",
                           dtype=dtype, num_prompts=prompts, samples=samples, num_heads=H,
                           head_dim=D, block_size=B, max_blocks_per_seq=mb,
                           prompt_range=prompt_range, gen_range=gen_range, num_kv_heads=Hkv)


def gpu_shared_step(w, status, out=None):
    """Cache write, host split of the tables, shared-prefix decode."""
    import paged_kv_cache_326_b200 as P
    gs = w.meta["samples"]
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=status)
    pt, pl, tt, tl = P.split_shared_prefix(w.block_tables.cpu(), w.context_lens.cpu(),
                                           w.block_size, gs)
    if out is None:
        out = torch.empty_like(w.q)
    P.pa_paged_attn_decode_shared(out, w.q, w.k_cache, w.v_cache, pt.cuda(), pl.cuda(),
                                  tt.cuda(), tl.cuda(), w.scale, gs, status=status)
    return out, (pt, pl, tt, tl)


CASES = [
    # dtype, D, B, prompts, samples, prompt range, generated range, heads
    (torch.float16, 128, 16, 3, 8, (5, 90), (1, 40), 4),
    (torch.bfloat16, 128, 8, 4, 3, (1, 70), (1, 30), 3),
    (torch.float16, 64, 32, 2, 16, (20, 130), (1, 50), 2),
    (torch.bfloat16, 64, 16, 5, 1, (1, 60), (1, 20), 2),
    (torch.float16, 128, 32, 3, 5, (2, 9), (1, 6), 2),   # prompts shorter than a block
    # groups of more than 16 texts: the prefix pass in subsets of at most 16
    (torch.float16, 128, 16, 2, 24, (30, 120), (1, 40), 3),   # 2 subsets of 12
    (torch.bfloat16, 64, 8, 1, 40, (10, 80), (1, 30), 2),     # 4 subsets of 10
    (torch.float16, 128, 16, 1, 17, (20, 60), (1, 20), 2),    # 17 subsets of 1
    (torch.float16, 128, 32, 2, 32, (40, 150), (1, 50), 2),   # 2 subsets of 16
]


@pytest.mark.parametrize("idx", range(len(CASES)),
                         ids=[f"{str(c[0])[6:]}-D{c[1]}-B{c[2]}-g{c[4]}" for c in CASES])
def test_shared_prefix_matches_oracle(idx):
    dtype, D, B, prompts, samples, pr, gr, H = CASES[idx]
    w = build_case(dtype, D, B, prompts, samples, pr, gr, H, seed=100 + idx)
    oi = oracle_inputs(w.q, w.k, w.v, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                       w.slot_mapping, B)
    st = new_status()
    out, split = gpu_shared_step(w, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    # the oracle's own split of the same (renumbered) tables, then its
    # shared-prefix attention
    kc, vc = oracle.cache_write(oi.k_cache, oi.v_cache, oi.k, oi.v, oi.slots, B)
    pt, pl, tt, tl = oracle.split_shared_prefix(oi.tables, oi.lens, B, samples)
    ref = oracle.paged_decode_shared(oi.q, kc, vc, pt, pl, tt, tl, samples, w.scale, B)
    c = compare(out, ref, dtype)
    assert c.ok, str(c)
    assert list(split[1].tolist()) == list(pl) and list(split[3].tolist()) == list(tl)


GQA_CASES = [
    # dtype, D, B, prompts, samples, prompt range, generated range, query heads, kv heads
    (torch.float16, 128, 16, 3, 8, (5, 90), (1, 40), 8, 1),     # 64 columns: 4 subsets of 16
    (torch.bfloat16, 128, 8, 2, 4, (1, 70), (1, 30), 16, 2),    # 32 columns a kv head
    (torch.float16, 64, 32, 2, 3, (20, 130), (1, 50), 6, 2),    # 9 columns
    (torch.float16, 128, 16, 2, 2, (30, 120), (1, 40), 64, 8),  # Llama-2-70B heads, 16 columns
]


@pytest.mark.parametrize("idx", range(len(GQA_CASES)),
                         ids=[f"{str(c[0])[6:]}-D{c[1]}-B{c[2]}-g{c[4]}-h{c[7]}kv{c[8]}"
                              for c in GQA_CASES])
def test_shared_prefix_grouped_query_matches_oracle(idx):
    """Grouped-query pools (pa_paged_attn_decode_shared_gqa): every output
    against the oracle's shared-prefix attention on the same pool."""
    dtype, D, B, prompts, samples, pr, gr, H, Hkv = GQA_CASES[idx]
    w = build_case(dtype, D, B, prompts, samples, pr, gr, H, seed=200 + idx, Hkv=Hkv)
    oi = oracle_inputs(w.q, w.k, w.v, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                       w.slot_mapping, B)
    st = new_status()
    out, split = gpu_shared_step(w, st)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    kc, vc = oracle.cache_write(oi.k_cache, oi.v_cache, oi.k, oi.v, oi.slots, B)
    pt, pl, tt, tl = oracle.split_shared_prefix(oi.tables, oi.lens, B, samples)
    ref = oracle.paged_decode_shared(oi.q, kc, vc, pt, pl, tt, tl, samples, w.scale, B)
    c = compare(out, ref, dtype)
    assert c.ok, str(c)


def test_shared_prefix_is_deterministic_and_close_to_plain_decode():
    import paged_kv_cache_326_b200 as P
    w = build_case(torch.float16, 128, 16, 4, 8, (40, 200), (1, 60), 8, seed=7)
    st = new_status()
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=st)
    pt, pl, tt, tl = [t.cuda() for t in P.split_shared_prefix(w.block_tables.cpu(),
                                                              w.context_lens.cpu(), 16, 8)]
    a = torch.empty_like(w.q)
    b = torch.empty_like(w.q)
    P.pa_paged_attn_decode_shared(a, w.q, w.k_cache, w.v_cache, pt, pl, tt, tl, w.scale, 8,
                                  status=st)
    P.pa_paged_attn_decode_shared(b, w.q, w.k_cache, w.v_cache, pt, pl, tt, tl, w.scale, 8,
                                  status=st)
    plain = torch.empty_like(w.q)
    P.pa_paged_attn_decode(plain, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                           w.scale, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(a, b), "shared-prefix decode is not reproducible"
    assert (a.float() - plain.float()).abs().max().item() <= 2e-3


def test_shared_prefix_empty_prefix_and_empty_text():
    """Groups with no shared block, and a text with no tokens (zeros)."""
    import paged_kv_cache_326_b200 as P
    S, H, D, B, N = 4, 2, 128, 16, 16
    g = torch.Generator(device="cuda").manual_seed(5)
    kc = torch.randn(N, H, B, D, device="cuda", generator=g).half()
    vc = torch.randn(N, H, B, D, device="cuda", generator=g).half()
    q = torch.randn(S, H, D, device="cuda", generator=g).half()
    pt = torch.tensor([[-1], [3]], dtype=torch.int32, device="cuda")
    pl = torch.tensor([0, 16], dtype=torch.int32, device="cuda")
    tt = torch.tensor([[1, 2], [-1, -1], [4, -1], [-1, -1]], dtype=torch.int32, device="cuda")
    tl = torch.tensor([20, 0, 7, 0], dtype=torch.int32, device="cuda")
    out = torch.full_like(q, float("nan"))
    st = new_status()
    P.pa_paged_attn_decode_shared(out, q, kc, vc, pt, pl, tt, tl, 0.1, 2, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = oracle.paged_decode_shared(q.float().cpu().numpy(), kc.float().cpu().numpy(),
                                     vc.float().cpu().numpy(), [[], [3]], [0, 16],
                                     [[1, 2], [], [4], []], [20, 0, 7, 0], 2, 0.1, B)
    assert torch.equal(out[1], torch.zeros_like(out[1])), "empty text is not zero"
    c = compare(out, ref, torch.float16)
    assert c.ok, str(c)


def test_shared_prefix_bad_block_sets_status():
    import paged_kv_cache_326_b200 as P
    S, H, D, B, N = 2, 2, 128, 16, 8
    kc = torch.zeros(N, H, B, D, device="cuda", dtype=torch.float16)
    q = torch.zeros(S, H, D, device="cuda", dtype=torch.float16)
    pt = torch.tensor([[N + 5]], dtype=torch.int32, device="cuda")
    pl = torch.tensor([16], dtype=torch.int32, device="cuda")
    tt = torch.tensor([[1], [2]], dtype=torch.int32, device="cuda")
    tl = torch.tensor([3, 3], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    st = new_status()
    P.pa_paged_attn_decode_shared(out, q, kc, kc, pt, pl, tt, tl, 0.1, 2, status=st)
    torch.cuda.synchronize()
    assert st.item() == -7
    assert torch.isfinite(out.float()).all()


def test_shared_prefix_full_size_sampled():
    """32 prompts x 8 samples, 40 heads x 128, B = 16, in the launch
    configuration the benchmark times; sampled outputs against the oracle's
    decode over the joined tables (equal to its shared-prefix form, bit for
    bit, by a CPU pin)."""
    import paged_kv_cache_326_b200 as P

    class Adapter:
        pass
    bm = P.BlockManager(8192, 16)
    Adapter.add_seq = staticmethod(bm.add_seq)
    Adapter.fork = staticmethod(bm.fork)
    Adapter.append_slot = staticmethod(bm.append_slot)
    Adapter.export = staticmethod(lambda ids, m: tuple(t.numpy() for t in bm.export(ids, m)))
    w = W.shared_prefix(Adapter, num_blocks=8192, seed=4, device="cuda")
    rng = np.random.default_rng(3)
    seqs = np.sort(rng.choice(w.q.shape[0], 12, replace=False))
    pairs = [(int(s), int(h)) for s in seqs for h in rng.choice(40, 3, replace=False)]
    oi = oracle_inputs(w.q, w.k, w.v, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                       w.slot_mapping, 16, seqs)
    st = new_status()
    out, _ = gpu_shared_step(w, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = run_oracle(oi, w.scale, 16, pairs)
    pos = {int(s): i for i, s in enumerate(seqs)}
    got = torch.stack([out[s, h] for s, h in pairs])
    want = np.stack([ref[pos[s], h] for s, h in pairs])
    c = compare(got, want, torch.float16)
    assert c.ok, str(c)
