"""The C++ prefix/tail splitter (pa_split_shared_prefix) against the oracle's
split, on tables the C++ block manager builds for forked prompts, and its
argument checks (CPU only)."""
import random

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins as P


def cpp_split(bt, lens, B, gs):
    import paged_kv_cache_326_b200 as PK
    pt, pl, tt, tl = PK.split_shared_prefix(torch.as_tensor(np.asarray(bt), dtype=torch.int32),
                                            torch.as_tensor(list(lens), dtype=torch.int32), B, gs)
    pt_rows = [[b for b in row if b >= 0] for row in pt.tolist()]
    tt_rows = [[b for b in row if b >= 0] for row in tt.tolist()]
    return pt_rows, pl.tolist(), tt_rows, tl.tolist()


def test_cpp_split_passes_the_worked_pins():
    P.pin_split_worked_example(cpp_split)


@pytest.mark.parametrize("seed", range(6))
def test_cpp_split_matches_oracle_on_forked_groups(seed):
    import paged_kv_cache_326_b200 as PK
    rng = random.Random(seed)
    B = rng.choice([4, 8, 16, 32])
    gs = rng.choice([1, 2, 3, 8])
    groups = rng.randint(1, 6)
    bm = PK.BlockManager(4096, B, shuffle_seed=seed + 1)
    ids = []
    for g in range(groups):
        root = g * 100
        bm.add_seq(root, rng.randint(0, 5 * B))
        members = [root] + [root + m for m in range(1, gs)]
        for m in members[1:]:
            bm.fork(root, m)
        for m in members:
            for _ in range(rng.randint(0 if gs > 1 else 1, 2 * B)):
                bm.append_slot(m)
        ids += members
    mb = 16
    bt, lens = bm.export(ids, mb)
    want = oracle.split_shared_prefix(bt.numpy(), lens.tolist(), B, gs)
    got = cpp_split(bt.numpy(), lens.tolist(), B, gs)
    assert got[1] == list(want[1]) and got[3] == list(want[3])
    assert got[0] == [list(r) for r in want[0]] and got[2] == [list(r) for r in want[2]]
    # the prefix blocks are the ones the whole group holds
    for g, row in enumerate(got[0]):
        for b in row:
            assert bm.refcount(b) >= gs


def test_cpp_split_rejects_bad_arguments():
    import paged_kv_cache_326_b200 as PK
    bt = torch.tensor([[1, 2], [1, 3]], dtype=torch.int32)
    with pytest.raises(ValueError):
        PK.split_shared_prefix(bt, torch.tensor([32, 32], dtype=torch.int32), 16, 3)
    with pytest.raises(PK.PagedAttnError):  # a length past the table
        PK.split_shared_prefix(bt, torch.tensor([33, 32], dtype=torch.int32), 16, 2)
    apart = torch.tensor([[1, 2], [4, 3]], dtype=torch.int32)
    with pytest.raises(PK.PagedAttnError):  # a tail longer than the tail table
        PK.split_shared_prefix(apart, torch.tensor([32, 32], dtype=torch.int32), 16, 2,
                               max_tail_blocks=1)


def test_shared_decode_rejects_bad_arguments_before_launch():
    """Argument errors return PA_ERR_INVALID before any CUDA call (no GPU)."""
    import paged_kv_cache_326_b200 as PK
    lib = PK.lib()
    bad = PK.binding.PA_ERR_INVALID
    args = dict(out=None, q=None, kc=None, vc=None, pt=None, pl=None, mp=4, tt=None, tl=None,
                mt=4, scale=0.1, G=2, gs=8, H=8, D=128, B=16, N=64, dt=0, ws=None, wsb=0,
                st=None, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return lib.pa_paged_attn_decode_shared(a["out"], a["q"], a["kc"], a["vc"], a["pt"], a["pl"],
                                               a["mp"], a["tt"], a["tl"], a["mt"], a["scale"],
                                               a["G"], a["gs"], a["H"], a["D"], a["B"], a["N"],
                                               a["dt"], a["ws"], a["wsb"], a["st"], a["stream"])
    assert call(G=0) == PK.binding.PA_OK          # nothing to do
    assert call() == bad                          # null pointers
    assert call(gs=17) == bad                     # more texts per group than tile columns
    assert call(gs=0) == bad
    assert call(G=513, gs=8) == bad               # more than 4,096 texts
    assert call(B=4) == bad                       # blocks of 4 do not suit the tensor cores
    assert call(D=96) == bad
    assert call(mp=0) == bad and call(mt=0) == bad
    assert lib.pa_paged_attn_decode_shared_workspace_size(2, 17, 8, 128, 16, 4, 4) == 0
    assert lib.pa_paged_attn_decode_shared_workspace_size(2, 8, 8, 128, 16, 0, 4) == 0
