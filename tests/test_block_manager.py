"""The C++ block manager (through the C ABI) against the pages' worked
example, the invariants, and the oracle's model (CPU only)."""
import random

import pytest

from oracle import BlockManagerModel
from tests import bm_checks as C


class CppManager:
    """Adapter: plain lists out of the binding's tensors."""

    def __init__(self, n, b, seed=0):
        import paged_kv_cache_326_b200 as P
        self.bm = P.BlockManager(n, b, seed)

    def add_seq(self, s, n):
        self.bm.add_seq(s, n)

    def fork(self, p, c):
        self.bm.fork(p, c)

    def append_slot(self, s):
        return self.bm.append_slot(s)

    def free_seq(self, s):
        self.bm.free_seq(s)

    def num_free(self):
        return self.bm.num_free()

    def refcount(self, b):
        return self.bm.refcount(b)

    def export(self, ids, mb):
        t, l = self.bm.export(ids, mb)
        return t.tolist(), l.tolist()


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_326_b200 import build
    build.build()


def test_golden_two_answers():
    C.run_golden_two_answers(lambda n, b: CppManager(n, b))


@pytest.mark.parametrize("seed", range(6))
def test_random_ops_keep_invariants(seed):
    C.random_ops(lambda n, b: CppManager(n, b, seed + 1), seed)


def test_errors():
    C.check_errors(lambda n, b: CppManager(n, b))


@pytest.mark.parametrize("seed", range(4))
def test_matches_model_exactly_in_block_order(seed):
    """Free list in block order: the same operations give the same slots,
    copies, tables and counts, bit for bit."""
    log_cpp = C.random_ops(lambda n, b: CppManager(n, b, 0), 100 + seed)
    log_model = C.random_ops(lambda n, b: BlockManagerModel(n, b), 100 + seed)
    assert log_cpp == log_model


@pytest.mark.parametrize("seed", range(3))
def test_matches_model_up_to_relabelling_when_shuffled(seed):
    """Shuffled free list: the two agree once physical block ids are
    relabelled consistently (which free block is handed out is the
    manager's choice; the pages fix only the structure)."""
    B = 4
    cpp = CppManager(40, B, 1234 + seed)
    model = BlockManagerModel(40, B)
    rnd = random.Random(seed)
    relabel = {}

    def same(a, b):
        if a < 0 or b < 0:
            assert a == b == -1 or (a < 0 and b < 0)
            return
        if a in relabel:
            assert relabel[a] == b
        else:
            assert b not in relabel.values()
            relabel[a] = b

    live, nid = [], 0
    for _ in range(300):
        op = rnd.choice(["add", "fork", "append", "append", "free"])
        try:
            if op == "add":
                n = rnd.randint(0, 9)
                model.add_seq(nid, n)
                cpp.add_seq(nid, n)
                live.append(nid)
                nid += 1
            elif op == "fork" and live:
                p = rnd.choice(live)
                model.fork(p, nid)
                cpp.fork(p, nid)
                live.append(nid)
                nid += 1
            elif op == "append" and live:
                s = rnd.choice(live)
                ms, msrc, mdst = model.append_slot(s)
                cs, csrc, cdst = cpp.append_slot(s)
                assert ms % B == cs % B
                same(cs // B, ms // B)
                same(csrc, msrc)
                same(cdst, mdst)
            elif op == "free" and live:
                s = rnd.choice(live)
                model.free_seq(s)
                cpp.free_seq(s)
                live.remove(s)
        except Exception as e:  # noqa: BLE001
            assert getattr(e, "kind", None) == "out_of_blocks"
            continue
        if live:
            mt, ml = model.export(live, 16)
            ct, cl = cpp.export(live, 16)
            assert ml == cl
            for mrow, crow in zip(mt, ct):
                for mb, cb in zip(mrow, crow):
                    same(cb, mb)
        assert model.num_free() == cpp.num_free()


def test_shared_prefix_workload_tables_agree_with_model():
    """The parallel-sampling workload built through the C++ manager and
    through the model gives the same tables, lengths, slots and copies."""
    from paged_kv_cache_326_b200 import workloads as W

    kw = dict(num_blocks=2048, num_prompts=3, samples=4, num_heads=2, head_dim=64,
              block_size=16, prompt_range=(20, 70), gen_range=(1, 40), max_blocks_per_seq=8)
    a = W.shared_prefix(CppManager(2048, 16), **kw)
    b = W.shared_prefix(BlockManagerModel(2048, 16), **kw)
    assert a.block_tables.tolist() == b.block_tables.tolist()
    assert a.context_lens.tolist() == b.context_lens.tolist()
    assert a.slot_mapping.tolist() == b.slot_mapping.tolist()
    assert a.meta["cow"] == b.meta["cow"]
    assert len(a.meta["cow"]) > 0
