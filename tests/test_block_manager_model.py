"""The oracle's block-manager model against the pages' worked example and the
invariants (CPU only)."""
import pytest

from oracle import BlockManagerModel
from tests import bm_checks as C


def make(n, b):
    return BlockManagerModel(n, b)


def test_golden_two_answers():
    C.run_golden_two_answers(make)


@pytest.mark.parametrize("seed", range(6))
def test_random_ops_keep_invariants(seed):
    C.random_ops(make, seed)


def test_errors():
    C.check_errors(make)


def test_eight_samples_copy_seven_times():
    """Eight samples of a prompt whose last block is partial: the first seven
    writers copy the shared block, the eighth finds count 1 and writes in
    place."""
    bm = BlockManagerModel(64, 16)
    bm.add_seq(0, 100)                      # 7 blocks, last one 4/16 full
    for k in range(1, 8):
        bm.fork(0, k)
    last = bm.export([0], 8)[0][0][6]
    cows = [bm.append_slot(k)[1:] for k in range(8)]
    assert [c for c in cows if c[0] >= 0] == [(last, 7 + i) for i in range(7)]
    assert cows[7] == (-1, -1)
    assert bm.refcount(last) == 1


def test_full_prompt_block_needs_no_copy():
    bm = BlockManagerModel(8, 4)
    bm.add_seq(0, 8)
    bm.fork(0, 1)
    slot, src, dst = bm.append_slot(1)
    assert (src, dst) == (-1, -1) and slot == 2 * 4
