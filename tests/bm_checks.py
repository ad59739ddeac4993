"""Block-manager checks shared by the model's tests and the C++ manager's
tests.  ``make(num_blocks, block_size)`` returns an object with the model's
methods; errors surface as an exception with a ``kind`` attribute."""
import random

from tests.oracle_pins import load_golden


def run_golden_two_answers(make):
    g = load_golden("cow_two_answers.json")
    bm = make(g["num_blocks"], g["block_size"])
    bm.add_seq(1, g["prompt_tokens"])
    bm.fork(1, 2)

    def state(expect):
        tables, _ = bm.export([1, 2], 4)
        got = {"answer1": [b for b in tables[0] if b >= 0],
               "answer2": [b for b in tables[1] if b >= 0]}
        assert got == expect["tables"], (got, expect["tables"])
        for b, c in expect["refcount"].items():
            assert bm.refcount(int(b)) == c, (b, bm.refcount(int(b)), c)
        assert bm.num_free() == expect["num_free"]

    state(g["after_fork"])
    assert tuple(bm.append_slot(1)) == (g["answer1_append"]["slot"], g["answer1_append"]["cow_src"],
                                        g["answer1_append"]["cow_dst"])
    state(g["after_answer1"])
    assert tuple(bm.append_slot(2)) == (g["answer2_append"]["slot"], g["answer2_append"]["cow_src"],
                                        g["answer2_append"]["cow_dst"])
    state(g["after_answer2"])
    bm.free_seq(1)
    bm.free_seq(2)
    assert bm.num_free() == g["after_free_both"]["num_free"]
    for b, c in g["after_free_both"]["refcount"].items():
        assert bm.refcount(int(b)) == c


def check_invariants(bm, live, num_blocks, block_size, max_blocks):
    """Free + distinct live blocks = pool; counts equal the number of tables
    holding the block; every text wastes less than one block (it receives a
    further block only once its current ones are full)."""
    if not live:
        assert bm.num_free() == num_blocks
        return
    tables, lens = bm.export(sorted(live), max_blocks)
    holders = {}
    for t, L in zip(tables, lens):
        blocks = [b for b in t if b >= 0]
        assert len(blocks) == -(-L // block_size), (blocks, L)
        assert len(blocks) * block_size - L < block_size
        for b in blocks:
            holders[b] = holders.get(b, 0) + 1
    for b, n in holders.items():
        assert bm.refcount(b) == n, (b, bm.refcount(b), n)
    assert bm.num_free() + len(holders) == num_blocks


def random_ops(make, seed, num_blocks=48, block_size=4, steps=400, max_blocks=64):
    """Random add / fork / append / free; invariants after every step; an
    operation refused for lack of blocks changes nothing."""
    rnd = random.Random(seed)
    bm = make(num_blocks, block_size)
    live = set()
    next_id = 0
    log = []
    for _ in range(steps):
        op = rnd.choice(["add", "fork", "append", "append", "append", "free"])
        before = (bm.num_free(), bm.export(sorted(live), max_blocks) if live else None)
        try:
            if op == "add":
                n = rnd.randint(0, 13)
                bm.add_seq(next_id, n)
                live.add(next_id)
                log.append(("add", next_id, n))
                next_id += 1
            elif op == "fork" and live:
                p = rnd.choice(sorted(live))
                bm.fork(p, next_id)
                live.add(next_id)
                log.append(("fork", p, next_id))
                next_id += 1
            elif op == "append" and live:
                s = rnd.choice(sorted(live))
                log.append(("append", s, tuple(bm.append_slot(s))))
            elif op == "free" and live:
                s = rnd.choice(sorted(live))
                bm.free_seq(s)
                live.discard(s)
                log.append(("free", s))
        except Exception as e:  # noqa: BLE001
            assert getattr(e, "kind", None) == "out_of_blocks", e
            after = (bm.num_free(), bm.export(sorted(live), max_blocks) if live else None)
            assert before == after, "refused operation changed the state"
            log.append(("refused", op))
        check_invariants(bm, live, num_blocks, block_size, max_blocks)
    return log


def check_errors(make):
    bm = make(4, 4)
    bm.add_seq(1, 8)
    for call, kind in ((lambda: bm.add_seq(1, 1), "exists"),
                       (lambda: bm.fork(9, 10), "no_seq"),
                       (lambda: bm.fork(1, 1), "exists"),
                       (lambda: bm.append_slot(7), "no_seq"),
                       (lambda: bm.free_seq(7), "no_seq"),
                       (lambda: bm.add_seq(2, 9), "out_of_blocks"),
                       (lambda: bm.export([1], 1), "table_full")):
        try:
            call()
        except Exception as e:  # noqa: BLE001
            assert getattr(e, "kind", None) == kind, (kind, e)
        else:
            raise AssertionError(f"expected {kind}")
    assert bm.num_free() == 2
