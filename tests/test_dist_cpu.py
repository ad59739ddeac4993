"""Multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from paged_kv_cache_326_b200 import dist
    r = dist.init("gloo", timeout_s=60)
    dist.barrier(r)
    times = dist.max_over_ranks(r, [1.0 + rank, 5.0 - rank])
    seed = dist.batch_seed(2, r)
    from paged_kv_cache_326_b200 import workloads as W
    lens = W.opt13b_batch64_lens(seed)
    dist.finish(r)
    q.put((rank, times, seed, lens[:4]))


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_max_and_run_independent_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=100) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    out.sort()
    # the slowest rank's time, the same on every rank
    assert out[0][1] == out[1][1] == [2.0, 5.0]
    # independent batches: distinct seeds and lengths
    assert out[0][2] != out[1][2] and out[0][3] != out[1][3]


def test_single_process_needs_no_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    from paged_kv_cache_326_b200 import dist
    r = dist.init("gloo")
    assert (r.world, r.rank) == (1, 0)
    assert dist.max_over_ranks(r, [3.0]) == [3.0]
