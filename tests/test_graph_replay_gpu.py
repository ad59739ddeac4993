"""Decode calls captured once in a CUDA graph and replayed.

A replay repeats the captured launches with the parameters they were
captured with, the grain counter's epoch among them.  Each call's last
kernel zeroes the counter, so every replay hands out its grains from zero.
Between replays the inputs change in place (lengths, tables, pool contents,
queries), and every replay is compared with the oracle on the inputs it saw.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_326_b200 import workloads as W
from tests.gpu_helpers import compare, new_status, oracle_inputs, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from paged_kv_cache_326_b200 import build
    build.build()
    import paged_kv_cache_326_b200 as P
    P.lib()
    return P


def _inputs(seed, num_kv_heads=None):
    # 16 texts x 8 query heads of 128, blocks of 16: a few thousand chunks, so
    # every warp's work comes in grains from the shared counter
    g = np.random.default_rng(seed)
    lens = [int(x) for x in g.integers(17, 600, size=16, endpoint=True)]
    return W.make_decode(f"replay{seed}", lens, num_heads=8, head_dim=128, block_size=16,
                         num_blocks=1024, dtype=torch.float16, seed=seed, device="cuda",
                         max_blocks_per_seq=40, num_kv_heads=num_kv_heads)


def _load(dst, src):
    """Copy every input of `src` into the tensors the graph was captured on."""
    for name in ("q", "k", "v", "k_cache", "v_cache", "block_tables", "context_lens",
                 "slot_mapping"):
        getattr(dst, name).copy_(getattr(src, name))


@pytest.mark.parametrize("kind", ["multi_head", "grouped_query", "one_launch_step"])
def test_replayed_decode_matches_oracle_each_time(P, kind):
    kv = 2 if kind == "grouped_query" else None
    live = _inputs(11, kv)
    out = torch.empty_like(live.q)
    status = new_status()
    S, H, D = live.q.shape
    if kv is None:
        ws_bytes = P.pa_paged_attn_decode_workspace_size(S, H, D, 16, live.max_blocks_per_seq)
    else:
        ws_bytes = P.binding.pa_paged_attn_decode_gqa_workspace_size(S, H, kv, D, 16,
                                                             live.max_blocks_per_seq)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")

    def step():
        if kind == "one_launch_step":
            P.pa_decode_step(out, live.q, live.k, live.v, live.k_cache, live.v_cache,
                             live.slot_mapping, live.block_tables, live.context_lens, live.scale,
                             workspace=ws, status=status)
            return
        P.pa_kv_cache_write(live.k, live.v, live.k_cache, live.v_cache, live.slot_mapping,
                            status=status)
        fn = P.pa_paged_attn_decode if kv is None else P.pa_paged_attn_decode_gqa
        fn(out, live.q, live.k_cache, live.v_cache, live.block_tables, live.context_lens,
           live.scale, workspace=ws, status=status)

    # warm-up outside capture (one-time host set-up), then restore the inputs
    fresh = _inputs(11, kv)
    step()
    torch.cuda.synchronize()
    _load(live, fresh)
    torch.cuda.synchronize()

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    for replay, seed in enumerate([11, 12, 13, 13]):
        src = _inputs(seed, kv)
        oi = oracle_inputs(src.q, src.k, src.v, src.k_cache, src.v_cache, src.block_tables,
                           src.context_lens, src.slot_mapping, 16)
        _load(live, src)
        out.fill_(float("nan"))
        status.zero_()
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert status.item() == 0, P.pa_status_string(status.item())
        c = compare(out, run_oracle(oi, src.scale, 16), torch.float16)
        assert c.ok, f"replay {replay + 1} (inputs {seed}): {c}"
    del graph
