"""Benchmark: one decode step of an OPT-13B-shaped layer, batch 64.

A step is the whole hot path once: the write of each text's new key/value,
then paged decode attention over every text's cache.  By default it is the
one-launch entry point pa_decode_step (write + attention in the decode
kernel, then the log-sum-exp merge kernel); ``--path calls`` times the two
calls pa_kv_cache_write + pa_paged_attn_decode instead.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--path fused|calls]

Prints one JSON line (rank 0).  ``value`` is KV bytes read per step / device
time per step (GB/s, whole job over all ranks); ``e2e`` repeats it with the
step's inputs copied from pinned host memory and the output copied back inside
the timed region.  Under torchrun each rank runs its own independent batch
(weak scaling, no collective on the data path).  ``--impl reference`` times the
fp64 CPU oracle on the host instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode KV HBM GB/s (% of B200 peak) and decode tokens/s, 1 GPU"
WORKLOAD = "opt13b_batch64"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
# Per workload: the committed ncu DRAM-traffic capture of its decode kernel and
# the sources that kernel is built from (the capture counts only while they
# are unchanged).
TRAFFIC = {
    "opt13b_batch64": (
        os.path.join(ROOT, "profiles", "paged_decode_opt13b_batch64_traffic.json"),
        ["paged_kv_cache_326_b200/csrc/paged_attn_decode.cu",
         "paged_kv_cache_326_b200/csrc/decode_common.cuh",
         "paged_kv_cache_326_b200/csrc/ptx.cuh", "paged_kv_cache_326_b200/csrc/dtype.cuh"]),
    "llama2_70b_gqa": (
        os.path.join(ROOT, "profiles", "paged_decode_mma_llama2_70b_gqa_traffic.json"),
        ["paged_kv_cache_326_b200/csrc/paged_attn_decode_mma.cu",
         "paged_kv_cache_326_b200/csrc/decode_common.cuh",
         "paged_kv_cache_326_b200/csrc/mma_ptx.cuh",
         "paged_kv_cache_326_b200/csrc/ptx.cuh", "paged_kv_cache_326_b200/csrc/dtype.cuh"]),
    "opt13b_batch64_fp8": (
        os.path.join(ROOT, "profiles", "paged_decode_fp8_opt13b_batch64_traffic.json"),
        ["paged_kv_cache_326_b200/csrc/paged_attn_decode_mma_fp8.cu",
         "paged_kv_cache_326_b200/csrc/decode_common.cuh",
         "paged_kv_cache_326_b200/csrc/fp8.cuh", "paged_kv_cache_326_b200/csrc/mma_ptx.cuh",
         "paged_kv_cache_326_b200/csrc/ptx.cuh", "paged_kv_cache_326_b200/csrc/dtype.cuh"]),
    "llama2_70b_gqa_fp8": (
        os.path.join(ROOT, "profiles", "paged_decode_mma_fp8_llama2_70b_gqa_fp8_traffic.json"),
        ["paged_kv_cache_326_b200/csrc/paged_attn_decode_mma_fp8.cu",
         "paged_kv_cache_326_b200/csrc/decode_common.cuh",
         "paged_kv_cache_326_b200/csrc/fp8.cuh", "paged_kv_cache_326_b200/csrc/mma_ptx.cuh",
         "paged_kv_cache_326_b200/csrc/ptx.cuh", "paged_kv_cache_326_b200/csrc/dtype.cuh"]),
    # the shared-prefix call: prefix pass + tail pass + merge, summed
    "shared_prefix": (
        os.path.join(ROOT, "profiles", "paged_decode_shared_prefix_c4_traffic.json"),
        ["paged_kv_cache_326_b200/csrc/shared_prefix.cu",
         "paged_kv_cache_326_b200/csrc/paged_attn_decode.cu",
         "paged_kv_cache_326_b200/csrc/paged_attn_decode_mma.cu",
         "paged_kv_cache_326_b200/csrc/decode_common.cuh",
         "paged_kv_cache_326_b200/csrc/mma_ptx.cuh",
         "paged_kv_cache_326_b200/csrc/ptx.cuh", "paged_kv_cache_326_b200/csrc/dtype.cuh"]),
}


def kernel_source_hash(workload: str) -> str:
    h = hashlib.sha256()
    for rel in TRAFFIC[workload][1]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs: copy, burst)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, an earlier copy measurement on B200)"


def traffic_per_launch(workload: str, path: str):
    """DRAM bytes per launch of the decode kernel from the committed ncu
    capture, if it was taken on this path and on the kernel as it is now;
    else None."""
    try:
        with open(TRAFFIC[workload][0]) as f:
            t = json.load(f)
        if t.get("kernel_source_hash") == kernel_source_hash(workload) and t.get("path") == path:
            return float(t["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max((num(r[3]) or 0) for r in rows)}


class StagedInputs:
    """A step's input tensors packed into one pinned host buffer (each piece
    256-byte aligned) and ``copies`` device buffers of the same layout, so a
    step moves all its inputs with one host-to-device copy."""

    def __init__(self, tensors, dev, copies: int = 2):
        offs, total = [], 0
        for t in tensors:
            total = -(-total // 256) * 256
            offs.append(total)
            total += t.numel() * t.element_size()
        self.nbytes = total
        self.host = torch.empty(total, dtype=torch.uint8).pin_memory()
        self.dev = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(copies)]

        def views(buf):
            return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                    for t, o in zip(tensors, offs)]
        for hv, t in zip(views(self.host), tensors):
            hv.copy_(t.cpu())
        self.views = [views(d) for d in self.dev]


def e2e_pipelined(run, staged: StagedInputs, outs, houts, steps: int, stream, copy_stream):
    """Time ``steps`` end-to-end steps on the device.  Step i: the copy stream
    uploads the inputs into device buffer i % 2 (once step i - 2 is done with
    it), the compute stream runs ``run(inputs, out)`` on it, and a second copy
    stream reads that step's output back into pinned host memory.  Uploads
    and readbacks have streams of their own, so step i + 1's upload does not
    queue behind step i's readback (which waits for step i's kernels): one
    step's copies overlap the neighbouring steps' kernels.  Returns ms/step."""
    n = len(staged.dev)
    read_stream = torch.cuda.Stream(device=stream.device)
    in_ready = [torch.cuda.Event() for _ in range(n)]
    computed = [torch.cuda.Event() for _ in range(n)]
    drained = [torch.cuda.Event() for _ in range(n)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    copy_stream.wait_stream(stream)
    read_stream.wait_stream(stream)
    for i in range(steps):
        b = i % n
        with torch.cuda.stream(copy_stream):
            if i >= n:
                copy_stream.wait_event(computed[b])
            staged.dev[b].copy_(staged.host, non_blocking=True)
            in_ready[b].record(copy_stream)
        stream.wait_event(in_ready[b])
        if i >= n:
            stream.wait_event(drained[b])
        run(staged.views[b], outs[b])
        computed[b].record(stream)
        with torch.cuda.stream(read_stream):
            read_stream.wait_event(computed[b])
            houts[b].copy_(outs[b], non_blocking=True)
            drained[b].record(read_stream)
    stream.wait_stream(copy_stream)
    stream.wait_stream(read_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def kv_bytes(context_lens, num_heads, head_dim, elem_bytes) -> int:
    from paged_kv_cache_326_b200.accounting import decode_kv_bytes
    return decode_kv_bytes(context_lens, num_heads, head_dim, elem_bytes)


def oracle_runner(w, num_pairs):
    """The oracle over the first ``num_pairs`` (text, head) pairs of the
    workload, in text-major order.  Inputs are prepared outside the timed
    region.  Returns (run, kv_bytes_of_the_sample)."""
    from threadpoolctl import threadpool_limits
    from tests.gpu_helpers import oracle_inputs, run_oracle, run_oracle_fp8
    H = w.num_heads
    pairs = [(p // H, p % H) for p in range(num_pairs)]
    seqs = sorted({s for s, _ in pairs})
    oi = oracle_inputs(w.q, w.k, w.v, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                       w.slot_mapping, w.block_size, seqs)
    lens = w.context_lens.tolist()
    full = num_pairs == len(seqs) * H
    # bytes of the KV cache the sample covers (each key/value head once)
    Hkv = w.k_cache.shape[1]
    cb = w.k_cache.element_size()
    if full:
        sample_bytes = sum(lens[s] for s in seqs) * 2 * Hkv * w.head_dim * cb
    else:
        sample_bytes = sum(lens[s] for s, _ in pairs) * 2 * w.head_dim * cb

    fp8 = w.k_cache.dtype == torch.uint8

    def run():
        with threadpool_limits(limits=1):
            if fp8:
                run_oracle_fp8(oi, w.scale, w.block_size, w.meta["k_scale"], w.meta["v_scale"],
                               None if full else pairs)
            else:
                run_oracle(oi, w.scale, w.block_size, None if full else pairs)
    return run, sample_bytes


def cpu_baseline(w, budget_s=12.0):
    """The oracle as it stands, on the host, over the whole batch, repeated
    until ``budget_s`` seconds of work (at least once)."""
    run, sample_bytes = oracle_runner(w, w.num_seqs * w.num_heads)
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 20:
            break
    return {"value": sample_bytes * reps / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"all {w.num_seqs} texts x {w.num_heads} query heads of the step ({w.name}), "
                      f"{reps} run(s), {el:.1f} s, numpy fp64, BLAS limited to 1 thread"}


def host_cores() -> dict:
    """What the host offers the oracle: usable cores, all cores, BLAS threads."""
    try:
        aff = len(os.sched_getaffinity(0))
    except Exception:
        aff = os.cpu_count() or 1
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()
                    if i.get("user_api") == "blas"), default=None)
    except Exception:
        blas = None
    return {"affinity_cores": aff, "cpu_count": os.cpu_count(), "blas_threads_default": blas}


def cpu_baseline_pool(w, budget_s=10.0, max_workers=128):
    """The oracle over the whole step, spread over the host's cores: one
    worker process per usable core (``python -m tests.oracle_pool_worker``,
    numpy and the oracle only, BLAS limited to one thread each).  The
    (text, head) pairs, in text-major order, are cut into one contiguous run
    per worker with about equal token counts; each worker holds the pool
    blocks of its texts and runs the cache write and its pairs.  A run is
    timed from the moment all workers are told to start until the last one
    is done; runs repeat until ``budget_s`` seconds have passed."""
    import pickle
    import threading

    from tests.gpu_helpers import oracle_inputs
    cores = host_cores()
    S, H = w.num_seqs, w.num_heads
    n = max(1, min(cores["affinity_cores"], max_workers, S * H))
    lens = w.context_lens.tolist()
    cost = [lens[s] for s in range(S) for _ in range(H)]
    total = sum(cost)
    cuts, acc = [0], 0
    for i, c in enumerate(cost):
        acc += c
        if len(cuts) < n and acc >= total * len(cuts) / n:
            cuts.append(i + 1)
    cuts.append(S * H)
    cuts = sorted(set(cuts))
    fp8 = w.k_cache.dtype == torch.uint8
    shares = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        pairs = [(p // H, p % H) for p in range(a, b)]
        seqs = sorted({s for s, _ in pairs})
        oi = oracle_inputs(w.q, w.k, w.v, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                           w.slot_mapping, w.block_size, seqs)
        pos = {s: i for i, s in enumerate(seqs)}
        shares.append({"q": oi.q, "k": oi.k, "v": oi.v, "k_cache": oi.k_cache,
                       "v_cache": oi.v_cache, "tables": oi.tables, "lens": oi.lens,
                       "slots": oi.slots, "scale": w.scale, "block_size": w.block_size,
                       "pairs": [(pos[s], h) for s, h in pairs],
                       "fp8": (w.meta["k_scale"], w.meta["v_scale"]) if fp8 else None})
    env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    procs = [subprocess.Popen([sys.executable, "-m", "tests.oracle_pool_worker"], cwd=ROOT,
                              env=env, stdin=subprocess.PIPE, stdout=subprocess.PIPE)
             for _ in shares]
    try:
        def send(p, x):
            pickle.dump(x, p.stdin, protocol=5)
            p.stdin.flush()
        ths = [threading.Thread(target=send, args=(p, x)) for p, x in zip(procs, shares)]
        for t in ths:
            t.start()
        for t in ths:
            t.join()
        del shares
        for p in procs:
            if p.stdout.readline().strip() != b"ready":
                raise RuntimeError("oracle worker failed to start")
        reps, spent = 0, 0.0
        while True:
            t0 = time.perf_counter()
            for p in procs:
                p.stdin.write(b"run\n")
                p.stdin.flush()
            for p in procs:
                if p.stdout.readline().strip() != b"done":
                    raise RuntimeError("oracle worker failed")
            spent += time.perf_counter() - t0
            reps += 1
            if spent >= budget_s or reps >= 200:
                break
    finally:
        for p in procs:
            try:
                p.stdin.write(b"quit\n")
                p.stdin.close()
            except Exception:
                pass
        for p in procs:
            try:
                p.wait(timeout=30)
            except Exception:
                p.kill()
    Hkv = w.k_cache.shape[1]
    step_bytes = sum(lens) * 2 * Hkv * w.head_dim * w.k_cache.element_size()
    return {"value": step_bytes * reps / spent / 1e9, "unit": "GB/s", "cores": len(procs),
            "kind": "oracle",
            "sample": f"all {S} texts x {H} query heads of the step ({w.name}) over "
                      f"{len(procs)} worker processes (one per usable core, contiguous runs of "
                      f"(text, head) pairs of about equal tokens), {reps} run(s), {spent:.1f} s, "
                      f"numpy fp64, BLAS limited to 1 thread per worker",
            **cores}


def time_call(fn, stream, reps=20, warm=3, flush=None):
    """Median and minimum device time (ms) of ``fn`` over ``reps`` calls after
    ``warm`` untimed ones, each bracketed by CUDA events on ``stream``;
    ``flush`` (if given) runs before each timed call, outside its events."""
    for _ in range(warm):
        fn()
    marks = []
    for _ in range(reps):
        if flush is not None:
            flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        marks.append((e0, e1))
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in marks]
    return statistics.median(ms), min(ms)


def oracle_check(w, out, seqs):
    """CPU-baseline leg of one configuration: the oracle (one core, fp64) over
    every head of the chosen texts, timed, and the GPU's outputs for them
    compared with its result (max-abs, max-rel over |ref| >= 0.2, and the
    tests' pass/fail rule)."""
    from threadpoolctl import threadpool_limits
    from tests.gpu_helpers import compare, oracle_inputs, run_oracle
    seqs = [int(s) for s in seqs]
    oi = oracle_inputs(w.q, w.k, w.v, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                       w.slot_mapping, w.block_size, seqs)
    t0 = time.perf_counter()
    with threadpool_limits(limits=1):
        ref = run_oracle(oi, w.scale, w.block_size)
    el = time.perf_counter() - t0
    c = compare(out.index_select(0, torch.as_tensor(seqs, device=out.device)), ref, w.q.dtype)
    lens = w.context_lens.tolist()
    kv = sum(lens[s] for s in seqs) * 2 * w.k_cache.shape[1] * w.head_dim * w.k_cache.element_size()
    return ({"max_abs": c.max_abs, "max_rel": c.max_rel, "ok": c.ok,
             "outputs_checked": len(seqs) * w.num_heads, "texts_checked": len(seqs)},
            {"value": kv / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
             "sample": f"{len(seqs)} seeded texts x {w.num_heads} heads, one run, {el:.2f} s"})


def sample_texts(w, n, seed):
    """n seeded texts of the batch, the longest one always among them (sorted)."""
    import numpy as np
    lens = w.context_lens.tolist()
    longest = max(range(len(lens)), key=lambda s: lens[s])
    rest = [s for s in range(len(lens)) if s != longest]
    rng = np.random.default_rng(seed)
    pick = rng.choice(len(rest), min(n - 1, len(rest)), replace=False)
    return sorted([longest] + [rest[int(i)] for i in pick])


def decode_step_config(P, w, stream, peak, flush=None):
    """pa_decode_step (write + attention, one launch, plus the merge kernel)
    on one workload: the call's device time and rates."""
    S, H, D = w.q.shape
    Hkv = w.k_cache.shape[1]
    eb = w.q.element_size()
    lens = w.context_lens.tolist()
    kv = kv_bytes(lens, Hkv, D, eb)
    nbytes = (kv + 2 * S * H * D * eb + sum(4 * -(-L // w.block_size) for L in lens) + 4 * S +
              2 * S * Hkv * D * 2 * eb + 8 * S)
    out = torch.empty_like(w.q)
    ws = P.binding.workspace_for(w.q, w.block_size, w.max_blocks_per_seq)
    status = torch.zeros(1, dtype=torch.int32, device=w.q.device)

    def fn():
        P.pa_decode_step(out, w.q, w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping,
                         w.block_tables, w.context_lens, w.scale, workspace=ws, status=status)
    med, mn = time_call(fn, stream, flush=flush)
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}")
    gbs = nbytes / (med * 1e-3) / 1e9
    return {"path": "pa_decode_step", "call_ms": med, "call_ms_min": mn,
            "algorithmic_bytes": nbytes, "kv_bytes": kv, "gbs": gbs,
            "kv_gbs": kv / (med * 1e-3) / 1e9, "frac_of_peak": gbs / peak,
            "decode_tokens_per_s": S / (med * 1e-3)}, out


def full_step_config(P, W, dev, stream, peak, with_oracle):
    """The 40-layer step (pa_decode_step per layer over one 42.9 GB pool).
    With the oracle: every head of 4 seeded texts at layers 0 and 39, from the
    first step on the initial pool (the oracle replays every layer's writes
    into the blocks those texts read, in layer order)."""
    import numpy as np
    fs = W.full_step(device=dev)
    S, H, D = fs.q[0].shape
    B, L = fs.block_size, fs.num_layers
    check_layers = [0, L - 1]
    seqs = np.sort(np.random.default_rng(5).choice(S, 4, replace=False))
    if with_oracle:
        sel = torch.as_tensor(seqs, device=dev)
        need = torch.unique(torch.cat([fs.block_tables[l].index_select(0, sel).flatten()
                                       for l in check_layers]))
        need = need[need >= 0]
        remap = torch.full((fs.k_cache.shape[0],), -1, dtype=torch.int64, device=dev)
        remap[need] = torch.arange(need.numel(), device=dev)
        kc = fs.k_cache.index_select(0, need).float().cpu().numpy()
        vc = fs.v_cache.index_select(0, need).float().cpu().numpy()
    out = torch.empty_like(fs.q[0])
    ws = P.binding.workspace_for(fs.q[0], B, fs.block_tables[0].shape[1])
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    kept = {}

    def step(keep=False):
        for layer in range(L):
            o = torch.empty_like(out) if keep and layer in check_layers else out
            P.pa_decode_step(o, fs.q[layer], fs.k[layer], fs.v[layer], fs.k_cache, fs.v_cache,
                             fs.slot_mapping[layer], fs.block_tables[layer], fs.context_lens,
                             fs.scale, workspace=ws, status=status)
            if keep and layer in check_layers:
                kept[layer] = o
    step(keep=True)
    med, mn = time_call(step, stream, reps=5, warm=2)
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}")
    lens = fs.context_lens.tolist()
    layer_kv = kv_bytes(lens, H, D, 2)
    per_layer = (layer_kv + 2 * S * H * D * 2 + 4 * S * H * D * 2 +
                 sum(4 * -(-x // B) for x in lens) + 12 * S)
    gbs = per_layer * L / (med * 1e-3) / 1e9
    rec = {"path": "pa_decode_step x 40 layers", "step_ms": med, "step_ms_min": mn,
           "call_ms": med / L, "algorithmic_bytes_per_layer": per_layer,
           "kv_bytes_per_step": layer_kv * L, "gbs": gbs,
           "kv_gbs": layer_kv * L / (med * 1e-3) / 1e9, "frac_of_peak": gbs / peak,
           "decode_tokens_per_s": S / (med * 1e-3),
           "pool": "one 131,072-block pool (42.9 GB) shared by the 40 layers, tables drawn "
                   "per layer, so blocks alias across layers"}
    if with_oracle:
        from threadpoolctl import threadpool_limits

        import oracle
        from tests.gpu_helpers import compare
        worst = {"max_abs": 0.0, "max_rel": 0.0, "ok": True, "outputs_checked": 0,
                 "texts_checked": len(seqs), "layers_checked": check_layers}
        t0 = time.perf_counter()
        done = 0
        with threadpool_limits(limits=1):
            for layer in check_layers:
                # the writes of the layers since the last check, in layer order
                ks, vs, slots = [], [], []
                for l2 in range(done, layer + 1):
                    sl = fs.slot_mapping[l2]
                    nb = remap[(sl // B).clamp(min=0)]
                    idx = torch.nonzero((sl >= 0) & (nb >= 0)).flatten()
                    ks.append(fs.k[l2].index_select(0, idx).float().cpu().numpy())
                    vs.append(fs.v[l2].index_select(0, idx).float().cpu().numpy())
                    slots.append((nb[idx] * B + sl[idx] % B).cpu().numpy())
                kc, vc = oracle.cache_write(kc, vc, np.concatenate(ks), np.concatenate(vs),
                                            np.concatenate(slots), B)
                done = layer + 1
                t = fs.block_tables[layer].index_select(0, sel).to(torch.int64)
                t = torch.where(t >= 0, remap[t.clamp(min=0)], torch.full_like(t, -1)).cpu().numpy()
                q = fs.q[layer].index_select(0, sel).float().cpu().numpy()
                ref = oracle.paged_decode(q, kc, vc, t,
                                          fs.context_lens.index_select(0, sel).cpu().numpy(),
                                          fs.scale, B)
                c = compare(kept[layer].index_select(0, sel), ref, torch.float16)
                worst["max_abs"] = max(worst["max_abs"], c.max_abs)
                worst["max_rel"] = max(worst["max_rel"], c.max_rel)
                worst["ok"] = worst["ok"] and c.ok
                worst["outputs_checked"] += len(seqs) * H
        el = time.perf_counter() - t0
        rec["parity"] = worst
        rec["cpu_baseline"] = {
            "value": sum(lens[s] for s in seqs) * 2 * H * D * 2 * len(check_layers) / el / 1e9,
            "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(seqs)} texts x {H} heads at layers {check_layers} with every "
                      f"layer's writes replayed, {el:.1f} s"}
    del fs
    torch.cuda.empty_cache()
    return rec


def other_configs(P, W, dev, stream, peak, with_oracle=True):
    """The other configurations of the study, each on the path the headline
    uses (or the shared-prefix call for the shared-prefix one): device time of
    the decode call, GB/s, fraction of the HBM peak (the headline's roofline
    peak, named in the line's roofline.peak_source), decode tokens/s, and, in the CPU-baseline leg, parity against the oracle on a
    seeded sample of outputs."""
    res = {}
    # tiny: 108 KB of KV, so L2 is flushed (a 256 MB write) before each call
    w = W.tiny(device=dev)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rec, out = decode_step_config(P, w, stream, peak, flush=lambda: flush_buf.zero_())
    rec["l2"] = "flushed before each call (256 MB write)"
    if with_oracle:
        rec["parity"], rec["cpu_baseline"] = oracle_check(w, out, range(w.num_seqs))
    res["tiny"] = rec
    del w, out, flush_buf
    # skewed lengths, bf16, blocks of 8, 16 and 32
    for B in (8, 16, 32):
        w = W.skewed(block_size=B, device=dev)
        rec, out = decode_step_config(P, w, stream, peak)
        if with_oracle:
            rec["parity"], rec["cpu_baseline"] = oracle_check(w, out, sample_texts(w, 24, 30 + B))
        res[f"skewed_b{B}"] = rec
        del w, out
        torch.cuda.empty_cache()
    # shared prefixes: 32 prompts x 8 samples built by the block manager
    w = shared_prefix_inputs(P, W, 4, dev)
    S, H, D = w.q.shape
    gs = w.meta["samples"]
    lens = w.context_lens.tolist()
    distinct = unique_kv_bytes(w, H, D, 2)
    logical = kv_bytes(lens, H, D, 2)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=status)
    split = P.split_shared_prefix(w.block_tables.cpu(), w.context_lens.cpu(), w.block_size, gs)
    pt, pl, tt, tl = [t.to(dev) for t in split]
    ws_sh = torch.empty(P.pa_paged_attn_decode_shared_workspace_size(
        pt.shape[0], gs, H, D, w.block_size, pt.shape[1], tt.shape[1]), dtype=torch.uint8,
        device=dev)
    out_sh = torch.empty_like(w.q)
    out_pl = torch.empty_like(w.q)
    ws = P.binding.workspace_for(w.q, w.block_size, w.max_blocks_per_seq)
    small = 2 * S * H * D * 2 + 4 * S
    tab_sh = 4 * len(split[1]) + sum(4 * -(-x // w.block_size) for x in split[1].tolist() +
                                     split[3].tolist())
    tab_pl = sum(4 * -(-x // w.block_size) for x in lens)
    for name, fn, out, tab in (
            ("shared_prefix_cascade",
             lambda: P.pa_paged_attn_decode_shared(out_sh, w.q, w.k_cache, w.v_cache, pt, pl, tt,
                                                   tl, w.scale, gs, workspace=ws_sh,
                                                   status=status), out_sh, tab_sh),
            ("shared_prefix_plain",
             lambda: P.pa_paged_attn_decode(out_pl, w.q, w.k_cache, w.v_cache, w.block_tables,
                                            w.context_lens, w.scale, workspace=ws,
                                            status=status), out_pl, tab_pl)):
        med, mn = time_call(fn, stream)
        if status.item() != 0:
            raise RuntimeError(f"device status {status.item()}")
        nbytes = distinct + small + tab
        gbs = nbytes / (med * 1e-3) / 1e9
        rec = {"path": ("pa_paged_attn_decode_shared (split by pa_split_shared_prefix)"
                        if name.endswith("cascade") else
                        "pa_paged_attn_decode over the joined tables"),
               "call_ms": med, "call_ms_min": mn, "algorithmic_bytes": nbytes,
               "distinct_kv_bytes": distinct, "logical_kv_bytes": logical, "gbs": gbs,
               "logical_kv_gbs": logical / (med * 1e-3) / 1e9,
               "frac_of_peak": gbs / peak, "counts": "distinct (block, row) KV bytes",
               "decode_tokens_per_s": S / (med * 1e-3)}
        if with_oracle:
            rec["parity"], rec["cpu_baseline"] = oracle_check(w, out, sample_texts(w, 24, 44))
        res[name] = rec
    del w, out_sh, out_pl, ws_sh, ws
    torch.cuda.empty_cache()
    res["full_step"] = full_step_config(P, W, dev, stream, peak, with_oracle)
    return res


def run_reference(args, world, rank):
    """The oracle timed as the reference arm: each step is the first n
    (text, head) pairs of the batch, n sized so warm-up + timed steps take
    about two minutes in all."""
    from paged_kv_cache_326_b200 import workloads as W
    if rank != 0:
        return 0
    w = W.opt13b_batch64(device="cpu")
    H = w.num_heads
    probe, _ = oracle_runner(w, H)
    t0 = time.perf_counter()
    probe()
    per_pair = (time.perf_counter() - t0) / H
    budget = min(2.0, 120.0 / (args.steps + args.warmup))
    n = int(max(1, min(w.num_seqs * H, budget / max(per_pair, 1e-6))))
    run, sample_bytes = oracle_runner(w, n)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t0
    ms = el / args.steps * 1e3
    value = sample_bytes / (el / args.steps) / 1e9
    desc = (f"first {n} (text, head) pairs of the {w.num_seqs}x{H} batch per step, "
            f"numpy fp64, 1 BLAS thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample": desc},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return (float(json.load(f)["bf16_tflops"]),
                    "measured (MEASURED_PEAKS.json bf16_tflops: cuBLAS dense, burst; fp16 runs "
                    "at the same tensor rate)")
    except Exception:
        return 1590.0, "fallback (1.59 PFLOP/s, an earlier cuBLAS bf16 measurement on B200)"


def run_prefill_bench(args, ranks, world, rank, local):
    """The prompt phase: 16 prompts of 2,048 tokens x 40 heads x 128, fp16 --
    each step stores the prompts' keys and values in their blocks and runs
    causal attention (pa_prefill)."""
    import paged_kv_cache_326_b200 as P
    from paged_kv_cache_326_b200 import dist, workloads as W
    P.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    w = W.opt13b_prefill(seed=dist.batch_seed(7, ranks), device=dev)
    T, H, D = w.q.shape
    flops = 4.0 * D * H * sum(L * (L + 1) / 2 for L in w.lens)   # causal QK^T and PV
    out = torch.empty_like(w.q)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        P.pa_prefill(out, w.q, w.k, w.v, w.cu_seqlens, w.max_seqlen, w.scale, w.k_cache,
                     w.v_cache, w.slot_mapping, status=status)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}")
    K = args.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        time.sleep(0.3)
        dist.barrier(ranks)
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(K):
            step()
        stop.record(stream)
        torch.cuda.synchronize()
        dist.barrier(ranks)
    clk = clocks.summary()
    ms_step = start.elapsed_time(stop) / K
    # end to end: q, k, v from pinned host memory, out back to the host
    hq, hk, hv = (t.cpu().pin_memory() for t in (w.q, w.k, w.v))
    hout = torch.empty_like(hq).pin_memory()
    Ke = max(1, K // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(Ke):
        w.q.copy_(hq, non_blocking=True)
        w.k.copy_(hk, non_blocking=True)
        w.v.copy_(hv, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / Ke
    # Prompt time against the reused fraction: the same prompts with their
    # first c tokens already in the cache (stored by the steps above), only
    # the other 2048 - c tokens computed (pa_prefill_with_prefix).
    sweep = []
    L0 = w.lens[0]
    for frac in (0.25, 0.5, 0.75):
        c = int(L0 * frac) // w.block_size * w.block_size
        n = L0 - c
        rows = torch.cat([torch.arange(int(w.cu_seqlens[s]) + c, int(w.cu_seqlens[s + 1]),
                                       device=dev) for s in range(len(w.lens))])
        qn, kn, vn = w.q[rows].contiguous(), w.k[rows].contiguous(), w.v[rows].contiguous()
        sn = w.slot_mapping[rows].contiguous()
        cun = torch.arange(0, (len(w.lens) + 1) * n, n, dtype=torch.int32, device=dev)
        cached = torch.full((len(w.lens),), c, dtype=torch.int32, device=dev)
        outn = torch.empty_like(qn)

        def reuse_step():
            P.pa_prefill_with_prefix(outn, qn, kn, vn, cun, n, w.scale, w.k_cache, w.v_cache,
                                     w.block_tables, cached, sn, status=status)
        med, mn = time_call(reuse_step, stream, reps=max(5, min(K, 20)))
        if status.item() != 0:
            raise RuntimeError(f"device status {status.item()}")
        fl = 4.0 * D * H * len(w.lens) * sum(c + i + 1 for i in range(n))
        sweep.append({"cached_tokens": c, "new_tokens": n, "ms": med, "ms_min": mn,
                      "ms_vs_no_reuse": med / ms_step, "tflops": fl / (med * 1e-3) / 1e12,
                      "new_tokens_per_s": len(w.lens) * n / (med * 1e-3)})
    # the attention without the store of the keys and values, for reference
    def attention_only():
        P.pa_prefill(out, w.q, w.k, w.v, w.cu_seqlens, w.max_seqlen, w.scale, status=status)
    attn_ms, attn_min = time_call(attention_only, stream, reps=max(5, min(K, 20)))
    ms_step, e2e_ms, attn_ms = dist.max_over_ranks(ranks, [ms_step, e2e_ms, attn_ms], dev)
    peak, peak_src = tensor_peak()
    tflops = flops / (ms_step * 1e-3) / 1e12
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    line = {
        "metric": "prefill TFLOP/s (causal attention, 4*D flops per query-key pair)",
        "value": world * tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "accumulate": "f32",
        "data": "synthetic",
        "config": {"workload": "opt13b_prefill", "prompts": len(w.lens), "prompt_len": w.lens[0],
                   "num_heads": H, "head_dim": D, "block_size": w.block_size,
                   "l2": "q, k, v, out 1.3 GB per step >> 126 MB L2",
                   "parallelism": f"independent prompts per GPU x{world}",
                   "path": "pa_prefill (causal attention; two warps of each CTA store the "
                           "prompts' keys and values in the same launch)"},
        "prefill_tokens_per_s": world * T / (ms_step * 1e-3),
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": tflops / peak, "traffic": None,
                     "kernel": "prefill_tc_kernel (tcgen05, TMEM accumulators; the one launch "
                               "of the step)",
                     "peak_source": peak_src, "algorithmic_flops_per_launch": flops},
        "attention_without_store": {"ms": attn_ms, "ms_min": attn_min,
                                    "tflops": attn_tflops},
        "reuse_sweep": sweep,
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": 3 * w.q.numel() * 2, "d2h_bytes_per_step": out.numel() * 2,
                "ms_per_step": e2e_ms},
        "gpu_launches": K,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        # one prompt's first 512 tokens, 4 heads: about ten seconds of host work
        L, Hs = 512, 4
        q = w.q[:L, :Hs].float().cpu().numpy()
        k = w.k[:L, :Hs].float().cpu().numpy()
        v = w.v[:L, :Hs].float().cpu().numpy()
        sample_flops = 4.0 * D * Hs * L * (L + 1) / 2
        reps, t0 = 0, time.perf_counter()
        while True:
            oracle.prefill(q, k, v, [0, L], w.scale)
            reps += 1
            el = time.perf_counter() - t0
            if el >= 10.0 or reps >= 200:
                break
        line["cpu_baseline"] = {
            "value": sample_flops * reps / el / 1e12, "unit": "TFLOP/s", "cores": 1,
            "kind": "oracle",
            "sample": f"one prompt's first {L} tokens x {Hs} heads, {reps} run(s), {el:.1f} s, "
                      f"numpy fp64 (BLAS threads as installed)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def read_probe_gbs(dev, gib: int = 4) -> float:
    """Read-only streaming ceiling of this GPU, measured in the same process:
    the median rate of the library's read probe (pa_read_probe) over a `gib`
    GiB buffer, larger than L2."""
    import paged_kv_cache_326_b200 as P
    buf = torch.empty(gib << 30, dtype=torch.uint8, device=dev)
    buf.fill_(1)
    sink = torch.empty(4096, dtype=torch.int32, device=dev)
    for _ in range(3):
        P.binding.pa_read_probe(buf, sink)
    times = []
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        P.binding.pa_read_probe(buf, sink)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    del buf
    torch.cuda.empty_cache()
    return (gib << 30) / (statistics.median(times) * 1e-3) / 1e9


def shared_prefix_inputs(P, W, seed, dev):
    """The shared-prefix workload built by the C++ block manager (copy-on-write
    copies applied while the samples generate)."""
    bm = P.BlockManager(8192, 16)

    class Adapter:
        add_seq = staticmethod(bm.add_seq)
        fork = staticmethod(bm.fork)
        append_slot = staticmethod(bm.append_slot)

        @staticmethod
        def export(ids, mb):
            t, l = bm.export(ids, mb)
            return t.numpy(), l.numpy()

    return W.shared_prefix(Adapter(), num_blocks=8192, seed=seed, device=dev)


def unique_kv_bytes(w, num_kv_heads, head_dim, elem_bytes) -> int:
    """KV bytes that the texts' reads cover, each stored (block, row) once."""
    import numpy as np
    tables = w.block_tables.cpu().numpy()
    lens = w.context_lens.cpu().numpy()
    B = w.block_size
    rows = {}
    for s in range(tables.shape[0]):
        L = int(lens[s])
        for j in range(-(-L // B)):
            b = int(tables[s, j])
            rows[b] = max(rows.get(b, 0), min(B, L - j * B))
    return sum(rows.values()) * 2 * num_kv_heads * head_dim * elem_bytes


def run_full_step(args, ranks, world, rank, local):
    """The full OPT-13B-shaped decode step: 40 layers x (write + attend) for
    256 texts, one 131,072-block pool (42.9 GB) shared by the layers; each
    layer streams its own ~5.5 GB of KV.  decode tokens/s = texts / step."""
    import paged_kv_cache_326_b200 as P
    from paged_kv_cache_326_b200 import dist, workloads as W
    P.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    fs = W.full_step(seed=dist.batch_seed(5, ranks), device=dev)
    S, H, D = fs.q[0].shape
    lens = fs.context_lens.tolist()
    layer_kv = kv_bytes(lens, H, D, 2)
    step_kv = layer_kv * fs.num_layers
    out = torch.empty_like(fs.q[0])
    ws = P.binding.workspace_for(fs.q[0], fs.block_size, fs.block_tables[0].shape[1])
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        for layer in range(fs.num_layers):
            P.pa_decode_step(out, fs.q[layer], fs.k[layer], fs.v[layer], fs.k_cache, fs.v_cache,
                             fs.slot_mapping[layer], fs.block_tables[layer], fs.context_lens,
                             fs.scale, workspace=ws, status=status)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}")
    K = args.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        time.sleep(0.3)
        dist.barrier(ranks)
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(K):
            step()
        stop.record(stream)
        torch.cuda.synchronize()
        dist.barrier(ranks)
    clk = clocks.summary()
    ms_step = start.elapsed_time(stop) / K
    # end to end: every layer's q, k, v and slots from pinned host memory, every
    # layer's output back to the host
    hq = [t.cpu().pin_memory() for t in fs.q]
    hk = [t.cpu().pin_memory() for t in fs.k]
    hv = [t.cpu().pin_memory() for t in fs.v]
    hs = [t.cpu().pin_memory() for t in fs.slot_mapping]
    hout = torch.empty_like(hq[0]).pin_memory()
    dq, dk, dv, dsl = (torch.empty_like(fs.q[0]), torch.empty_like(fs.k[0]),
                       torch.empty_like(fs.v[0]), torch.empty_like(fs.slot_mapping[0]))
    Ke = max(1, min(K, 10))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        for layer in range(fs.num_layers):
            dq.copy_(hq[layer], non_blocking=True)
            dk.copy_(hk[layer], non_blocking=True)
            dv.copy_(hv[layer], non_blocking=True)
            dsl.copy_(hs[layer], non_blocking=True)
            P.pa_decode_step(out, dq, dk, dv, fs.k_cache, fs.v_cache, dsl,
                             fs.block_tables[layer], fs.context_lens, fs.scale, workspace=ws,
                             status=status)
            hout.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / Ke
    ms_step, e2e_ms = dist.max_over_ranks(ranks, [ms_step, e2e_ms], dev)
    peak, peak_src = hbm_peak()
    per_layer_bytes = (layer_kv + 2 * S * H * D * 2 + 4 * S * H * D * 2 +
                       sum(4 * -(-L // fs.block_size) for L in lens) + 12 * S)
    achieved = per_layer_bytes * fs.num_layers / (ms_step * 1e-3) / 1e9
    h2d = fs.num_layers * sum(t.numel() * t.element_size() for t in (hq[0], hk[0], hv[0], hs[0]))
    d2h = fs.num_layers * hout.numel() * hout.element_size()
    line = {
        "metric": METRIC, "value": world * step_kv / (ms_step * 1e-3) / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "accumulate": "f32", "data": "synthetic",
        "config": {"workload": "full_step", "layers": fs.num_layers, "num_seqs": S,
                   "num_heads": H, "head_dim": D, "block_size": fs.block_size,
                   "context_lens": "uniform [64, 2048], seed 5+rank",
                   "num_blocks": fs.k_cache.shape[0], "kv_bytes_per_step": step_kv,
                   "pool": "one 131,072-block pool shared by the 40 layers (tables drawn per layer)",
                   "l2": "inputs larger than L2 (5.5 GB of KV per layer)",
                   "parallelism": f"independent batch per GPU x{world}",
                   "path": "pa_decode_step per layer"},
        "decode_tokens_per_s": world * S / (ms_step * 1e-3),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "pa_decode_step x 40 layers (decode kernel + merge kernel)",
                     "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": per_layer_bytes},
        "e2e": {"value": world * step_kv / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": 2 * fs.num_layers * K,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_cow_copy(args, ranks, world, rank, local):
    """Copy-on-write bursts: each step copies one burst of 224 whole blocks
    (32 prompts x 7 samples, 40 heads x 16 x 128 fp16, K and V) with
    pa_copy_blocks; bursts rotate over 8 disjoint sets of blocks."""
    import numpy as np
    import paged_kv_cache_326_b200 as P
    from paged_kv_cache_326_b200 import dist, workloads as W
    P.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    kc, vc, bursts = W.cow_bursts(seed=dist.batch_seed(4, ranks), device=dev)
    N, H, B, D = kc.shape
    block_bytes = H * B * D * kc.element_size()
    n = bursts[0].shape[0]
    # Least DRAM traffic a burst needs: each distinct source block read once
    # (its 7 copies share one read), each destination written once; K and V.
    uniq_src = bursts[0][:, 0].unique().numel()
    step_bytes = (uniq_src + n) * 2 * block_bytes
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(i):
        P.pa_copy_blocks(kc, vc, kc, vc, bursts[i % len(bursts)], status=status)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        time.sleep(0.3)
        dist.barrier(ranks)
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(K):
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
        stop.record(stream)
        torch.cuda.synchronize()
        dist.barrier(ranks)
    clk = clocks.summary()
    ms_step = start.elapsed_time(stop) / K
    kernel_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))

    # end to end: each step's pairs uploaded from pinned host memory, the
    # status word read back
    hpairs = [b.cpu().pin_memory() for b in bursts]
    dpairs = torch.empty_like(bursts[0])
    hstat = torch.zeros(1, dtype=torch.int32).pin_memory()
    Ke = max(1, K // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(Ke):
        dpairs.copy_(hpairs[i % len(hpairs)], non_blocking=True)
        P.pa_copy_blocks(kc, vc, kc, vc, dpairs, status=status)
        hstat.copy_(status, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / Ke
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}")
    # The write ceiling for a launch of this size: the write-only probe on
    # the same number of bytes as a burst writes, rotating over as many
    # buffers as there are bursts (so L2 holds the same share of them).
    write_bytes = n * 2 * block_bytes
    wbuf = torch.empty(len(bursts) * write_bytes, dtype=torch.uint8, device=dev)
    wslices = [wbuf[i * write_bytes:(i + 1) * write_bytes] for i in range(len(bursts))]
    for i in range(3):
        P.binding.pa_write_probe(wslices[i % len(wslices)])
    wev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(max(K, 20))]
    for i, (e0, e1) in enumerate(wev):
        e0.record(stream)
        P.binding.pa_write_probe(wslices[i % len(wslices)])
        e1.record(stream)
    torch.cuda.synchronize()
    probe_ms = statistics.median(a.elapsed_time(b) for a, b in wev)
    del wbuf, wslices
    ms_step, e2e_ms, kernel_ms, probe_ms = dist.max_over_ranks(
        ranks, [ms_step, e2e_ms, kernel_ms, probe_ms], dev)
    peak, peak_src = hbm_peak()
    achieved = step_bytes / (kernel_ms * 1e-3) / 1e9
    write_gbs = write_bytes / (kernel_ms * 1e-3) / 1e9
    probe_gbs = write_bytes / (probe_ms * 1e-3) / 1e9
    line = {
        "metric": "paged block copy GB/s (distinct blocks read + blocks written)",
        "value": world * step_bytes / (ms_step * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": "cow_copy", "pairs_per_step": n, "num_heads": H,
                   "block_size": B, "head_dim": D, "block_bytes": block_bytes,
                   "num_blocks": N, "bursts": len(bursts),
                   "l2": f"{len(bursts)} disjoint bursts in rotation "
                         f"({len(bursts) * step_bytes / 1e9:.2f} GB of blocks >> 126 MB L2)",
                   "parallelism": f"independent pool per GPU x{world}"},
        "kernel_ms": {"copy_blocks": kernel_ms},
        "write_ceiling": {"probe_ms": probe_ms, "probe_gbs": probe_gbs,
                          "copy_write_gbs": write_gbs, "frac": write_gbs / probe_gbs,
                          "how": f"pa_write_probe over {write_bytes} bytes (a burst's "
                                 f"destination blocks), {len(bursts)} buffers in rotation, "
                                 "median launch"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None, "kernel": "copy_blocks_kernel",
                     "peak_source": peak_src, "algorithmic_bytes_per_launch": step_bytes},
        "e2e": {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": dpairs.numel() * 4, "d2h_bytes_per_step": 4,
                "ms_per_step": e2e_ms},
        "gpu_launches": K,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        pairs = bursts[0].cpu().numpy()
        used = np.unique(pairs)
        remap = {int(b): i for i, b in enumerate(used)}
        local_pairs = [(remap[int(a)], remap[int(b)]) for a, b in pairs]
        sk = kc[torch.as_tensor(used, device=dev)].cpu().numpy()
        sv = vc[torch.as_tensor(used, device=dev)].cpu().numpy()
        reps, t0 = 0, time.perf_counter()
        while True:
            oracle.copy_blocks(sk, sv, sk, sv, local_pairs)
            reps += 1
            el = time.perf_counter() - t0
            if el >= 10.0 or reps >= 200:
                break
        line["cpu_baseline"] = {
            "value": step_bytes * reps / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"burst 0 ({n} pairs) on a host pool of the {len(used)} blocks it names, "
                      f"{reps} run(s), {el:.1f} s, numpy"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the tiny, skewed, shared-prefix and 40-layer configurations that "
                         "the default run reports under other_configs")
    ap.add_argument("--path", choices=["fused", "calls"], default=None,
                    help="fused: one launch stores the new tokens and attends "
                         "(pa_decode_step, pa_decode_step_fp8; multi-head pools); calls: the "
                         "write, then the decode (default for the 8-bit and grouped-query "
                         "workloads)")
    ap.add_argument("--kv-dtype", choices=["f16", "fp8"], default="f16",
                    help="fp8: the step over 8-bit E4M3 caches (batch-64 OPT-13B, or with "
                         "--workload llama2_70b_gqa the grouped-query step)")
    ap.add_argument("--shared-path", choices=["cascade", "plain"], default="cascade",
                    help="shared_prefix workload: pa_paged_attn_decode_shared over the split "
                         "tables (cascade) or pa_paged_attn_decode over the joined ones (plain)")
    ap.add_argument("--gqa-kernel", choices=["auto", "cores", "tensor"], default="auto",
                    help="grouped-query workload: kernel choice (PA_OPT_GQA_KERNEL)")
    ap.add_argument("--workload", choices=["opt13b_batch64", "llama2_70b_gqa", "cow_copy",
                                           "prefill", "skewed", "shared_prefix", "full_step"],
                    default="opt13b_batch64",
                    help="llama2_70b_gqa: 64 query heads on 8 key/value heads (two calls); "
                         "cow_copy: copy-on-write bursts of whole blocks (pa_copy_blocks); "
                         "prefill: the prompt phase of 16 prompts of 2,048 tokens (pa_prefill); "
                         "skewed: 256 texts, lognormal lengths, bf16; shared_prefix: 32 prompts "
                         "x 8 samples built by the block manager; full_step: 40 layers x 256 "
                         "texts over one 42.9 GB pool")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    from paged_kv_cache_326_b200 import dist
    ranks = dist.init("gloo" if args.impl == "reference" else "nccl")
    world, rank, local = ranks.world, ranks.rank, ranks.local
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        dist.finish(ranks)
        return rc

    if args.workload == "cow_copy":
        rc = run_cow_copy(args, ranks, world, rank, local)
        dist.finish(ranks)
        return rc
    if args.workload == "prefill":
        rc = run_prefill_bench(args, ranks, world, rank, local)
        dist.finish(ranks)
        return rc
    if args.workload == "full_step":
        rc = run_full_step(args, ranks, world, rank, local)
        dist.finish(ranks)
        return rc

    import paged_kv_cache_326_b200 as P
    from paged_kv_cache_326_b200 import workloads as W
    P.lib()   # fails loudly if the library was not built
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    gqa = args.workload == "llama2_70b_gqa"
    P.pa_set_option(P.PA_OPT_GQA_KERNEL, {"auto": 0, "cores": 1, "tensor": 2}[args.gqa_kernel])
    gqa_kernel = "CUDA-core" if args.gqa_kernel == "cores" else "tensor-core"
    fp8 = args.kv_dtype == "fp8"
    if args.path is None:
        args.path = "calls" if (gqa or fp8) else "fused"
    if gqa:
        args.path = "calls"   # the one-launch step is multi-head only
        w = (W.llama2_70b_gqa_fp8 if fp8 else W.llama2_70b_gqa)(
            seed=dist.batch_seed(6, ranks), device=dev)
    elif fp8:
        w = W.opt13b_batch64_fp8(seed=dist.batch_seed(2, ranks), device=dev)
    elif args.workload == "skewed":
        w = W.skewed(seed=dist.batch_seed(3, ranks), device=dev)
    elif args.workload == "shared_prefix":
        w = shared_prefix_inputs(P, W, dist.batch_seed(4, ranks), dev)
    else:
        w = W.opt13b_batch64(seed=dist.batch_seed(2, ranks), device=dev)
    S, H, D = w.q.shape
    Hkv = w.k_cache.shape[1]
    eb = w.q.element_size()
    cb = w.k_cache.element_size()                 # cache bytes per number (1 for 8-bit)
    lens = w.context_lens.tolist()
    step_kv = kv_bytes(lens, Hkv, D, cb)
    logical_kv = step_kv
    if args.workload == "shared_prefix":
        # texts share their prompt's blocks: count each stored row once
        step_kv = unique_kv_bytes(w, Hkv, D, cb)
    decode_bytes = step_kv + 2 * S * H * D * eb + sum(4 * -(-L // w.block_size) for L in lens) + 4 * S
    write_bytes = 2 * S * Hkv * D * (eb + cb) + 8 * S   # k, v read and stored; slots
    cascade = args.workload == "shared_prefix" and args.shared_path == "cascade"
    if cascade:
        # the host splits the exported tables once per step, as it exports
        # them: a prefix per prompt, a tail per sample
        args.path = "calls"
        gs = w.meta["samples"]
        split = P.split_shared_prefix(w.block_tables.cpu(), w.context_lens.cpu(), w.block_size, gs)
        split_d = [t.to(dev) for t in split]
        pl, tl = split[1].tolist(), split[3].tolist()
        decode_bytes = (step_kv + 2 * S * H * D * eb + 4 * S + 4 * len(pl) +
                        sum(4 * -(-L // w.block_size) for L in pl + tl))
    fused = args.path == "fused"
    if fused:
        decode_bytes += write_bytes
    out0 = torch.empty_like(w.q)
    ws = P.binding.workspace_for(w.q, w.block_size, w.max_blocks_per_seq, Hkv)
    if cascade:
        ws_shared = torch.empty(P.pa_paged_attn_decode_shared_workspace_size(
            len(pl), gs, H, D, w.block_size, split[0].shape[1], split[2].shape[1]),
            dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def write_part(k, v, slots):
        if fused:
            return
        if fp8:
            P.pa_kv_cache_write_fp8(k, v, w.k_cache, w.v_cache, slots, w.meta["k_scale"],
                                    w.meta["v_scale"], status=status)
        elif not fused:
            P.pa_kv_cache_write(k, v, w.k_cache, w.v_cache, slots, status=status)

    def decode_part(q, k, v, slots, tables, lens, shared_tables=None, out_=None):
        out = out_ if out_ is not None else out0
        if cascade:
            pt, pl_d, tt, tl_d = shared_tables if shared_tables is not None else split_d
            P.pa_paged_attn_decode_shared(out, q, w.k_cache, w.v_cache, pt, pl_d, tt, tl_d,
                                          w.scale, gs, workspace=ws_shared, status=status)
        elif fused and fp8:
            P.pa_decode_step_fp8(out, q, k, v, w.k_cache, w.v_cache, slots, tables, lens,
                                 w.scale, w.meta["k_scale"], w.meta["v_scale"], workspace=ws,
                                 status=status)
        elif fused:
            P.pa_decode_step(out, q, k, v, w.k_cache, w.v_cache, slots, tables, lens, w.scale,
                             workspace=ws, status=status)
        elif gqa and fp8:
            P.pa_paged_attn_decode_fp8(out, q, w.k_cache, w.v_cache, tables, lens, w.scale,
                                       w.meta["k_scale"], w.meta["v_scale"], workspace=ws,
                                       status=status)
        elif gqa:
            P.pa_paged_attn_decode_gqa(out, q, w.k_cache, w.v_cache, tables, lens, w.scale,
                                       workspace=ws, status=status)
        elif fp8:
            P.pa_paged_attn_decode_fp8(out, q, w.k_cache, w.v_cache, tables, lens, w.scale,
                                       w.meta["k_scale"], w.meta["v_scale"], workspace=ws,
                                       status=status)
        else:
            P.pa_paged_attn_decode(out, q, w.k_cache, w.v_cache, tables, lens, w.scale,
                                   workspace=ws, status=status)

    def step():
        write_part(w.k, w.v, w.slot_mapping)
        decode_part(w.q, w.k, w.v, w.slot_mapping, w.block_tables, w.context_lens)

    def barrier():
        dist.barrier(ranks)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}: {P.pa_status_string(status.item())}")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        time.sleep(0.3)
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(K):
            ev[i][0].record(stream)
            write_part(w.k, w.v, w.slot_mapping)
            ev[i][1].record(stream)
            decode_part(w.q, w.k, w.v, w.slot_mapping, w.block_tables, w.context_lens)
            ev[i][2].record(stream)
        stop.record(stream)
        torch.cuda.synchronize()
        barrier()
    clk = clocks.summary()
    total_ms = start.elapsed_time(stop)
    decode_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(K))
    write_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))

    # end to end: each step's inputs from pinned host memory (one packed copy),
    # its output back to pinned host memory, copies overlapped with the
    # neighbouring steps' kernels on a second stream
    if cascade:   # the split tables stand in for the joined ones
        inputs = [w.q, w.k, w.v, w.slot_mapping, *split_d]
    else:
        inputs = [w.q, w.k, w.v, w.slot_mapping, w.block_tables, w.context_lens]
    staged = StagedInputs(inputs, dev)
    outs = [torch.empty_like(w.q) for _ in staged.dev]
    houts = [torch.empty(w.q.shape, dtype=w.q.dtype).pin_memory() for _ in staged.dev]
    h2d = staged.nbytes
    d2h = outs[0].numel() * outs[0].element_size()

    def e2e_run(x, o):
        if cascade:
            q, k, v, slots, pt, pl_d, tt, tl_d = x
            write_part(k, v, slots)
            decode_part(q, k, v, slots, None, None, shared_tables=(pt, pl_d, tt, tl_d), out_=o)
        else:
            q, k, v, slots, tables, lens = x
            write_part(k, v, slots)
            decode_part(q, k, v, slots, tables, lens, out_=o)

    copy_stream = torch.cuda.Stream(dev)
    Ke = max(3, min(K, 1000))
    e2e_pipelined(e2e_run, staged, outs, houts, 3, stream, copy_stream)
    barrier()
    e2e_ms = e2e_pipelined(e2e_run, staged, outs, houts, Ke, stream, copy_stream)
    barrier()
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}: {P.pa_status_string(status.item())}")

    ms_step = total_ms / K
    ms_step, e2e_ms, decode_ms = dist.max_over_ranks(ranks, [ms_step, e2e_ms, decode_ms], dev)

    peak, peak_src = hbm_peak()
    achieved = decode_bytes / (decode_ms * 1e-3) / 1e9
    value = world * step_kv / (ms_step * 1e-3) / 1e9
    probe_gbs = read_probe_gbs(dev)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.q.dtype == torch.bfloat16 else "f16", "accumulate": "f32",
        "data": "synthetic",
        "config": {"workload": args.workload + ("_fp8" if fp8 else ""), "num_seqs": S,
                   "num_heads": H,
                   "kv_cache": ("e4m3, per-tensor scales k %g, v %g" %
                                (w.meta["k_scale"], w.meta["v_scale"]) if fp8 else "f16"),
                   "num_kv_heads": Hkv, "head_dim": D, "block_size": w.block_size,
                   "context_lens": ("uniform [128, 4096], seed 6+rank" if gqa else
                                    "lognormal (median 300, sigma 1.0) clipped [16, 2048], 8 at "
                                    "2,048, seed 3+rank" if args.workload == "skewed" else
                                    "prompts U[256, 1024] x 8 samples, generated U[1, 256], "
                                    "seed 4+rank" if args.workload == "shared_prefix" else
                                    "uniform [128, 2048], seed 2+rank"),
                   "num_blocks": w.num_blocks, "kv_bytes_per_step": step_kv,
                   "l2": "inputs larger than L2 (KV read per step >> 126 MB)",
                   "parallelism": f"independent batch per GPU x{world}",
                   "path": ("pa_kv_cache_write + pa_paged_attn_decode_shared (tables split "
                            "by pa_split_shared_prefix)" if cascade else
                            "pa_decode_step_fp8" if fused and fp8 else
                            "pa_decode_step" if fused else
                            "pa_kv_cache_write_fp8 + pa_paged_attn_decode_fp8 (grouped-query "
                            "pools)" if gqa and fp8 else
                            f"pa_kv_cache_write + pa_paged_attn_decode_gqa ({gqa_kernel})" if gqa
                            else "pa_kv_cache_write_fp8 + pa_paged_attn_decode_fp8" if fp8
                            else "pa_kv_cache_write + pa_paged_attn_decode")},
        "decode_tokens_per_s": world * S / (ms_step * 1e-3),
        **({"logical_kv_gbs": world * logical_kv / (ms_step * 1e-3) / 1e9,
            "value_counts": "distinct (block, row) KV bytes; logical_kv_gbs counts every "
                            "text's reads"} if args.workload == "shared_prefix" else {}),
        "pct_of_nominal_8tbs": 100.0 * (value / world) / NOMINAL_HBM_GBS,
        # the decode call against three ceilings: the nominal spec, the
        # measured copy bandwidth, and a read-only stream measured here
        "ceilings": {"nominal_gbs": NOMINAL_HBM_GBS, "measured_copy_gbs": peak,
                     "read_probe_gbs": probe_gbs,
                     "decode_frac_of": {"nominal": achieved / NOMINAL_HBM_GBS,
                                        "measured_copy": achieved / peak,
                                        "read_probe": achieved / probe_gbs}},
        "kernel_ms": ({"pa_decode_step_fp8" if fp8 else "pa_decode_step": decode_ms} if fused else
                      {"kv_cache_write": write_ms, "paged_attn_decode": decode_ms}),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": traffic_per_launch(args.workload + ("_fp8" if fp8 else ""),
                                                   args.path),
                     "kernel": ("pa_paged_attn_decode_shared (prefix pass on the tensor cores, "
                                "tail pass, merge kernel)" if cascade else
                                "pa_decode_step_fp8 (8-bit decode kernel with the cache write, "
                                "+ merge kernel)" if fused and fp8 else
                                "pa_decode_step (decode kernel with the cache write, + merge kernel)"
                                if fused else
                                "pa_paged_attn_decode_fp8 (8-bit grouped-query decode kernel + "
                                "merge kernel)" if gqa and fp8 else
                                f"pa_paged_attn_decode_gqa ({gqa_kernel} decode kernel + merge kernel)" if gqa
                                else "pa_paged_attn_decode_fp8 (8-bit decode kernel + merge kernel)" if fp8
                                else "pa_paged_attn_decode (decode kernel + merge kernel)"),
                     "peak_source": peak_src, "algorithmic_bytes_per_launch": decode_bytes},
        "e2e": {"value": world * step_kv / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": (2 if fused else 4 if cascade else 3) * K,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        single = cpu_baseline(w)
        try:
            line["cpu_baseline"] = cpu_baseline_pool(w)
            line["cpu_baseline"]["single_core"] = single
        except Exception as e:   # the pool is a report, never a reason to lose the line
            line["cpu_baseline"] = dict(single, pool_error=str(e)[:200], **host_cores())
    if (world == 1 and args.workload == "opt13b_batch64" and not fp8 and args.path == "fused"
            and not args.no_other_configs):
        del w, staged, outs, houts, ws
        torch.cuda.empty_cache()
        line["other_configs"] = other_configs(P, W, dev, stream, peak,
                                              with_oracle=not args.no_cpu_baseline)
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.finish(ranks)
    return 0


if __name__ == "__main__":
    sys.exit(main())
