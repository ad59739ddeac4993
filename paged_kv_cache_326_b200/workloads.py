"""Seeded synthetic inputs for paged decode attention.

This module only *generates inputs*: context lengths, block tables, the
contents of the KV pool, the new token's q/k/v and the slot it is written to.
It holds none of the attention arithmetic.  Both the CUDA path (through the
tests and the bench) and the CPU oracle (through the tests) are fed from here,
and it imports neither.

Shapes and distributions follow the OPT-13B example of "The KV Cache and
PagedAttention" (§800 KB a Token: 40 layers, 5,120 = 40 heads x 128 numbers,
2-byte floats, texts up to 2,048 tokens) and its default block of 16 tokens
(§Like Pages of Memory).  Every value is N(0, 1) cast to the storage dtype.

Layout of the pool (chosen here; the pages only say that every block stores
keys and values for the same count of tokens): ``k_cache`` and ``v_cache`` are each
``[num_blocks][num_heads][block_size][head_dim]``.

Decode-step convention: ``context_lens[s]`` counts the token written in this
step, which sits at position ``context_lens[s] - 1``; ``slot_mapping[s]`` is
that position's slot.  Pool rows that hold no earlier token (the tail of the
last block, the new token's own row and every block no table references) are
filled with NaN so that a kernel that reads them is caught.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, List, Optional, Sequence, Tuple

import numpy as np
import torch

NAN16 = float("nan")


@dataclass
class DecodeInputs:
    """One decode step's inputs (one layer)."""

    name: str
    q: torch.Tensor              # [S][H][D] dt
    k: torch.Tensor              # [S][H][D] dt, key of the token written this step
    v: torch.Tensor              # [S][H][D] dt
    k_cache: torch.Tensor        # [N][H][B][D] dt
    v_cache: torch.Tensor        # [N][H][B][D] dt
    block_tables: torch.Tensor   # [S][max_blocks] int32, -1 past the last block
    context_lens: torch.Tensor   # [S] int32, includes the token written this step
    slot_mapping: torch.Tensor   # [S] int64
    scale: float                 # exactly representable in fp32
    block_size: int
    seed: int
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return self.q.shape[0]

    @property
    def num_heads(self) -> int:
        return self.q.shape[1]

    @property
    def head_dim(self) -> int:
        return self.q.shape[2]

    @property
    def num_blocks(self) -> int:
        return self.k_cache.shape[0]

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]

    @property
    def dtype(self) -> torch.dtype:
        return self.q.dtype


def fp32_scale(head_dim: int) -> float:
    """1/sqrt(head_dim) rounded to fp32, so both sides see the same number."""
    return float(np.float32(1.0 / math.sqrt(head_dim)))


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, dtype, gen, device, chunk_elems: int = 1 << 28) -> torch.Tensor:
    """N(0,1) in fp32, cast to ``dtype``; generated in slices along dim 0 so a
    40 GB pool never needs an fp32 copy of itself."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(shape[0], -1)
    row = flat.shape[1]
    step = max(1, chunk_elems // max(row, 1))
    for i in range(0, shape[0], step):
        j = min(shape[0], i + step)
        flat[i:j] = torch.randn((j - i, row), generator=gen, device=device,
                                dtype=torch.float32).to(dtype)
    return out


def blocks_needed(length: int, block_size: int) -> int:
    return -(-int(length) // block_size)


def _poison_unwritten(k_cache, v_cache, history_fill: torch.Tensor, block_size: int):
    """NaN every pool row at or past ``history_fill[block]`` (rows that hold
    no earlier token).  ``history_fill`` is an int64 tensor on the pool's device."""
    N = k_cache.shape[0]
    rows = torch.arange(block_size, device=k_cache.device)
    dead = rows[None, :] >= history_fill[:, None]            # [N][B]
    mask = dead[:, None, :, None]                            # [N][1][B][1]
    step = 4096
    for i in range(0, N, step):
        j = min(N, i + step)
        k_cache[i:j].masked_fill_(mask[i:j], NAN16)
        v_cache[i:j].masked_fill_(mask[i:j], NAN16)


def history_fill_of(tables: Sequence[torch.Tensor], lens: Sequence[torch.Tensor],
                    num_blocks: int, block_size: int, device) -> torch.Tensor:
    """For every physical block, how many leading rows hold an earlier token
    in at least one of the given (table, lens) sets.  Earlier tokens of text s
    are positions < lens[s] - 1."""
    fill = torch.zeros(num_blocks, dtype=torch.int64, device=device)
    for bt, ln in zip(tables, lens):
        bt = bt.to(device=device, dtype=torch.int64)
        hist = (ln.to(device=device, dtype=torch.int64) - 1).clamp(min=0)   # [S]
        j = torch.arange(bt.shape[1], device=device, dtype=torch.int64)
        rows = (hist[:, None] - j[None, :] * block_size).clamp(0, block_size)  # [S][MB]
        valid = bt >= 0
        fill.scatter_reduce_(0, bt[valid], rows[valid], reduce="amax")
    return fill


def slots_of(block_tables: torch.Tensor, positions: torch.Tensor, block_size: int) -> torch.Tensor:
    """Slot of token ``positions[s]`` of text s: physical block of its logical
    block, times the block size, plus its place in the block."""
    pos = positions.to(torch.int64)
    phys = block_tables.to(torch.int64).gather(1, (pos.clamp(min=0) // block_size)[:, None])[:, 0]
    return torch.where(pos >= 0, phys * block_size + pos % block_size,
                       torch.full_like(pos, -1))


def make_decode(name: str, context_lens: Sequence[int], num_heads: int, head_dim: int,
                block_size: int, num_blocks: int, dtype: torch.dtype, seed: int,
                device="cpu", max_blocks_per_seq: Optional[int] = None,
                block_order: Optional[torch.Tensor] = None,
                poison: bool = True, num_kv_heads: Optional[int] = None) -> DecodeInputs:
    """Generic single-layer decode step.

    Physical blocks are handed to the texts, in text order, from a seeded
    random permutation of the pool (or from ``block_order`` if given).  With
    ``num_kv_heads`` < ``num_heads`` the pool and the new k, v hold only the
    shared key/value heads (grouped-query attention)."""
    num_kv_heads = num_heads if num_kv_heads is None else num_kv_heads
    dev = torch.device(device)
    g_cpu = _gen(seed, "cpu")
    lens = [int(x) for x in context_lens]
    S = len(lens)
    nb = [blocks_needed(L, block_size) for L in lens]
    if max_blocks_per_seq is None:
        max_blocks_per_seq = max([1] + nb)
    need = sum(nb)
    if need > num_blocks:
        raise ValueError(f"{name}: pool of {num_blocks} blocks < {need} needed")
    order = block_order if block_order is not None else torch.randperm(num_blocks, generator=g_cpu)
    tables = torch.full((S, max_blocks_per_seq), -1, dtype=torch.int32)
    at = 0
    for s in range(S):
        tables[s, :nb[s]] = order[at:at + nb[s]].to(torch.int32)
        at += nb[s]
    lens_t = torch.tensor(lens, dtype=torch.int32)
    g = _gen(seed + 1000003, dev)
    shape_pool = (num_blocks, num_kv_heads, block_size, head_dim)
    k_cache = _randn(shape_pool, dtype, g, dev)
    v_cache = _randn(shape_pool, dtype, g, dev)
    q = _randn((S, num_heads, head_dim), dtype, g, dev)
    k = _randn((S, num_kv_heads, head_dim), dtype, g, dev)
    v = _randn((S, num_kv_heads, head_dim), dtype, g, dev)
    tables_d = tables.to(dev)
    lens_d = lens_t.to(dev)
    if poison:
        fill = history_fill_of([tables_d], [lens_d], num_blocks, block_size, dev)
        _poison_unwritten(k_cache, v_cache, fill, block_size)
    slots = slots_of(tables_d, lens_d.to(torch.int64) - 1, block_size)
    return DecodeInputs(name=name, q=q, k=k, v=v, k_cache=k_cache, v_cache=v_cache,
                        block_tables=tables_d, context_lens=lens_d, slot_mapping=slots,
                        scale=fp32_scale(head_dim), block_size=block_size, seed=seed)


# ---------------------------------------------------------------------------
# The five named workloads
# ---------------------------------------------------------------------------

def tiny(seed: int = 1, device="cpu", dtype=torch.float16) -> DecodeInputs:
    """Tiny paged decode, one layer: 4 texts of 5, 9, 16 and 23 tokens, 8 heads
    of 64, blocks of 4 (the drawings' size), a pool of 64 blocks handed out in
    seeded random order, fp16, and the write of the 4 new tokens."""
    return make_decode("tiny", [5, 9, 16, 23], num_heads=8, head_dim=64, block_size=4,
                       num_blocks=64, dtype=dtype, seed=seed, device=device)


def llama2_70b_gqa(seed: int = 6, device="cpu", dtype=torch.float16, num_seqs: int = 64,
                   num_blocks: int = 12288) -> DecodeInputs:
    """One layer of a Llama-2-70B-shaped decode ("The KV Cache and
    PagedAttention", section "What Came After": 64 query heads sharing 8
    key/value heads): head_dim 128, blocks of 16, lengths uniform in
    [128, 4096] (Llama 2's context), fp16."""
    g = np.random.default_rng(seed)
    lens = [int(x) for x in g.integers(128, 4096, size=num_seqs, endpoint=True)]
    return make_decode("llama2_70b_gqa", lens, num_heads=64, head_dim=128, block_size=16,
                       num_blocks=num_blocks, dtype=dtype, seed=seed, device=device,
                       max_blocks_per_seq=4096 // 16, num_kv_heads=8)


def opt13b_batch64_lens(seed: int = 2) -> List[int]:
    g = np.random.default_rng(seed)
    return [int(x) for x in g.integers(128, 2048, size=64, endpoint=True)]


def opt13b_batch64(seed: int = 2, device="cpu", dtype=torch.float16,
                   num_blocks: int = 8192) -> DecodeInputs:
    """OPT-13B-shaped layer, batch 64: 40 heads of 128, blocks of 16, lengths
    uniform in [128, 2048], shuffled physical blocks, fp16."""
    return make_decode("opt13b_batch64", opt13b_batch64_lens(seed), num_heads=40, head_dim=128,
                       block_size=16, num_blocks=num_blocks, dtype=dtype, seed=seed,
                       device=device, max_blocks_per_seq=2048 // 16)


def skewed_lens(seed: int = 3, num_seqs: int = 256, median: int = 300, sigma: float = 1.0,
                lo: int = 16, hi: int = 2048, num_full: int = 8) -> List[int]:
    g = np.random.default_rng(seed)
    x = np.exp(g.normal(math.log(median), sigma, size=num_seqs))
    lens = np.clip(np.rint(x), lo, hi).astype(np.int64)
    full = g.choice(num_seqs, size=num_full, replace=False)
    lens[full] = hi
    return [int(v) for v in lens]


def skewed(seed: int = 3, block_size: int = 16, device="cpu", dtype=torch.bfloat16) -> DecodeInputs:
    """Skewed lengths: 256 texts, lognormal lengths (median 300, sigma 1.0)
    clipped to [16, 2048], 8 texts at 2,048, bf16, pool 1.5x what is needed."""
    lens = skewed_lens(seed)
    need = sum(blocks_needed(L, block_size) for L in lens)
    return make_decode(f"skewed_b{block_size}", lens, num_heads=40, head_dim=128,
                       block_size=block_size, num_blocks=(3 * need + 1) // 2, dtype=dtype,
                       seed=seed, device=device, max_blocks_per_seq=2048 // block_size)


class _Allocator:
    """What ``shared_prefix`` needs from a block manager (the C++ one through
    its binding, or the oracle's model)."""

    def add_seq(self, seq_id: int, num_tokens: int) -> None: ...
    def fork(self, parent: int, child: int) -> None: ...
    def append_slot(self, seq_id: int) -> Tuple[int, int, int]: ...
    def export(self, seq_ids: Sequence[int], max_blocks_per_seq: int): ...


def shared_prefix_plan(seed: int = 4, num_prompts: int = 32, samples: int = 8,
                       prompt_lo: int = 256, prompt_hi: int = 1024,
                       gen_lo: int = 1, gen_hi: int = 256):
    """Prompt and generated lengths for parallel sampling: per prompt a length
    in [256, 1024], per sample a generated length in [1, 256].  The generated
    length counts the token written in the measured step."""
    g = np.random.default_rng(seed)
    prompts = [int(x) for x in g.integers(prompt_lo, prompt_hi, size=num_prompts, endpoint=True)]
    gens = [[int(x) for x in g.integers(gen_lo, gen_hi, size=samples, endpoint=True)]
            for _ in range(num_prompts)]
    return prompts, gens


def shared_prefix(allocator, num_blocks: int, seed: int = 4, device="cpu",
                  dtype=torch.float16, num_prompts: int = 32, samples: int = 8,
                  num_heads: int = 40, head_dim: int = 128, block_size: int = 16,
                  max_blocks_per_seq: int = (1024 + 256 + 15) // 16,
                  prompt_range=(256, 1024), gen_range=(1, 256),
                  num_kv_heads: Optional[int] = None) -> DecodeInputs:
    """Shared-prefix parallel sampling, built by driving a block manager.

    Per prompt: add the prompt, fork it into ``samples`` texts, then append the
    samples' generated tokens one at a time, interleaved across samples (each
    append may copy a shared partial block, per "Shared, Copied on Write").  The
    last append of every sample is the token written in the measured step.

    Block copies that the manager asks for are applied to the pool here, as a
    setup step: rows that already hold tokens are copied from source to
    destination.  ``meta['cow']`` lists them in order.  ``num_kv_heads``
    below ``num_heads`` gives grouped-query pools."""
    dev = torch.device(device)
    Hkv = num_heads if num_kv_heads is None else num_kv_heads
    prompts, gens = shared_prefix_plan(seed, num_prompts, samples, *prompt_range, *gen_range)
    seq_ids: List[int] = []
    cows: List[Tuple[int, int, int]] = []      # (src, dst, rows filled when copied)
    last_slot = {}
    for pi, P in enumerate(prompts):
        base = pi * samples
        allocator.add_seq(base, P)
        for k in range(1, samples):
            allocator.fork(base, base + k)
        ids = [base + k for k in range(samples)]
        seq_ids += ids
        tokens = {i: P for i in ids}
        remaining = {i: gens[pi][i - base] for i in ids}
        # interleave: round r appends one token to every sample still generating
        while any(r > 0 for r in remaining.values()):
            for i in ids:
                if remaining[i] == 0:
                    continue
                slot, src, dst = allocator.append_slot(i)
                if src >= 0:
                    cows.append((src, dst, tokens[i] % block_size))
                tokens[i] += 1
                remaining[i] -= 1
                if remaining[i] == 0:
                    last_slot[i] = slot
    tables, lens = allocator.export(seq_ids, max_blocks_per_seq)
    tables = torch.as_tensor(np.asarray(tables), dtype=torch.int32)
    lens = torch.as_tensor(np.asarray(lens), dtype=torch.int32)
    S = len(seq_ids)
    g = _gen(seed + 1000003, dev)
    shape_pool = (num_blocks, Hkv, block_size, head_dim)
    k_cache = _randn(shape_pool, dtype, g, dev)
    v_cache = _randn(shape_pool, dtype, g, dev)
    for src, dst, rows in cows:
        if rows:
            k_cache[dst, :, :rows] = k_cache[src, :, :rows]
            v_cache[dst, :, :rows] = v_cache[src, :, :rows]
    q = _randn((S, num_heads, head_dim), dtype, g, dev)
    k = _randn((S, Hkv, head_dim), dtype, g, dev)
    v = _randn((S, Hkv, head_dim), dtype, g, dev)
    tables_d, lens_d = tables.to(dev), lens.to(dev)
    fill = history_fill_of([tables_d], [lens_d], num_blocks, block_size, dev)
    _poison_unwritten(k_cache, v_cache, fill, block_size)
    slots = torch.tensor([last_slot[i] for i in seq_ids], dtype=torch.int64, device=dev)
    return DecodeInputs(name="shared_prefix", q=q, k=k, v=v, k_cache=k_cache, v_cache=v_cache,
                        block_tables=tables_d, context_lens=lens_d, slot_mapping=slots,
                        scale=fp32_scale(head_dim), block_size=block_size, seed=seed,
                        meta={"cow": cows, "prompts": prompts, "gens": gens,
                              "samples": samples})


@dataclass
class FullStepInputs:
    """A 40-layer decode step over one pool that all layers share."""

    k_cache: torch.Tensor
    v_cache: torch.Tensor
    context_lens: torch.Tensor                # [S] int32 (same in every layer)
    block_tables: List[torch.Tensor]          # per layer [S][max_blocks] int32
    slot_mapping: List[torch.Tensor]          # per layer [S] int64
    q: List[torch.Tensor]
    k: List[torch.Tensor]
    v: List[torch.Tensor]
    scale: float
    block_size: int
    seed: int

    @property
    def num_layers(self) -> int:
        return len(self.block_tables)


def full_step(seed: int = 5, device="cpu", dtype=torch.float16, num_layers: int = 40,
              num_seqs: int = 256, num_heads: int = 40, head_dim: int = 128,
              block_size: int = 16, num_blocks: int = 131072,
              len_range=(64, 2048)) -> FullStepInputs:
    """Full OPT-13B-shaped decode step: ``num_layers`` x (write + attend), batch
    256, lengths uniform in [64, 2048], one pool of ``num_blocks`` blocks.

    The 40 layers' caches do not fit one B200 as 40 separate pools of this
    size, so all layers share the one pool: each layer draws its own tables
    from a seeded permutation of the pool (distinct blocks within a layer,
    independent across layers, so blocks alias across layers).  Each layer
    streams its own ~5.5 GB, so the HBM bytes per step are those of 40 pools."""
    dev = torch.device(device)
    g_np = np.random.default_rng(seed)
    lens = [int(x) for x in g_np.integers(len_range[0], len_range[1], size=num_seqs, endpoint=True)]
    max_blocks = blocks_needed(len_range[1], block_size)
    lens_d = torch.tensor(lens, dtype=torch.int32, device=dev)
    nb = [blocks_needed(L, block_size) for L in lens]
    g_cpu = _gen(seed, "cpu")
    tables = []
    for _ in range(num_layers):
        order = torch.randperm(num_blocks, generator=g_cpu)
        t = torch.full((num_seqs, max_blocks), -1, dtype=torch.int32)
        at = 0
        for s in range(num_seqs):
            t[s, :nb[s]] = order[at:at + nb[s]].to(torch.int32)
            at += nb[s]
        tables.append(t.to(dev))
    g = _gen(seed + 1000003, dev)
    shape_pool = (num_blocks, num_heads, block_size, head_dim)
    k_cache = _randn(shape_pool, dtype, g, dev)
    v_cache = _randn(shape_pool, dtype, g, dev)
    fill = history_fill_of(tables, [lens_d] * num_layers, num_blocks, block_size, dev)
    _poison_unwritten(k_cache, v_cache, fill, block_size)
    qs, ks, vs, slots = [], [], [], []
    for layer in range(num_layers):
        qs.append(_randn((num_seqs, num_heads, head_dim), dtype, g, dev))
        ks.append(_randn((num_seqs, num_heads, head_dim), dtype, g, dev))
        vs.append(_randn((num_seqs, num_heads, head_dim), dtype, g, dev))
        slots.append(slots_of(tables[layer], lens_d.to(torch.int64) - 1, block_size))
    return FullStepInputs(k_cache=k_cache, v_cache=v_cache, context_lens=lens_d,
                          block_tables=tables, slot_mapping=slots, q=qs, k=ks, v=vs,
                          scale=fp32_scale(head_dim), block_size=block_size, seed=seed)


def cow_bursts(seed: int = 4, device="cpu", dtype=torch.float16, num_bursts: int = 8,
               prompts: int = 32, samples: int = 8, num_heads: int = 40, head_dim: int = 128,
               block_size: int = 16, num_blocks: int = 8192):
    """Copy-on-write bursts at the OPT-13B layer shape: in each burst, every
    one of ``prompts`` prompts has its partial last block copied for
    ``samples - 1`` of its samples (the last one writes in place), i.e. the
    copies of one decode step right after parallel sampling forks.  Sources
    and destinations of all bursts are distinct blocks drawn from a seeded
    permutation of the pool, so rotating through the bursts touches about
    ``num_bursts * prompts * samples`` blocks (far more than L2 holds).

    Returns (k_cache, v_cache, [pairs of each burst as [n][2] int32])."""
    dev = torch.device(device)
    per = prompts * samples
    if num_bursts * per > num_blocks:
        raise ValueError("pool too small for the bursts")
    order = torch.randperm(num_blocks, generator=_gen(seed, "cpu"))
    bursts = []
    for b in range(num_bursts):
        ids = order[b * per:(b + 1) * per].view(prompts, samples)
        src = ids[:, :1].expand(prompts, samples - 1)
        dst = ids[:, 1:]
        bursts.append(torch.stack([src.reshape(-1), dst.reshape(-1)], dim=1)
                      .to(torch.int32).contiguous().to(dev))
    g = _gen(seed + 1000003, dev)
    shape = (num_blocks, num_heads, block_size, head_dim)
    return _randn(shape, dtype, g, dev), _randn(shape, dtype, g, dev), bursts


# ---------------------------------------------------------------------------
# 8-bit (E4M3) caches
# ---------------------------------------------------------------------------

# Per-tensor scales of the 8-bit workloads: N(0,1) numbers divided by them
# spread over about +-100, well inside E4M3's +-448, so no code saturates.
FP8_K_SCALE = 0.05
FP8_V_SCALE = 0.04
NAN_CODE = 0x7F


def to_codes(x: torch.Tensor, scale: float) -> torch.Tensor:
    """E4M3 codes (uint8) of x / scale through torch's float8_e4m3fn cast
    (round to nearest even), computed in fp32 on x's device."""
    return (x.float() / scale).to(torch.float8_e4m3fn).view(torch.uint8)


def make_decode_fp8(name: str, context_lens: Sequence[int], num_heads: int, head_dim: int,
                    block_size: int, num_blocks: int, dtype: torch.dtype, seed: int,
                    device="cpu", max_blocks_per_seq: Optional[int] = None,
                    k_scale: float = FP8_K_SCALE, v_scale: float = FP8_V_SCALE,
                    num_kv_heads: Optional[int] = None) -> DecodeInputs:
    """make_decode with 8-bit caches: the pools hold E4M3 codes of seeded
    N(0,1) numbers over the scales (``meta['k_scale']``, ``meta['v_scale']``);
    rows that hold no earlier token hold the NaN code.  q, k, v stay in
    ``dtype``; ``num_kv_heads`` below ``num_heads`` gives grouped-query
    pools."""
    w = make_decode(name, context_lens, num_heads, head_dim, block_size, num_blocks, dtype, seed,
                    device, max_blocks_per_seq, poison=False, num_kv_heads=num_kv_heads)
    dev = w.q.device
    g = _gen(seed + 2000003, dev)
    shape = w.k_cache.shape
    kc = torch.empty(shape, dtype=torch.uint8, device=dev)
    vc = torch.empty(shape, dtype=torch.uint8, device=dev)
    for dst, sc in ((kc, k_scale), (vc, v_scale)):
        flat = dst.view(shape[0], -1)
        step = max(1, (1 << 26) // flat.shape[1])
        for i in range(0, shape[0], step):
            j = min(shape[0], i + step)
            flat[i:j] = to_codes(torch.randn((j - i, flat.shape[1]), generator=g, device=dev), sc)
    fill = history_fill_of([w.block_tables], [w.context_lens], num_blocks, block_size, dev)
    rows = torch.arange(block_size, device=dev)
    dead = (rows[None, :] >= fill[:, None])[:, None, :, None]
    kc.masked_fill_(dead, NAN_CODE)
    vc.masked_fill_(dead, NAN_CODE)
    w.k_cache, w.v_cache = kc, vc
    w.name = name
    w.meta.update(k_scale=k_scale, v_scale=v_scale)
    return w


def llama2_70b_gqa_fp8(seed: int = 6, device="cpu", num_seqs: int = 64,
                       num_blocks: int = 12288) -> DecodeInputs:
    """The Llama-2-70B-shaped grouped-query step (64 query heads over 8
    key/value heads, head_dim 128, blocks of 16, lengths uniform in
    [128, 4096]) over 8-bit caches."""
    g = np.random.default_rng(seed)
    lens = [int(x) for x in g.integers(128, 4096, size=num_seqs, endpoint=True)]
    return make_decode_fp8("llama2_70b_gqa_fp8", lens, num_heads=64, head_dim=128,
                           block_size=16, num_blocks=num_blocks, dtype=torch.float16, seed=seed,
                           device=device, max_blocks_per_seq=4096 // 16, num_kv_heads=8)


def opt13b_batch64_fp8(seed: int = 2, device="cpu") -> DecodeInputs:
    """The batch-64 OPT-13B-shaped step (lengths, tables, q, k, v as
    opt13b_batch64) over 8-bit caches."""
    return make_decode_fp8("opt13b_batch64_fp8", opt13b_batch64_lens(seed), num_heads=40,
                           head_dim=128, block_size=16, num_blocks=8192, dtype=torch.float16,
                           seed=seed, device=device, max_blocks_per_seq=128)


# ---------------------------------------------------------------------------
# Prompt phase (prefill)
# ---------------------------------------------------------------------------

@dataclass
class PrefillInputs:
    """Packed prompts: prompt s is rows cu_seqlens[s]..cu_seqlens[s+1]-1."""

    name: str
    q: torch.Tensor             # [T][H][D]
    k: torch.Tensor             # [T][H_kv][D]
    v: torch.Tensor             # [T][H_kv][D]
    cu_seqlens: torch.Tensor    # [S+1] int32
    max_seqlen: int
    k_cache: torch.Tensor       # [N][H_kv][B][D], NaN before the store
    v_cache: torch.Tensor
    slot_mapping: torch.Tensor  # [T] int64: each token's slot through its prompt's table
    block_tables: torch.Tensor  # [S][max_blocks] int32
    scale: float
    block_size: int
    lens: List[int]


def make_prefill(name: str, lens: Sequence[int], num_heads: int, num_kv_heads: int,
                 head_dim: int, dtype: torch.dtype, seed: int, device="cpu",
                 block_size: int = 16, spare_blocks: int = 8) -> PrefillInputs:
    """Seeded N(0,1) prompts packed back to back; each prompt gets blocks from
    a seeded permutation of a pool with ``spare_blocks`` extra blocks, and
    token t of prompt s has slot table[s][t // B] * B + t % B."""
    dev = torch.device(device)
    lens = [int(x) for x in lens]
    T, S = sum(lens), len(lens)
    nb = [blocks_needed(L, block_size) for L in lens]
    N = sum(nb) + spare_blocks
    order = torch.randperm(N, generator=_gen(seed, "cpu"))
    mb = max([1] + nb)
    tables = torch.full((S, mb), -1, dtype=torch.int32)
    slots = torch.empty(T, dtype=torch.int64)
    at = pos = 0
    for s, L in enumerate(lens):
        tables[s, :nb[s]] = order[at:at + nb[s]].to(torch.int32)
        at += nb[s]
        t = torch.arange(L)
        slots[pos:pos + L] = tables[s, t // block_size].to(torch.int64) * block_size + t % block_size
        pos += L
    g = _gen(seed + 1000003, dev)
    q = _randn((max(T, 1), num_heads, head_dim), dtype, g, dev)[:T]
    k = _randn((max(T, 1), num_kv_heads, head_dim), dtype, g, dev)[:T]
    v = _randn((max(T, 1), num_kv_heads, head_dim), dtype, g, dev)[:T]
    cache_shape = (N, num_kv_heads, block_size, head_dim)
    k_cache = torch.full(cache_shape, NAN16, dtype=dtype, device=dev)
    v_cache = torch.full(cache_shape, NAN16, dtype=dtype, device=dev)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    return PrefillInputs(name=name, q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                         cu_seqlens=cu.to(dev), max_seqlen=max([0] + lens), k_cache=k_cache,
                         v_cache=v_cache, slot_mapping=slots.to(dev), block_tables=tables.to(dev),
                         scale=fp32_scale(head_dim), block_size=block_size, lens=lens)


def opt13b_prefill(seed: int = 7, device="cpu", num_prompts: int = 16,
                   prompt_len: int = 2048) -> PrefillInputs:
    """OPT-13B-shaped prompt phase: 16 prompts of 2,048 tokens (the model's
    longest), 40 heads of 128, fp16, blocks of 16."""
    return make_prefill("opt13b_prefill", [prompt_len] * num_prompts, num_heads=40,
                        num_kv_heads=40, head_dim=128, dtype=torch.float16, seed=seed,
                        device=device)
