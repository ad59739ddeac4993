"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
hand the oracle the same inputs, compare with the stated tolerance."""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

import oracle

# Attention tolerance (fp16/bf16 out, fp32 accumulate):
#   fp16: max |gpu - ref| <= 2e-3 and max relative error <= 1e-2, the relative
#         error taken over outputs with |ref| >= 0.2 (= atol / rtol);
#   bf16: |gpu - ref| <= 2e-3 + 1e-2 * |ref| element-wise.  (Rounding the exact
#         result to bf16 alone costs up to 2^-8 |x|, above 2e-3 at |x| ~ 1, so
#         the absolute bound cannot hold alone for any correct bf16 kernel.)
ATOL = 2e-3
RTOL = 1e-2


@dataclass
class Closeness:
    max_abs: float
    max_rel: float
    ok: bool

    def __str__(self):
        return f"max_abs={self.max_abs:.3e} max_rel={self.max_rel:.3e} ok={self.ok}"


def compare(got: torch.Tensor, ref: np.ndarray, dtype: torch.dtype,
            mask: Optional[np.ndarray] = None) -> Closeness:
    g = got.float().cpu().numpy().astype(np.float64)
    if mask is not None:
        g, ref = g[mask], ref[mask]
    err = np.abs(g - ref)
    big = np.abs(ref) >= ATOL / RTOL
    max_abs = float(err.max()) if err.size else 0.0
    max_rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    if not np.isfinite(g).all():
        return Closeness(float("inf"), float("inf"), False)
    if dtype == torch.float16:
        ok = max_abs <= ATOL and max_rel <= RTOL
    else:
        ok = bool((err <= ATOL + RTOL * np.abs(ref)).all())
    return Closeness(max_abs, max_rel, ok)


def host_f32(t: torch.Tensor) -> np.ndarray:
    """Exact widening of fp16/bf16 to float32 on the host."""
    return t.detach().float().cpu().numpy()


@dataclass
class OracleInputs:
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray
    tables: np.ndarray
    lens: np.ndarray
    slots: np.ndarray
    seqs: np.ndarray


def oracle_inputs(q, k, v, k_cache, v_cache, block_tables, context_lens, slot_mapping,
                  block_size: int, seqs: Optional[Sequence[int]] = None) -> OracleInputs:
    """Copy to the host only the pool blocks that the chosen texts reference,
    renumbered 0..n-1 (renumbering is pinned not to change the oracle's
    output), and the writes that land in them.  Call BEFORE the GPU step: the
    pool must be the pre-write one.  8-bit (uint8) pools are copied as raw
    codes."""
    S = q.shape[0]
    seqs = np.arange(S) if seqs is None else np.asarray(seqs)
    sel = torch.as_tensor(seqs, device=block_tables.device, dtype=torch.long)
    t = block_tables.index_select(0, sel).to(torch.int64)
    used = torch.unique(t[t >= 0])
    N = k_cache.shape[0]
    remap = torch.full((N,), -1, dtype=torch.int64, device=block_tables.device)
    remap[used] = torch.arange(used.numel(), device=block_tables.device)
    new_t = torch.where(t >= 0, remap[t.clamp(min=0)], torch.full_like(t, -1))
    slots = slot_mapping.to(torch.int64)
    blk = (slots // block_size).clamp(min=0, max=N - 1)
    nb = torch.where(slots >= 0, remap[blk], torch.full_like(slots, -1))
    new_slots = torch.where(nb >= 0, nb * block_size + slots % block_size, torch.full_like(slots, -1))
    pool = (lambda t: t.cpu().numpy()) if k_cache.dtype == torch.uint8 else host_f32
    return OracleInputs(
        q=host_f32(q.index_select(0, sel)), k=host_f32(k), v=host_f32(v),
        k_cache=pool(k_cache.index_select(0, used)),
        v_cache=pool(v_cache.index_select(0, used)),
        tables=new_t.cpu().numpy(), lens=context_lens.index_select(0, sel).cpu().numpy(),
        slots=new_slots.cpu().numpy(), seqs=seqs)


def run_oracle(oi: OracleInputs, scale: float, block_size: int, pairs=None) -> np.ndarray:
    """Oracle decode step (write, then attend) for the selected texts."""
    kc, vc = oracle.cache_write(oi.k_cache, oi.v_cache, oi.k, oi.v, oi.slots, block_size)
    local_pairs = None
    if pairs is not None:
        pos = {int(s): i for i, s in enumerate(oi.seqs)}
        local_pairs = [(pos[int(s)], int(h)) for s, h in pairs]
    return oracle.paged_decode(oi.q, kc, vc, oi.tables, oi.lens, scale, block_size, local_pairs)


def run_oracle_fp8(oi: OracleInputs, scale: float, block_size: int, k_scale: float,
                   v_scale: float, pairs=None) -> np.ndarray:
    """Oracle decode step over 8-bit caches (quantizing write, then attend)."""
    kc, vc = oracle.cache_write_fp8(oi.k_cache, oi.v_cache, oi.k, oi.v, oi.slots, block_size,
                                    k_scale, v_scale)
    local_pairs = None
    if pairs is not None:
        pos = {int(s): i for i, s in enumerate(oi.seqs)}
        local_pairs = [(pos[int(s)], int(h)) for s, h in pairs]
    return oracle.paged_decode_fp8(oi.q, kc, vc, oi.tables, oi.lens, scale, block_size, k_scale,
                                   v_scale, local_pairs)


def gpu_step_fp8(w, status=None, out=None):
    """Quantizing write, then decode, over the workload's 8-bit caches."""
    import paged_kv_cache_326_b200 as P
    ks, vs = w.meta["k_scale"], w.meta["v_scale"]
    P.pa_kv_cache_write_fp8(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, ks, vs, status=status)
    if out is None:
        out = torch.empty_like(w.q)
    P.pa_paged_attn_decode_fp8(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                               w.scale, ks, vs, status=status)
    return out


def gpu_step(w, status=None, out=None):
    import paged_kv_cache_326_b200 as P
    P.pa_kv_cache_write(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, status=status)
    if out is None:
        out = torch.empty_like(w.q)
    P.pa_paged_attn_decode(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                           w.scale, status=status)
    return out


def gpu_step_fused(w, status=None, out=None):
    """The same step through the one-launch entry point pa_decode_step."""
    import paged_kv_cache_326_b200 as P
    if out is None:
        out = torch.empty_like(w.q)
    P.pa_decode_step(out, w.q, w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, w.block_tables,
                     w.context_lens, w.scale, status=status)
    return out


def new_status(device="cuda"):
    return torch.zeros(1, dtype=torch.int32, device=device)
