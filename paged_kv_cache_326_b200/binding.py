"""Python binding of libpagedattn.so (ctypes): argument marshalling only.

Every function carries the name of the C entry point it calls (see
include/pagedattn.h for the definitions).  Tensors are torch tensors; the
binding checks their device, dtype and contiguity, reads the sizes from their
shapes and passes raw pointers and the current CUDA stream.  All arithmetic
runs in the library's CUDA kernels.  There is no fallback: if the shared
library is missing, loading it raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Dict, Optional, Sequence, Tuple

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedattn.so")

PA_OK = 0
PA_ERR_INVALID = -1
PA_ERR_CUDA = -2
PA_ERR_OUT_OF_BLOCKS = -3
PA_ERR_NO_SEQ = -4
PA_ERR_EXISTS = -5
PA_ERR_TABLE_FULL = -6
PA_ERR_BAD_BLOCK = -7
PA_ERR_BAD_LEN = -8
PA_ERR_BAD_SLOT = -9
PA_ERR_TIMEOUT = -10
PA_ERR_CORRUPT = -11
PA_ERR_TOO_LARGE = -12

PA_F16 = 0
PA_BF16 = 1
PA_E4M3 = 2

PA_OPT_WAIT_LIMIT_NS = 1
PA_OPT_DECODE_WARPS = 2
PA_OPT_GQA_KERNEL = 3
PA_OPT_PREFILL_KERNEL = 4
PA_OPT_PREFIX_KEY_BITS = 5
PA_OPT_FP8_KERNEL = 6

_KIND = {PA_ERR_INVALID: "invalid", PA_ERR_CUDA: "cuda", PA_ERR_OUT_OF_BLOCKS: "out_of_blocks",
         PA_ERR_NO_SEQ: "no_seq", PA_ERR_EXISTS: "exists", PA_ERR_TABLE_FULL: "table_full",
         PA_ERR_CORRUPT: "corrupt", PA_ERR_TOO_LARGE: "too_large"}


class PagedAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.kind = _KIND.get(code, "error")
        super().__init__(f"{where}: {pa_status_string(code)} ({code})")


_lib = None
_lock = threading.Lock()

_vp, _i32, _i64, _u64, _f32, _sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                     ctypes.c_uint64, ctypes.c_float, ctypes.c_size_t)

_SIGNATURES = {
    "pa_status_string": (ctypes.c_char_p, [_i32]),
    "pa_set_option": (_i32, [_i32, _i64]),
    "pa_kv_cache_write": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _i32,
                                 _vp, _vp]),
    "pa_paged_attn_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "pa_paged_attn_decode": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _f32, _i32, _i32, _i32, _i32,
                                    _i32, _i64, _i32, _vp, _sz, _vp, _vp]),
    "pa_paged_attn_decode_gqa_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "pa_paged_attn_decode_gqa": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _f32, _i32, _i32, _i32, _i32,
                                        _i32, _i32, _i64, _i32, _vp, _sz, _vp, _vp]),
    "pa_decode_step": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _f32, _i32, _i32, _i32,
                              _i32, _i32, _i64, _i32, _vp, _sz, _vp, _vp]),
    "pa_decode_step_fp8": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _f32, _f32, _f32,
                                  _i32, _i32, _i32, _i32, _i32, _i64, _i32, _vp, _sz, _vp, _vp]),
    "pa_paged_attn_decode_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _f32, _i32, _i32, _i32,
                                            _i32, _i32, _i64, _i32, _vp, _vp]),
    "pa_kv_cache_write_fp8": (_i32, [_vp, _vp, _vp, _vp, _vp, _f32, _f32, _i32, _i32, _i32, _i32,
                                     _i64, _i32, _vp, _vp]),
    "pa_paged_attn_decode_fp8": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _f32, _f32, _f32, _i32, _i32,
                                        _i32, _i32, _i32, _i64, _i32, _vp, _sz, _vp, _vp]),
    "pa_paged_attn_decode_fp8_gqa": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _f32, _f32, _f32, _i32,
                                            _i32, _i32, _i32, _i32, _i32, _i64, _i32, _vp, _sz,
                                            _vp, _vp]),
    "pa_prefill": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _f32, _i32,
                          _i32, _i32, _i32, _i64, _i32, _vp, _vp]),
    "pa_prefill_with_prefix": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                      _i32, _i32, _i32, _f32, _i32, _i32, _i32, _i32, _i64,
                                      _i32, _vp, _vp]),
    "pa_read_probe": (_i32, [_vp, _sz, _vp, _i32, _vp]),
    "pa_exp2_probe": (_i32, [_vp, _vp, _i64, _i32, _vp]),
    "pa_write_probe": (_i32, [_vp, _sz, _vp]),
    "pa_copy_blocks": (_i32, [_vp, _vp, _i64, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _i32, _i32,
                              _vp, _vp]),
    "pa_paged_attn_decode_shared_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32,
                                                           _i32]),
    "pa_paged_attn_decode_shared": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32,
                                           _f32, _i32, _i32, _i32, _i32, _i32, _i64, _i32, _vp,
                                           _sz, _vp, _vp]),
    "pa_paged_attn_decode_shared_gqa_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32,
                                                               _i32, _i32, _i32]),
    "pa_paged_attn_decode_shared_gqa": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                                               _i32, _f32, _i32, _i32, _i32, _i32, _i32, _i32,
                                               _i64, _i32, _vp, _sz, _vp, _vp]),
    "pa_split_shared_prefix": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _i32, _vp, _vp,
                                      _i32, _vp]),
    "pa_bm_create": (_vp, [_i64, _i32, _u64]),
    "pa_bm_destroy": (None, [_vp]),
    "pa_bm_add_seq": (_i32, [_vp, _i64, _i32]),
    "pa_bm_fork": (_i32, [_vp, _i64, _i64]),
    "pa_bm_append_slot": (_i32, [_vp, _i64, ctypes.POINTER(_i64), ctypes.POINTER(ctypes.c_int32),
                                 ctypes.POINTER(ctypes.c_int32)]),
    "pa_bm_free_seq": (_i32, [_vp, _i64]),
    "pa_bm_num_free": (_i64, [_vp]),
    "pa_bm_refcount": (_i32, [_vp, ctypes.c_int32]),
    "pa_bm_num_tokens": (_i64, [_vp, _i64]),
    "pa_bm_export": (_i32, [_vp, _vp, _i32, _vp, _i32, _vp]),
    "pa_bm_add_seq_tokens": (_i32, [_vp, _i64, _vp, _i32, ctypes.POINTER(ctypes.c_int)]),
    "pa_bm_num_cached_blocks": (_i64, [_vp]),
}


def lib() -> ctypes.CDLL:
    """The loaded library (built by ``python -m paged_kv_cache_326_b200.build``)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(f"{LIB_PATH} is missing: build it with "
                                      "`python -m paged_kv_cache_326_b200.build`")
                l = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in _SIGNATURES.items():
                    fn = getattr(l, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = l
    return _lib


def _check(code: int, where: str) -> None:
    if code != PA_OK:
        raise PagedAttnError(code, where)


def pa_status_string(code: int) -> str:
    return lib().pa_status_string(int(code)).decode()


def pa_set_option(key: int, value: int) -> None:
    _check(lib().pa_set_option(int(key), int(value)), "pa_set_option")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: fp16 or bf16")


def _cuda(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream, device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _status_ptr(status: Optional[torch.Tensor]) -> Optional[int]:
    if status is None:
        return None
    return _cuda(status, "status", torch.int32)


def pa_kv_cache_write(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                      status: Optional[torch.Tensor] = None, stream=None) -> None:
    """k, v: [T][H][D]; caches [N][H][B][D]; slot_mapping [T] int64."""
    T, H, D = k.shape
    N, H2, B, D2 = k_cache.shape
    if v.shape != k.shape or v_cache.shape != k_cache.shape or (H2, D2) != (H, D):
        raise ValueError("shape mismatch between k/v and the caches")
    if slot_mapping.shape != (T,):
        raise ValueError("slot_mapping must be [num_tokens]")
    for t in (v, k_cache, v_cache):
        if t.dtype != k.dtype:
            raise TypeError("k, v and the caches must share a dtype")
    code = lib().pa_kv_cache_write(
        _cuda(k, "k"), _cuda(v, "v"), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
        _cuda(slot_mapping, "slot_mapping", torch.int64), T, H, D, B, N, _dtype_code(k),
        _status_ptr(status), _stream(stream, k.device))
    _check(code, "pa_kv_cache_write")


def _codes(t: torch.Tensor, name: str) -> int:
    """An 8-bit cache pool: uint8 or float8_e4m3fn, on the GPU."""
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError(f"{name} must hold 8-bit codes (uint8 or float8_e4m3fn), got {t.dtype}")
    return _cuda(t, name)


def pa_kv_cache_write_fp8(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor,
                          v_cache: torch.Tensor, slot_mapping: torch.Tensor, k_scale: float,
                          v_scale: float, status: Optional[torch.Tensor] = None,
                          stream=None) -> None:
    """k, v: [T][H][D] fp16/bf16; 8-bit caches [N][H][B][D]; slot_mapping [T]
    int64; per-tensor scales."""
    T, H, D = k.shape
    N, H2, B, D2 = k_cache.shape
    if v.shape != k.shape or v_cache.shape != k_cache.shape or (H2, D2) != (H, D):
        raise ValueError("shape mismatch between k/v and the caches")
    if slot_mapping.shape != (T,) or v.dtype != k.dtype:
        raise ValueError("slot_mapping must be [num_tokens]; k and v must share a dtype")
    code = lib().pa_kv_cache_write_fp8(
        _cuda(k, "k"), _cuda(v, "v"), _codes(k_cache, "k_cache"), _codes(v_cache, "v_cache"),
        _cuda(slot_mapping, "slot_mapping", torch.int64), float(k_scale), float(v_scale), T, H, D,
        B, N, _dtype_code(k), _status_ptr(status), _stream(stream, k.device))
    _check(code, "pa_kv_cache_write_fp8")


def pa_paged_attn_decode_fp8(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                             v_cache: torch.Tensor, block_tables: torch.Tensor,
                             context_lens: torch.Tensor, scale: float, k_scale: float,
                             v_scale: float, workspace: Optional[torch.Tensor] = None,
                             status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out, q: [S][H][D] fp16/bf16; 8-bit caches [N][H_kv][B][D].  H_kv == H
    is multi-head attention (pa_paged_attn_decode_fp8); a divisor of H is
    grouped-query attention (pa_paged_attn_decode_fp8_gqa)."""
    S, H, D = q.shape
    N, Hkv, B, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or D2 != D or H % Hkv:
        raise ValueError("shape mismatch (num_heads must be a multiple of num_kv_heads)")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S][max_blocks], context_lens [S]")
    if out.dtype != q.dtype:
        raise TypeError("q and out must share a dtype")
    MB = block_tables.shape[1]
    if workspace is None:
        workspace = workspace_for(q, B, MB, Hkv)
    args = (_cuda(out, "out"), _cuda(q, "q"), _codes(k_cache, "k_cache"),
            _codes(v_cache, "v_cache"), _cuda(block_tables, "block_tables", torch.int32),
            _cuda(context_lens, "context_lens", torch.int32), float(scale), float(k_scale),
            float(v_scale), S, H)
    tail = (D, B, MB, N, _dtype_code(q), _cuda(workspace, "workspace"),
            workspace.numel() * workspace.element_size(), _status_ptr(status),
            _stream(stream, q.device))
    if Hkv == H:
        code = lib().pa_paged_attn_decode_fp8(*args, *tail)
        _check(code, "pa_paged_attn_decode_fp8")
    else:
        code = lib().pa_paged_attn_decode_fp8_gqa(*args, Hkv, *tail)
        _check(code, "pa_paged_attn_decode_fp8_gqa")
    return out


def pa_prefill(out: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
               cu_seqlens: torch.Tensor, max_seqlen: int, scale: float,
               k_cache: Optional[torch.Tensor] = None, v_cache: Optional[torch.Tensor] = None,
               slot_mapping: Optional[torch.Tensor] = None,
               status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Prompt phase over packed prompts: out, q [T][H][D]; k, v [T][H_kv][D];
    cu_seqlens [S+1] int32.  With caches and slot_mapping [T] int64, the
    prompts' keys and values are stored in their blocks first."""
    T, H, D = q.shape
    Tk, Hkv, Dk = k.shape
    if out.shape != q.shape or v.shape != k.shape or Tk != T or Dk != D or H % Hkv:
        raise ValueError("shape mismatch")
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be [num_seqs + 1]")
    for t in (out, k, v):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v and out must share a dtype")
    S = cu_seqlens.numel() - 1
    B, N, kc, vc, sm = 16, 0, None, None, None
    if k_cache is not None:
        N, Hc, B, Dc = k_cache.shape
        if v_cache is None or slot_mapping is None or v_cache.shape != k_cache.shape or \
                (Hc, Dc) != (Hkv, D) or slot_mapping.shape != (T,) or k_cache.dtype != q.dtype:
            raise ValueError("caches must be [N][H_kv][B][D] of q's dtype with slot_mapping [T]")
        kc, vc = _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache")
        sm = _cuda(slot_mapping, "slot_mapping", torch.int64)
    code = lib().pa_prefill(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), kc, vc, sm,
        _cuda(cu_seqlens, "cu_seqlens", torch.int32), S, T, int(max_seqlen), float(scale), H, Hkv,
        D, B, N, _dtype_code(q), _status_ptr(status), _stream(stream, q.device))
    _check(code, "pa_prefill")
    return out


def pa_prefill_with_prefix(out: torch.Tensor, q: torch.Tensor, k: torch.Tensor,
                           v: torch.Tensor, cu_seqlens: torch.Tensor, max_seqlen: int,
                           scale: float, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           block_tables: torch.Tensor, cached_lens: torch.Tensor,
                           slot_mapping: Optional[torch.Tensor] = None,
                           status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Prompt phase of prompts whose first cached_lens[s] tokens are stored
    in the caches (blocks block_tables[s]): out, q [T][H][D] and k, v
    [T][H_kv][D] hold the other tokens; slot_mapping [T] int64 (optional)
    stores their keys and values."""
    T, H, D = q.shape
    Tk, Hkv, Dk = k.shape
    if out.shape != q.shape or v.shape != k.shape or Tk != T or Dk != D or H % Hkv:
        raise ValueError("shape mismatch")
    S = cu_seqlens.numel() - 1
    N, Hc, B, Dc = k_cache.shape
    if v_cache.shape != k_cache.shape or (Hc, Dc) != (Hkv, D) or k_cache.dtype != q.dtype:
        raise ValueError("caches must be [N][H_kv][B][D] of q's dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or cached_lens.shape != (S,):
        raise ValueError("block_tables must be [S][max_blocks], cached_lens [S]")
    sm = None
    if slot_mapping is not None:
        if slot_mapping.shape != (T,):
            raise ValueError("slot_mapping must be [T]")
        sm = _cuda(slot_mapping, "slot_mapping", torch.int64)
    for t in (out, k, v):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v and out must share a dtype")
    code = lib().pa_prefill_with_prefix(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"),
        _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"), sm,
        _cuda(cu_seqlens, "cu_seqlens", torch.int32),
        _cuda(block_tables, "block_tables", torch.int32),
        _cuda(cached_lens, "cached_lens", torch.int32), S, T, int(max_seqlen),
        block_tables.shape[1], float(scale), H, Hkv, D, B, N, _dtype_code(q),
        _status_ptr(status), _stream(stream, q.device))
    _check(code, "pa_prefill_with_prefix")
    return out


def pa_read_probe(buf: torch.Tensor, sink: torch.Tensor, stream=None) -> None:
    """Read every byte of the CUDA tensor `buf` once (the HBM read ceiling);
    sink: a CUDA int32 tensor of at least 4 x the SM count words."""
    nbytes = buf.numel() * buf.element_size()
    _check(lib().pa_read_probe(_cuda(buf, "buf"), nbytes & ~15, _cuda(sink, "sink", torch.int32),
                               sink.numel(), _stream(stream, buf.device)), "pa_read_probe")


def pa_write_probe(buf: torch.Tensor, stream=None) -> None:
    """Write the whole (contiguous, device) buffer once: the write ceiling."""
    _check(lib().pa_write_probe(_cuda(buf, "buf"), buf.numel() * buf.element_size(),
                                _stream(stream, buf.device)), "pa_write_probe")


def pa_exp2_probe(x: torch.Tensor, y: torch.Tensor, method: int, stream=None) -> None:
    """y = 2^x (float32 device tensors) by the softmax polynomial (method 0)
    or the exponential unit (method 1)."""
    if x.shape != y.shape:
        raise ValueError("x and y must have one shape")
    _check(lib().pa_exp2_probe(_cuda(x, "x", torch.float32), _cuda(y, "y", torch.float32),
                               x.numel(), int(method), _stream(stream, x.device)),
           "pa_exp2_probe")


def _pool(t: torch.Tensor, name: str) -> int:
    """A pool the GPU can address: a CUDA tensor, or a pinned CPU tensor (the
    library checks the mapping before launch)."""
    if not isinstance(t, torch.Tensor) or not (t.is_cuda or t.is_pinned()):
        raise TypeError(f"{name} must be a CUDA tensor or a pinned CPU tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def pa_copy_blocks(src_k: torch.Tensor, src_v: torch.Tensor, dst_k: torch.Tensor,
                   dst_v: torch.Tensor, block_pairs: torch.Tensor,
                   status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Pools [N][H][B][D] (source and destination may differ in N, or be the
    same tensors); block_pairs [n][2] int32 (source block, destination
    block), on the GPU."""
    Ns, H, B, D = src_k.shape
    Nd = dst_k.shape[0]
    if (src_v.shape != src_k.shape or dst_k.shape[1:] != src_k.shape[1:] or
            dst_v.shape != dst_k.shape):
        raise ValueError("pool shapes differ")
    if block_pairs.dim() != 2 or block_pairs.shape[1] != 2:
        raise ValueError("block_pairs must be [n][2]")
    for t in (src_v, dst_k, dst_v):
        if t.dtype != src_k.dtype:
            raise TypeError("pools must share a dtype")
    dev = block_pairs.device
    dt = PA_E4M3 if src_k.dtype in (torch.uint8, torch.float8_e4m3fn) else _dtype_code(src_k)
    code = lib().pa_copy_blocks(
        _pool(src_k, "src_k"), _pool(src_v, "src_v"), Ns, _pool(dst_k, "dst_k"),
        _pool(dst_v, "dst_v"), Nd, _cuda(block_pairs, "block_pairs", torch.int32),
        block_pairs.shape[0], H, D, B, dt, _status_ptr(status), _stream(stream, dev))
    _check(code, "pa_copy_blocks")


def pa_paged_attn_decode_workspace_size(num_seqs: int, num_heads: int, head_dim: int,
                                        block_size: int, max_blocks_per_seq: int) -> int:
    return int(lib().pa_paged_attn_decode_workspace_size(num_seqs, num_heads, head_dim,
                                                          block_size, max_blocks_per_seq))


_ws_cache: Dict[Tuple[int, int], torch.Tensor] = {}


def pa_paged_attn_decode_gqa_workspace_size(num_seqs: int, num_heads: int, num_kv_heads: int,
                                            head_dim: int, block_size: int,
                                            max_blocks_per_seq: int) -> int:
    return int(lib().pa_paged_attn_decode_gqa_workspace_size(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq))


def workspace_for(q: torch.Tensor, block_size: int, max_blocks_per_seq: int,
                  num_kv_heads: Optional[int] = None) -> torch.Tensor:
    """A cached device workspace big enough for these sizes (allocated by
    torch, never by the library)."""
    S, H, D = q.shape
    if num_kv_heads is None or num_kv_heads == H:
        need = pa_paged_attn_decode_workspace_size(S, H, D, block_size, max_blocks_per_seq)
    else:
        need = pa_paged_attn_decode_gqa_workspace_size(S, H, num_kv_heads, D, block_size,
                                                       max_blocks_per_seq)
    if need == 0:
        raise PagedAttnError(PA_ERR_INVALID, "pa_paged_attn_decode_workspace_size")
    key = (q.device.index if q.device.index is not None else torch.cuda.current_device(), need)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        _ws_cache[key] = ws
    return ws


def pa_paged_attn_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                         v_cache: torch.Tensor, block_tables: torch.Tensor,
                         context_lens: torch.Tensor, scale: float,
                         workspace: Optional[torch.Tensor] = None,
                         status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out, q: [S][H][D]; caches [N][H][B][D]; block_tables [S][max_blocks]
    int32; context_lens [S] int32."""
    S, H, D = q.shape
    N, H2, B, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or (H2, D2) != (H, D):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S][max_blocks], context_lens [S]")
    for t in (out, k_cache, v_cache):
        if t.dtype != q.dtype:
            raise TypeError("q, out and the caches must share a dtype")
    MB = block_tables.shape[1]
    if workspace is None:
        workspace = workspace_for(q, B, MB)
    code = lib().pa_paged_attn_decode(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
        _cuda(block_tables, "block_tables", torch.int32),
        _cuda(context_lens, "context_lens", torch.int32), float(scale), S, H, D, B, MB, N,
        _dtype_code(q), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _status_ptr(status), _stream(stream, q.device))
    _check(code, "pa_paged_attn_decode")
    return out


def pa_paged_attn_decode_gqa(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                             v_cache: torch.Tensor, block_tables: torch.Tensor,
                             context_lens: torch.Tensor, scale: float,
                             workspace: Optional[torch.Tensor] = None,
                             status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Grouped-query decode: out, q [S][H][D]; caches [N][H_kv][B][D] with H a
    multiple of H_kv (query head h reads key/value head h // (H / H_kv))."""
    S, H, D = q.shape
    N, Hkv, B, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or D2 != D or H % Hkv:
        raise ValueError("shape mismatch (num_heads must be a multiple of num_kv_heads)")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S][max_blocks], context_lens [S]")
    for t in (out, k_cache, v_cache):
        if t.dtype != q.dtype:
            raise TypeError("q, out and the caches must share a dtype")
    MB = block_tables.shape[1]
    if workspace is None:
        workspace = workspace_for(q, B, MB, Hkv)
    code = lib().pa_paged_attn_decode_gqa(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
        _cuda(block_tables, "block_tables", torch.int32),
        _cuda(context_lens, "context_lens", torch.int32), float(scale), S, H, Hkv, D, B, MB, N,
        _dtype_code(q), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _status_ptr(status), _stream(stream, q.device))
    _check(code, "pa_paged_attn_decode_gqa")
    return out


def pa_paged_attn_decode_shared_workspace_size(num_groups: int, group_size: int, num_heads: int,
                                               head_dim: int, block_size: int,
                                               max_prefix_blocks: int, max_tail_blocks: int,
                                               num_kv_heads: Optional[int] = None) -> int:
    if num_kv_heads is None or num_kv_heads == num_heads:
        return int(lib().pa_paged_attn_decode_shared_workspace_size(
            num_groups, group_size, num_heads, head_dim, block_size, max_prefix_blocks,
            max_tail_blocks))
    return int(lib().pa_paged_attn_decode_shared_gqa_workspace_size(
        num_groups, group_size, num_heads, num_kv_heads, head_dim, block_size,
        max_prefix_blocks, max_tail_blocks))


def pa_paged_attn_decode_shared(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                                v_cache: torch.Tensor, prefix_tables: torch.Tensor,
                                prefix_lens: torch.Tensor, tail_tables: torch.Tensor,
                                tail_lens: torch.Tensor, scale: float, group_size: int,
                                workspace: Optional[torch.Tensor] = None,
                                status: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
    """Decode for groups of ``group_size`` consecutive texts sharing a prefix:
    out, q [G*group_size][H][D]; caches [N][H_kv][B][D] (H_kv == H:
    multi-head; a divisor of H: grouped-query, pa_paged_attn_decode_shared_gqa);
    prefix_tables [G][max_prefix_blocks], prefix_lens [G]; tail_tables
    [G*group_size][max_tail_blocks], tail_lens [G*group_size] (int32)."""
    S, H, D = q.shape
    N, Hkv, B, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or D2 != D or H % Hkv:
        raise ValueError("shape mismatch (num_heads must be a multiple of num_kv_heads)")
    if group_size < 1 or S % group_size:
        raise ValueError("the number of texts must be a multiple of group_size")
    G = S // group_size
    if prefix_tables.dim() != 2 or prefix_tables.shape[0] != G or prefix_lens.shape != (G,):
        raise ValueError("prefix_tables must be [G][max_prefix_blocks], prefix_lens [G]")
    if tail_tables.dim() != 2 or tail_tables.shape[0] != S or tail_lens.shape != (S,):
        raise ValueError("tail_tables must be [S][max_tail_blocks], tail_lens [S]")
    for t in (out, k_cache, v_cache):
        if t.dtype != q.dtype:
            raise TypeError("q, out and the caches must share a dtype")
    MP, MT = prefix_tables.shape[1], tail_tables.shape[1]
    if workspace is None:
        need = pa_paged_attn_decode_shared_workspace_size(G, group_size, H, D, B, MP, MT, Hkv)
        if need == 0:
            raise PagedAttnError(PA_ERR_INVALID, "pa_paged_attn_decode_shared_workspace_size")
        key = (q.device.index if q.device.index is not None else torch.cuda.current_device(),
               need)
        workspace = _ws_cache.get(key)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
            _ws_cache[key] = workspace
    head = (_cuda(out, "out"), _cuda(q, "q"), _cuda(k_cache, "k_cache"),
            _cuda(v_cache, "v_cache"), _cuda(prefix_tables, "prefix_tables", torch.int32),
            _cuda(prefix_lens, "prefix_lens", torch.int32), MP,
            _cuda(tail_tables, "tail_tables", torch.int32),
            _cuda(tail_lens, "tail_lens", torch.int32), MT, float(scale), G, int(group_size), H)
    tail = (D, B, N, _dtype_code(q), _cuda(workspace, "workspace"),
            workspace.numel() * workspace.element_size(), _status_ptr(status),
            _stream(stream, q.device))
    if Hkv == H:
        _check(lib().pa_paged_attn_decode_shared(*head, *tail), "pa_paged_attn_decode_shared")
    else:
        _check(lib().pa_paged_attn_decode_shared_gqa(*head, Hkv, *tail),
               "pa_paged_attn_decode_shared_gqa")
    return out


def split_shared_prefix(block_tables: torch.Tensor, context_lens: torch.Tensor,
                        block_size: int, group_size: int, max_prefix_blocks: Optional[int] = None,
                        max_tail_blocks: Optional[int] = None):
    """Host: cut block tables of groups of ``group_size`` consecutive texts
    into (prefix_tables, prefix_lens, tail_tables, tail_lens), CPU int32
    tensors, with pa_split_shared_prefix."""
    bt = block_tables.detach().to("cpu", torch.int32).contiguous()
    cl = context_lens.detach().to("cpu", torch.int32).contiguous()
    S, MB = bt.shape
    if cl.shape != (S,) or group_size < 1 or S % group_size:
        raise ValueError("block_tables [S][max_blocks], context_lens [S], S % group_size == 0")
    MP = MB if max_prefix_blocks is None else int(max_prefix_blocks)
    MT = MB if max_tail_blocks is None else int(max_tail_blocks)
    G = S // group_size
    pt = torch.empty((G, MP), dtype=torch.int32)
    pl = torch.empty(G, dtype=torch.int32)
    tt = torch.empty((S, MT), dtype=torch.int32)
    tl = torch.empty(S, dtype=torch.int32)
    _check(lib().pa_split_shared_prefix(bt.data_ptr(), cl.data_ptr(), S, MB, int(block_size),
                                        int(group_size), pt.data_ptr(), MP, pl.data_ptr(),
                                        tt.data_ptr(), MT, tl.data_ptr()),
           "pa_split_shared_prefix")
    return pt, pl, tt, tl


def pa_decode_step(out: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   k_cache: torch.Tensor, v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                   block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                   workspace: Optional[torch.Tensor] = None,
                   status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Cache write of each text's new token plus decode attention, one launch.
    q, k, v, out: [S][H][D]; slot_mapping [S] int64 (the slot of position
    context_lens[s] - 1)."""
    S, H, D = q.shape
    N, H2, B, D2 = k_cache.shape
    if (out.shape != q.shape or k.shape != q.shape or v.shape != q.shape
            or v_cache.shape != k_cache.shape or (H2, D2) != (H, D)):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S][max_blocks], context_lens [S]")
    if slot_mapping.shape != (S,):
        raise ValueError("slot_mapping must be [num_seqs]")
    for t in (out, k, v, k_cache, v_cache):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, out and the caches must share a dtype")
    MB = block_tables.shape[1]
    if workspace is None:
        workspace = workspace_for(q, B, MB)
    code = lib().pa_decode_step(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), _cuda(k_cache, "k_cache"),
        _cuda(v_cache, "v_cache"), _cuda(slot_mapping, "slot_mapping", torch.int64),
        _cuda(block_tables, "block_tables", torch.int32),
        _cuda(context_lens, "context_lens", torch.int32), float(scale), S, H, D, B, MB, N,
        _dtype_code(q), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _status_ptr(status), _stream(stream, q.device))
    _check(code, "pa_decode_step")
    return out


def pa_decode_step_fp8(out: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                       k_cache: torch.Tensor, v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                       block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                       k_scale: float, v_scale: float, workspace: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """pa_decode_step over 8-bit caches [N][H][B][D] (uint8 codes): each
    text's new token is stored quantized and attended in one launch.
    q, k, v, out: [S][H][D] fp16/bf16; slot_mapping [S] int64."""
    S, H, D = q.shape
    N, H2, B, D2 = k_cache.shape
    if (out.shape != q.shape or k.shape != q.shape or v.shape != q.shape
            or v_cache.shape != k_cache.shape or (H2, D2) != (H, D)):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S][max_blocks], context_lens [S]")
    if slot_mapping.shape != (S,):
        raise ValueError("slot_mapping must be [num_seqs]")
    for t in (out, k, v):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v and out must share a dtype")
    MB = block_tables.shape[1]
    if workspace is None:
        workspace = workspace_for(q, B, MB)
    code = lib().pa_decode_step_fp8(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"),
        _codes(k_cache, "k_cache"), _codes(v_cache, "v_cache"),
        _cuda(slot_mapping, "slot_mapping", torch.int64),
        _cuda(block_tables, "block_tables", torch.int32),
        _cuda(context_lens, "context_lens", torch.int32), float(scale), float(k_scale),
        float(v_scale), S, H, D, B, MB, N, _dtype_code(q), _cuda(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _status_ptr(status),
        _stream(stream, q.device))
    _check(code, "pa_decode_step_fp8")
    return out


def pa_paged_attn_decode_noalloc(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                                 v_cache: torch.Tensor, block_tables: torch.Tensor,
                                 context_lens: torch.Tensor, scale: float,
                                 status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """pa_paged_attn_decode with the library's own static 16 MiB scratch: for
    callers that cannot allocate device memory.  Calls that may overlap on
    the GPU share that scratch and race.  Raises PagedAttnError with code
    PA_ERR_TOO_LARGE when the sizes need more scratch than it holds."""
    S, H, D = q.shape
    N, H2, B, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or (H2, D2) != (H, D):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S][max_blocks], context_lens [S]")
    for t in (out, k_cache, v_cache):
        if t.dtype != q.dtype:
            raise TypeError("q, out and the caches must share a dtype")
    code = lib().pa_paged_attn_decode_noalloc(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
        _cuda(block_tables, "block_tables", torch.int32),
        _cuda(context_lens, "context_lens", torch.int32), float(scale), S, H, D, B,
        block_tables.shape[1], N, _dtype_code(q), _status_ptr(status), _stream(stream, q.device))
    _check(code, "pa_paged_attn_decode_noalloc")
    return out


# aliases under the names the method's description uses
kv_cache_write = pa_kv_cache_write
paged_attn_decode = pa_paged_attn_decode


class BlockManager:
    """Host block manager (pa_bm_* in the C ABI)."""

    def __init__(self, num_blocks: int, block_size: int, shuffle_seed: int = 0):
        self._h = lib().pa_bm_create(int(num_blocks), int(block_size), int(shuffle_seed))
        if not self._h:
            raise PagedAttnError(PA_ERR_INVALID, "pa_bm_create")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id: int, num_tokens: int) -> None:
        _check(lib().pa_bm_add_seq(self._h, int(seq_id), int(num_tokens)), "pa_bm_add_seq")

    def add_seq_tokens(self, seq_id: int, tokens: Sequence[int]) -> int:
        """A new text from its prompt's token ids, taking over cached blocks
        of an earlier text that began the same way.  Returns the number of
        leading tokens whose blocks were taken over."""
        t = torch.tensor(list(tokens), dtype=torch.int32)
        cached = ctypes.c_int(0)
        _check(lib().pa_bm_add_seq_tokens(self._h, int(seq_id), t.data_ptr() if t.numel() else None,
                                          int(t.numel()), ctypes.byref(cached)),
               "pa_bm_add_seq_tokens")
        return cached.value

    def num_cached_blocks(self) -> int:
        return int(lib().pa_bm_num_cached_blocks(self._h))

    def fork(self, parent: int, child: int) -> None:
        _check(lib().pa_bm_fork(self._h, int(parent), int(child)), "pa_bm_fork")

    def append_slot(self, seq_id: int) -> Tuple[int, int, int]:
        slot = ctypes.c_int64()
        src = ctypes.c_int32()
        dst = ctypes.c_int32()
        _check(lib().pa_bm_append_slot(self._h, int(seq_id), ctypes.byref(slot), ctypes.byref(src),
                                       ctypes.byref(dst)), "pa_bm_append_slot")
        return slot.value, src.value, dst.value

    def free_seq(self, seq_id: int) -> None:
        _check(lib().pa_bm_free_seq(self._h, int(seq_id)), "pa_bm_free_seq")

    def num_free(self) -> int:
        return int(lib().pa_bm_num_free(self._h))

    def refcount(self, block: int) -> int:
        r = lib().pa_bm_refcount(self._h, int(block))
        if r < 0:
            raise PagedAttnError(r, "pa_bm_refcount")
        return r

    def num_tokens(self, seq_id: int) -> int:
        r = int(lib().pa_bm_num_tokens(self._h, int(seq_id)))
        if r < 0:
            raise PagedAttnError(r, "pa_bm_num_tokens")
        return r

    def export(self, seq_ids: Sequence[int], max_blocks_per_seq: int):
        """(block_tables [n][max_blocks] int32, context_lens [n] int32) as CPU tensors."""
        n = len(seq_ids)
        ids = torch.tensor(list(seq_ids), dtype=torch.int64)
        tables = torch.empty((n, max_blocks_per_seq), dtype=torch.int32)
        lens = torch.empty(n, dtype=torch.int32)
        _check(lib().pa_bm_export(self._h, ids.data_ptr(), n, tables.data_ptr(),
                                  int(max_blocks_per_seq), lens.data_ptr()), "pa_bm_export")
        return tables, lens
