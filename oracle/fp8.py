"""CPU oracle: the 8-bit floating-point KV cache (E4M3), exact.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT (see oracle/__init__.py).

"The KV Cache and PagedAttention", §What Came After: storing each cached
number in 8 bits instead of 16 halves the cache, so about twice the tokens
fit.  The pages fix neither the format nor the scaling; the readings here
(also in the design notes):
  * format E4M3 with finite values only: 1 sign bit, 4 exponent bits (bias
    7), 3 mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6;
    the all-ones code S.1111.111 is NaN and there are no infinities, so the
    largest finite magnitude is 1.75 * 2^8 = 448;
  * one fp32 scale per cache tensor (k_scale, v_scale): a stored code c
    stands for value(c) * scale;
  * a new key or value x (fp16/bf16) is stored as the code nearest to the
    fp32 quotient x / scale (IEEE division in fp32), ties to the even code,
    magnitudes past 448 saturating to 448, NaN to NaN (0x7F);
  * decode attention over such a cache is the plain attention of
    paged_attention.py over the dequantized values value(c) * scale.

Pinned by tests/test_oracle.py: torch's float8_e4m3fn cast (an independent
implementation) on every fp16 value and on random fp32 within range; the
format's closed-form constants (448, 2^-6, 2^-9, the NaN codes); saturation
and signed zeros; and attention over a cache whose values are exactly
representable, which must equal attention over the same values in fp16.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from .paged_attention import paged_decode

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """The number an E4M3 code stands for (NaN for S.1111.111)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


# All 128 non-negative codes and their values; the finite ones (0x00-0x7E)
# increase strictly with the code.
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = np.array([e4m3_value(c) for c in _POS_CODES], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Values (fp64) of an array of uint8 codes."""
    table = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """uint8 codes of the values x (fp32 or wider; each value taken exactly):
    round to nearest, ties to the even code, saturating past 448, NaN to
    0x7F, sign kept (so -0.0 is 0x80)."""
    x = np.asarray(x, dtype=np.float64)
    nan = np.isnan(x)
    sign = np.where(np.signbit(x), 0x80, 0).astype(np.int64)
    a = np.minimum(np.abs(np.where(nan, 0.0, x)), E4M3_MAX)
    # neighbouring codes: hi = first code whose value is >= a, lo = the one below
    hi = np.searchsorted(_POS_VALUES, a, side="left")
    lo = np.maximum(hi - 1, 0)
    exact = _POS_VALUES[hi] == a
    d_lo = a - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - a
    take_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(exact, hi, np.where(take_lo, lo, hi))
    out = (sign | code).astype(np.uint8)
    out[nan] = 0x7F
    return out


def quantize(x: np.ndarray, scale: float) -> np.ndarray:
    """Codes for fp16/bf16 values x (given as their exact fp32 values): the
    fp32 quotient x / scale, then e4m3_encode."""
    q = np.asarray(x, dtype=np.float32) / np.float32(scale)
    return e4m3_encode(q.astype(np.float32))


def cache_write_fp8(k_cache: np.ndarray, v_cache: np.ndarray, k: np.ndarray, v: np.ndarray,
                    slot_mapping: Sequence[int], block_size: int, k_scale: float,
                    v_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Copies of the uint8 code pools ``[N][H][B][D]`` with token t's key and
    value, quantized, at slot ``slot_mapping[t]`` (negative: skipped).  k, v
    are ``[T][H][D]`` exact fp32 values of the fp16/bf16 inputs."""
    kc = k_cache.copy()
    vc = v_cache.copy()
    for t, slot in enumerate(slot_mapping):
        slot = int(slot)
        if slot < 0:
            continue
        block, place = divmod(slot, block_size)
        kc[block, :, place, :] = quantize(k[t], k_scale)
        vc[block, :, place, :] = quantize(v[t], v_scale)
    return kc, vc


def paged_decode_fp8(q, k_codes, v_codes, block_tables, context_lens, scale, block_size,
                     k_scale, v_scale, pairs=None) -> np.ndarray:
    """Decode attention over E4M3 caches: the plain paged attention over the
    dequantized pools value(code) * scale, fp64."""
    kd = e4m3_decode(k_codes) * float(np.float32(k_scale))
    vd = e4m3_decode(v_codes) * float(np.float32(v_scale))
    return paged_decode(q, kd, vd, block_tables, context_lens, scale, block_size, pairs)
