"""NVFP4 two-level quantiser, plain NumPy (test infrastructure: part of the oracle).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the GPU library never does, and this file
shares no code with it.

What it computes (the FFN-down workload's quantisation: each run of 16 elements
gets an E4M3 scale from its largest magnitude over 6, and the tensor an FP32
scale from its largest magnitude over 6 x 448; in the two-level reading the block
scale is taken relative to the per-tensor scale).
The pages fix FP32 for the per-tensor scale, so every step below is an IEEE
FP32 operation, round to nearest even, in this order:

    x      = the BF16 input, widened to FP32 (exact)
    amax   = max |x| over the tensor                         (exact)
    g      = amax / 2688            (6 * 448 = 2688; g = 1 when amax = 0)
    for each block b of 16 consecutive k of a row:
      amax_b = max |x| over the block                        (exact)
      q      = amax_b / (6 * g)     (the product 6 * g rounded first)
      s_b    = the E4M3 byte nearest to q, ties to the even mantissa, values
               above 448 giving 448 (satfinite); s = its value
      den    = s * g
      t      = x / den              (not formed when den = 0: t = +-0, x's sign)
      code   = sign(t) << 3 | the E2M1 magnitude nearest to |t|, ties to the
               even mantissa, values above 6 giving 6 (satfinite)

The E4M3 and E2M1 value tables come from the oracle's field-definition decoders
(``oracle.e4m3_value``, ``oracle.e2m1_value``).  Layouts as everywhere: packed
codes ``uint8[rows, K/2]`` (even k in the low nibble), scales ``uint8[rows, K/16]``.
"""
from __future__ import annotations

import functools

import numpy as np

from . import e2m1_value, e4m3_value

F32 = np.float32
E4M3_SAT_BYTE = 0x7E  # 448, the largest finite E4M3 value


@functools.lru_cache(maxsize=None)
def _tables():
    e4 = np.array([e4m3_value(b) for b in range(0x7F)], dtype=np.float64)  # 0x00..0x7E
    e2 = np.array([e2m1_value(c) for c in range(8)], dtype=np.float64)     # 0, .5, ..., 6
    return e4, e2


def nearest_even(a: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Index of the entry of the increasing table `values` nearest to each a >= 0;
    ties go to the even index (the even mantissa: both tables step the mantissa
    by one per index); a above the last entry gives the last index."""
    a = np.asarray(a, dtype=np.float64)
    hi = np.searchsorted(values, a, side="left")          # values[hi-1] < a <= values[hi]
    hi = np.clip(hi, 1, len(values) - 1)
    lo = hi - 1
    d_lo = a - values[lo]
    d_hi = values[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(a >= values[-1], len(values) - 1, idx)
    idx = np.where(a <= values[0], 0, idx)
    return idx.astype(np.int64)


def e4m3_rne_satfinite(q: np.ndarray) -> np.ndarray:
    """Non-negative FP32 -> E4M3 byte (nearest, ties to even, saturating at 448)."""
    e4, _ = _tables()
    return nearest_even(q, e4).astype(np.uint8)


def e2m1_rne_satfinite(t: np.ndarray) -> np.ndarray:
    """FP32 -> 4-bit E2M1 code: the nearest magnitude (ties to even, saturating at 6)
    with t's sign bit (so -0 and small negatives that round to zero give code 8)."""
    t = np.asarray(t, dtype=F32)
    _, e2 = _tables()
    mag = nearest_even(np.abs(t), e2).astype(np.uint8)
    return mag | (np.signbit(t).astype(np.uint8) << 3)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(F32)


def quantize_nvfp4_bf16(x_bits: np.ndarray, amax=None):
    """Quantise a BF16 matrix (uint16 bit patterns [rows, K], K % 16 == 0).

    `amax` is the tensor's max |x| when these rows are a sample of a larger
    tensor (None: taken over these rows).
    Returns (packed codes uint8[rows, K/2], scales uint8[rows, K/16], g as FP32)."""
    bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, K = bits.shape
    if K % 16 != 0:
        raise ValueError("K must be a multiple of 16")
    x = bf16_to_f32(bits)
    if amax is None:
        amax = F32(np.max(np.abs(x))) if x.size else F32(0.0)
    amax = F32(amax)
    g = F32(amax / F32(2688.0)) if amax > 0 else F32(1.0)
    xb = x.reshape(rows, K // 16, 16)
    amax_b = np.max(np.abs(xb), axis=2).astype(F32) if x.size else np.zeros((rows, K // 16), F32)
    q = (amax_b / F32(F32(6.0) * g)).astype(F32)
    s_bytes = e4m3_rne_satfinite(q)
    e4, _ = _tables()
    s = e4[s_bytes.astype(np.int64)].astype(F32)
    den = (s * g).astype(F32)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(den > 0, xb / np.where(den > 0, den, F32(1.0)), xb * F32(0.0)).astype(F32)
    codes = e2m1_rne_satfinite(t).reshape(rows, K)
    packed = np.ascontiguousarray(codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, np.ascontiguousarray(s_bytes), g
