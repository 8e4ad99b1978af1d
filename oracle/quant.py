"""Oracle: int4 group quantization and FP8 (e4m3) row quantization.

TEST INFRASTRUCTURE ONLY (see the package docstring).
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# int4, groups of 128 along the last axis
# ---------------------------------------------------------------------------


def int4_row_quantize(w: np.ndarray, group_size: int = 128):
    """Quantize fp32 ``w[..., K]`` to int4 codes with one fp32 scale per group.

    Follows [P1] "FP8 / Int4 混合量化" (the int4_row_quantize listing), step
    by step in the pages' order, in fp32 as the listing's tensors are:
      1. view w as rows of ``group_size`` consecutive elements of the last axis;
      2. m = max |w| over the group;
      3. scale = max(m, 1e-6) / 8            (1e-6 as an fp32 constant);
      4. q = clamp(round(w / scale), -8, 7)  (IEEE fp32 division, round half
         to even as torch's ``round`` does; the asymmetric clamp is kept);
      5. return q as int8 and the scales.
    Returns (q int8 [..., K], scales fp32 [..., K // group_size]).
    """
    w = np.asarray(w, dtype=np.float32)
    K = w.shape[-1]
    if K % group_size:
        raise ValueError("last dimension %d is not a multiple of %d" % (K, group_size))
    groups = w.reshape(-1, group_size)
    m = np.abs(groups).max(axis=1, keepdims=True)
    scales = np.maximum(m, np.float32(1e-6)) / np.float32(8.0)
    q = np.clip(np.rint(groups / scales), -8, 7).astype(np.int8)
    return q.reshape(w.shape), scales.reshape(w.shape[:-1] + (K // group_size,))


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Two codes per byte: byte j = (q[2j] & 0xF) | (q[2j+1] & 0xF) << 4.

    Reading (the pages return unpacked int8): two's-complement nibbles, the
    even K index in the low nibble.
    """
    q = np.asarray(q, dtype=np.int8)
    if q.shape[-1] % 2:
        raise ValueError("odd number of codes")
    lo = q[..., 0::2].astype(np.uint8) & 0xF
    hi = q[..., 1::2].astype(np.uint8) & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(codes: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_int4`: uint8 [..., K/2] -> int8 [..., K]."""
    codes = np.asarray(codes, dtype=np.uint8)
    lo = (codes & 0xF).astype(np.int16)
    hi = (codes >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def dequant_int4(q: np.ndarray, scales: np.ndarray, group_size: int = 128) -> np.ndarray:
    """w_hat = q * scale, zero point 0 ([P2] "量化环节做了什么": the int4
    matmul is given zeros_like(scale) as its zero points).  fp64 result."""
    q = np.asarray(q, dtype=np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float64), group_size, axis=-1)
    return q * s


# ---------------------------------------------------------------------------
# FP8 e4m3 ("fn": no infinities, 0x7F / 0xFF are NaN, largest finite 448)
# ---------------------------------------------------------------------------


def _e4m3_table() -> np.ndarray:
    """Value of every e4m3 code (fp64), from the format's definition:
    sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
    holds subnormals m/8 * 2^-6; S.1111.111 is NaN."""
    vals = np.empty(256, dtype=np.float64)
    for c in range(256):
        sign = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


E4M3_VALUES = _e4m3_table()
E4M3_MAX = 448.0
_POS = E4M3_VALUES[:0x7F]          # codes 0x00..0x7E, strictly increasing


def fp8_e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Encode finite values to e4m3: nearest representable value, ties to the
    code with an even mantissa, magnitudes beyond 448 saturate to 448, the sign
    bit copied from the input (so -0 and tiny negatives give 0x80)."""
    x = np.asarray(x)
    a = np.abs(x.astype(np.float64))
    hi = np.searchsorted(_POS, a, side="left").clip(0, len(_POS) - 1)
    lo = (hi - 1).clip(0, None)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 0x7E, code).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << 7
    return (code | sign).astype(np.uint8)


def fp8_e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


def fp8_row_quantize(x: np.ndarray, num_valid_rows: int | None = None,
                     scale_ub: float = float("inf")):
    """Per-row FP8 quantization of ``x[R, C]`` (bf16 or fp32 values).

    [P2] "量化环节做了什么" names the operation (quantize_fp8_per_row with a
    valid-row count and an activation-scale upper bound) but not its formula.
    Reading, in fp32 (the kernel's precision, so both sides take the same
    rounding decisions):
      a = min(max_c |x[r, c]|, scale_ub);  s = max(a, 1e-12) / 448;
      q = e4m3(x / s) with IEEE division, round to nearest even, saturating;
      rows r >= num_valid_rows get q = 0 and s = 0.
    Returns (q uint8 [R, C], s fp32 [R]).
    """
    xf = np.asarray(x, dtype=np.float32)
    R = xf.shape[0]
    nv = R if num_valid_rows is None else int(num_valid_rows)
    a = np.abs(xf).max(axis=1) if xf.shape[1] else np.zeros(R, np.float32)
    a = np.minimum(a, np.float32(scale_ub))
    s = np.maximum(a, np.float32(1e-12)) / np.float32(E4M3_MAX)
    q = fp8_e4m3_encode(xf / s[:, None])
    q[nv:] = 0
    s = s.astype(np.float32)
    s[nv:] = 0.0
    return q, s


def dequant_fp8_rows(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """w_hat[r, c] = e4m3_value(q[r, c]) * s[r] in fp64."""
    return fp8_e4m3_decode(q) * np.asarray(s, dtype=np.float64)[:, None]
