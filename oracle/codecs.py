"""Low-precision read-copy codecs (oracle; test infrastructure).

[summary ¶4]: ReplaySSM keeps a high-precision checkpoint for the recurrence
and a low-precision copy of it for reads, and reports NVFP4 reads on top of a
higher-precision recurrence.  The pages give no block format, so the two read
copies are read as follows:

* FP8 row copy: for each row r (the contraction vector of one output element)
  s_r = amax_r / 448 in fp32, code = E4M3_RNE_satfinite(x / s_r) in fp32;
  an all-zero row has s_r = 0 and all codes 0.  Value = E4M3(code) * s_r.
* NVFP4 copy: for each block of 16 consecutive elements of a row
  s_b = E4M3_RNE_satfinite(amax_b / 6) (an E4M3 code), code =
  E2M1_RNE_satfinite(x / E4M3(s_b)); when s_b decodes to 0 the whole block is
  coded 0.  Value = E2M1(code) * E4M3(s_b).  No second per-tensor scale.

Every division and rounding decision is taken in fp32 (the precision the
kernel takes it in) so that codes can be compared bit for bit.

Element formats (OCP "8-bit Floating Point Specification (OFP8)" E4M3 and
OCP "Microscaling Formats (MX) Specification v1.0" FP4 E2M1):
* E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities; only
  S.1111.111 is NaN; largest finite 448; subnormals m/8 * 2^-6.
* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; magnitudes
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no NaN or infinity.
Encoders round to nearest with ties to the even code (even mantissa), clamp
finite overflow to the largest finite magnitude (satfinite) and keep the sign
of the input (a negative value that rounds to zero becomes -0).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def _e4m3_magnitudes() -> np.ndarray:
    """Values of the 127 finite non-negative codes 0x00..0x7E, increasing."""
    vals = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        vals.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


def _e2m1_magnitudes() -> np.ndarray:
    """Values of the 8 non-negative codes 0x0..0x7, increasing."""
    vals = []
    for c in range(8):
        e, m = c >> 1, c & 1
        vals.append(m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1))
    return np.array(vals, dtype=np.float64)


E4M3_VALUES = _e4m3_magnitudes()
E2M1_VALUES = _e2m1_magnitudes()


def _round_to_table(a: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest table entry to each a >= 0, ties to the even index."""
    idx = np.searchsorted(table, a, side="left")
    idx = np.clip(idx, 1, len(table) - 1)
    lo, hi = table[idx - 1], table[idx]
    dlo, dhi = a - lo, hi - a
    lower_even = ((idx - 1) % 2) == 0
    return np.where(dlo < dhi, idx - 1,
                    np.where(dlo > dhi, idx, np.where(lower_even, idx - 1, idx)))


def e4m3_encode(x) -> np.ndarray:
    """fp32/fp64 values -> E4M3 codes (uint8), RNE, satfinite, sign kept."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    code = _round_to_table(np.minimum(a, E4M3_MAX), E4M3_VALUES)
    sign = np.signbit(x).astype(np.int64)
    return (code.astype(np.int64) | (sign << 7)).astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    mag = E4M3_VALUES[np.minimum(code & 0x7F, 0x7E)]
    mag = np.where((code & 0x7F) == 0x7F, np.nan, mag)
    return np.where(code & 0x80, -mag, mag)


def e2m1_encode(x) -> np.ndarray:
    """fp32/fp64 values -> E2M1 codes (uint8 0..15), RNE, satfinite, sign kept."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    code = _round_to_table(np.minimum(a, E2M1_MAX), E2M1_VALUES)
    sign = np.signbit(x).astype(np.int64)
    return (code.astype(np.int64) | (sign << 3)).astype(np.uint8)


def e2m1_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    mag = E2M1_VALUES[code & 7]
    return np.where(code & 8, -mag, mag)


def fp8_row_quantize(rows):
    """rows [..., n] fp32 -> (codes uint8 [..., n], scales fp32 [...])."""
    r = np.asarray(rows, dtype=np.float32)
    amax = np.max(np.abs(r), axis=-1)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (r / s[..., None]).astype(np.float32)
    codes = e4m3_encode(q)
    codes = np.where((s == 0)[..., None], np.uint8(0), codes).astype(np.uint8)
    return codes, s


def fp8_row_dequantize(codes, scales) -> np.ndarray:
    return e4m3_decode(codes) * np.asarray(scales, np.float64)[..., None]


def nvfp4_quantize(rows):
    """rows [..., n] fp32, n % 16 == 0 -> (codes uint8 [..., n] (0..15),
    block scale codes uint8 [..., n/16] (E4M3))."""
    r = np.asarray(rows, dtype=np.float32)
    n = r.shape[-1]
    if n % 16:
        raise ValueError("row length must be a multiple of 16")
    blk = r.reshape(r.shape[:-1] + (n // 16, 16))
    amax = np.max(np.abs(blk), axis=-1)
    s_code = e4m3_encode((amax / np.float32(E2M1_MAX)).astype(np.float32))
    s_val = e4m3_decode(s_code).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (blk / s_val[..., None]).astype(np.float32)
    codes = e2m1_encode(q)
    codes = np.where((s_val == 0)[..., None], np.uint8(0), codes).astype(np.uint8)
    return codes.reshape(r.shape), s_code


def nvfp4_dequantize(codes, scale_codes) -> np.ndarray:
    codes = np.asarray(codes)
    n = codes.shape[-1]
    vals = e2m1_decode(codes).reshape(codes.shape[:-1] + (n // 16, 16))
    return (vals * e4m3_decode(scale_codes)[..., None]).reshape(codes.shape)
