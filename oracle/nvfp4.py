"""FP64 decoding of NVFP4 expert weights and the NVFP4 activation quantiser (test
infrastructure, part of the oracle).

Storage, per expert matrix W[e] of shape [out, in] (Muse Spark Open deep dive, §7.3 bytes
bullet and §7.4 NVFP4 paragraph: 4-bit values, one FP8 E4M3 scale per 16 weights,
0.5625 bytes per weight):
  * codes  uint8 [out, in/2], two 4-bit values per byte, the low nibble holding the even
    element;
  * scales uint8 [out, in/16], one E4M3 byte per block of 16 consecutive weights of a row;
  * one float32 scale per matrix.
The weight is decode_e2m1(code) * decode_e4m3(scale) * matrix_scale.

The 4-bit value is FP4 E2M1 of the OCP Microscaling (MX) formats specification v1.0: sign,
2 exponent bits with bias 1, 1 mantissa bit, subnormal when the exponent is 0, no infinities
or NaN. E4M3 (deep dive §7.4: 4 exponent bits, 3 mantissa bits) is the OCP 8-bit float of
the same specification: bias 7, subnormal when the exponent is 0, S.1111.111 is NaN, no
infinities, largest value 448.

Activations of the W4A4 mode (deep dive §7.4: the released checkpoint quantises both
operands of the expert GEMMs) use the same element and block formats without a tensor
scale: per block of 16 consecutive values of a row, scale = E4M3(amax / 6) (amax / 6 one
float32 division, as the kernels do it) and code = the E2M1 value nearest to the exact
quotient value / scale, both with ties to even, E2M1 saturating at 6. The quotient is taken
in float64, which orders it exactly against the E2M1 midpoints: scale has 4 significant
bits, so a value that is not exactly a midpoint times scale differs from it by at least one
float32 unit, far more than float64 rounding.
"""
from __future__ import annotations

import numpy as np

__all__ = ["decode_e2m1", "decode_e4m3", "unpack_nibbles", "dequantize_nvfp4", "NVFP4_BYTES_PER_WEIGHT",
           "round_e4m3", "round_e2m1", "quantize_activations_nvfp4", "dequantize_activations_nvfp4"]

# 4 bits per value plus one byte per 16 values
NVFP4_BYTES_PER_WEIGHT = 0.5 + 1.0 / 16.0


def decode_e2m1(code) -> np.ndarray:
    """Value of 4-bit E2M1 codes (any integer array with values 0..15)."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where((c >> 3) & 1, -1.0, 1.0)
    e = (c >> 1) & 3
    m = (c & 1).astype(np.float64)
    mag = np.where(e == 0, m * 0.5, np.exp2(e - 1.0) * (1.0 + m / 2.0))
    return sign * mag


def decode_e4m3(byte) -> np.ndarray:
    """Value of E4M3 bytes (NaN for S.1111.111)."""
    b = np.asarray(byte, dtype=np.int64)
    sign = np.where((b >> 7) & 1, -1.0, 1.0)
    e = (b >> 3) & 15
    m = (b & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, np.exp2(e - 7.0) * (1.0 + m / 8.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def unpack_nibbles(packed) -> np.ndarray:
    """[..., n/2] bytes -> [..., n] codes, low nibble first."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


def dequantize_nvfp4(codes, scales, matrix_scale) -> np.ndarray:
    """FP64 weights [out, in] of one matrix from its codes, block scales and matrix scale.

    The decoders are applied through tables of their values on every code and byte (the
    same numbers, looked up instead of recomputed per element, so a full-size layer
    decodes in seconds). The three factors have 3, 4 and 24 significant bits, so their
    product is exact in float64 whatever the order of the multiplications."""
    vals = _E2M1_ALL[unpack_nibbles(codes)]
    rows, n = vals.shape[:-1], vals.shape[-1]
    blk = _E4M3_ALL[np.asarray(scales, dtype=np.uint8)] * float(matrix_scale)
    return (vals.reshape(rows + (n // 16, 16)) * blk[..., None]).reshape(rows + (n,))


# every code's and every byte's value: decode_e2m1 on 0..15, decode_e4m3 on 0..255
_E2M1_ALL = decode_e2m1(np.arange(16))
_E4M3_ALL = decode_e4m3(np.arange(256))
# the 127 finite non-negative E4M3 values in byte order (bytes 0x00 .. 0x7E), increasing
_E4M3_POS = decode_e4m3(np.arange(127))
# the 8 E2M1 magnitudes in code order (codes 0 .. 7), increasing
_E2M1_POS = decode_e2m1(np.arange(8))


def _nearest_even(table: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Index of the entry of the increasing table nearest to each v >= 0 (ties to the
    even index, values past the end to the last entry)."""
    v = np.asarray(v, dtype=np.float64)
    hi = np.clip(np.searchsorted(table, v, side="left"), 1, len(table) - 1)
    lo = hi - 1
    dl, dh = v - table[lo], table[hi] - v
    pick = np.where(dl < dh, lo, np.where(dh < dl, hi, np.where(lo % 2 == 0, lo, hi)))
    return np.where(v >= table[-1], len(table) - 1, pick)


def round_e4m3(v) -> np.ndarray:
    """E4M3 byte nearest to each non-negative value (ties to even, saturating at 448)."""
    return _nearest_even(_E4M3_POS, v).astype(np.uint8)


def round_e2m1(q) -> np.ndarray:
    """4-bit E2M1 code nearest to each value (ties to even, saturating at +-6); the sign
    bit is set only for a negative value whose magnitude code is not 0."""
    q = np.asarray(q, dtype=np.float64)
    mag = _nearest_even(_E2M1_POS, np.abs(q)).astype(np.uint8)
    return np.where((q < 0) & (mag > 0), mag | 8, mag).astype(np.uint8)


def quantize_activations_nvfp4(x, ref=None, rel_tol: float = 2.0 ** -7, adopted=None):
    """Rows [..., n] (n a multiple of 16; values exactly representable in float32) ->
    (codes uint8 [..., n/2] low nibble first, scales uint8 E4M3 [..., n/16]).

    ref: optional (codes, scales) of the same rows from another implementation whose input
    may differ from x by accumulation-order rounding. Where a decision of ref differs from
    this one, it is adopted only if this input lies within rel_tol (relative) of the rounding
    boundary between the two neighbouring values -- for a scale, amax / 6 near the midpoint of
    two adjacent E4M3 values; for a code, value / scale near the midpoint of two adjacent E2M1
    values of the same sign -- since then both decisions are correct for inputs that close;
    any other difference raises ValueError. adopted (a one-element list) counts adoptions."""
    x32 = np.asarray(x, dtype=np.float32)
    blocks = x32.reshape(x32.shape[:-1] + (x32.shape[-1] // 16, 16))
    amax = np.max(np.abs(blocks), axis=-1)                          # exact
    s = (amax / np.float32(6.0)).astype(np.float32)                  # one float32 division
    sbyte = round_e4m3(s.astype(np.float64))
    if ref is not None:
        rs = np.asarray(ref[1], dtype=np.uint8).reshape(sbyte.shape)
        diff = rs != sbyte
        if diff.any():
            mid = (decode_e4m3(rs[diff]) + decode_e4m3(sbyte[diff])) / 2.0
            sv = s[diff].astype(np.float64)
            near = (np.abs(rs[diff].astype(int) - sbyte[diff].astype(int)) == 1) & (np.abs(sv - mid) <= rel_tol * sv)
            if not near.all():
                raise ValueError(f"{int((~near).sum())} scale bytes differ away from a rounding boundary")
            sbyte = np.where(diff, rs, sbyte)
            if adopted is not None:
                adopted[0] += int(diff.sum())
    sdec = decode_e4m3(sbyte)                                        # exact
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(sdec[..., None] > 0, blocks.astype(np.float64) / sdec[..., None], 0.0)
    codes = round_e2m1(q).reshape(x32.shape)
    if ref is not None:
        rc = unpack_nibbles(np.asarray(ref[0], dtype=np.uint8)).reshape(codes.shape)
        diff = rc != codes
        if diff.any():
            qd = q.reshape(codes.shape)[diff]
            a, b = codes[diff].astype(int), rc[diff].astype(int)
            same_side = ((a & 8) == (b & 8)) | ((a & 7) == 0) | ((b & 7) == 0)
            adjacent = same_side & (np.abs((a & 7) - (b & 7)) == 1)
            mid = (np.abs(decode_e2m1(a)) + np.abs(decode_e2m1(b))) / 2.0
            near = adjacent & (np.abs(np.abs(qd) - mid) <= rel_tol * np.abs(qd))
            if not near.all():
                raise ValueError(f"{int((~near).sum())} codes differ away from a rounding boundary")
            codes = np.where(diff, rc, codes)
            if adopted is not None:
                adopted[0] += int(diff.sum())
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, sbyte


def dequantize_activations_nvfp4(codes, scales) -> np.ndarray:
    """FP64 values [..., n] of quantised activations."""
    vals = decode_e2m1(unpack_nibbles(codes))
    return vals * np.repeat(decode_e4m3(scales), 16, axis=-1)
