"""FP64 decoding of NVFP4 expert weights (test infrastructure, part of the oracle).

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
"""
from __future__ import annotations

import numpy as np

__all__ = ["decode_e2m1", "decode_e4m3", "unpack_nibbles", "dequantize_nvfp4", "NVFP4_BYTES_PER_WEIGHT"]

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
    """FP64 weights [out, in] of one matrix from its codes, block scales and matrix scale."""
    vals = decode_e2m1(unpack_nibbles(codes))
    blk = np.repeat(decode_e4m3(scales), 16, axis=-1)
    return vals * blk * float(matrix_scale)
