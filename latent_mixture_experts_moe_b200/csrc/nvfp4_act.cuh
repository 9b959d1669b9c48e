// nvfp4_act.cuh -- NVFP4 quantisation of the expert GEMMs' activation operands (W4A4 mode).
//
// The released checkpoint quantises both operands of the expert GEMMs (Muse Spark Open deep
// dive §7.4): per block of 16 consecutive values of a row, one E4M3 scale and sixteen 4-bit
// E2M1 codes (OCP Microscaling formats v1.0). Here, with no tensor-wide scale:
//   scale = E4M3(amax / 6), code_i = the E2M1 value nearest to the exact quotient v_i / scale
// both with ties to even, E2M1 saturating at +-6; amax / 6 is one IEEE float32 division on
// the float32 values of the stored bfloat16 activation. The code needs no division: the
// rounding boundaries of v / scale are the E2M1 midpoints t times scale, products of at most
// 3 and 4 significant bits and so exact in float32, and |v| is compared with them. Codes
// are packed two per byte, the low nibble holding the even element, the same packing as the
// NVFP4 expert weights.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace muse {

// Exact value of an E4M3 byte (bias 7, subnormal when the exponent field is 0; the NaN
// pattern S.1111.111 decodes to NaN).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v;
  if (e == 15u && m == 7u) {
    v = __int_as_float(0x7FC00000);
  } else if (e == 0u) {
    v = static_cast<float>(m) * 0.001953125f;  // m * 2^-9
  } else {
    v = __int_as_float(static_cast<int>(((e + 120u) << 23) | (m << 20)));
  }
  return (b & 0x80u) ? -v : v;
}

// One block of 16 bf16 values, given as 8 packed pairs, -> 8 code bytes (two words, element
// 2i in the low nibble of byte i) and the E4M3 scale byte. A code's magnitude index counts the
// E2M1 midpoints t = 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 (between the magnitudes 0, 0.5, 1,
// 1.5, 2, 3, 4, 6) below |v| / s, a value exactly on a midpoint going to the neighbour with an
// even index; the sign bit is set only on a nonzero magnitude. Two values per instruction: |v| and
// the boundaries t * s are compared as bf16 pairs (exact: v is bf16, and t * s has at most
// 3 + 4 significant bits), the comparison results (1.0 or 0.0) summed as bf16 pairs, and
// each count k (0..7) read from the bits of k + 128.0 (= 2^7 (1 + k / 128): k is the low
// mantissa bits).
__device__ __forceinline__ void quant_block16_bf16(const uint32_t (&w)[8], uint2& codes, uint32_t& sbyte) {
  __nv_bfloat162 mx = __floats2bfloat162_rn(0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a = w[i] & 0x7FFF7FFFu;
    mx = __hmax2(mx, *reinterpret_cast<const __nv_bfloat162*>(&a));
  }
  const float amax = fmaxf(__low2float(mx), __high2float(mx));
  sbyte = f32_to_e4m3_rn_satfinite(amax / 6.0f);
  const float s = e4m3_to_f32(sbyte);
  uint32_t out[2] = {0u, 0u};
  if (s > 0.0f) {
    const float t[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
    __nv_bfloat162 b[7];
#pragma unroll
    for (int j = 0; j < 7; ++j) b[j] = __float2bfloat162_rn(t[j] * s);  // exact
    const __nv_bfloat162 bias = __float2bfloat162_rn(128.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t au = w[i] & 0x7FFF7FFFu;
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&au);
      // midpoints with an even upper neighbour (0.75, 1.75, 3.5) count at equality
      __nv_bfloat162 cnt = __hadd2(__hgt2(a, b[0]), __hge2(a, b[1]));
      cnt = __hadd2(cnt, __hgt2(a, b[2]));
      cnt = __hadd2(cnt, __hge2(a, b[3]));
      cnt = __hadd2(cnt, __hgt2(a, b[4]));
      cnt = __hadd2(cnt, __hge2(a, b[5]));
      cnt = __hadd2(cnt, __hgt2(a, b[6]));
      const __nv_bfloat162 kb = __hadd2(cnt, bias);
      const uint32_t k2 = *reinterpret_cast<const uint32_t*>(&kb);
      const uint32_t k_lo = k2 & 7u, k_hi = (k2 >> 16) & 7u;
      const uint32_t c_lo = k_lo | (((w[i] >> 15) & 1u) && k_lo ? 8u : 0u);
      const uint32_t c_hi = k_hi | ((w[i] >> 31) && k_hi ? 8u : 0u);
      out[i >> 2] |= (c_lo | (c_hi << 4)) << (8 * (i & 3));
    }
  }
  codes = make_uint2(out[0], out[1]);
}

// Quantise rows of bf16 activations of K values (K a multiple of 16) into codes
// [rows, K/2] and scales [rows, K/16]. Rows whose row_token is negative (an expert's padding
// rows of h) get zero codes and scales; without row_token every row is quantised, and
// total_rows may be NULL, rows_host giving the count. One block per row, grid-strided; one
// thread per block of 16 values (two 16-byte loads, one 8-byte and one 1-byte store).
__global__ void k_quant_rows_nvfp4(const int* __restrict__ row_token, const int* __restrict__ total_rows,
                                   int rows_host, const __nv_bfloat16* __restrict__ src, int K,
                                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int R = total_rows != nullptr ? *total_rows : rows_host;
  const int nb = K / 16;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    const bool live = row_token == nullptr || row_token[r] >= 0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
      uint2 c = make_uint2(0u, 0u);
      uint32_t sb = 0u;
      if (live) {
        const uint4* p = reinterpret_cast<const uint4*>(src + static_cast<int64_t>(r) * K + b * 16);
        const uint4 u0 = p[0], u1 = p[1];
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        quant_block16_bf16(w, c, sb);
      }
      *reinterpret_cast<uint2*>(codes + static_cast<int64_t>(r) * (K / 2) + b * 8) = c;
      scales[static_cast<int64_t>(r) * nb + b] = static_cast<uint8_t>(sb);
    }
  }
}

// Dispatch of the quantised latent: row r of the expert-ordered code and scale matrices is
// token row_token[r]'s row of the token-ordered ones (zeros for padding rows). The latent is
// quantised once per token and its bytes copied k times, instead of quantising every copy.
// One block per row, grid-strided; 16-byte vectors (K / 32 of codes, K / 256 of scales).
__global__ void k_gather_nvfp4_rows(const int* __restrict__ row_token, const int* __restrict__ total_rows,
                                    const uint4* __restrict__ codes_tok, const uint4* __restrict__ scales_tok,
                                    uint4* __restrict__ codes, uint4* __restrict__ scales, int K) {
  const int R = *total_rows;
  const int vc = K / 32, vs = K / 256;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    const int tok = row_token[r];
    for (int i = threadIdx.x; i < vc + vs; i += blockDim.x) {
      const bool is_code = i < vc;
      const int j = is_code ? i : i - vc;
      const uint4* src = is_code ? codes_tok + static_cast<int64_t>(tok) * vc : scales_tok + static_cast<int64_t>(tok) * vs;
      uint4* dst = is_code ? codes + static_cast<int64_t>(r) * vc : scales + static_cast<int64_t>(r) * vs;
      dst[j] = tok >= 0 ? src[j] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

}  // namespace muse
