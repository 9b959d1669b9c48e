// route_kernels.cuh -- the non-GEMM steps of the latent-MoE block:
//   router logits in FP32 FMA (float32 workloads only), top-k selection and weights,
//   token -> expert permutation (histogram, padded prefix sum, device tile lists,
//   stable rank), gather into expert order, and the per-expert-RMSNorm weighted combine.
// All of them are deterministic: integer atomics only for counts, fixed-order FP32 sums.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "gemm_umma.cuh"

namespace muse {

__device__ __forceinline__ float neg_inf() { return -__int_as_float(0x7f800000); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Exclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024); *total
// receives the block sum. Every thread of the block must call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_tot[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  __syncthreads();
  if (lane == 31) warp_tot[w] = inc;
  __syncthreads();
  if (w == 0) {
    int x = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += u;
    }
    warp_tot[lane] = x;  // inclusive over warps
  }
  __syncthreads();
  const int before = (w == 0) ? 0 : warp_tot[w - 1];
  *total = warp_tot[nw - 1];
  return before + inc - v;
}

// --------------------------------------------------------------------------------------
// (a1, float32 workloads) router logits l[t, e] = sum_d W_router[e, d] x[t, d] in FP32
// FMA, so routing decisions of float32 inputs see FP32 and not TF32 products.
// One block per token, a warp per expert, lanes stride over d, fixed-order reduction.
// --------------------------------------------------------------------------------------
__global__ void k_router_logits_f32(const float* __restrict__ x, const float* __restrict__ Wr,
                                    int D, int E, float* __restrict__ logits) {
  const int t = blockIdx.x;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float* xr = x + static_cast<int64_t>(t) * D;
  for (int e = w; e < E; e += nw) {
    const float* wr = Wr + static_cast<int64_t>(e) * D;
    float s = 0.0f;
    for (int d = lane; d < D; d += 32) s = fmaf(wr[d], xr[d], s);
    s = warp_sum(s);
    if (lane == 0) logits[static_cast<int64_t>(t) * E + e] = s;
  }
}

// --------------------------------------------------------------------------------------
// (a2) top-k selection and routing weights, one warp per token.
// key = l + b (softmax mode) or sigmoid(scale*l) + b (sigmoid mode); the k largest keys
// are taken one at a time by a warp argmax with ties to the lower expert index, so
// slot j holds the j-th largest key. Weights use the unbiased logits:
//   softmax: g_j = exp(l_j - m) / sum_S exp(l - m)  (softmax over E renormalised on S)
//   sigmoid: g_j = rsf * s_j / (sum_S s + 1e-15)
// --------------------------------------------------------------------------------------
// NPL: key slots per lane (E <= 32 * NPL; NPL a power of two up to 32).
template <int NPL>
__global__ void k_topk(const float* __restrict__ logits, int T, int E, int k,
                       const float* __restrict__ bias, int mode, float scale, float rsf,
                       int* __restrict__ idx_out, float* __restrict__ w_out,
                       int* __restrict__ user_idx, float* __restrict__ user_w) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;  // warp-uniform
  const float* l = logits + static_cast<int64_t>(t) * E;
  float key[NPL];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    key[i] = neg_inf();
    const int e = lane + 32 * i;
    if (e < E) {
      const float li = l[e];
      float kv = (mode == 0) ? li : 1.0f / (1.0f + expf(-scale * li));
      if (bias != nullptr) kv += bias[e];
      key[i] = (kv == kv) ? kv : neg_inf();  // a NaN key never wins over a number
    } else {
      taken |= 1u << i;
    }
  }
  int my_sel = 0;
  for (int j = 0; j < k; ++j) {
    float bk = neg_inf();
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      if (!((taken >> i) & 1u) && (key[i] > bk || (key[i] == bk && e < bi))) {
        bk = key[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ok > bk || (ok == bk && oi < bi)) {
        bk = ok;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) my_sel = bi;
  }
  const bool mine = lane < k;
  const float lj = mine ? l[my_sel] : 0.0f;
  float g;
  if (mode == 0) {
    const float m = warp_max(mine ? lj : neg_inf());
    const float pj = mine ? expf(lj - m) : 0.0f;
    g = pj / warp_sum(pj);
  } else {
    const float sj = mine ? 1.0f / (1.0f + expf(-scale * lj)) : 0.0f;
    g = rsf * sj / (warp_sum(sj) + 1e-15f);
  }
  if (mine) {
    const int64_t o = static_cast<int64_t>(t) * k + lane;
    idx_out[o] = my_sel;
    w_out[o] = g;
    if (user_idx != nullptr) user_idx[o] = my_sel;
    if (user_w != nullptr) user_w[o] = g;
  }
}

// --------------------------------------------------------------------------------------
// (a3) permutation, step 1: tokens per expert (integer atomics: exact, order-free).
// --------------------------------------------------------------------------------------
__global__ void k_expert_hist(const int* __restrict__ idx, int n, int E, int* __restrict__ counts,
                              uint32_t* status) {
  extern __shared__ int hist[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int a = blockIdx.x * blockDim.x + threadIdx.x; a < n; a += gridDim.x * blockDim.x) {
    const int e = idx[a];
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
      atomicAdd(&hist[e], 1);
    else
      record_status(status, kStatusDevice, 0x1000u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x)
    if (hist[i]) atomicAdd(&counts[i], hist[i]);
}

// --------------------------------------------------------------------------------------
// (a3) step 2 (one block, thread per expert): padded row offsets (each expert's rows
// rounded up to a multiple of 16, the MMA's N granularity), the two grouped-GEMM tile
// lists (gate/up tiles step_gu features apart, down tiles step_dn apart) and the padding
// rows' token = -1. An expert's n rows split into
// ceil(n / BN) near-equal chunks of a multiple of 16 rows; tiles are ordered expert,
// feature tile, chunk, so the chunks sharing one weight tile run side by side. Also
// zeroes the tile counters the CTA-pair GEMMs of the forward claim tiles from.
// --------------------------------------------------------------------------------------
__global__ void k_build_tiles(const int* __restrict__ counts, int E, int BN, int mt_gu, int step_gu, int mt_dn,
                              int step_dn, int* __restrict__ offsets, int4* __restrict__ tiles_gu,
                              int* __restrict__ ntiles_gu, int4* __restrict__ tiles_dn,
                              int* __restrict__ ntiles_dn, int* __restrict__ tile_counters,
                              int* __restrict__ row_token) {
  const int e = threadIdx.x;
  const int n = (e < E) ? counts[e] : 0;
  const int padded = (n + 15) & ~15;
  int total_rows, total_gu, total_dn;
  const int off = block_exclusive_scan(padded, &total_rows);
  const int nch = (n + BN - 1) / BN;
  const int chunk = nch ? ((((n + nch - 1) / nch) + 15) & ~15) : 0;
  const int gu_off = block_exclusive_scan(nch * mt_gu, &total_gu);
  const int dn_off = block_exclusive_scan(nch * mt_dn, &total_dn);
  if (e < E) {
    offsets[e] = off;
    for (int ft = 0; ft < mt_gu; ++ft)
      for (int ch = 0; ch < nch; ++ch)
        tiles_gu[gu_off + ft * nch + ch] = make_int4(e, ft * step_gu, off + ch * chunk, min(chunk, n - ch * chunk));
    for (int ft = 0; ft < mt_dn; ++ft)
      for (int ch = 0; ch < nch; ++ch)
        tiles_dn[dn_off + ft * nch + ch] = make_int4(e, ft * step_dn, off + ch * chunk, min(chunk, n - ch * chunk));
    for (int r = off + n; r < off + padded; ++r) row_token[r] = -1;
  }
  if (threadIdx.x == 0) {
    offsets[E] = total_rows;
    *ntiles_gu = total_gu;
    *ntiles_dn = total_dn;
    for (int i = 0; i < 4; ++i) tile_counters[i] = 0;  // the CTA-pair GEMMs of this forward
  }
}

// --------------------------------------------------------------------------------------
// (a3) step 3 (block per expert): stable rank of each assignment a = t*k + j among the
// assignments to the same expert, in increasing a (token ascending, slot ascending):
// row = offsets[e] + rank; inv[a] = row, row_token[row] = t.
// --------------------------------------------------------------------------------------
__global__ void k_assign_rows(const int* __restrict__ idx, int n, int k, const int* __restrict__ counts,
                              const int* __restrict__ offsets, int* __restrict__ inv,
                              int* __restrict__ row_token) {
  // Warp w owns the contiguous segment [w * seg, (w + 1) * seg) of the assignments (seg a
  // multiple of 32). Pass 1 counts the segment's assignments to this expert with ballots;
  // an exclusive scan over the warps gives each segment's first rank; pass 2 walks the
  // segment again and numbers the matches in order (rank = first + matches before it).
  __shared__ int seg_count[32];
  const int e = blockIdx.x;
  const int cnt = counts[e];
  if (cnt == 0) return;  // block-uniform
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int seg = ((n + nw - 1) / nw + 31) & ~31;
  const int a0 = w * seg, a1 = min(n, a0 + seg);
  int mine = 0;
  for (int a = a0 + lane; a - lane < a1; a += 32) {
    const bool hit = a < a1 && idx[a] == e;
    mine += __popc(__ballot_sync(0xffffffffu, hit));
  }
  if (lane == 0) seg_count[w] = mine;
  __syncthreads();
  int first = 0;
  for (int i = 0; i < w; ++i) first += seg_count[i];
  const int base_row = offsets[e];
  const unsigned below = (1u << lane) - 1u;
  for (int a = a0 + lane; a - lane < a1; a += 32) {
    const bool hit = a < a1 && idx[a] == e;
    const unsigned b = __ballot_sync(0xffffffffu, hit);
    if (hit) {
      const int row = base_row + first + __popc(b & below);
      inv[a] = row;
      row_token[row] = a / k;
    }
    first += __popc(b);
  }
}

// Sum over the block in a fixed order (a butterfly inside each warp, then every warp
// sums the warp totals the same way), so equal inputs give equal bits on every run and
// every thread receives the total. part: 32 floats of shared memory.
__device__ __forceinline__ float block_sum(float v, float* part) {
  v = warp_sum(v);
  __syncthreads();  // part may still be read by a previous call
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = v;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  float t = lane < static_cast<int>(blockDim.x >> 5) ? part[lane] : 0.0f;
  return warp_sum(t);
}

// --------------------------------------------------------------------------------------
// Centred RMSNorm of rows of n elements (one block per row, FP32 statistics):
//   out = in / sqrt(mean(in^2) + eps) * (1 + w)
// Used for the pages' pre_expert_norm on z (in place, in == out) and for the feed-
// forward sublayer's pre-norm on x (deep dive §2.1 step 6, §5.3 table). Two passes over
// the row: the second re-reads it from cache.
// --------------------------------------------------------------------------------------
template <typename T>
__global__ void k_rmsnorm_rows(const T* in, T* out, const T* __restrict__ w, int n, float eps) {
  constexpr int VEC = 16 / sizeof(T);
  __shared__ float part[32];
  const T* irow = in + static_cast<int64_t>(blockIdx.x) * n;
  T* orow = out + static_cast<int64_t>(blockIdx.x) * n;
  float ss = 0.0f;
  for (int c = threadIdx.x * VEC; c < n; c += blockDim.x * VEC) {
    const uint4 v = *reinterpret_cast<const uint4*>(irow + c);
    const T* vv = reinterpret_cast<const T*>(&v);
#pragma unroll
    for (int i = 0; i < VEC; ++i) ss = fmaf(to_f32(vv[i]), to_f32(vv[i]), ss);
  }
  const float scale = 1.0f / sqrtf(block_sum(ss, part) / static_cast<float>(n) + eps);
  for (int c = threadIdx.x * VEC; c < n; c += blockDim.x * VEC) {
    const uint4 v = *reinterpret_cast<const uint4*>(irow + c);
    const uint4 gv = *reinterpret_cast<const uint4*>(w + c);
    const T* vv = reinterpret_cast<const T*>(&v);
    const T* gg = reinterpret_cast<const T*>(&gv);
    uint4 ov;
    T* oo = reinterpret_cast<T*>(&ov);
#pragma unroll
    for (int i = 0; i < VEC; ++i) oo[i] = from_f32<T>(to_f32(vv[i]) * scale * (1.0f + to_f32(gg[i])));
    *reinterpret_cast<uint4*>(orow + c) = ov;
  }
}

// --------------------------------------------------------------------------------------
// Feed-forward sublayer, after the unpooler (deep dive §2.1 step 7, §5.2, §5.3), in place
// on out = f; a block covers kFinishRows tokens x kFinishThreads vectors of channels, so
// each thread computes its channels' gate coefficients once for many tokens:
//   post norm (post_gain != NULL): v = f * (1 + w), fn = v / sqrt(mean(v^2) + post_eps),
//     mean(v^2) from the unpooler epilogue's partial sums ss[t, 0 .. D/32) of squares of
//     the FP32 accumulator times (1 + w), the scale applied to the stored f;
//   residual gate (gate != NULL): out = alpha * x + beta * fn, beta = sigmoid(g / T),
//     alpha = sqrt(max(sigmoid(-g / T) * (1 + beta), gate_eps)), coefficients in FP32.
// --------------------------------------------------------------------------------------
constexpr int kFinishRows = 32;     // tokens per block
constexpr int kFinishThreads = 256;  // one 16-byte vector of channels per thread

template <typename T>
__global__ void __launch_bounds__(kFinishThreads) k_ffn_finish(
    T* __restrict__ out, const T* __restrict__ x, const float* __restrict__ ss, int ss_ld,
    const T* __restrict__ post_gain, float post_eps, const float* __restrict__ gate, float inv_temp,
    float gate_eps, int D, int T_rows) {
  constexpr int VEC = 16 / sizeof(T);
  __shared__ float scale_s[kFinishRows];
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kFinishRows;  // x: token blocks (up to 2^31 - 1)
  const int rows = min(kFinishRows, T_rows - static_cast<int>(t0));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // post-norm scale of each of the block's tokens: one warp per token, fixed order
  for (int r = warp; r < rows; r += kFinishThreads / 32) {
    float sc = 1.0f;
    if (post_gain != nullptr) {
      float s = 0.0f;
      for (int i = lane; i < ss_ld; i += 32) s += ss[(t0 + r) * ss_ld + i];
      sc = 1.0f / sqrtf(warp_sum(s) / static_cast<float>(D) + post_eps);
    }
    if (lane == 0) scale_s[r] = sc;
  }
  __syncthreads();
  const int c = (blockIdx.y * kFinishThreads + threadIdx.x) * VEC;  // y: channel slices
  if (c >= D) return;
  // this thread's channels: gain and gate coefficients, once for all rows
  float gain[VEC], alpha[VEC], beta[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    gain[i] = 1.0f;
    alpha[i] = 0.0f;
    beta[i] = 1.0f;
  }
  if (post_gain != nullptr) {
    const uint4 gv4 = *reinterpret_cast<const uint4*>(post_gain + c);
    const T* gv = reinterpret_cast<const T*>(&gv4);
#pragma unroll
    for (int i = 0; i < VEC; ++i) gain[i] = 1.0f + to_f32(gv[i]);
  }
  if (gate != nullptr) {
#pragma unroll
    for (int i = 0; i < VEC; i += 4) {
      const float4 g4 = *reinterpret_cast<const float4*>(gate + c + i);
      const float gg[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float wg = gg[j] * inv_temp;
        beta[i + j] = 1.0f / (1.0f + expf(-wg));
        alpha[i + j] = sqrtf(fmaxf((1.0f / (1.0f + expf(wg))) * (1.0f + beta[i + j]), gate_eps));
      }
    }
  }
  // rows four at a time: loads first, then arithmetic and stores
  for (int r0 = 0; r0 < rows; r0 += 4) {
    uint4 fv4[4], xv4[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      fv4[j] = make_uint4(0, 0, 0, 0);
      xv4[j] = make_uint4(0, 0, 0, 0);
      if (r0 + j < rows) {
        fv4[j] = *reinterpret_cast<const uint4*>(out + (t0 + r0 + j) * D + c);
        if (gate != nullptr) xv4[j] = *reinterpret_cast<const uint4*>(x + (t0 + r0 + j) * D + c);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (r0 + j >= rows) break;
      const T* fv = reinterpret_cast<const T*>(&fv4[j]);
      const T* xv = reinterpret_cast<const T*>(&xv4[j]);
      const float sc = scale_s[r0 + j];
      uint4 ov;
      T* oo = reinterpret_cast<T*>(&ov);
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        const float f = to_f32(fv[i]) * gain[i] * sc;
        oo[i] = from_f32<T>(gate != nullptr ? alpha[i] * to_f32(xv[i]) + beta[i] * f : f);
      }
      *reinterpret_cast<uint4*>(out + (t0 + r0 + j) * D + c) = ov;
    }
  }
}

// bf16 -> f16, two or eight values at a time (round to nearest even, saturating): exact for
// magnitudes 2^-14 .. 65504 (f16's normal range holds every 8-bit bf16 significand);
// smaller values round to f16's subnormal grid of 2^-24, larger ones saturate at +-65504.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  const float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  return make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
}

// --------------------------------------------------------------------------------------
// (a3) gather: Zp[row] = z[row_token[row]] (zeros for padding rows), 16-byte vectors;
// one block per row (grid-strided), every thread moving several independent vectors.
// kToF16: the rows are converted from bf16 to f16 on the way (the NVFP4-weight W4A16
// path, whose tensor-core operands are f16).
// --------------------------------------------------------------------------------------
template <bool kToF16 = false>
__global__ void k_gather_rows(const int* __restrict__ row_token, const int* __restrict__ total_rows,
                              const uint4* __restrict__ z, uint4* __restrict__ zp, int vec_per_row) {
  // (z and zp never overlap)
  const int R = *total_rows;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    const int tok = row_token[r];
    uint4* dst = zp + static_cast<int64_t>(r) * vec_per_row;
    if (tok >= 0) {
      const uint4* src = z + static_cast<int64_t>(tok) * vec_per_row;
      // four vectors in flight per thread: all loads issued before the stores
      for (int c0 = threadIdx.x; c0 < vec_per_row; c0 += 4 * blockDim.x) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + u * blockDim.x;
          if (c < vec_per_row) v[u] = src[c];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + u * blockDim.x;
          if (c < vec_per_row) {
            if constexpr (kToF16) v[u] = bf16x8_to_f16x8(v[u]);
            dst[c] = v[u];
          }
        }
      }
    } else {
      for (int c = threadIdx.x; c < vec_per_row; c += blockDim.x) dst[c] = make_uint4(0, 0, 0, 0);
    }
  }
}

// --------------------------------------------------------------------------------------
// (a8 + a9) per-expert RMSNorm applied inside the weighted combine, one block per token:
//   c[t] = sum_j g_j * y_j / sqrt(ss_j / L + eps) * (1 + gamma[e_j])
// j in routing order, FP32 accumulation, 16-byte loads. ss_j is the sum of the row's
// L/32 partial sums of squares (fixed order) written by the down-projection epilogue;
// in input-scaled mode those partials were taken of y * (1 + gamma) instead of y.
// --------------------------------------------------------------------------------------
template <typename T>
__global__ void k_combine(const int* __restrict__ topk_idx, const float* __restrict__ topk_w,
                          const int* __restrict__ inv, const float* __restrict__ ss, int ss_ld,
                          const T* __restrict__ Y, const T* __restrict__ gamma, int64_t gamma_stride,
                          int L, int k, float eps, T* __restrict__ c) {
  constexpr int VEC = 16 / sizeof(T);
  __shared__ float scale_s[32];
  __shared__ int pos_s[32];
  __shared__ int e_s[32];
  const int t = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  // the k row scales in parallel, one warp per selected row
  for (int j = warp; j < k; j += nw) {
    const int64_t a = static_cast<int64_t>(t) * k + j;
    const int pos = inv[a];
    float s = 0.0f;
    for (int i = lane; i < ss_ld; i += 32) s += ss[static_cast<int64_t>(pos) * ss_ld + i];
    s = warp_sum(s);
    if (lane == 0) {
      scale_s[j] = topk_w[a] * (1.0f / sqrtf(s / static_cast<float>(L) + eps));
      pos_s[j] = pos;
      e_s[j] = topk_idx[a];
    }
  }
  __syncthreads();
  for (int f0 = threadIdx.x * VEC; f0 < L; f0 += blockDim.x * VEC) {
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.0f;
#pragma unroll 8
    for (int j = 0; j < k; ++j) {
      const uint4 yv = *reinterpret_cast<const uint4*>(Y + static_cast<int64_t>(pos_s[j]) * L + f0);
      const uint4 gv = *reinterpret_cast<const uint4*>(gamma + e_s[j] * gamma_stride + f0);
      const T* yy = reinterpret_cast<const T*>(&yv);
      const T* gg = reinterpret_cast<const T*>(&gv);
      const float sj = scale_s[j];
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = fmaf(sj * (1.0f + to_f32(gg[v])), to_f32(yy[v]), acc[v]);
    }
    uint4 ov;
    T* oo = reinterpret_cast<T*>(&ov);
#pragma unroll
    for (int v = 0; v < VEC; ++v) oo[v] = from_f32<T>(acc[v]);
    *reinterpret_cast<uint4*>(c + static_cast<int64_t>(t) * L + f0) = ov;
  }
}

// --------------------------------------------------------------------------------------
// Split-K GEMM: out[i] = sum over the S K-ranges of part[s * n + i] (i < n = T * M), summed
// in range order so that equal inputs give equal bits, converted to the output type.
// Grid-strided over groups of 4 elements (n is a multiple of 4: M is a multiple of 128).
// --------------------------------------------------------------------------------------
template <typename TOut>
__global__ void k_splitk_reduce(const float4* __restrict__ part, int64_t n4, int S, TOut* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 acc = part[i];
    for (int s = 1; s < S; ++s) {
      const float4 v = part[static_cast<int64_t>(s) * n4 + i];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if constexpr (sizeof(TOut) == 4) {
      reinterpret_cast<float4*>(out)[i] = acc;
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&lo);
      w.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(out)[i] = w;
    }
  }
}

// --------------------------------------------------------------------------------------
// Expert parallelism over G ranks, rank r owning experts [r * E_loc, (r + 1) * E_loc).
// The latent of a token crosses to each rank that owns one of its experts (one row per
// selected expert, 2 L bytes); the expert outputs and their partial sums of squares
// come back; the per-expert norm and the weighted combine run on the token's own rank.
// --------------------------------------------------------------------------------------

// Send plan (one block, a thread per expert): the T*k assignments in expert-major order
// without padding, offsets[e] = number of assignments to experts below e. Because the
// owners' expert ranges are contiguous and ascending, that order is also rank-major:
// rank r's rows are [offsets[r * E_loc], offsets[(r + 1) * E_loc]), rank_counts[r] of
// them. Also zeroes the tile counters of the pooler and unpooler GEMMs, as k_build_tiles
// does in the single-GPU forward.
__global__ void k_ep_plan(const int* __restrict__ counts, int E, int E_loc, int G, int* __restrict__ offsets,
                          int* __restrict__ rank_counts, int* __restrict__ tile_counters) {
  const int e = threadIdx.x;
  const int n = (e < E) ? counts[e] : 0;
  int total;
  const int off = block_exclusive_scan(n, &total);
  if (e < E) offsets[e] = off;
  if (threadIdx.x == 0) {
    offsets[E] = total;
    for (int i = 0; i < 4; ++i) tile_counters[i] = 0;
  }
  __syncthreads();  // offsets visible to the whole block
  for (int r = threadIdx.x; r < G; r += blockDim.x) rank_counts[r] = offsets[(r + 1) * E_loc] - offsets[r * E_loc];
}

// Send buffer: assignment a = t*k + j to expert e = idx[a] goes to row inv[a] (its place
// in the send plan) as a copy of z's row t, tagged with e's index on its owning rank,
// e - E_loc * (e / E_loc). One block per assignment, grid-strided; 16-byte vectors.
__global__ void k_ep_pack(const int* __restrict__ idx, const int* __restrict__ inv, int n, int k, int E_loc,
                          const uint4* __restrict__ z, int vec_per_row, uint4* __restrict__ send_z,
                          int* __restrict__ send_expert) {
  for (int a = blockIdx.x; a < n; a += gridDim.x) {
    const int pos = inv[a];
    const uint4* src = z + static_cast<int64_t>(a / k) * vec_per_row;
    uint4* dst = send_z + static_cast<int64_t>(pos) * vec_per_row;
    for (int c = threadIdx.x; c < vec_per_row; c += blockDim.x) dst[c] = src[c];
    if (threadIdx.x == 0) send_expert[pos] = idx[a] % E_loc;
  }
}

// An expert shard's results in the order its rows were received: ret_y[r] = y[inv[r]]
// and ret_ss[r] = ss[inv[r]] (the L/32 partial sums of squares). A row whose expert
// index was out of range has no slot (inv[r] < 0, the histogram recorded the error) and
// gets zeros. One block per row, grid-strided; 16-byte vectors.
__global__ void k_ep_unpermute(const int* __restrict__ inv, int R, const uint4* __restrict__ y,
                               const uint4* __restrict__ ss, int vec_y, int vec_ss, uint4* __restrict__ ret_y,
                               uint4* __restrict__ ret_ss) {
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    const int row = inv[r];
    for (int c = threadIdx.x; c < vec_y + vec_ss; c += blockDim.x) {
      const bool is_y = c < vec_y;
      const int j = is_y ? c : c - vec_y;
      const int vpr = is_y ? vec_y : vec_ss;
      const uint4* src = (is_y ? y : ss) + static_cast<int64_t>(row) * vpr;
      uint4* dst = (is_y ? ret_y : ret_ss) + static_cast<int64_t>(r) * vpr;
      dst[j] = row >= 0 ? src[j] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// --------------------------------------------------------------------------------------
// Self-test of the bounded waits: one thread waits on an mbarrier that nothing will ever
// complete, through the same mbar_wait the GEMMs use, with a short limit; the timeout is
// recorded in status (a completed wait would be recorded as a device error).
// --------------------------------------------------------------------------------------
__global__ void k_selftest_wait(uint64_t limit_ns, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (mbar_wait(smem_u32(&bar), 0u, &abort_flag, status, 0x5E1Fu, limit_ns))
      record_status(status, kStatusDevice, 0x5E1Fu);
  }
}

}  // namespace muse
