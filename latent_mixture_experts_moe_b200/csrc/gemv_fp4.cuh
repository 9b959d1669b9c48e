// gemv_fp4.cuh -- the grouped expert GEMMs with NVFP4 weights and 16-bit activations at
// decode-sized tiles (at most 16 token rows per tile, typically 1..8):
//
//   C[token, f] = mscale[e] * sum_k (e2m1(code[f, k]) * e4m3(scale[f, k / 16])) * X[token, k]
//
// With a few tokens per expert the layer streams 4-bit weights from HBM and each weight
// takes part in a few multiply-adds. A tcgen05 MMA reads its A operand -- the weights,
// expanded to f16 -- from tensor or shared memory: 2 bytes moved on chip for every 0.5 byte
// read from HBM, which holds the tensor-memory kernel near a third of the HBM rate at decode.
// Here the expanded weights never leave registers: consumer warps convert the codes in
// registers (cvt.rn.f16x2.e2m1x2, the block scale applied by one exact f16x2 multiply, as in
// the tensor-memory kernel) and hand them to the warp-level MMA mma.sync.m16n8k16 as its A
// fragment (f16 operands, FP32 accumulation), the tokens as its N = 8 columns.
//
// Roles (288 threads, one CTA per SM, persistent over the tile list): warp 0 lane 0 is the
// TMA producer; consumer warp wc = 0..7 (warp 1 + wc) owns weight rows 16 wc .. 16 wc + 15
// of the tile's 128 (of both gate and up for SwiGLU). A ring stage carries 256 K elements of
// two weight matrices (gate/up) or 512 of one (down): per matrix a 128-row x 32-byte code box
// per 64-element k-block and a 128-row x 16-byte box of block scales per 256 elements, and
// the tile's token rows as one 16-row x 128-byte box per k-block (128-byte swizzle).
//
// The MMA's K order is free as long as A and B agree, so lane (g, t) of a warp (g = lane / 4,
// t = lane % 4) takes whole 16-weight blocks: block t of each 64-element k-block, rows g and
// g + 8 of its M-tile, four weights per MMA step, and the matching 16 activations of token
// g of each 8-token group. Every shared-memory read is conflict-free: code rows are 32 bytes
// apart (lanes (g, t) read 8 bytes at 32 g + 8 t), a scale row is one 16-byte broadcast, and
// the swizzle puts the token rows of lanes (0|1, t) on distinct 16-byte chunks.
// Every wait is bounded (ptx.cuh); a consumer that gives up still meets its warps at the
// store epilogue's named barriers, where they agree to leave the tile loop together.
#pragma once

#include <cuda_fp16.h>

#include "gemm_umma.cuh"
#include "gemm_umma_fp4.cuh"

namespace muse {

constexpr int kGemvThreads = 288;        // producer warp + 8 consumer warps
constexpr int kGemvMaxTokens = 16;       // token rows per tile (one 16-row token box)
constexpr int kGemvKGroup = 256;         // K elements per block-scale box (16 blocks)

struct GemvMaps {
  CUtensorMap codes[2];   // [E * rows, K/2] u8, 128-row x 32-byte boxes (gate, up; or down twice)
  CUtensorMap scales[2];  // [E * rows, K/16] u8, 128-row x 16-byte boxes
  CUtensorMap x;          // [R, K] 16-bit activation rows, 16-row x 128-byte boxes, 128-byte swizzle
};

struct GemvArgs {
  const int4* tiles;           // {expert, m0, row0, n}, n <= kGemvMaxTokens
  const int* num_tiles;        // device count
  const float* mscale[2];      // per-expert matrix scales
  int rows_per_group;          // weight rows per expert (I for gate/up, L for down)
  int K;                       // input width (multiple of kGemvKGroup)
  void* out;                   // SwiGLU: __half h [rows, ld_out]; store: bf16 y [rows, ld_out]
  int64_t ld_out;
  float* ss;                   // store: sums of squares [rows, ss_ld], one per 32 features
  int ss_ld;
  const __nv_bfloat16* ss_gain;  // optional gain offsets: squares of y * (1 + gain)
  int64_t ss_gain_stride;
  uint32_t* status;
};

template <int MATS>
struct GemvShape {
  // a stage holds SG groups of 256 K elements: one for two weight matrices (gate/up), two for
  // one (down), so that a consumer warp has the same work per stage either way
  static constexpr int kSG = MATS == 2 ? 1 : 2;
  static constexpr int kKB = 4 * kSG;                                  // 64-element k-blocks per stage
  static constexpr int kKStage = kGemvKGroup * kSG;                    // K elements per stage
  static constexpr uint32_t kCodeBox = 128u * 32u;                    // one 64-element k-block
  static constexpr uint32_t kScaleBox = 128u * 16u;                   // 16 blocks = 256 K elements
  static constexpr uint32_t kXBox = 16u * 128u;                       // 16 tokens x 64 elements
  static constexpr uint32_t kCodeOff = 0;
  static constexpr uint32_t kScaleOff = kCodeOff + kKB * kCodeBox * MATS;
  static constexpr uint32_t kXOff = kScaleOff + kSG * kScaleBox * MATS;
  static constexpr uint32_t kStageBytes = kXOff + kKB * kXBox;        // k-blocks x 1 token box
  static constexpr uint32_t kSsBytes = 8u * 16u * 4u;                 // store epilogue partials
  static constexpr int kSmemBudget = 227 * 1024 - 1024 - static_cast<int>(kSsBytes) - 256;
  static constexpr int kStagesFit = kSmemBudget / static_cast<int>(kStageBytes);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + kSsBytes + 256;
  static_assert(kXOff % 1024 == 0 && kStageBytes % 1024 == 0, "swizzled token boxes need 1024-byte alignment");
  static_assert(kStages >= 2, "ring too small");
};

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// E4M3 byte `sel` (0..3) of w as an f16 value in both halves (exact)
__device__ __forceinline__ uint32_t e4m3_bcast_f16x2(uint32_t w, uint32_t sel) {
  return e4m3x2_to_f16x2(__byte_perm(w, 0u, sel | (sel << 4)));
}

// One consumer warp's share of a tile: rows 16 wc .. 16 wc + 15 of each weight matrix, NB8
// groups of 8 tokens. Returns false when a wait gave up.
template <int EPI, int NB8>
__device__ __forceinline__ bool gemv_consume(const GemvArgs& p, uint8_t* smem, uint32_t bar0, int& stage,
                                             uint32_t& phase, volatile int* abort_flag, int wc, int lane, int e,
                                             int m0, int row0, int n, int nstages) {
  constexpr int MATS = (EPI == EPI_SWIGLU) ? 2 : 1;
  using S = GemvShape<MATS>;
  constexpr int kStages = S::kStages;
  const int g = lane >> 2, t = lane & 3;
  // with one 8-token group, two accumulator sets (even and odd k-blocks) halve the chain of
  // dependent MMAs per accumulator; they are summed before the epilogue
  constexpr int CH = NB8 == 1 ? 2 : 1;
  float acc[MATS][NB8][CH][4];
#pragma unroll
  for (int m = 0; m < MATS; ++m)
#pragma unroll
    for (int j8 = 0; j8 < NB8; ++j8)
#pragma unroll
      for (int c = 0; c < CH; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][j8][c][i] = 0.0f;
  const uint32_t r_lo = static_cast<uint32_t>(16 * wc + g);  // this lane's rows in the 128-row boxes
  const uint32_t sel_t = static_cast<uint32_t>(t);
  bool ok = true;
  for (int s = 0; s < nstages; ++s) {
    // (every lane waits; a failure in any lane fails the whole warp, which stays converged)
    if (!__all_sync(0xffffffffu, mbar_wait(bar0 + 8u * stage, phase, abort_flag, p.status, 0xD00u + stage))) {
      ok = false;
      break;
    }
    const uint8_t* st = smem + static_cast<uint32_t>(stage) * S::kStageBytes;
    // the block scales of rows r_lo and r_lo + 8 for this stage: 16 per group, per matrix
    uint4 sw[MATS][S::kSG][2];
#pragma unroll
    for (int m = 0; m < MATS; ++m)
#pragma unroll
      for (int sg = 0; sg < S::kSG; ++sg) {
        const uint8_t* sb = st + S::kScaleOff + (m * S::kSG + sg) * S::kScaleBox;
        sw[m][sg][0] = *reinterpret_cast<const uint4*>(sb + r_lo * 16u);
        sw[m][sg][1] = *reinterpret_cast<const uint4*>(sb + (r_lo + 8u) * 16u);
      }
#pragma unroll
    for (int j = 0; j < S::kKB; ++j) {   // k-block of 64 elements; this lane's block in it: t
      // activations: token g of each 8-token group, elements 16 t .. 16 t + 15 of the k-block
      uint32_t xv[NB8][8];
#pragma unroll
      for (int j8 = 0; j8 < NB8; ++j8) {
        const uint32_t row = static_cast<uint32_t>(8 * j8 + g);   // row in the 16-row box
        const uint8_t* xb = st + S::kXOff + j * S::kXBox + row * 128u;
        const uint4 v0 = *reinterpret_cast<const uint4*>(xb + (((2u * t) ^ (row & 7u)) << 4));
        const uint4 v1 = *reinterpret_cast<const uint4*>(xb + (((2u * t + 1u) ^ (row & 7u)) << 4));
        xv[j8][0] = v0.x; xv[j8][1] = v0.y; xv[j8][2] = v0.z; xv[j8][3] = v0.w;
        xv[j8][4] = v1.x; xv[j8][5] = v1.y; xv[j8][6] = v1.z; xv[j8][7] = v1.w;
      }
#pragma unroll
      for (int m = 0; m < MATS; ++m) {
        const uint8_t* cb = st + S::kCodeOff + (S::kKB * m + j) * S::kCodeBox;
        const uint2 c_lo = *reinterpret_cast<const uint2*>(cb + r_lo * 32u + 8u * t);
        const uint2 c_hi = *reinterpret_cast<const uint2*>(cb + (r_lo + 8u) * 32u + 8u * t);
        const uint4& q_lo = sw[m][j / 4][0];
        const uint4& q_hi = sw[m][j / 4][1];
        const uint32_t w_lo = j % 4 == 0 ? q_lo.x : j % 4 == 1 ? q_lo.y : j % 4 == 2 ? q_lo.z : q_lo.w;
        const uint32_t w_hi = j % 4 == 0 ? q_hi.x : j % 4 == 1 ? q_hi.y : j % 4 == 2 ? q_hi.z : q_hi.w;
        const uint32_t s_lo = e4m3_bcast_f16x2(w_lo, sel_t), s_hi = e4m3_bcast_f16x2(w_hi, sel_t);
        uint32_t a_lo[8], a_hi[8];   // byte b of the block -> weights 2b, 2b + 1
        e2m1x8_to_f16x2(c_lo.x, a_lo[0], a_lo[1], a_lo[2], a_lo[3]);
        e2m1x8_to_f16x2(c_lo.y, a_lo[4], a_lo[5], a_lo[6], a_lo[7]);
        e2m1x8_to_f16x2(c_hi.x, a_hi[0], a_hi[1], a_hi[2], a_hi[3]);
        e2m1x8_to_f16x2(c_hi.y, a_hi[4], a_hi[5], a_hi[6], a_hi[7]);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          a_lo[q] = f16x2_mul(a_lo[q], s_lo);
          a_hi[q] = f16x2_mul(a_hi[q], s_hi);
        }
        // step q: weights 4q .. 4q + 3 of the block (bytes 2q, 2q + 1) against activations
        // 4q .. 4q + 3 -- this lane's MMA columns k = 2t, 2t + 1 and 2t + 8, 2t + 9
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j8 = 0; j8 < NB8; ++j8)
            mma_f16_16816(acc[m][j8][j % CH], a_lo[2 * q], a_hi[2 * q], a_lo[2 * q + 1], a_hi[2 * q + 1],
                          xv[j8][2 * q], xv[j8][2 * q + 1]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar0 + 8u * (kStages + stage));
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
#pragma unroll
  for (int m = 0; m < MATS; ++m)
#pragma unroll
    for (int j8 = 0; j8 < NB8; ++j8)
#pragma unroll
      for (int c = 1; c < CH; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][j8][0][i] += acc[m][j8][c][i];
  // epilogue: lane (g, t) holds rows f_lo = m0 + 16 wc + g and f_lo + 8, tokens 8 j8 + 2 t, + 1
  const int f_lo = m0 + 16 * wc + g;
  if constexpr (EPI == EPI_SWIGLU) {
    if (!ok) return false;
    const float ms_g = p.mscale[0][e], ms_u = p.mscale[1][e];
    __half* hout = reinterpret_cast<__half*>(p.out);
#pragma unroll
    for (int j8 = 0; j8 < NB8; ++j8)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = 8 * j8 + 2 * t + (i & 1);
        const int f = f_lo + 8 * (i >> 1);
        if (tok < n) {
          const float h = silu_tanh(acc[0][j8][0][i] * ms_g) * (acc[1][j8][0][i] * ms_u);
          hout[(static_cast<int64_t>(row0) + tok) * p.ld_out + f] = f32_to_f16_sat(h);
        }
      }
  } else {
    const float ms = p.mscale[0][e];
    __nv_bfloat16* yout = reinterpret_cast<__nv_bfloat16*>(p.out);
    float gain[2] = {1.0f, 1.0f};
    if (p.ss_gain != nullptr) {
      gain[0] = 1.0f + __bfloat162float(p.ss_gain[e * p.ss_gain_stride + f_lo]);
      gain[1] = 1.0f + __bfloat162float(p.ss_gain[e * p.ss_gain_stride + f_lo + 8]);
    }
    float* ssred = reinterpret_cast<float*>(smem + static_cast<uint32_t>(kStages) * S::kStageBytes);  // [8][16]
#pragma unroll
    for (int j8 = 0; j8 < NB8; ++j8) {
      float sq[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int tok = 8 * j8 + 2 * t + c;
        const float y0 = acc[0][j8][0][c] * ms, y1 = acc[0][j8][0][2 + c] * ms;
        if (ok && tok < n) {
          yout[(static_cast<int64_t>(row0) + tok) * p.ld_out + f_lo] = __float2bfloat16_rn(y0);
          yout[(static_cast<int64_t>(row0) + tok) * p.ld_out + f_lo + 8] = __float2bfloat16_rn(y1);
        }
        const float u0 = y0 * gain[0], u1 = y1 * gain[1];
        float v = u0 * u0 + u1 * u1;
        // over the warp's 16 rows: the lanes of equal t
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        sq[c] = v;
      }
      if (g == 0) {
        ssred[wc * 16 + 8 * j8 + 2 * t] = sq[0];
        ssred[wc * 16 + 8 * j8 + 2 * t + 1] = sq[1];
      }
    }
    // consumer warps 2 q and 2 q + 1 hold the two 16-row halves of 32-feature group q
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if ((wc & 1) == 0 && ok && lane < n) {
      const float v = ssred[wc * 16 + lane] + ssred[(wc + 1) * 16 + lane];
      p.ss[(static_cast<int64_t>(row0) + lane) * p.ss_ld + ((m0 + 16 * wc) >> 5)] = v;
    }
    // the second barrier also ORs the warps' failures, so that all consumer warps leave the
    // tile loop together (none may wait at a named barrier for a warp that has left)
    uint32_t any_failed;
    asm volatile(
        "{\n\t.reg .pred f, a;\n\tsetp.ne.u32 f, %1, 0;\n\tbar.red.or.pred a, 1, 256, f;\n\t"
        "selp.u32 %0, 1, 0, a;\n\t}"
        : "=r"(any_failed)
        : "r"(ok ? 0u : 1u)
        : "memory");
    ok = any_failed == 0;
  }
  return ok;
}

// (one CTA per SM; nine warps put three on one SM quarter, whose 16K registers allow 170 a thread)
template <int EPI>
__global__ void __launch_bounds__(kGemvThreads, 1) k_fp4_gemv(const __grid_constant__ GemvMaps maps, const GemvArgs p) {
  constexpr int MATS = (EPI == EPI_SWIGLU) ? 2 : 1;
  using S = GemvShape<MATS>;
  constexpr int kStages = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // after the ring: the store epilogue's partials [8][16] floats, barriers, abort flag
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * S::kStageBytes + S::kSsBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kStages);
  const uint32_t bar0 = smem_u32(bars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar0 + 8u * s, 1);                  // full: producer arrival + bytes
      mbar_init(bar0 + 8u * (kStages + s), 8);      // empty: one arrival per consumer warp
    }
    *abort_flag = 0;
    fence_mbar_init();
    for (int m = 0; m < MATS; ++m) {
      prefetch_tmap(&maps.codes[m]);
      prefetch_tmap(&maps.scales[m]);
    }
    prefetch_tmap(&maps.x);
  }
  __syncthreads();
  const int num_tiles = *p.num_tiles;
  // (a last stage past K reads zeros: the tensor maps fill outside the matrices)
  const int nstages = (p.K + S::kKStage - 1) / S::kKStage;
  if (warp == 0) {
    if (lane == 0) {
      const uint64_t evict_first = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int ti = blockIdx.x; ok && ti < num_tiles; ti += gridDim.x) {
        const int4 tile = p.tiles[ti];
        const int a_row = tile.x * p.rows_per_group + tile.y;
        // (tiles hold at most 16 rows; a longer one is recorded and cut, never overrun)
        if (tile.w > kGemvMaxTokens) record_status(p.status, kStatusDevice, 0x6E00u);
        const uint32_t bytes = (S::kKB * S::kCodeBox + S::kSG * S::kScaleBox) * MATS + S::kKB * S::kXBox;
        for (int s = 0; s < nstages; ++s) {
          if (!mbar_wait(bar0 + 8u * (kStages + stage), phase ^ 1u, abort_flag, p.status, 0xE00u + stage)) {
            ok = false;
            break;
          }
          const uint32_t full = bar0 + 8u * stage;
          const uint32_t st = smem_u32(smem + static_cast<uint32_t>(stage) * S::kStageBytes);
          mbar_arrive_expect_tx(full, bytes);
#pragma unroll
          for (int m = 0; m < MATS; ++m) {
#pragma unroll
            for (int j = 0; j < S::kKB; ++j)
              tma_load_2d_hint(st + S::kCodeOff + (S::kKB * m + j) * S::kCodeBox, &maps.codes[m], full,
                               (S::kKStage / 2) * s + 32 * j, a_row, evict_first);
#pragma unroll
            for (int sg = 0; sg < S::kSG; ++sg)
              tma_load_2d_hint(st + S::kScaleOff + (m * S::kSG + sg) * S::kScaleBox, &maps.scales[m], full,
                               (S::kKStage / 16) * s + 16 * sg, a_row, evict_first);
          }
          for (int j = 0; j < S::kKB; ++j)
            tma_load_2d(st + S::kXOff + j * S::kXBox, &maps.x, full, S::kKStage * s + 64 * j, tile.z);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) mbar_wait_drain(bar0 + 8u * s, (issued_phase >> s) & 1u);
      }
    }
    __syncwarp();
  } else {
    const int wc = warp - 1;
    int stage = 0;
    uint32_t phase = 0;
    for (int ti = blockIdx.x; ti < num_tiles; ti += gridDim.x) {
      const int4 tile = p.tiles[ti];
      const int n = min(tile.w, kGemvMaxTokens);
      bool ok;
      if (n <= 8)
        ok = gemv_consume<EPI, 1>(p, smem, bar0, stage, phase, abort_flag, wc, lane, tile.x, tile.y, tile.z, n,
                                  nstages);
      else
        ok = gemv_consume<EPI, 2>(p, smem, bar0, stage, phase, abort_flag, wc, lane, tile.x, tile.y, tile.z, n,
                                  nstages);
      if (!ok) break;
    }
  }
}

}  // namespace muse
