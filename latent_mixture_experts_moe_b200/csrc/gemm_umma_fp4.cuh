// gemm_umma_fp4.cuh -- the grouped expert GEMMs with NVFP4 expert weights (W4A16):
//
//   C[token, f] = mscale[e] * sum_k (e2m1(code[f, k]) * e4m3(scale[f, k / 16])) * X[token, k]
//
// Weights stay 4-bit in HBM (0.5 B per weight + one E4M3 byte per 16 weights). TMA brings the
// packed codes of a 128-row x 64-K tile (4 KB) and the token tile into shared memory; eight
// converter warps expand each code row into 64 f16 values and write them straight into
// TENSOR MEMORY, where the UMMA takes its A operand (kind::f16 with A in TMEM: 128 lanes x 32
// columns per 64-K tile, two K elements per column). The expansion is two hardware
// conversions per pair of weights' worth of work: cvt.rn.f16x2.e2m1x2 turns a code byte into
// two f16 values, cvt.rn.f16x2.e4m3x2 turns two block-scale bytes into f16, and one f16x2
// multiply applies the scale -- exact, since a code value (2 significant bits) times an E4M3
// scale (4 bits) is a normal f16 number (2^-10 .. 2688). The token operand is therefore f16
// too (the gather converts the bf16 latent rows; this kernel's SwiGLU epilogue writes h as
// f16 for the down projection), exact for activations of magnitude 2^-14 .. 65504. The
// dequantised weights never touch shared memory. The per-matrix FP32 scale multiplies the
// FP32 accumulator in the epilogue.
//
// Roles (448 threads, one CTA per SM): warp 0 TMA producer (codes + token tile, a deep ring:
// 4-bit stages are small), warp 1 TMEM owner + UMMA issuer, warps 2..5 epilogue, warps 6..13
// converters (warp w expands weight rows 32*(w%4) .. +31 -- the TMEM lanes it may write -- of
// tile (w-6)/4; block scales read from global memory 8 k-blocks at a time). With four
// converted slots (decode-sized tiles) a converter warp issues the TMEM store of k-block j,
// expands k-block j+1, and only then waits for the store and hands slot j to the UMMA, so
// each store's latency hides behind the next expansion; with two (prefill tiles) it hands
// each slot over as soon as its store completes. TMEM columns: accumulators from 0,
// converted weight slots (32 * MT columns each) after them. Barriers: per TMA stage full (bytes) / empty (UMMA commit); per converted slot
// conv (converter warps) / cfree (UMMA commit). Every wait is bounded (ptx.cuh).
#pragma once

#include "gemm_umma.cuh"

namespace muse {

struct Fp4Args {
  const uint8_t* scales_a;   // E4M3 block scales of the matrix behind maps.a  [rows, scale_ld]
  const uint8_t* scales_a2;  // ... behind maps.a2 (gate/up: the up matrix; else = scales_a)
  const float* mscale_a;     // per-group (expert) matrix scales of maps.a
  const float* mscale_a2;
  int scale_ld;              // bytes per weight row of block scales (K / 16)
};

template <int BN, int EPI, int MT>
struct Fp4Shape {
  static_assert(BN == 32 || BN == 128 || BN == 192, "token tiles of 32, 128 or 192 rows");
  static constexpr uint32_t kCodeBytes = 128u * 32u;  // packed codes of 128 rows x 64 K
  static constexpr uint32_t kBBytes = static_cast<uint32_t>(BN) * 128u;
  static constexpr uint32_t kStageBytes = kBBytes + kCodeBytes * MT;   // TMA ring stage
  static constexpr int kSmemBudget = 227 * 1024 - 1024 - 1024;         // alignment, barriers
  static constexpr int kStagesFit = kSmemBudget / static_cast<int>(kStageBytes);
  static constexpr int kStages = kStagesFit > 16 ? 16 : kStagesFit;
  static constexpr int kAccStages = MT == 2 ? 1 : 2;
  static constexpr uint32_t kAccCols = static_cast<uint32_t>(BN) * MT;
  static constexpr uint32_t kTmemCols = 512;
  // converted weight tiles in the TMEM columns the accumulators leave, up to 4 slots
  static constexpr uint32_t kConvCols = 32u * MT;         // TMEM columns per slot
  static constexpr uint32_t kConvCol0 = kAccCols * kAccStages;
  static constexpr int kConvFit = static_cast<int>((kTmemCols - kConvCol0) / kConvCols);
  static constexpr int kConvSlots = kConvFit > 4 ? 4 : kConvFit;
  // With 4 slots a converter warp hands slot j to the UMMA only after expanding k-block
  // j + 1, so the TMEM store's latency hides behind that expansion. With 2 slots (192-token
  // tiles) it hands each slot over as soon as its store completes: a late hand-over would
  // leave the UMMA one expansion behind with no other slot to work on (measured: the T=4096
  // NVFP4 step 5.37 -> 4.70 ms with the early hand-over there).
  static constexpr bool kLateHandOver = kConvSlots >= 4;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + 1024;
  static_assert(kConvSlots >= 2, "no TMEM room for converted weight tiles");
  static_assert(kStages >= 2, "tile too large for the shared-memory ring");
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
  static_assert(EPI != EPI_SWIGLU || MT == 2, "SwiGLU needs the gate and up accumulators");
};

// warps 0 producer, 1 UMMA issuer, 2..5 epilogue, 6..13 converters (with MT = 1, 10..13 idle)
constexpr int kFp4Threads = 448;

// 8 E2M1 codes (one 32-bit word; byte b holds K elements 2b (low nibble) and 2b + 1) -> 4
// words of f16 pairs, the lower K element in the low half
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2,
                                                uint32_t& o3) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
      : "r"(w));
}

// two E4M3 bytes (the low 16 bits of v, byte 0 first) -> f16 pair, byte 0 in the low half
// (exact: E4M3 values have 4 significant bits and lie in 2^-9 .. 448; S.1111.111 -> NaN)
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(r) : "r"(v));
  return r;
}

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// One 64-weight row segment (32 code bytes at `codes`, its 4 E4M3 block scales in s4, the
// first in the low byte) -> 32 words of f16 pairs (K elements 2j, 2j+1 in word j), the TMEM
// column order of the A operand.
// `flip` (bit 2 of the row): which 16-byte half of the row is read first. Rows are 32 bytes
// apart, so the 8 lanes of a 16-byte load phase cover 4 rows' worth of banks twice unless
// lanes 4..7 of each 8 start on the other half -- then every phase is conflict-free.
__device__ __forceinline__ void expand_row(const uint8_t* codes, uint32_t s4, bool flip, uint32_t (&out)[32]) {
  const uint4 p = *reinterpret_cast<const uint4*>(codes + (flip ? 16 : 0));
  const uint4 q = *reinterpret_cast<const uint4*>(codes + (flip ? 0 : 16));
  const uint4 c0 = flip ? q : p, c1 = flip ? p : q;
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const uint32_t s01 = e4m3x2_to_f16x2(s4), s23 = e4m3x2_to_f16x2(s4 >> 16);
  // each block scale in both halves of a word: blocks of 16 weights = 2 code words
  const uint32_t sc[4] = {__byte_perm(s01, 0u, 0x1010u), __byte_perm(s01, 0u, 0x3232u), __byte_perm(s23, 0u, 0x1010u),
                          __byte_perm(s23, 0u, 0x3232u)};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t a0, a1, a2, a3;
    e2m1x8_to_f16x2(words[i], a0, a1, a2, a3);
    out[4 * i + 0] = f16x2_mul(a0, sc[i >> 1]);
    out[4 * i + 1] = f16x2_mul(a1, sc[i >> 1]);
    out[4 * i + 2] = f16x2_mul(a2, sc[i >> 1]);
    out[4 * i + 3] = f16x2_mul(a3, sc[i >> 1]);
  }
}

// f32 -> f16, round to nearest even, saturating at +-65504 (the h the down projection reads)
__device__ __forceinline__ __half f32_to_f16_sat(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.f16.f32 %0, %1;" : "=h"(r) : "f"(v));
  return __ushort_as_half(r);
}

template <int BN, int EPI, int MT>
__global__ void __launch_bounds__(kFp4Threads, 1)
    k_umma_gemm_fp4(const __grid_constant__ TmaMaps maps, const GemmArgs p, const Fp4Args q4) {
  using S = Fp4Shape<BN, EPI, MT>;
  using TOut = __nv_bfloat16;
  constexpr int kStages = S::kStages;
  constexpr bool kDual = (MT == 2);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kConv = S::kConvSlots;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * S::kStageBytes);
  // bars: full[kStages], empty[kStages], conv[kConv], cfree[kConv], acc_full[2], acc_empty[2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 2 * kConv + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto conv_bar = [&](int c) { return bar0 + 8u * (2 * kStages + c); };
  auto cfree_bar = [&](int c) { return bar0 + 8u * (2 * kStages + kConv + c); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 * kConv + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 * kConv + 2 + a); };
  auto b_tile = [&](int s) { return smem + s * S::kStageBytes; };
  auto code_tile = [&](int s, int m) { return smem + s * S::kStageBytes + S::kBBytes + m * S::kCodeBytes; };
  // TMEM column of converted weight tile m of slot c
  auto conv_col = [&](int c, int m) { return S::kConvCol0 + static_cast<uint32_t>(c) * S::kConvCols + 32u * m; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int c = 0; c < kConv; ++c) {
      mbar_init(conv_bar(c), 4 * MT);
      mbar_init(cfree_bar(c), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf_bar(a), 1);
      mbar_init(acce_bar(a), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.a);
    if (kDual) prefetch_tmap(&maps.a2);
    for (int i = 0; i < 5 && (16 << i) <= BN; ++i) prefetch_tmap(&maps.b[i]);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int num_tiles = *p.num_tiles_dev;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        int g, m0, row0, n;
        gemm_tile(p, t, BN, g, m0, row0, n);
        const int nb16 = (n + 15) >> 4;
        const uint32_t bytes = S::kCodeBytes * MT + static_cast<uint32_t>(nb16) * 2048u;
        const int a_row = g * p.rows_per_group + m0;
        const int a2_row = EPI == EPI_SWIGLU ? a_row : a_row + 128;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status, 0x900u + stage)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), bytes);
          tma_load_2d(smem_u32(code_tile(stage, 0)), &maps.a, full_bar(stage), kb * 32, a_row);
          if (kDual) tma_load_2d(smem_u32(code_tile(stage, 1)), &maps.a2, full_bar(stage), kb * 32, a2_row);
          const uint32_t sB = smem_u32(b_tile(stage));
          const int kc = kb * 64;
          int j16 = 0;
#pragma unroll
          for (int i = 3; i >= 0; --i) {
            if ((16 << i) <= BN && (nb16 >> i) & 1) {
              tma_load_2d(sB + 2048u * j16, &maps.b[i], full_bar(stage), kc, row0 + 16 * j16);
              j16 += 1 << i;
            }
          }
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
          if (issued_mask & (1u << s)) mbar_wait_drain(full_bar(s), (issued_phase >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA issuer
    if (lane == 0) {
      int stage = 0, cs = 0;
      uint32_t phase = 0, cphase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        int g, m0, row0, n;
        gemm_tile(p, t, BN, g, m0, row0, n);
        const uint32_t N = static_cast<uint32_t>((n + 15) & ~15);
        const uint32_t idesc = idesc_f32acc(0u, 128u, N);  // f16 A (TMEM) and B (shared memory)
        if (!mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag, p.status, 0xA00u + acc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc) * S::kAccCols;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status, 0xB00u + stage) ||
              !mbar_wait(conv_bar(cs), cphase, abort_flag, p.status, 0xC00u + cs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sB = smem_u32(b_tile(stage));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            const uint64_t db = sdesc_k_sw128(sB + 32u * kk);
            umma_ts_bf16(d, tmem_base + conv_col(cs, 0) + 8u * kk, db, idesc, accum);
            if (kDual) umma_ts_bf16(d + BN, tmem_base + conv_col(cs, 1) + 8u * kk, db, idesc, accum);
          }
          issued_any = true;
          tc_commit(empty_bar(stage));
          tc_commit(cfree_bar(cs));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
          if (++cs == kConv) {
            cs = 0;
            cphase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(accf_bar(acc));
        if (S::kAccStages == 2) {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        } else {
          acc_phase ^= 1u;
        }
      }
      if (!ok && issued_any) {
        tc_commit(accf_bar(acc));
        mbar_wait_drain(accf_bar(acc), acc_phase);
      }
    }
    __syncwarp();
  } else if (warp >= 6) {
    // ---------------------------------------------------------------- converters
    const int mat = (warp - 6) >> 2;  // which 128-row weight tile: 0 = maps.a, 1 = maps.a2
    const int quad = warp & 3;        // TMEM lane quadrant this warp may write
    const int r = quad * 32 + lane;   // weight row (= TMEM lane) this thread expands
    if (mat < MT) {
      int stage = 0, cs = 0;
      uint32_t phase = 0, cphase = 0;
      bool ok = true;
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        int g, m0, row0, n;
        gemm_tile(p, t, BN, g, m0, row0, n);
        const int a_row = g * p.rows_per_group + m0;
        const int row = (mat == 0 ? a_row : (EPI == EPI_SWIGLU ? a_row : a_row + 128)) + r;
        const uint8_t* sc = (mat == 0 ? q4.scales_a : q4.scales_a2) + static_cast<int64_t>(row) * q4.scale_ld;
        // the row's block scales for 8 k-blocks are one 32-byte sector: two 16-byte loads
        // (when rows are 16-byte aligned), the next sector loaded while this one is used
        auto load8 = [&](int kb0, uint32_t (&dst)[8]) {
          if (kb0 + 8 <= p.k_blocks && (q4.scale_ld & 15) == 0) {  // 16-byte aligned rows
            const uint4 u0 = *reinterpret_cast<const uint4*>(sc + 4 * kb0);
            const uint4 u1 = *reinterpret_cast<const uint4*>(sc + 4 * kb0 + 16);
            dst[0] = u0.x; dst[1] = u0.y; dst[2] = u0.z; dst[3] = u0.w;
            dst[4] = u1.x; dst[5] = u1.y; dst[6] = u1.z; dst[7] = u1.w;
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = kb0 + j < p.k_blocks ? *reinterpret_cast<const uint32_t*>(sc + 4 * (kb0 + j)) : 0u;
          }
        };
        uint32_t cur[8], nxt[8];
        load8(0, cur);
        // k-block j: expand into v, then (late hand-over) finish k-block j - 1 -- wait for its
        // TMEM store, hand its slot to the UMMA -- then store k-block j; with the early
        // hand-over the store is finished right away. pend: a store not yet handed over.
        bool pend = false;
        int pend_cs = 0;
        auto hand_over = [&]() {
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(conv_bar(pend_cs));
          pend = false;
        };
        for (int kb0 = 0; ok && kb0 < p.k_blocks; kb0 += 8) {
          if (kb0 + 8 < p.k_blocks) load8(kb0 + 8, nxt);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int kb = kb0 + j;
            if (kb < p.k_blocks) {
              const bool ready = mbar_wait(full_bar(stage), phase, abort_flag, p.status, 0xD00u + stage) &&
                                 mbar_wait(cfree_bar(cs), cphase ^ 1u, abort_flag, p.status, 0xF00u + cs);
              if (!__all_sync(0xffffffffu, ready)) {
                ok = false;
              } else {
                tc_fence_after();
                uint32_t v[32];
                expand_row(code_tile(stage, mat) + r * 32, cur[j], (r & 4) != 0, v);
                if (pend) hand_over();
                tmem_st32(lane_base + conv_col(cs, mat), v);
                pend = true;
                pend_cs = cs;
                if (!S::kLateHandOver) hand_over();
                if (++stage == kStages) {
                  stage = 0;
                  phase ^= 1u;
                }
                if (++cs == kConv) {
                  cs = 0;
                  cphase ^= 1u;
                }
              }
            }
            if (!ok) break;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) cur[j] = nxt[j];
        }
        if (pend) hand_over();  // the tile's last k-block (also on the abort path: the store is in flight)
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int g, m0, row0, n;
      gemm_tile(p, t, BN, g, m0, row0, n);
      const bool ready = mbar_wait(accf_bar(acc), acc_phase, abort_flag, p.status, 0xE00u + acc);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc) * S::kAccCols;
      TOut* out = reinterpret_cast<TOut*>(p.out);
      const int nchunks = (n + 31) >> 5;
      const float ms_a = q4.mscale_a[g];
      if constexpr (EPI == EPI_SWIGLU) {
        // h = SiLU(gate) * up, written as f16 (the down projection's f16 token operand)
        const float ms_u = q4.mscale_a2[g];
        const int f = m0 + q * 32 + lane;
        const bool f_ok = f < p.m_valid;
        __half* hout = reinterpret_cast<__half*>(p.out);
        for (int c = 0; c < nchunks; ++c) {
          uint32_t v[32], u[32];
          tmem_ld32(taddr + 32u * c, v);
          tmem_ld32(taddr + BN + 32u * c, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = c * 32 + i;
            const float h = silu_tanh(__uint_as_float(v[i]) * ms_a) * (__uint_as_float(u[i]) * ms_u);
            if (tok < n && f_ok) hout[(static_cast<int64_t>(row0) + tok) * p.ld_out + f] = f32_to_f16_sat(h);
          }
        }
      } else {
#pragma unroll
        for (int half = 0; half < MT; ++half) {
          const int f = m0 + half * 128 + q * 32 + lane;
          const bool f_ok = f < p.m_valid;
          float gain1 = 1.0f;
          if (EPI == EPI_STORE_SS && p.ss_gain != nullptr && f_ok)
            gain1 = 1.0f + to_f32(reinterpret_cast<const __nv_bfloat16*>(p.ss_gain)[g * p.ss_gain_group_stride + f]);
          for (int c = 0; c < nchunks; ++c) {
            uint32_t v[32];
            tmem_ld32(taddr + static_cast<uint32_t>(half * BN) + 32u * c, v);
            tmem_ld_wait();
            float yv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) yv[i] = __uint_as_float(v[i]) * ms_a;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int tok = c * 32 + i;
              if (tok < n && f_ok) out[(static_cast<int64_t>(row0) + tok) * p.ld_out + f] = from_f32<TOut>(yv[i]);
            }
            if constexpr (EPI == EPI_STORE_SS) {
              float sq[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float y = yv[i] * gain1;
                sq[i] = f_ok ? y * y : 0.0f;
              }
              const float tot = transpose_reduce32(sq, lane);
              const int tok = c * 32 + lane;
              if (tok < n) p.ss[(static_cast<int64_t>(row0) + tok) * p.ss_ld + ((m0 + half * 128) >> 5) + q] = tot;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(acc));
      if (S::kAccStages == 2) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

}  // namespace muse
