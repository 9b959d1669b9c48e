// gemm_umma_w4a4.cuh -- the grouped expert GEMMs with both operands NVFP4 (W4A4):
//
//   C[token, f] = mscale[e] * sum_k e2m1(w[f, k]) e4m3(ws[f, k/16]) * e2m1(x[token, k]) e4m3(xs[token, k/16])
//
// The tensor core reads the 4-bit codes and their block scales directly
// (tcgen05.mma kind::mxf4nvf4 with one E4M3 scale per 16 elements): nothing is expanded, so
// the weights cross HBM, shared memory and the tensor datapath at 0.5625 bytes each.
//
// Per TMA stage (K = 256 elements, 128 bytes of codes per row): the weight codes of one or
// two 128-row tiles and the token tile's codes, 128-byte swizzled, K-major; the weight rows'
// and tokens' scale bytes (16 per row) as plain row-major boxes. Four scale warps copy the
// scale bytes from shared memory into TMEM in the layout the MMA reads (see umma_mxf4nvf4):
// weight row m's word for MMA kk at lane m, column sfa + 4 kk + m / 32 -- written by the
// warp of m's lane quadrant; token row n's word at column sfb + 4 kk + n / 32 in every lane
// quadrant (each scale warp writes the same words into its own quadrant).
//
// Roles (448 threads, one CTA per SM): warp 0 TMA producer, warp 1 TMEM owner + UMMA
// issuer, warps 2..5 scale warps (warp w serves lane quadrant w % 4), warps 6..13 epilogue
// in two groups of four taking alternate 32-token chunks (the 4-bit main loop is short, so
// the single-buffered accumulator's drain must be too).
// Barriers: per TMA stage full (bytes) / empty (UMMA commit -- after the scale warps have
// read the stage, since the UMMA waits for them); per TMEM scale slot sfull (4 scale
// warps) / sfree (UMMA commit); accumulator full / empty. Every wait is bounded (ptx.cuh).
// Tiles: with a tile counter the producer claims the CTA's next tile from it (atomicAdd)
// and hands the index to the other roles through a 4-slot ring in shared memory, so CTAs
// that free up one after the other take consecutive tiles -- the token chunks of one
// expert's weight tile start together and DRAM delivers the tile once; without a counter,
// static round robin.
#pragma once

#include "gemm_umma.cuh"

namespace muse {

struct W4A4Maps {
  CUtensorMap a;     // weight codes [E * rows, K / 2] uint8, box 128 B x 128 rows, 128-B swizzle
  CUtensorMap a2;    // second weight matrix (gate/up: the up projection; else = a)
  CUtensorMap b;     // token codes [R, K / 2] uint8, box 128 B x BN rows, 128-B swizzle
  CUtensorMap sfa;   // weight scales [E * rows, K / 16] uint8, box 16 B x 128 rows
  CUtensorMap sfa2;
  CUtensorMap sfb;   // token scales [R, K / 16] uint8, box 16 B x BN rows
};

struct W4A4Args {
  const float* mscale_a;   // per-expert matrix scales of the weights behind maps.a
  const float* mscale_a2;  // ... behind maps.a2
};

template <int BN, int EPI, int MT>
struct W4A4Shape {
  static_assert(BN == 32 || BN == 128, "token tiles of 32 or 128 rows");
  static_assert(EPI != EPI_SWIGLU || MT == 2, "SwiGLU needs the gate and up accumulators");
  static constexpr uint32_t kCodeBytes = 128u * 128u;                     // 128 rows x 256 K
  static constexpr uint32_t kBBytes = static_cast<uint32_t>(BN) * 128u;
  static constexpr uint32_t kSfaBytes = 128u * 16u;
  static constexpr uint32_t kSfbBytes = static_cast<uint32_t>(BN) * 16u;
  static constexpr uint32_t kTxBytes = kCodeBytes * MT + kBBytes + kSfaBytes * MT + kSfbBytes;
  static constexpr uint32_t kStageBytes = (kTxBytes + 1023u) & ~1023u;    // swizzled tiles stay 1024-aligned
  static constexpr int kSmemBudget = 227 * 1024 - 1024 - 512;
  static constexpr int kStagesFit = kSmemBudget / static_cast<int>(kStageBytes);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kAccStages = MT == 2 ? 1 : 2;
  static constexpr uint32_t kAccCols = static_cast<uint32_t>(BN) * MT;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM scale slots after the accumulators: per slot 16 columns per weight tile (4 MMAs x 4
  // lane-quadrant columns) and 16 for the tokens (4 MMAs x up to 4 columns of 32 rows)
  static constexpr uint32_t kSfCol0 = kAccCols * kAccStages;
  static constexpr uint32_t kSlotCols = 16u * MT + 16u;
  static constexpr int kSlotsFit = static_cast<int>((kTmemCols - kSfCol0) / kSlotCols);
  static constexpr int kSlots = kSlotsFit > 4 ? 4 : kSlotsFit;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + 512;
  static_assert(kStages >= 2, "tile too large for the shared-memory ring");
  static_assert(kSlots >= 2, "no TMEM room for the scale slots");
  static constexpr int kSched = 4;
  static constexpr int kSchedReaders = 1 + 4 + 8;  // UMMA thread, scale warps, epilogue warps
  static_assert(8 * (2 * kStages + 2 * kSlots + 4 + 2 * kSched) + 8 + 4 * kSched <= 512, "barrier area");
};

constexpr int kW4A4Threads = 448;

template <int BN, int EPI, int MT>
__global__ void __launch_bounds__(kW4A4Threads, 1)
    k_umma_gemm_w4a4(const __grid_constant__ W4A4Maps maps, const GemmArgs p, const W4A4Args q) {
  using S = W4A4Shape<BN, EPI, MT>;
  using TOut = __nv_bfloat16;
  constexpr int kStages = S::kStages;
  constexpr int kSlots = S::kSlots;
  constexpr bool kDual = (MT == 2);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * S::kStageBytes);
  // bars: full[kStages], empty[kStages], sfull[kSlots], sfree[kSlots], accf[2], acce[2],
  // tfull[kSched], tempty[kSched]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 2 * kSlots + 4 + 2 * S::kSched);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* tile_ring = reinterpret_cast<volatile int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto sfull_bar = [&](int c) { return bar0 + 8u * (2 * kStages + c); };
  auto sfree_bar = [&](int c) { return bar0 + 8u * (2 * kStages + kSlots + c); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 * kSlots + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 * kSlots + 2 + a); };
  auto tfull_bar = [&](int i) { return bar0 + 8u * (2 * kStages + 2 * kSlots + 4 + i); };
  auto tempty_bar = [&](int i) { return bar0 + 8u * (2 * kStages + 2 * kSlots + 4 + S::kSched + i); };
  // stage layout: weight codes (MT x 16 KB), token codes, weight scales (MT x 2 KB), token scales
  auto code_tile = [&](int s, int m) { return smem + s * S::kStageBytes + m * S::kCodeBytes; };
  auto b_tile = [&](int s) { return smem + s * S::kStageBytes + MT * S::kCodeBytes; };
  auto sfa_tile = [&](int s, int m) { return b_tile(s) + S::kBBytes + m * S::kSfaBytes; };
  auto sfb_tile = [&](int s) { return b_tile(s) + S::kBBytes + MT * S::kSfaBytes; };
  // TMEM columns of scale slot c
  auto sfa_col = [&](int c, int m) { return S::kSfCol0 + static_cast<uint32_t>(c) * S::kSlotCols + 16u * m; };
  auto sfb_col = [&](int c) { return S::kSfCol0 + static_cast<uint32_t>(c) * S::kSlotCols + 16u * MT; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int c = 0; c < kSlots; ++c) {
      mbar_init(sfull_bar(c), 4);
      mbar_init(sfree_bar(c), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf_bar(a), 1);
      mbar_init(acce_bar(a), 8);  // 8 epilogue warps
    }
    for (int i = 0; i < S::kSched; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), S::kSchedReaders);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.a);
    prefetch_tmap(&maps.b);
    prefetch_tmap(&maps.sfa);
    prefetch_tmap(&maps.sfb);
    if (kDual) {
      prefetch_tmap(&maps.a2);
      prefetch_tmap(&maps.sfa2);
    }
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
  const bool dyn = p.tile_counter != nullptr;

  // The CTA's i-th tile: -1 past the end, -2 when a wait gave up. The producer claims and
  // publishes it; the other roles receive it (one thread or a whole warp) and free the slot
  // (one arrival per thread or warp).
  auto claim_publish = [&](int i) -> int {
    int t = dyn ? atomicAdd(p.tile_counter, 1) : static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    if (t >= num_tiles) t = -1;
    if (!dyn) return t;
    const int sl = i % S::kSched;
    const uint32_t ph = static_cast<uint32_t>(i / S::kSched) & 1u;
    if (!mbar_wait(tempty_bar(sl), ph ^ 1u, abort_flag, p.status, 0x1700u + sl)) return -2;
    tile_ring[sl] = t;
    mbar_arrive(tfull_bar(sl));
    return t;
  };
  auto receive = [&](int i, uint32_t code) -> int {
    if (!dyn) {
      const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
      return t < num_tiles ? t : -1;
    }
    const int sl = i % S::kSched;
    const uint32_t ph = static_cast<uint32_t>(i / S::kSched) & 1u;
    if (!mbar_wait(tfull_bar(sl), ph, abort_flag, p.status, code + sl)) return -2;
    return tile_ring[sl];
  };
  auto release = [&](int i) {
    if (dyn) mbar_arrive(tempty_bar(i % S::kSched));
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int t = claim_publish(i);
        if (t == -2) {
          ok = false;
          break;
        }
        if (t < 0) break;
        int g, m0, row0, n;
        gemm_tile(p, t, BN, g, m0, row0, n);
        const int a_row = g * p.rows_per_group + m0;
        const int a2_row = EPI == EPI_SWIGLU ? a_row : a_row + 128;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status, 0x1000u + stage)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, S::kTxBytes);
          tma_load_2d(smem_u32(code_tile(stage, 0)), &maps.a, fb, kb * 128, a_row);
          if (kDual) tma_load_2d(smem_u32(code_tile(stage, 1)), &maps.a2, fb, kb * 128, a2_row);
          tma_load_2d(smem_u32(b_tile(stage)), &maps.b, fb, kb * 128, row0);
          tma_load_2d(smem_u32(sfa_tile(stage, 0)), &maps.sfa, fb, kb * 16, a_row);
          if (kDual) tma_load_2d(smem_u32(sfa_tile(stage, 1)), &maps.sfa2, fb, kb * 16, a2_row);
          tma_load_2d(smem_u32(sfb_tile(stage)), &maps.sfb, fb, kb * 16, row0);
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
      for (int i = 0; ok; ++i) {
        const int t = receive(i, 0x1800u);
        if (t == -2) {
          ok = false;
          break;
        }
        release(i);
        if (t < 0) break;
        int g, m0, row0, n;
        gemm_tile(p, t, BN, g, m0, row0, n);
        const uint32_t N = static_cast<uint32_t>((n + 15) & ~15);
        const uint32_t idesc = idesc_mxf4nvf4(128u, N);
        if (!mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag, p.status, 0x1100u + acc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc) * S::kAccCols;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status, 0x1200u + stage) ||
              !mbar_wait(sfull_bar(cs), cphase, abort_flag, p.status, 0x1300u + cs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sB = smem_u32(b_tile(stage));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            const uint64_t db = sdesc_k_sw128(sB + 32u * kk);
            const uint32_t sfb = tmem_base + sfb_col(cs) + 4u * kk;
            umma_mxf4nvf4(d, sdesc_k_sw128(smem_u32(code_tile(stage, 0)) + 32u * kk), db, idesc,
                          tmem_base + sfa_col(cs, 0) + 4u * kk, sfb, accum);
            if (kDual)
              umma_mxf4nvf4(d + BN, sdesc_k_sw128(smem_u32(code_tile(stage, 1)) + 32u * kk), db, idesc,
                            tmem_base + sfa_col(cs, 1) + 4u * kk, sfb, accum);
          }
          issued_any = true;
          tc_commit(empty_bar(stage));
          tc_commit(sfree_bar(cs));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
          if (++cs == kSlots) {
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
  } else if (warp < 6) {
    // ---------------------------------------------------------------- scale warps (2..5)
    const int quad = warp & 3;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    int stage = 0, cs = 0;
    uint32_t phase = 0, cphase = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      int t = receive(i, 0x1900u);
      if (!__all_sync(0xffffffffu, t != -2)) break;
      t = __shfl_sync(0xffffffffu, t, 0);
      __syncwarp();
      if (lane == 0) release(i);
      if (t < 0) break;
      for (int kb = 0; kb < p.k_blocks; ++kb) {
        const bool ready = mbar_wait(full_bar(stage), phase, abort_flag, p.status, 0x1400u + stage) &&
                           mbar_wait(sfree_bar(cs), cphase ^ 1u, abort_flag, p.status, 0x1500u + cs);
        if (!__all_sync(0xffffffffu, ready)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // weight rows 32 * quad + lane: MMA kk reads column sfa + 4 kk + quad of this lane
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint4 w = *reinterpret_cast<const uint4*>(sfa_tile(stage, m) + (quad * 32 + lane) * 16);
          const uint32_t col = lane_base + sfa_col(cs, m) + static_cast<uint32_t>(quad);
          tmem_st_x1(col + 0u, w.x);
          tmem_st_x1(col + 4u, w.y);
          tmem_st_x1(col + 8u, w.z);
          tmem_st_x1(col + 12u, w.w);
        }
        // token rows 32 j + lane: MMA kk reads column sfb + 4 kk + j, in every quadrant
        if constexpr (BN == 32) {
          const uint4 w = *reinterpret_cast<const uint4*>(sfb_tile(stage) + lane * 16);
          const uint32_t col = lane_base + sfb_col(cs);
          tmem_st_x1(col + 0u, w.x);
          tmem_st_x1(col + 4u, w.y);
          tmem_st_x1(col + 8u, w.z);
          tmem_st_x1(col + 12u, w.w);
        } else {
          uint4 w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const uint4*>(sfb_tile(stage) + (32 * j + lane) * 16);
          const uint32_t col = lane_base + sfb_col(cs);
          tmem_st_x4(col + 0u, w[0].x, w[1].x, w[2].x, w[3].x);
          tmem_st_x4(col + 4u, w[0].y, w[1].y, w[2].y, w[3].y);
          tmem_st_x4(col + 8u, w[0].z, w[1].z, w[2].z, w[3].z);
          tmem_st_x4(col + 12u, w[0].w, w[1].w, w[2].w, w[3].w);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sfull_bar(cs));
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
        if (++cs == kSlots) {
          cs = 0;
          cphase ^= 1u;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (6..13)
    const int qd = warp & 3;
    const int grp = (warp - 6) >> 2;  // chunks c with c % 2 == grp
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int i = 0;; ++i) {
      int t = receive(i, 0x1A00u);
      if (!__all_sync(0xffffffffu, t != -2)) break;
      t = __shfl_sync(0xffffffffu, t, 0);
      __syncwarp();
      if (lane == 0) release(i);
      if (t < 0) break;
      int g, m0, row0, n;
      gemm_tile(p, t, BN, g, m0, row0, n);
      const bool ready = mbar_wait(accf_bar(acc), acc_phase, abort_flag, p.status, 0x1600u + acc);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) +
                             static_cast<uint32_t>(acc) * S::kAccCols;
      TOut* out = reinterpret_cast<TOut*>(p.out);
      const int nchunks = (n + 31) >> 5;
      const float ms_a = q.mscale_a[g];
      if constexpr (EPI == EPI_SWIGLU) {
        const float ms_u = q.mscale_a2[g];
        const int f = m0 + qd * 32 + lane;
        const bool f_ok = f < p.m_valid;
        for (int c = grp; c < nchunks; c += 2) {
          uint32_t v[32], u[32];
          tmem_ld32(taddr + 32u * c, v);
          tmem_ld32(taddr + BN + 32u * c, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = c * 32 + i;
            const float a = __uint_as_float(v[i]) * ms_a;
            const float h = __fdividef(a, 1.0f + __expf(-a)) * (__uint_as_float(u[i]) * ms_u);  // SiLU(gate) * up
            if (tok < n && f_ok) out[(static_cast<int64_t>(row0) + tok) * p.ld_out + f] = from_f32<TOut>(h);
          }
        }
      } else {
#pragma unroll
        for (int half = 0; half < MT; ++half) {
          const int f = m0 + half * 128 + qd * 32 + lane;
          const bool f_ok = f < p.m_valid;
          const float ms = half == 0 ? ms_a : q.mscale_a2[g];
          float gain1 = 1.0f;
          if (EPI == EPI_STORE_SS && p.ss_gain != nullptr && f_ok)
            gain1 = 1.0f + to_f32(reinterpret_cast<const __nv_bfloat16*>(p.ss_gain)[g * p.ss_gain_group_stride + f]);
          for (int c = grp; c < nchunks; c += 2) {
            uint32_t v[32];
            tmem_ld32(taddr + static_cast<uint32_t>(half * BN) + 32u * c, v);
            tmem_ld_wait();
            float yv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) yv[i] = __uint_as_float(v[i]) * ms;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int tok = c * 32 + i;
              if (tok < n && f_ok) out[(static_cast<int64_t>(row0) + tok) * p.ld_out + f] = from_f32<TOut>(yv[i]);
            }
            if constexpr (EPI == EPI_STORE_SS) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float y = yv[i] * gain1;
                yv[i] = f_ok ? y * y : 0.0f;
              }
              const float tot = transpose_reduce32(yv, lane);
              const int tok = c * 32 + lane;
              if (tok < n) p.ss[(static_cast<int64_t>(row0) + tok) * p.ss_ld + ((m0 + half * 128) >> 5) + qd] = tot;
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
