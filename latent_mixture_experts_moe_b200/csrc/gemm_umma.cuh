// gemm_umma.cuh -- persistent, warp-specialised tcgen05 GEMM for every dense contraction
// of the latent-MoE block (router logits, pooler, expert gate/up, expert down, unpooler).
//
//   C[token, f] = sum_k W[f, k] * X[token, k]         (both operands K-contiguous)
//
// Weights are the UMMA "A" operand (M = 128 output features per tile) and tokens the
// "B" operand (N = tokens per tile, 16..BN, a runtime value), so one kernel serves a
// decode batch (a few tokens per expert: N = 16) and a prefill batch (N up to 256)
// without padding the token side to 128. The accumulator tile lives in TMEM as
// 128 lanes (features) x N columns (tokens) of FP32.
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: A tile 128 x 128 B (+ a second A tile for gate/up) and the
//               token tile in at most 5 boxes of 16..256 rows (one box for a full tile),
//               128-byte swizzle, into a STAGES-deep ring guarded by full/empty mbarriers;
//   warp 1      TMEM allocator and UMMA issuer (one thread): 4 x K=16 (bf16) or K=8 (tf32)
//               MMAs per stage, tcgen05.commit frees the stage; a commit per tile hands
//               the accumulator to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, then one of
//               EPI_STORE   y -> out (activation dtype, or float32 for router logits)
//               EPI_SWIGLU  SiLU(gate) * up -> H (two accumulators, same lanes)
//               EPI_STORE_SS  y -> Y plus per-token partial sums of y^2 over the warp's
//                             32 features (for the per-expert RMSNorm), from the FP32
//                             accumulator before rounding.
// With MT = 2 two 128-row weight tiles share each token tile (256 features per CTA tile,
// or gate + up of 128 features); with MT = 1 the TMEM accumulator is double-buffered so
// the epilogue of tile i overlaps the MMAs of tile i+1.
//
// Work list: either a device-built list of int4 {group, m0, row0, n} (grouped expert
// GEMMs; built by the routing kernels, never read by the host) or implicit dense
// tiling over (M/128) x ceil(T/BN) tiles. Tiles are strided over the persistent grid.
//
// Every mbarrier wait is bounded (see ptx.cuh): a timeout records MUSE_ERR_TIMEOUT in
// the workspace status word, all roles stop, in-flight copies and MMAs are drained with
// bounded waits, and TMEM is freed before the CTA exits.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace muse {

enum EpiMode : int { EPI_STORE = 0, EPI_SWIGLU = 1, EPI_STORE_SS = 2 };

struct GemmArgs {
  const int4* tiles;         // grouped: device tile list; nullptr: dense implicit tiling
  const int* num_tiles_dev;  // grouped: device tile count
  int num_tiles;             // dense: m_tiles * ceil(T / BN)
  int m_tiles;               // dense: tiles along M
  int m_step;                // dense: features per tile (128 * MT)
  int rows_per_group;        // rows of A per group (expert); A row = group * this + m0
  int m_valid;               // valid output features per group (stores masked beyond)
  int T;                     // dense: token rows of B
  int k_blocks;              // K / (128 bytes of elements)
  void* out;                 // output [rows, ld_out]
  int64_t ld_out;
  float* ss;                 // EPI_STORE_SS: partial sums [rows, ss_ld]
  int ss_ld;
  const void* ss_gain;       // EPI_STORE_SS: optional gain offsets; squares y*(1+gain)
  int64_t ss_gain_group_stride;  // elements between groups' gains (0 = shared)
  uint32_t* status;          // workspace status word
  int* tile_counter;         // CTA-pair kernel: tiles are claimed from this counter (zero
                             // before the launch); nullptr: static round robin over pairs
  int k_splits;              // one-CTA dense GEMM: K divided into this many equal ranges of
                             // k-blocks (0 or 1: none); range s writes its FP32 partial
                             // product to (float*)out + s * split_stride
  int64_t split_stride;
  int m_group;               // dense tiling: weight tiles per group (0: none). Tiles run group by
                             // group, each group's m-tiles side by side for every token chunk,
                             // so the weights a wave of CTAs streams stay within the group
};

// Split-K decode of launch tile t (dense tiling): range s = t / base of base tile t % base,
// base = num_tiles / k_splits, over k-blocks [kb0, kb1). Without splits: the whole K.
__device__ __forceinline__ void split_range(const GemmArgs& p, int num_tiles, int& t, int& s, int& kb0, int& kb1) {
  if (p.k_splits > 1) {
    const int base = num_tiles / p.k_splits;
    const int per = p.k_blocks / p.k_splits;  // the host splits only evenly
    s = t / base;
    t -= s * base;
    kb0 = s * per;
    kb1 = kb0 + per;
  } else {
    s = 0;
    kb0 = 0;
    kb1 = p.k_blocks;
  }
}

template <typename TIn>
struct ElemTraits;
template <>
struct ElemTraits<__nv_bfloat16> {
  static constexpr bool kTF32 = false;
  static constexpr uint32_t kFmt = 1;  // bf16
};
template <>
struct ElemTraits<float> {
  static constexpr bool kTF32 = true;
  static constexpr uint32_t kFmt = 2;  // tf32
};

__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }
template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }

// MT = 128-row weight tiles per CTA: 2 puts two accumulators behind one token tile
// (gate and up for EPI_SWIGLU; two adjacent 128-feature blocks otherwise), which halves
// the operand bytes the CTA loads per MMA cycle compared with MT = 1.
template <int BN, int EPI, int MT>
struct GemmShape {
  static constexpr bool kDual = (MT == 2);
  static_assert(MT == 1 || MT == 2, "MT is 1 or 2");
  static_assert(EPI != EPI_SWIGLU || MT == 2, "SwiGLU needs the gate and up accumulators");
  static constexpr uint32_t kABytes = 128u * 128u;              // 128 rows x 128 B
  static constexpr uint32_t kBBytes = static_cast<uint32_t>(BN) * 128u;
  static constexpr uint32_t kStageBytes = kABytes * (kDual ? 2u : 1u) + kBBytes;
  static constexpr int kSmemBudget = 227 * 1024 - 1024 - 256;   // minus alignment slack, barriers
  static constexpr int kStagesFit = kSmemBudget / static_cast<int>(kStageBytes);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kAccStages = kDual ? 1 : 2;
  static constexpr uint32_t kAccCols = kDual ? 2u * BN : static_cast<uint32_t>(BN);
  static constexpr uint32_t kColsNeeded = kAccCols * kAccStages;
  static constexpr uint32_t kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64
                                        : kColsNeeded <= 128 ? 128 : kColsNeeded <= 256 ? 256 : 512;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + 256;
  static_assert(kStages >= 2, "tile too large for the shared-memory ring");
  static_assert(kColsNeeded <= 512, "accumulators exceed TMEM");
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be 32..256, multiple of 32");
};

__device__ __forceinline__ void gemm_tile(const GemmArgs& p, int t, int BN, int& g, int& m0, int& row0,
                                          int& n) {
  if (p.tiles != nullptr) {
    const int4 v = p.tiles[t];
    g = v.x;
    m0 = v.y;
    row0 = v.z;
    n = v.w;
  } else {
    int mt = t % p.m_tiles;
    int ch = t / p.m_tiles;
    if (p.m_group > 0 && p.m_group < p.m_tiles) {
      const int chunks = (p.T + BN - 1) / BN;
      const int gi = t / (p.m_group * chunks);        // group (the last one may hold fewer m-tiles)
      const int r = t - gi * p.m_group * chunks;
      const int gsz = min(p.m_group, p.m_tiles - gi * p.m_group);
      mt = gi * p.m_group + r % gsz;
      ch = r / gsz;
    }
    g = 0;
    m0 = mt * p.m_step;
    row0 = ch * BN;
    n = min(BN, p.T - row0);
  }
}

// Sum over the 32 lanes of each of 32 registers: afterwards lane l holds the total of
// register l (butterfly exchange of halves, 31 shuffles for 32 sums).
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// Tensor maps of one launch: the weight operand (a second one for the up projection)
// and the token operand with boxes of 16 << i rows, i = 0..4, so that a tile of n rows
// loads in popcount(ceil(n / 16)) copies (one copy for a full 256-row tile).
struct TmaMaps {
  CUtensorMap a;
  CUtensorMap a2;
  CUtensorMap b[5];
  CUtensorMap out;  // output [rows, features], 16-row x 128-feature boxes (CTA-pair bf16 stores)
};

template <typename TIn, typename TOut, int BN, int EPI, int MT>
__global__ void __launch_bounds__(192, 1) k_umma_gemm(const __grid_constant__ TmaMaps maps, const GemmArgs p) {
  using S = GemmShape<BN, EPI, MT>;
  constexpr bool kDual = S::kDual;
  constexpr int kStages = S::kStages;
  constexpr bool kTF32 = ElemTraits<TIn>::kTF32;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * S::kStageBytes);
  // bars: full[kStages], empty[kStages], acc_full[2], acc_empty[2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * kStages + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 + a); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
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
  const int num_tiles = (p.tiles != nullptr) ? *p.num_tiles_dev : p.num_tiles;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // per stage, for the abort drain
      bool ok = true;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        int g, m0, row0, n, tb = t, ks, kb0, kb1;
        split_range(p, num_tiles, tb, ks, kb0, kb1);
        gemm_tile(p, tb, BN, g, m0, row0, n);
        const int nb16 = (n + 15) >> 4;
        const uint32_t bytes = S::kABytes * (kDual ? 2u : 1u) + static_cast<uint32_t>(nb16) * 2048u;
        const int a_row = g * p.rows_per_group + m0;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status, 0x100u + stage)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), bytes);
          const uint32_t sA = smem_u32(smem + stage * S::kStageBytes);
          const int kc = kb * static_cast<int>(128 / sizeof(TIn));
          tma_load_2d(sA, &maps.a, full_bar(stage), kc, a_row);
          // second weight tile: the up projection at the same rows, or the next 128 rows
          if (kDual) tma_load_2d(sA + S::kABytes, &maps.a2, full_bar(stage), kc, EPI == EPI_SWIGLU ? a_row : a_row + 128);
          const uint32_t sB = sA + S::kABytes * (kDual ? 2u : 1u);
          // largest boxes first: 16-row block offset j16 advances by each box's height
          int j16 = 0;
#pragma unroll
          for (int i = 4; i >= 0; --i) {
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
        // let every copy this thread started land before the CTA can exit
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) mbar_wait_drain(full_bar(s), (issued_phase >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        int g, m0, row0, n, tb = t, ks, kb0, kb1;
        split_range(p, num_tiles, tb, ks, kb0, kb1);
        gemm_tile(p, tb, BN, g, m0, row0, n);
        const uint32_t N = static_cast<uint32_t>((n + 15) & ~15);
        const uint32_t idesc = idesc_f32acc(ElemTraits<TIn>::kFmt, 128u, N);
        if (!mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag, p.status, 0x200u + acc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc) * S::kAccCols;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status, 0x300u + stage)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(smem + stage * S::kStageBytes);
          const uint32_t sB = sA + S::kABytes * (kDual ? 2u : 1u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t accum = (kb > kb0 || kk > 0) ? 1u : 0u;
            const uint64_t db = sdesc_k_sw128(sB + 32u * kk);
            umma<kTF32>(d, sdesc_k_sw128(sA + 32u * kk), db, idesc, accum);
            if (kDual) umma<kTF32>(d + BN, sdesc_k_sw128(sA + S::kABytes + 32u * kk), db, idesc, accum);
          }
          issued_any = true;
          tc_commit(empty_bar(stage));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
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
        // wait until every MMA issued so far has finished writing TMEM
        tc_commit(accf_bar(acc));
        mbar_wait_drain(accf_bar(acc), acc_phase);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int g, m0, row0, n, tb = t, ks, kb0, kb1;
      split_range(p, num_tiles, tb, ks, kb0, kb1);
      gemm_tile(p, tb, BN, g, m0, row0, n);
      // every lane waits; the vote keeps the warp converged for the .sync.aligned loads
      const bool ready = mbar_wait(accf_bar(acc), acc_phase, abort_flag, p.status, 0x400u + acc);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc) * S::kAccCols;
      TOut* out = reinterpret_cast<TOut*>(p.out) + static_cast<int64_t>(ks) * p.split_stride;
      const int nchunks = (n + 31) >> 5;
      if constexpr (EPI == EPI_SWIGLU) {
        const int f = m0 + q * 32 + lane;  // output feature of this thread (within group)
        const bool f_ok = f < p.m_valid;
        for (int c = 0; c < nchunks; ++c) {
          uint32_t v[32], u[32];
          tmem_ld32(taddr + 32u * c, v);
          tmem_ld32(taddr + BN + 32u * c, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = c * 32 + i;
            const float a = __uint_as_float(v[i]);
            const float h = a / (1.0f + __expf(-a)) * __uint_as_float(u[i]);
            if (tok < n && f_ok) out[(static_cast<int64_t>(row0) + tok) * p.ld_out + f] = from_f32<TOut>(h);
          }
        }
      } else {
#pragma unroll
        for (int half = 0; half < MT; ++half) {
          const int f = m0 + half * 128 + q * 32 + lane;
          const bool f_ok = f < p.m_valid;
          float gain1 = 1.0f;
          if (EPI == EPI_STORE_SS && p.ss_gain != nullptr && f_ok)
            gain1 = 1.0f + to_f32(reinterpret_cast<const TIn*>(p.ss_gain)[g * p.ss_gain_group_stride + f]);
          for (int c = 0; c < nchunks; ++c) {
            uint32_t v[32];
            tmem_ld32(taddr + static_cast<uint32_t>(half * BN) + 32u * c, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int tok = c * 32 + i;
              if (tok < n && f_ok)
                out[(static_cast<int64_t>(row0) + tok) * p.ld_out + f] = from_f32<TOut>(__uint_as_float(v[i]));
            }
            if constexpr (EPI == EPI_STORE_SS) {
              float sq[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float y = __uint_as_float(v[i]) * gain1;
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
