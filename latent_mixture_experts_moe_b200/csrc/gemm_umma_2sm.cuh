// gemm_umma_2sm.cuh -- the same contraction as gemm_umma.cuh on a CTA pair (a cluster of
// two CTAs on one TPC) with cta_group::2 UMMAs, for tiles of up to 256 tokens (prefill):
//
//   the pair tile is 256 (or 512) output features x N <= 256 tokens; each CTA stages
//   128 weight rows per weight tile and HALF of the token tile (N/2 rows) in its own
//   shared memory; the leader CTA (cluster rank 0) issues M = 256 MMAs that read both
//   CTAs' tiles, and each CTA's TMEM receives its own 128 feature rows x N columns.
//
// Per SM and MMA cycle this moves 48 bytes of operands (gate/up; 512-feature down tiles)
// or 64 (256-feature tiles) instead of 64 / 96 for one CTA, and the ring holds more
// stages. Synchronisation:
//   * both CTAs' TMA copies complete on the LEADER's full barrier (cta_group::2 form of the
//     copy, no multicast); only the leader posts the expected bytes of both halves;
//   * the leader's tcgen05.commit multicasts "stage free" to both CTAs' empty barriers and
//     "accumulator ready" to both CTAs' accumulator barriers;
//   * both CTAs' epilogue warps release the accumulator on the leader's barrier (8 arrivals,
//     remote ones through the cluster window);
//   * a cluster barrier after initialisation and before TMEM is freed keeps each CTA alive
//     while its partner may still touch its barriers, shared memory or TMEM.
// Tile scheduling: with a tile counter the leader's producer claims the pair's next tile
// from it (atomicAdd) when it is about to load it, and hands the index to every role of
// both CTAs through a 4-deep ring in shared memory (the partner's copy is written through
// the cluster window; full / empty mbarriers per slot). Pairs that become free one after
// the other take consecutive tiles, and the tile list orders the token chunks of one
// expert's feature tile side by side, so the pairs that share a weight tile stream it at
// the same time and DRAM delivers it once (a static round robin lets them drift apart by
// more than L2 can bridge). Without a counter the pairs take tiles round robin.
// Every wait is bounded as in gemm_umma.cuh.
#pragma once

#include <type_traits>

#include "gemm_umma.cuh"

namespace muse {

template <int EPI, int MT>
struct Gemm2Shape {
  static constexpr bool kDual = (MT == 2);
  static_assert(MT == 1 || MT == 2, "MT is 1 or 2");
  static_assert(EPI != EPI_SWIGLU || MT == 2, "SwiGLU needs the gate and up accumulators");
  static constexpr int kBN = 256;                               // tokens per pair tile
  static constexpr uint32_t kABytes = 128u * 128u;              // 128 weight rows x 128 B
  static constexpr uint32_t kBBytes = 128u * 128u;              // 128 token rows x 128 B
  static constexpr uint32_t kStageBytes = kABytes * MT + kBBytes;
  // output staging for TMA stores: per epilogue group 2 buffers x 32 token rows x 128
  // features of bf16
  static constexpr uint32_t kOutBufBytes = 32u * 128u * 2u;
  static constexpr uint32_t kOutBytes = 2u * 2u * kOutBufBytes;
  static constexpr int kSmemBudget = 227 * 1024 - 1024 - 512 - static_cast<int>(kOutBytes);
  static constexpr int kStagesFit = kSmemBudget / static_cast<int>(kStageBytes);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kAccStages = kDual ? 1 : 2;
  static constexpr uint32_t kAccCols = 256u * MT;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + kOutBytes + 512;
  // tile-index ring (dynamic scheduling): slots, and the readers of each slot -- the
  // leader's UMMA thread and 8 epilogue warps, the partner's producer and 8 epilogue warps
  static constexpr int kSched = 4;
  static constexpr int kSchedReaders = 1 + 8 + 1 + 8;
  static_assert(8 * (2 * kStages + 4 + 2 * kSched) + 8 + 4 * kSched <= 512, "barrier area");
  // output features covered by one pair tile
  static constexpr int kFeatStep = (EPI == EPI_SWIGLU) ? 256 : 256 * MT;
  static_assert(kAccCols * kAccStages <= kTmemCols, "accumulators exceed TMEM");
};

// 10 warps: 0 TMA producer, 1 TMEM owner + UMMA issuer (leader), 2..9 epilogue in two
// groups of four (one warp per TMEM lane quadrant each) taking alternate token chunks
constexpr int kPairThreads = 320;

template <typename TOut, int EPI, int MT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    k_umma_gemm_2sm(const __grid_constant__ TmaMaps maps, const GemmArgs p) {
  using S = Gemm2Shape<EPI, MT>;
  using TIn = __nv_bfloat16;
  constexpr bool kDual = S::kDual;
  constexpr int kStages = S::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* out_stage = smem + kStages * S::kStageBytes;  // 1024-aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + S::kOutBytes);
  constexpr bool kTmaStore = std::is_same<TOut, __nv_bfloat16>::value;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 4 + 2 * S::kSched);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* sched_ring = reinterpret_cast<volatile int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * kStages + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 + a); };
  auto sfull_bar = [&](int s) { return bar0 + 8u * (2 * kStages + 4 + s); };
  auto sempty_bar = [&](int s) { return bar0 + 8u * (2 * kStages + 4 + S::kSched + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf_bar(a), 1);
      mbar_init(acce_bar(a), 16);  // 8 epilogue warps in each CTA of the pair
    }
    for (int s = 0; s < S::kSched; ++s) {
      mbar_init(sfull_bar(s), 1);
      mbar_init(sempty_bar(s), S::kSchedReaders);  // used on the leader
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.a);
    if (kDual) prefetch_tmap(&maps.a2);
    for (int i = 0; i < 4; ++i) prefetch_tmap(&maps.b[i]);
    if (kTmaStore) prefetch_tmap(&maps.out);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), S::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // partner barriers are initialised before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int num_tiles = (p.tiles != nullptr) ? *p.num_tiles_dev : p.num_tiles;
  const bool dyn = (p.tile_counter != nullptr);

  // The pair's i-th tile: -1 past the end, -2 when a wait gave up. The leader's producer
  // claims and publishes it; every other role receives it and then frees the slot.
  auto claim_tile = [&](int i) -> int {
    const int t = dyn ? atomicAdd(p.tile_counter, 1) : pair + i * npairs;
    return t < num_tiles ? t : -1;
  };
  auto publish_tile = [&](int i, int t) -> bool {
    if (!dyn) return true;
    const int s = i % S::kSched;
    const uint32_t ph = static_cast<uint32_t>(i / S::kSched) & 1u;
    if (!mbar_wait<true>(sempty_bar(s), ph ^ 1u, abort_flag, p.status, 0x900u + s)) return false;
    sched_ring[s] = t;
    st_shared_cluster_u32(mapa_shared(smem_u32(const_cast<int*>(sched_ring + s)), 1), static_cast<uint32_t>(t));
    mbar_arrive(sfull_bar(s));
    mbar_arrive_cluster(mapa_shared(sfull_bar(s), 1));  // release: orders the store above
    return true;
  };
  auto receive_tile = [&](int i, uint32_t code) -> int {
    if (!dyn) {
      const int t = pair + i * npairs;
      return t < num_tiles ? t : -1;
    }
    const int s = i % S::kSched;
    const uint32_t ph = static_cast<uint32_t>(i / S::kSched) & 1u;
    if (!mbar_wait<true>(sfull_bar(s), ph, abort_flag, p.status, code + s)) return -2;
    return sched_ring[s];
  };
  auto release_tile = [&](int i) {
    if (!dyn) return;
    const uint32_t b = sempty_bar(i % S::kSched);
    if (leader) {
      mbar_arrive(b);
    } else {
      mbar_arrive_cluster(mapa_shared(b, 0));
    }
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        int t;
        if (leader) {
          t = claim_tile(i);
          if (!publish_tile(i, t)) {
            ok = false;
            break;
          }
        } else {
          t = receive_tile(i, 0x940u);
          if (t == -2) {
            ok = false;
            break;
          }
          release_tile(i);
        }
        if (t < 0) break;
        int g, m0, row0, n;
        gemm_tile(p, t, S::kBN, g, m0, row0, n);
        // N = n rounded up to 16 (the M = 256 MMA's N granularity); each CTA stages N / 2
        // token rows, a multiple of 8, loaded as 16-row boxes: the last box may carry 8 rows
        // past the half (the partner's first rows, or zero fill past the tensor), which
        // still lie inside the stage's 128-row B area and count in the expected bytes
        const int N = (n + 15) & ~15;
        const int half = N >> 1;             // token rows the MMA reads from this CTA
        const int nb16 = (half + 15) >> 4;   // 1..8 boxes of 16 rows
        const uint32_t bytes_pair = 2u * (S::kABytes * MT + static_cast<uint32_t>(nb16) * 2048u);
        const int a_row = g * p.rows_per_group + m0 + static_cast<int>(rank) * 128;
        const int a2_row = (EPI == EPI_SWIGLU) ? a_row : a_row + 256;
        const int b_row = row0 + static_cast<int>(rank) * half;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait<true>(empty_bar(stage), phase ^ 1u, abort_flag, p.status, 0x500u + stage)) {
            ok = false;
            break;
          }
          const uint32_t fb = mapa_shared(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), bytes_pair);
          const uint32_t sA = smem_u32(smem + stage * S::kStageBytes);
          const int kc = kb * 64;
          tma_load_2d_pair(sA, &maps.a, fb, kc, a_row);
          if (kDual) tma_load_2d_pair(sA + S::kABytes, &maps.a2, fb, kc, a2_row);
          const uint32_t sB = sA + S::kABytes * MT;
          int j16 = 0;
#pragma unroll
          for (int i = 3; i >= 0; --i) {
            if ((nb16 >> i) & 1) {
              tma_load_2d_pair(sB + 2048u * j16, &maps.b[i], fb, kc, b_row + 16 * j16);
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
      if (!ok && leader) {
        // the leader's full barriers count both CTAs' copies: let them land
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) mbar_wait_drain(full_bar(s), (issued_phase >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA issuer (leader)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int i = 0; ok; ++i) {
        const int t = receive_tile(i, 0x980u);
        if (t == -2) {
          ok = false;
          break;
        }
        release_tile(i);
        if (t < 0) break;
        int g, m0, row0, n;
        gemm_tile(p, t, S::kBN, g, m0, row0, n);
        const uint32_t N = static_cast<uint32_t>((n + 15) & ~15);
        const uint32_t idesc = idesc_f32acc(1u, 256u, N);
        if (!mbar_wait<true>(acce_bar(acc), acc_phase ^ 1u, abort_flag, p.status, 0x600u + acc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc) * S::kAccCols;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait<true>(full_bar(stage), phase, abort_flag, p.status, 0x700u + stage)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(smem + stage * S::kStageBytes);
          const uint32_t sB = sA + S::kABytes * MT;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            const uint64_t db = sdesc_k_sw128(sB + 32u * kk);
            umma_pair_bf16(d, sdesc_k_sw128(sA + 32u * kk), db, idesc, accum);
            if (kDual) umma_pair_bf16(d + 256u, sdesc_k_sw128(sA + S::kABytes + 32u * kk), db, idesc, accum);
          }
          issued_any = true;
          tc_commit_pair(empty_bar(stage), 0x3);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(accf_bar(acc), 0x3);
        if (S::kAccStages == 2) {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        } else {
          acc_phase ^= 1u;
        }
      }
      if (!ok && issued_any) {
        tc_commit_pair(accf_bar(acc), 0x3);
        mbar_wait_drain(accf_bar(acc), acc_phase);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    // bf16 outputs go through a double-buffered shared tile [32 tokens][128 features] and
    // leave as TMA stores of 16-row boxes (one thread issues them); a 16-row box never
    // reaches past an expert's 16-padded rows, and TMA clips at the tensor's edge.
    const int q = warp & 3;
    const int fl = q * 32 + lane;  // feature of this thread within the CTA's 128
    const int grp = (warp - 2) >> 2;  // epilogue group: chunks c with c % 2 == grp
    const bool elected = ((warp & ~4) == 2 && lane == 0);  // warp 2 or 6
    uint8_t* grp_stage = out_stage + grp * 2 * S::kOutBufBytes;
    int sbuf = 0;
    auto emit = [&](const float (&val)[32], int c, int col0, int row0, int n, bool f_ok, int f) {
      TOut* out = reinterpret_cast<TOut*>(p.out);
      if constexpr (kTmaStore) {
        if (elected) bulk_wait_group_read<1>();  // the buffer's previous store has read it
        epilogue_group_bar_sync(grp);
        __nv_bfloat16* buf = reinterpret_cast<__nv_bfloat16*>(grp_stage + sbuf * S::kOutBufBytes);
#pragma unroll
        for (int i = 0; i < 32; ++i) buf[i * 128 + fl] = __float2bfloat16_rn(val[i]);
        fence_proxy_async_smem();
        epilogue_group_bar_sync(grp);
        if (elected) {
          const uint32_t src = smem_u32(buf);
          if (c * 32 < n) tma_store_2d(&maps.out, src, col0, row0 + c * 32);
          if (c * 32 + 16 < n) tma_store_2d(&maps.out, src + S::kOutBufBytes / 2, col0, row0 + c * 32 + 16);
          bulk_commit_group();
        }
        sbuf ^= 1;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int tok = c * 32 + i;
          if (tok < n && f_ok) out[(static_cast<int64_t>(row0) + tok) * p.ld_out + f] = from_f32<TOut>(val[i]);
        }
      }
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int i = 0;; ++i) {
      int t = receive_tile(i, 0x9C0u);
      if (!__all_sync(0xffffffffu, t != -2)) break;
      t = __shfl_sync(0xffffffffu, t, 0);
      __syncwarp();
      if (lane == 0) release_tile(i);
      if (t < 0) break;
      int g, m0, row0, n;
      gemm_tile(p, t, S::kBN, g, m0, row0, n);
      const bool ready = mbar_wait<true>(accf_bar(acc), acc_phase, abort_flag, p.status, 0x800u + acc);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc) * S::kAccCols;
      const int nchunks = (n + 31) >> 5;
      const int col_cta = m0 + static_cast<int>(rank) * 128;  // first feature of this CTA
      // This group's chunks are c = grp, grp + 2, ... < nchunks (m of them). TMEM loads are
      // issued one step ahead of the arithmetic that uses them, into two register buffers,
      // with the loops unrolled so that no buffer is carried around a loop. (10 warps per
      // CTA leave 168 registers a thread: three warps share one quarter of the register
      // file on two of the four schedulers.)
      const int m = nchunks > grp ? (nchunks - grp + 1) >> 1 : 0;
      if constexpr (EPI == EPI_SWIGLU) {
        // per chunk two steps of 16 tokens; buffers hold gate and up of one step
        const int f = col_cta + fl;
        const bool f_ok = f < p.m_valid;
        constexpr int kMaxM = S::kBN / 64;
        auto load = [&](int c, int half, uint32_t (&gu)[32]) {
          const uint32_t a = taddr + static_cast<uint32_t>(32 * c + 16 * half);
          tmem_ld16(a, *reinterpret_cast<uint32_t(*)[16]>(&gu[0]));
          tmem_ld16(a + 256u, *reinterpret_cast<uint32_t(*)[16]>(&gu[16]));
        };
        auto swiglu16 = [&](const uint32_t (&gu)[32], float* hv) {
#pragma unroll
          for (int i = 0; i < 16; ++i) hv[i] = silu_tanh(__uint_as_float(gu[i])) * __uint_as_float(gu[16 + i]);
        };
        uint32_t ba[32], bb[32];
        if (m > 0) load(grp, 0, ba);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < kMaxM; ++j) {
          if (j >= m) break;
          const int c = grp + 2 * j;
          float hv[32];
          load(c, 1, bb);
          swiglu16(ba, hv);
          tmem_ld_wait();
          if (j + 1 < m) load(c + 2, 0, ba);
          swiglu16(bb, hv + 16);
          emit(hv, c, col_cta, row0, n, f_ok, f);
          tmem_ld_wait();
        }
      } else {
        float gain1[MT];
        bool fok[MT];
#pragma unroll
        for (int h = 0; h < MT; ++h) {
          const int f = col_cta + h * 256 + fl;
          fok[h] = f < p.m_valid;
          gain1[h] = 1.0f;
          if (EPI == EPI_STORE_SS && p.ss_gain != nullptr && fok[h])
            gain1[h] = 1.0f + to_f32(reinterpret_cast<const TIn*>(p.ss_gain)[g * p.ss_gain_group_stride + f]);
        }
        constexpr int kItems = MT * (S::kBN / 64);
        const int valid = MT * m;  // item j: chunk grp + 2 * (j / MT), accumulator half j % MT
        auto addr = [&](int j) {
          return taddr + static_cast<uint32_t>((j % MT) * 256 + 32 * (grp + 2 * (j / MT)));
        };
        auto process = [&](const uint32_t (&v)[32], int j) {
          const int h = j % MT;
          const int c = grp + 2 * (j / MT);
          float yv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) yv[i] = __uint_as_float(v[i]);
          emit(yv, c, col_cta + h * 256, row0, n, fok[h], col_cta + h * 256 + fl);
          if constexpr (EPI == EPI_STORE_SS) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float y = yv[i] * gain1[h];
              yv[i] = fok[h] ? y * y : 0.0f;
            }
            const float tot = transpose_reduce32(yv, lane);
            const int tok = c * 32 + lane;
            if (tok < n) p.ss[(static_cast<int64_t>(row0) + tok) * p.ss_ld + ((col_cta + h * 256) >> 5) + q] = tot;
          }
        };
        uint32_t va[32], vb[32];
        if (valid > 0) tmem_ld32(addr(0), va);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < kItems; j += 2) {
          if (j >= valid) break;
          if (j + 1 < valid) tmem_ld32(addr(j + 1), vb);
          process(va, j);
          tmem_ld_wait();
          if (j + 1 >= valid) break;
          if (j + 2 < valid) tmem_ld32(addr(j + 2), va);
          process(vb, j + 1);
          tmem_ld_wait();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(acce_bar(acc), 0));
      if (S::kAccStages == 2) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        acc_phase ^= 1u;
      }
    }
    if (kTmaStore && elected) bulk_wait_group_all();  // stores done before the CTA leaves
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its partner may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::kTmemCols);
  }
}

}  // namespace muse
