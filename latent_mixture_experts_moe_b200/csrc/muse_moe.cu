// muse_moe.cu -- C ABI of the latent-MoE block forward pass (see include/muse_moe.h).
//
// One forward call validates its arguments, carves the caller's workspace and enqueues
// eleven kernels on the caller's stream:
//   router logits (tcgen05 GEMM; FP32 FMA for float32 inputs) -> top-k + weights ->
//   expert histogram -> padded offsets + tile lists -> stable row assignment ->
//   pooler (tcgen05 GEMM) -> gather into expert order -> gate/up grouped GEMM with
//   SiLU(gate)*up epilogue -> down grouped GEMM with sum-of-squares epilogue ->
//   per-expert RMSNorm + weighted combine -> unpooler (tcgen05 GEMM).
// No host synchronisation, no device allocation, no host read of routing results.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "muse_moe.h"
#include "gemm_umma.cuh"
#include "gemm_umma_2sm.cuh"
#include "gemm_umma_fp4.cuh"
#include "gemm_umma_w4a4.cuh"
#include "gemv_fp4.cuh"
#include "nvfp4_act.cuh"
#include "route_kernels.cuh"

using namespace muse;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------- tile sizing
// tokens per grouped-GEMM tile: small tiles when experts see few tokens (decode)
bool w4a4(const muse_moe_config& c) { return c.act_format == MUSE_ACT_NVFP4; }
#ifndef MUSE_NVFP4_TILE_TOKENS
#define MUSE_NVFP4_TILE_TOKENS 192  // W4A16 prefill tiles: 128 or 192 tokens
#endif
// NVFP4 weights with 16-bit activations and a few rows per expert (decode): both expert GEMMs
// run on the register-fed MMA kernel (gemv_fp4.cuh) -- 128 features and at most 16 token
// rows per tile; K a multiple of its 256-element stage
bool fp4_gemv(const muse_moe_config& c) {
  return c.expert_weights == MUSE_EXPERTS_NVFP4 && !w4a4(c) && c.T * c.top_k <= 4 * c.E && c.L % 256 == 0 &&
         c.I % 256 == 0;
}
int grouped_bn(const muse_moe_config& c) {
  if (fp4_gemv(c)) return 16;
  if ((c.T * c.top_k) <= 32 * c.E) return 32;
  if (w4a4(c)) return 128;  // W4A4: accumulators leave TMEM room for scales
  // NVFP4 weights: accumulators leave TMEM room for converted weight slots
  return c.expert_weights == MUSE_EXPERTS_NVFP4 ? MUSE_NVFP4_TILE_TOKENS : 256;
}
int dense_bn(const muse_moe_config& c) { return c.T <= 32 ? 32 : 256; }

struct Layout {
  muse_moe_workspace_layout pub;
  size_t tiles_gu, tiles_dn, ntiles;  // int4 lists; int[8]: tile counts [0..1], tile counters [4..7]
  size_t zt_codes, zt_scales;         // W4A4: the latent quantised in token order [T, L/2], [T, L/16]
  size_t splitk, splitk_bytes;        // FP32 partial products of split-K dense GEMMs (0 bytes: none)
  int64_t max_tiles_gu, max_tiles_dn;
};

size_t act_size(const muse_moe_config& c) { return c.dtype == MUSE_BF16 ? 2 : 4; }

// Which buffers a workspace holds: those of the whole forward, or of one side of the
// expert-parallel split -- the token's own rank (routing, send plan, pooler, combine,
// unpooler) or an expert shard (grouped GEMMs over the rows it received; c.T = rows).
// Buffers a role does not use have offset 0 and no bytes.
enum class Role { kFull, kHome, kExperts };

Layout make_layout(const muse_moe_config& c, Role role = Role::kFull) {
  Layout l{};
  const bool home = role != Role::kExperts, grouped = role != Role::kHome;
  const int64_t T = c.T, E = c.E, k = c.top_k;
  const int64_t assign = T * k;
  // rows of the expert-ordered buffers: each expert's rows padded to 16 (home: the send
  // plan, unpadded)
  const int64_t rows =
      grouped ? static_cast<int64_t>(align_up(static_cast<size_t>(assign + 15 * std::min<int64_t>(E, assign)), 16))
              : assign;
  const int bn = grouped_bn(c);
  const int64_t chunks = cdiv(assign, bn) + std::min<int64_t>(E, assign);
  l.max_tiles_gu = grouped ? chunks * (c.I / 128) : 0;
  l.max_tiles_dn = grouped ? chunks * (c.L / 128) : 0;
  const size_t as = act_size(c);
  size_t o = 0;
  auto take = [&](bool used, size_t bytes) -> size_t {
    if (!used) return 0;
    const size_t at = o;
    o = align_up(o + bytes, kAlign);
    return at;
  };
  l.pub.status = take(true, 16);
  l.pub.expert_count = take(true, sizeof(int32_t) * E);
  l.pub.expert_offset = take(true, sizeof(int32_t) * (E + 1));
  l.ntiles = take(true, sizeof(int32_t) * 8);
  l.pub.logits = take(home, sizeof(float) * T * E);
  l.pub.topk_idx = take(home, sizeof(int32_t) * assign);
  l.pub.topk_w = take(home, sizeof(float) * assign);
  l.pub.inv = take(true, sizeof(int32_t) * assign);
  l.pub.row_token = take(true, sizeof(int32_t) * rows);
  l.tiles_gu = take(grouped, sizeof(int4) * l.max_tiles_gu);
  l.tiles_dn = take(grouped, sizeof(int4) * l.max_tiles_dn);
  l.pub.z = take(home, as * T * c.L);
  l.pub.zp = take(grouped, as * rows * c.L);
  l.pub.h = take(grouped, as * rows * c.I);
  l.pub.y = take(grouped, as * rows * c.L);
  l.pub.ss = take(grouped, sizeof(float) * rows * (c.L / 32));
  l.pub.c = take(home, as * T * c.L);
  l.pub.xn = take(home && c.ffn_pre_gain != nullptr, as * T * c.D);
  l.pub.ss_out = take(home && c.ffn_post_gain != nullptr, sizeof(float) * T * (c.D / 32));
  const bool q = grouped && w4a4(c);
  l.zt_codes = take(q, T * (c.L / 2));
  l.zt_scales = take(q, T * (c.L / 16));
  l.pub.zq_codes = take(q, rows * (c.L / 2));
  l.pub.zq_scales = take(q, rows * (c.L / 16));
  l.pub.hq_codes = take(q, rows * (c.I / 2));
  l.pub.hq_scales = take(q, rows * (c.I / 16));
  // split-K partials of the dense GEMMs (router, pooler, unpooler) when one of them has a K
  // of 64 k-blocks or more: up to 32 ranges of T x M floats, at most 8 MiB -- decode-sized
  // outputs; larger ones cost more in partial traffic than the extra CTAs win
  const int64_t kb_max = std::max(c.D, c.L) * static_cast<int64_t>(as) / 128;
  l.splitk_bytes = (home && kb_max >= 64)
                       ? std::min<size_t>(size_t(8) << 20, sizeof(float) * 32 * T * std::max({c.D, c.L, c.E}))
                       : 0;
  l.splitk = take(l.splitk_bytes > 0, l.splitk_bytes);
  l.pub.total = o;
  l.pub.rows = rows;
  return l;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

muse_status validate_sizes(const muse_moe_config* c) {
  if (c == nullptr) return MUSE_ERR_INVALID_ARG;
  if (c->T < 1 || c->D < 1 || c->L < 1 || c->I < 1 || c->E < 1) return MUSE_ERR_INVALID_ARG;
  if (c->top_k < 1 || c->top_k > c->E) return MUSE_ERR_INVALID_ARG;
  if (c->dtype != MUSE_F32 && c->dtype != MUSE_BF16) return MUSE_ERR_INVALID_ARG;
  if (!(c->eps >= 0.0f)) return MUSE_ERR_INVALID_ARG;
  if (c->router_mode != MUSE_ROUTER_SOFTMAX && c->router_mode != MUSE_ROUTER_SIGMOID) return MUSE_ERR_INVALID_ARG;
  if (c->norm_mode != MUSE_NORM_CENTRED && c->norm_mode != MUSE_NORM_INPUT_SCALED) return MUSE_ERR_INVALID_ARG;
  if (c->top_k > 32 || c->E > 1024) return MUSE_ERR_UNSUPPORTED;
  if (c->D % 128 || c->L % 128 || c->I % 128) return MUSE_ERR_UNSUPPORTED;
  if (c->L > 8192 || c->D > 65536 || c->I > 65536) return MUSE_ERR_UNSUPPORTED;
  // 32-bit row / coordinate arithmetic inside the kernels
  if (c->T * c->top_k + 16 * c->E > (int64_t(1) << 30) || c->E * std::max(c->I, c->L) > (int64_t(1) << 31) - 1)
    return MUSE_ERR_UNSUPPORTED;
  if (c->T > (int64_t(1) << 24)) return MUSE_ERR_UNSUPPORTED;
  if (c->expert_weights != MUSE_EXPERTS_DENSE && c->expert_weights != MUSE_EXPERTS_NVFP4) return MUSE_ERR_INVALID_ARG;
  if (c->expert_weights == MUSE_EXPERTS_NVFP4 && c->dtype != MUSE_BF16) return MUSE_ERR_UNSUPPORTED;
  if (c->act_format != MUSE_ACT_BF16 && c->act_format != MUSE_ACT_NVFP4) return MUSE_ERR_INVALID_ARG;
  if (c->act_format == MUSE_ACT_NVFP4 &&
      (c->expert_weights != MUSE_EXPERTS_NVFP4 || c->L % 256 != 0 || c->I % 256 != 0))
    return MUSE_ERR_UNSUPPORTED;
  return MUSE_OK;
}

bool valid_nvfp4(const void* w) {
  const muse_nvfp4_weight* q = static_cast<const muse_nvfp4_weight*>(w);
  return q != nullptr && q->codes != nullptr && q->block_scales != nullptr && q->matrix_scale != nullptr &&
         aligned16(q->codes) && aligned16(q->block_scales) && (reinterpret_cast<uintptr_t>(q->matrix_scale) & 3u) == 0;
}

// ---------------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// K-major 2-D map over rows x K elements, box = box_rows x 128 bytes, 128-byte swizzle;
// rows beyond the tensor read as zeros.
bool make_map(CUtensorMap* m, const void* base, bool bf16, int64_t K, int64_t rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const uint32_t es = bf16 ? 2 : 4;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * es};
  cuuint32_t box[2] = {128u / es, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed 4-bit codes: rows x (K/2) bytes, boxes of 128 rows x 32 bytes (64 weights),
// no swizzle (the converter warps read them).
bool make_code_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {32u, 128u};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Byte matrix rows x cols (uint8: packed codes or E4M3 scales), boxes of box_rows rows x
// box_cols bytes, 128-byte swizzle for code tiles the UMMA reads, none for scale boxes.
bool make_u8_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows,
                 bool swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map for TMA stores: rows x cols bf16 row-major, boxes of 16 rows x 128 columns,
// no swizzle (the epilogue stages tiles row-major in shared memory).
bool make_out_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {128u, 16u};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// ---------------------------------------------------------------------- GEMM launch
template <typename TIn, typename TOut, int BN, int EPI, int MT>
cudaError_t launch_gemm(const TmaMaps& maps, const GemmArgs& args, int grid, cudaStream_t st) {
  auto kern = k_umma_gemm<TIn, TOut, BN, EPI, MT>;
  const size_t smem = GemmShape<BN, EPI, MT>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, 192, smem, st>>>(maps, args);
  return cudaGetLastError();
}

template <typename TIn, typename TOut, int EPI>
cudaError_t launch_gemm_bn(int bn, int mt, const TmaMaps& maps, const GemmArgs& args, int grid, cudaStream_t st) {
  if constexpr (EPI == EPI_SWIGLU) {
    if (bn == 32) return launch_gemm<TIn, TOut, 32, EPI, 2>(maps, args, grid, st);
    return launch_gemm<TIn, TOut, 256, EPI, 2>(maps, args, grid, st);
  } else {
    if (bn == 32) return mt == 2 ? launch_gemm<TIn, TOut, 32, EPI, 2>(maps, args, grid, st)
                                 : launch_gemm<TIn, TOut, 32, EPI, 1>(maps, args, grid, st);
    if constexpr (EPI == EPI_STORE) {
      if (bn == 128) return launch_gemm<TIn, TOut, 128, EPI, 1>(maps, args, grid, st);
    }
    return mt == 2 ? launch_gemm<TIn, TOut, 256, EPI, 2>(maps, args, grid, st)
                   : launch_gemm<TIn, TOut, 256, EPI, 1>(maps, args, grid, st);
  }
}

template <int BN, int EPI, int MT>
cudaError_t launch_gemm_fp4_t(const TmaMaps& maps, const GemmArgs& args, const Fp4Args& q4, int grid, cudaStream_t st) {
  auto kern = k_umma_gemm_fp4<BN, EPI, MT>;
  const size_t smem = Fp4Shape<BN, EPI, MT>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kFp4Threads, smem, st>>>(maps, args, q4);
  return cudaGetLastError();
}

template <int BN, int EPI>
cudaError_t launch_gemm_fp4_bn(int mt, const TmaMaps& maps, const GemmArgs& args, const Fp4Args& q4, int grid,
                               cudaStream_t st) {
  if constexpr (EPI == EPI_SWIGLU) {
    return launch_gemm_fp4_t<BN, EPI, 2>(maps, args, q4, grid, st);
  } else {
    return mt == 2 ? launch_gemm_fp4_t<BN, EPI, 2>(maps, args, q4, grid, st)
                   : launch_gemm_fp4_t<BN, EPI, 1>(maps, args, q4, grid, st);
  }
}

template <int EPI>
cudaError_t launch_gemm_fp4(int bn, int mt, const TmaMaps& maps, const GemmArgs& args, const Fp4Args& q4, int grid,
                            cudaStream_t st) {
  if (bn == 32) return launch_gemm_fp4_bn<32, EPI>(mt, maps, args, q4, grid, st);
  if (bn == 128) return launch_gemm_fp4_bn<128, EPI>(mt, maps, args, q4, grid, st);
  return launch_gemm_fp4_bn<192, EPI>(mt, maps, args, q4, grid, st);
}

// NVFP4 weights, 16-bit activations, decode-sized tiles: the register-fed MMA kernel. Maps:
// the codes and block scales of one or two weight matrices [rows_w, K] and the activation rows.
bool make_gemv_maps(GemvMaps* m, const muse_nvfp4_weight* w, const muse_nvfp4_weight* w2, int64_t rows_w,
                    const void* x, int64_t R, int64_t K) {
  std::memset(m, 0, sizeof(*m));
  return make_code_map(&m->codes[0], w->codes, rows_w, K) && make_code_map(&m->codes[1], w2->codes, rows_w, K) &&
         make_u8_map(&m->scales[0], w->block_scales, rows_w, K / 16, 16, 128, false) &&
         make_u8_map(&m->scales[1], w2->block_scales, rows_w, K / 16, 16, 128, false) &&
         make_map(&m->x, x, true, K, R, 16);
}

template <int EPI>
cudaError_t launch_gemv_fp4(const GemvMaps& maps, const GemvArgs& args, int grid, cudaStream_t st) {
  auto kern = k_fp4_gemv<EPI>;
  const size_t smem = GemvShape<EPI == EPI_SWIGLU ? 2 : 1>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kGemvThreads, smem, st>>>(maps, args);
  return cudaGetLastError();
}

template <int BN, int EPI>
cudaError_t launch_gemm_w4a4_t(const W4A4Maps& maps, const GemmArgs& args, const W4A4Args& q, int grid,
                               cudaStream_t st) {
  auto kern = k_umma_gemm_w4a4<BN, EPI, 2>;
  const size_t smem = W4A4Shape<BN, EPI, 2>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kW4A4Threads, smem, st>>>(maps, args, q);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_gemm_w4a4(int bn, const W4A4Maps& maps, const GemmArgs& args, const W4A4Args& q, int grid,
                             cudaStream_t st) {
  return bn == 32 ? launch_gemm_w4a4_t<32, EPI>(maps, args, q, grid, st)
                  : launch_gemm_w4a4_t<128, EPI>(maps, args, q, grid, st);
}

// W4A4 maps: weight codes and scales of one or two matrices ([rows_w, K/2], [rows_w, K/16]),
// token codes and scales ([R, K/2], [R, K/16]) in boxes of bn rows.
bool make_w4a4_maps(W4A4Maps* m, const muse_nvfp4_weight* w, const muse_nvfp4_weight* w2, int64_t rows_w,
                    const void* codes, const void* scales, int64_t R, int64_t K, int bn) {
  std::memset(m, 0, sizeof(*m));
  return make_u8_map(&m->a, w->codes, rows_w, K / 2, 128, 128, true) &&
         make_u8_map(&m->a2, w2->codes, rows_w, K / 2, 128, 128, true) &&
         make_u8_map(&m->b, codes, R, K / 2, 128, bn, true) &&
         make_u8_map(&m->sfa, w->block_scales, rows_w, K / 16, 16, 128, false) &&
         make_u8_map(&m->sfa2, w2->block_scales, rows_w, K / 16, 16, 128, false) &&
         make_u8_map(&m->sfb, scales, R, K / 16, 16, bn, false);
}

template <typename TOut, int EPI, int MT>
cudaError_t launch_gemm_2sm(const TmaMaps& maps, const GemmArgs& args, int pairs, cudaStream_t st) {
  auto kern = k_umma_gemm_2sm<TOut, EPI, MT>;
  const size_t smem = Gemm2Shape<EPI, MT>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<2 * pairs, kPairThreads, smem, st>>>(maps, args);
  return cudaGetLastError();
}

// How a GEMM is tiled: on one SM (mt weight tiles of 128 rows per CTA) or on a CTA pair
// (cta_group::2; 256 * mt features per pair tile, tiles of up to 256 tokens).
struct GemmPlan {
  bool pair;
  int mt;
  int step;  // output features per tile
};

// weight operand map(s) with 128-row boxes and the token operand with 16..256-row boxes
bool make_maps(TmaMaps* m, const void* a, const void* a2, int64_t a_rows, const void* b, int64_t b_rows, int64_t K,
               bool bf16) {
  std::memset(m, 0, sizeof(*m));
  if (!make_map(&m->a, a, bf16, K, a_rows, 128)) return false;
  if (!make_map(&m->a2, a2 ? a2 : a, bf16, K, a_rows, 128)) return false;
  for (int i = 0; i < 5; ++i)
    if (!make_map(&m->b[i], b, bf16, K, b_rows, 16 << i)) return false;
  return true;
}

GemmArgs base_args(uint32_t* status) {
  GemmArgs g{};
  g.status = status;
  return g;
}

// Sum-of-squares partials of a dense GEMM's output (EPI_STORE_SS): ss[t, f / 32] over
// 32-column groups of (acc * (1 + gain[f])).
struct DenseSS {
  float* ss = nullptr;
  int ld = 0;
  const void* gain = nullptr;
};

// Scratch for split-K partial products (null: K is never split).
struct SplitK {
  float* buf = nullptr;
  size_t bytes = 0;
};

// dense C[T, M] = X[T, K] W[M, K]^T
template <typename TIn, typename TOut, int EPI = EPI_STORE>
muse_status dense_gemm(const void* W, int64_t M, const void* X, int64_t T, int64_t K, void* out, int bn,
                       uint32_t* status, int* tile_counter, cudaStream_t st, DenseSS sq = DenseSS{},
                       SplitK sk = SplitK{}) {
  TmaMaps maps;
  const bool bf = sizeof(TIn) == 2;
  if (!make_maps(&maps, W, nullptr, M, X, T, K, bf)) return MUSE_ERR_CUDA;
  GemmArgs g = base_args(status);
  const int nsm = sm_count();
  g.rows_per_group = 0;
  g.m_valid = static_cast<int>(M);
  g.T = static_cast<int>(T);
  g.k_blocks = static_cast<int>(cdiv(K * sizeof(TIn), 128));
  g.out = out;
  g.ld_out = M;
  g.ss = sq.ss;
  g.ss_ld = sq.ld;
  g.ss_gain = sq.gain;
  g.ss_gain_group_stride = 0;
  // a CTA pair per 256 features x 256 tokens when that fills at least one wave of pairs;
  // 512 features (two weight tiles per CTA, so each staged token tile feeds twice the
  // MMAs) when the width allows
  if (bf && bn == 256 && cdiv(M, 256) * cdiv(T, 256) >= nsm / 2) {
    if (sizeof(TOut) == 2 && !make_out_map(&maps.out, out, T, M)) return MUSE_ERR_CUDA;
    const bool wide = sizeof(TOut) == 2 && M % 512 == 0;
    g.m_step = wide ? 512 : 256;
    g.m_tiles = static_cast<int>(cdiv(M, g.m_step));
    g.num_tiles = static_cast<int>(g.m_tiles * cdiv(T, 256));
    // when the weights are at least as large as the token operand (the unpooler: 67 MB each
    // at T = 8192), tiles run by groups of weight tiles holding ~32 MB, so that a wave of
    // pairs re-reads its weights from L2 (unpooler DRAM bytes 2.42x -> 1.61x of the
    // algorithmic ones); otherwise (the pooler reads 134 MB of x against 67 MB of weights)
    // token chunk by token chunk, each chunk's weight tiles side by side
    if (M >= T)
      g.m_group = static_cast<int>(
          std::max<int64_t>(1, (int64_t(32) << 20) / (g.m_step * K * static_cast<int64_t>(sizeof(TIn)))));
    g.tile_counter = tile_counter;
    const int pairs = std::min(g.num_tiles, nsm / 2);
    if constexpr (sizeof(TOut) == 2) {
      if (wide) return launch_gemm_2sm<TOut, EPI, 2>(maps, g, pairs, st) == cudaSuccess ? MUSE_OK : MUSE_ERR_CUDA;
    }
    return launch_gemm_2sm<TOut, EPI, 1>(maps, g, pairs, st) == cudaSuccess ? MUSE_OK : MUSE_ERR_CUDA;
  }
  // two 128-row weight tiles per CTA when that still leaves at least a full wave of tiles
  const int mt = (cdiv(M, 256) * cdiv(T, bn) >= nsm) ? 2 : 1;
  g.m_step = 128 * mt;
  g.m_tiles = static_cast<int>(cdiv(M, g.m_step));
  // 128-token tiles when 256-token ones would fill at most half the SMs (the router: E = 256
  // features x T / 256 token tiles)
  if (EPI == EPI_STORE && bn == 256 && mt == 1 && 2 * g.m_tiles * cdiv(T, 256) <= nsm) bn = 128;
  g.num_tiles = static_cast<int>(g.m_tiles * cdiv(T, bn));
  // K split into S equal ranges while the tiles of all ranges still fit one wave: each
  // range writes its FP32 partial product, k_splitk_reduce sums them in range order
  int S = 1;
  if (EPI == EPI_STORE && sk.buf != nullptr && M % 4 == 0) {
    while (2 * S * g.num_tiles <= nsm && g.k_blocks % (2 * S) == 0 && g.k_blocks / (2 * S) >= 4 &&
           sizeof(float) * static_cast<size_t>(2 * S) * T * M <= sk.bytes)
      S *= 2;
  }
  if (S > 1) {
    g.k_splits = S;
    g.split_stride = T * M;
    g.out = sk.buf;
    g.ld_out = M;
    g.num_tiles *= S;
    if (launch_gemm_bn<TIn, float, EPI_STORE>(bn, mt, maps, g, std::min(g.num_tiles, nsm), st) != cudaSuccess)
      return MUSE_ERR_CUDA;
    const int64_t n4 = T * M / 4;
    const int rgrid = static_cast<int>(std::min<int64_t>(cdiv(n4, 256), 4 * nsm));
    k_splitk_reduce<TOut><<<rgrid, 256, 0, st>>>(reinterpret_cast<const float4*>(sk.buf), n4, S,
                                                 static_cast<TOut*>(out));
    return cudaGetLastError() == cudaSuccess ? MUSE_OK : MUSE_ERR_CUDA;
  }
  const int grid = std::min(g.num_tiles, nsm);
  return launch_gemm_bn<TIn, TOut, EPI>(bn, mt, maps, g, grid, st) == cudaSuccess ? MUSE_OK : MUSE_ERR_CUDA;
}

// Grouped-GEMM plans. gate/up: a CTA pair per 256 features when tiles hold up to 256
// tokens (bf16), else one CTA per 128 features (gate and up accumulators). down: a pair
// per 512 features (two accumulators) or 256, else one CTA per 256 or 128 features.
GemmPlan plan_gate_up(const muse_moe_config& c, int bn_g) {
  if (c.expert_weights == MUSE_EXPERTS_NVFP4) return {false, 2, 128};
  if (c.dtype == MUSE_BF16 && bn_g == 256 && c.I % 256 == 0) return {true, 2, 256};
  return {false, 2, 128};
}
GemmPlan plan_down(const muse_moe_config& c, int bn_g) {
  if (w4a4(c)) return {false, 2, 256};
  if (fp4_gemv(c)) return {false, 1, 128};
  if (c.expert_weights == MUSE_EXPERTS_NVFP4) return c.L % 256 == 0 ? GemmPlan{false, 2, 256} : GemmPlan{false, 1, 128};
  if (c.dtype == MUSE_BF16 && bn_g == 256 && c.L % 512 == 0) return {true, 2, 512};
  if (c.dtype == MUSE_BF16 && bn_g == 256 && c.L % 256 == 0) return {true, 1, 256};
  if (bn_g == 256 && c.L % 256 == 0) return {false, 2, 256};
  return {false, 1, 128};
}

// the last CUDA error a call of this thread returned MUSE_ERR_CUDA for
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

#define MUSE_CK(x)                          \
  do {                                      \
    const cudaError_t muse_e_ = (x);        \
    if (muse_e_ != cudaSuccess) {           \
      g_last_cuda_error = muse_e_;          \
      return MUSE_ERR_CUDA;                 \
    }                                       \
  } while (0)

#define MUSE_TRY(x)                     \
  do {                                  \
    const muse_status s_ = (x);         \
    if (s_ != MUSE_OK) return s_;       \
  } while (0)

// One pass of kernels over a workspace: its buffers, the stream and the optional stage
// events (recorded after each launch of the full forward; null on the expert-parallel
// entry points).
template <typename T>
struct Pass {
  const muse_moe_config& c;
  const Layout& lay;
  cudaStream_t st;
  void* const* events;
  int stage = 0;
  int nsm;
  uint8_t* ws;
  uint32_t* status;
  int *counts, *offsets, *ntiles, *topk_idx, *inv, *row_token;
  float* topk_w;
  Pass(const muse_moe_config& c_, const Layout& l, cudaStream_t s, void* const* ev)
      : c(c_), lay(l), st(s), events(ev), nsm(sm_count()), ws(static_cast<uint8_t*>(c_.workspace)) {
    status = ptr<uint32_t>(l.pub.status);
    counts = ptr<int>(l.pub.expert_count);
    offsets = ptr<int>(l.pub.expert_offset);
    ntiles = ptr<int>(l.ntiles);
    topk_idx = ptr<int>(l.pub.topk_idx);
    topk_w = ptr<float>(l.pub.topk_w);
    inv = ptr<int>(l.pub.inv);
    row_token = ptr<int>(l.pub.row_token);
  }
  uint8_t* at(size_t off) const { return ws + off; }
  SplitK splitk() const {
    SplitK k;
    if (lay.splitk_bytes > 0) {
      k.buf = reinterpret_cast<float*>(ws + lay.splitk);
      k.bytes = lay.splitk_bytes;
    }
    return k;
  }
  template <typename U>
  U* ptr(size_t off) const { return reinterpret_cast<U*>(ws + off); }
  cudaError_t mark() {
    if (events == nullptr) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[stage++]), st);
  }
};

// status word and expert histogram zeroed; the first stage event
template <typename T>
muse_status begin(Pass<T>& p) {
  MUSE_CK(cudaMemsetAsync(p.status, 0, 16, p.st));
  MUSE_CK(cudaMemsetAsync(p.counts, 0, sizeof(int) * p.c.E, p.st));
  MUSE_CK(p.mark());
  return MUSE_OK;
}

// feed-forward sublayer pre-norm (optional), (a1) router logits, (a2) top-k and weights;
// *xin: the rows the router and the pooler read (x, or its normalisation)
template <typename T>
muse_status route(Pass<T>& p, const void* x, const void* W_router, const void** xin) {
  const muse_moe_config& c = p.c;
  const int64_t Tn = c.T, D = c.D, E = c.E, k = c.top_k;
  *xin = x;
  if (c.ffn_pre_gain != nullptr) {
    T* xn = p.template ptr<T>(p.lay.pub.xn);
    k_rmsnorm_rows<T><<<static_cast<unsigned>(Tn), 256, 0, p.st>>>(reinterpret_cast<const T*>(x), xn,
                                                                   reinterpret_cast<const T*>(c.ffn_pre_gain),
                                                                   static_cast<int>(D), c.ffn_pre_eps);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(p.mark());
    *xin = xn;
  }
  float* logits = p.template ptr<float>(p.lay.pub.logits);
  if (sizeof(T) == 2) {
    MUSE_TRY((dense_gemm<T, float>(W_router, E, *xin, Tn, D, logits, dense_bn(c), p.status, nullptr, p.st, DenseSS{},
                                   p.splitk())));
  } else {
    k_router_logits_f32<<<static_cast<unsigned>(Tn), 256, 0, p.st>>>(reinterpret_cast<const float*>(*xin),
                                                                    reinterpret_cast<const float*>(W_router),
                                                                    static_cast<int>(D), static_cast<int>(E), logits);
    MUSE_CK(cudaGetLastError());
  }
  MUSE_CK(p.mark());
  {
    // key slots per lane: E / 32 rounded up to a power of two (E <= 1024)
    const int npl = E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : E <= 256 ? 8 : E <= 512 ? 16 : 32;
    auto kern = npl == 1 ? k_topk<1> : npl == 2 ? k_topk<2> : npl == 4 ? k_topk<4> : npl == 8 ? k_topk<8>
              : npl == 16 ? k_topk<16> : k_topk<32>;
    kern<<<static_cast<unsigned>(cdiv(Tn * 32, 256)), 256, 0, p.st>>>(
        logits, static_cast<int>(Tn), static_cast<int>(E), static_cast<int>(k), c.router_bias, c.router_mode,
        c.router_logit_scale, c.routed_scaling, p.topk_idx, p.topk_w, c.topk_idx_out, c.topk_w_out);
    MUSE_CK(cudaGetLastError());
  }
  MUSE_CK(p.mark());
  return MUSE_OK;
}

// (a3) expert histogram of n assignments (out-of-range indices are counted nowhere and
// recorded in the status word)
template <typename T>
muse_status hist(Pass<T>& p, const int* idx, int64_t n) {
  const int grid = static_cast<int>(std::min<int64_t>(cdiv(n, 256), 4 * p.nsm));
  k_expert_hist<<<grid, 256, sizeof(int) * p.c.E, p.st>>>(idx, static_cast<int>(n), static_cast<int>(p.c.E), p.counts,
                                                            p.status);
  MUSE_CK(cudaGetLastError());
  MUSE_CK(p.mark());
  return MUSE_OK;
}

// (a3) padded expert offsets, grouped-GEMM tile lists and the stable row of each of the n
// assignments idx (k per token)
template <typename T>
muse_status permute(Pass<T>& p, const int* idx, int64_t n, int k) {
  const muse_moe_config& c = p.c;
  const int bn_g = grouped_bn(c);
  const GemmPlan pgu = plan_gate_up(c, bn_g), pdn = plan_down(c, bn_g);
  const int threads = static_cast<int>(align_up(static_cast<size_t>(c.E), 32));
  k_build_tiles<<<1, threads, 0, p.st>>>(p.counts, static_cast<int>(c.E), bn_g, static_cast<int>(c.I / pgu.step),
                                         pgu.step, static_cast<int>(c.L / pdn.step), pdn.step, p.offsets,
                                         p.template ptr<int4>(p.lay.tiles_gu), p.ntiles,
                                         p.template ptr<int4>(p.lay.tiles_dn), p.ntiles + 1, p.ntiles + 4,
                                         p.row_token);
  MUSE_CK(cudaGetLastError());
  MUSE_CK(p.mark());
  k_assign_rows<<<static_cast<unsigned>(c.E), 1024, 0, p.st>>>(idx, static_cast<int>(n), k, p.counts, p.offsets,
                                                               p.inv, p.row_token);
  MUSE_CK(cudaGetLastError());
  MUSE_CK(p.mark());
  return MUSE_OK;
}

// (a4) pooler, then the pages' pre_expert_norm on z (optional)
template <typename T>
muse_status pool(Pass<T>& p, const void* xin, const void* W_pool) {
  const muse_moe_config& c = p.c;
  T* z = p.template ptr<T>(p.lay.pub.z);
  MUSE_TRY((dense_gemm<T, T>(W_pool, c.L, xin, c.T, c.D, z, dense_bn(c), p.status, p.ntiles + 6, p.st, DenseSS{},
                             p.splitk())));
  MUSE_CK(p.mark());
  if (c.pre_norm_gain != nullptr) {
    k_rmsnorm_rows<T><<<static_cast<unsigned>(c.T), 256, 0, p.st>>>(
        z, z, reinterpret_cast<const T*>(c.pre_norm_gain), static_cast<int>(c.L), c.pre_norm_eps);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(p.mark());
  }
  return MUSE_OK;
}

// (a5) gather of the latent rows zsrc [nsrc, L] into expert order (W4A4: quantised to
// NVFP4 once per source row, then the codes gathered), (a6) gate/up + SwiGLU, (a7) down
// projection + sum-of-squares partials, over the tiles permute() listed
template <typename T>
muse_status experts(Pass<T>& p, const T* zsrc, int64_t nsrc, const void* W_gate, const void* W_up,
                    const void* W_down, const void* gamma) {
  const muse_moe_config& c = p.c;
  const Layout& lay = p.lay;
  cudaStream_t st = p.st;
  const bool bf = sizeof(T) == 2;
  const int64_t L = c.L, I = c.I, E = c.E;
  const int nsm = p.nsm;
  const int bn_g = grouped_bn(c);
  const GemmPlan pdn = plan_down(c, bn_g), pgu = plan_gate_up(c, bn_g);
  T* zp = p.template ptr<T>(lay.pub.zp);
  T* h = p.template ptr<T>(lay.pub.h);
  T* y = p.template ptr<T>(lay.pub.y);
  float* ss = p.template ptr<float>(lay.pub.ss);
  const bool q4a = w4a4(c);
  uint8_t* zq_codes = p.at(lay.pub.zq_codes);
  uint8_t* zq_scales = p.at(lay.pub.zq_scales);
  uint8_t* hq_codes = p.at(lay.pub.hq_codes);
  uint8_t* hq_scales = p.at(lay.pub.hq_scales);
  const int quant_grid = static_cast<int>(std::min<int64_t>(lay.pub.rows, 16 * nsm));
  if (q4a) {
    uint8_t* zt_codes = p.at(lay.zt_codes);
    uint8_t* zt_scales = p.at(lay.zt_scales);
    k_quant_rows_nvfp4<<<static_cast<unsigned>(std::min<int64_t>(nsrc, 16 * nsm)), 256, 0, st>>>(
        nullptr, nullptr, static_cast<int>(nsrc), reinterpret_cast<const __nv_bfloat16*>(zsrc), static_cast<int>(L),
        zt_codes, zt_scales);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(p.mark());
    k_gather_nvfp4_rows<<<quant_grid, 128, 0, st>>>(p.row_token, p.offsets + E,
                                                    reinterpret_cast<const uint4*>(zt_codes),
                                                    reinterpret_cast<const uint4*>(zt_scales),
                                                    reinterpret_cast<uint4*>(zq_codes),
                                                    reinterpret_cast<uint4*>(zq_scales), static_cast<int>(L));
    MUSE_CK(cudaGetLastError());
    MUSE_CK(p.mark());
  } else {
    const int vpr = static_cast<int>(L * sizeof(T) / 16);
    const int rows_grid = static_cast<int>(std::min<int64_t>(lay.pub.rows, 16 * nsm));
    // NVFP4 weights with bf16 activations (W4A16): the expert GEMMs' operands are f16, so the
    // gathered rows are converted on the way (zp and h then hold f16)
    if (c.expert_weights == MUSE_EXPERTS_NVFP4)
      k_gather_rows<true><<<rows_grid, 128, 0, st>>>(p.row_token, p.offsets + E, reinterpret_cast<const uint4*>(zsrc),
                                                     reinterpret_cast<uint4*>(zp), vpr);
    else
      k_gather_rows<false><<<rows_grid, 128, 0, st>>>(p.row_token, p.offsets + E, reinterpret_cast<const uint4*>(zsrc),
                                                      reinterpret_cast<uint4*>(zp), vpr);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(p.mark());
  }
  const int64_t R = lay.pub.rows;
  const bool fp4 = c.expert_weights == MUSE_EXPERTS_NVFP4;
  // (a6) gate/up + SwiGLU
  {
    TmaMaps maps;
    Fp4Args q4{};
    if (q4a) {
      // W4A4: its maps are built at the launch below
    } else if (fp4) {
      const muse_nvfp4_weight* wg = static_cast<const muse_nvfp4_weight*>(W_gate);
      const muse_nvfp4_weight* wu = static_cast<const muse_nvfp4_weight*>(W_up);
      std::memset(&maps, 0, sizeof(maps));
      if (!make_code_map(&maps.a, wg->codes, E * I, L) || !make_code_map(&maps.a2, wu->codes, E * I, L)) return MUSE_ERR_CUDA;
      for (int i = 0; i < 5; ++i)
        if (!make_map(&maps.b[i], zp, bf, L, R, 16 << i)) return MUSE_ERR_CUDA;
      q4 = Fp4Args{static_cast<const uint8_t*>(wg->block_scales), static_cast<const uint8_t*>(wu->block_scales),
                   wg->matrix_scale, wu->matrix_scale, static_cast<int>(L / 16)};
    } else if (!make_maps(&maps, W_gate, W_up, E * I, zp, R, L, bf)) {
      return MUSE_ERR_CUDA;
    }
    GemmArgs g = base_args(p.status);
    g.tiles = p.template ptr<int4>(lay.tiles_gu);
    g.num_tiles_dev = p.ntiles;
    g.tile_counter = p.ntiles + 4;
    g.rows_per_group = static_cast<int>(I);
    g.m_valid = static_cast<int>(I);
    g.k_blocks = static_cast<int>(L * sizeof(T) / 128);
    g.out = h;
    g.ld_out = I;
    if (q4a) {
      W4A4Maps wm;
      const muse_nvfp4_weight* wg = static_cast<const muse_nvfp4_weight*>(W_gate);
      const muse_nvfp4_weight* wu = static_cast<const muse_nvfp4_weight*>(W_up);
      if (!make_w4a4_maps(&wm, wg, wu, E * I, zq_codes, zq_scales, R, L, bn_g)) return MUSE_ERR_CUDA;
      const W4A4Args wq{wg->matrix_scale, wu->matrix_scale};
      g.k_blocks = static_cast<int>(L / 256);
      MUSE_CK(launch_gemm_w4a4<EPI_SWIGLU>(bn_g, wm, g, wq, nsm, st));
    } else if (fp4_gemv(c)) {
      const muse_nvfp4_weight* wg = static_cast<const muse_nvfp4_weight*>(W_gate);
      const muse_nvfp4_weight* wu = static_cast<const muse_nvfp4_weight*>(W_up);
      GemvMaps vm;
      if (!make_gemv_maps(&vm, wg, wu, E * I, zp, R, L)) return MUSE_ERR_CUDA;
      GemvArgs v{};
      v.tiles = g.tiles;
      v.num_tiles = g.num_tiles_dev;
      v.mscale[0] = wg->matrix_scale;
      v.mscale[1] = wu->matrix_scale;
      v.rows_per_group = static_cast<int>(I);
      v.K = static_cast<int>(L);
      v.out = h;
      v.ld_out = I;
      v.status = p.status;
      MUSE_CK(launch_gemv_fp4<EPI_SWIGLU>(vm, v, nsm, st));
    } else if (fp4) {
      MUSE_CK(launch_gemm_fp4<EPI_SWIGLU>(bn_g, 2, maps, g, q4, nsm, st));
    } else if (pgu.pair) {
      if (!make_out_map(&maps.out, h, R, I)) return MUSE_ERR_CUDA;
      MUSE_CK((launch_gemm_2sm<T, EPI_SWIGLU, 2>(maps, g, nsm / 2, st)));
    } else {
      MUSE_CK((launch_gemm_bn<T, T, EPI_SWIGLU>(bn_g, 2, maps, g, nsm, st)));
    }
    MUSE_CK(p.mark());
  }
  // W4A4: quantise h (already in expert order) for the down projection
  if (q4a) {
    k_quant_rows_nvfp4<<<quant_grid, 256, 0, st>>>(p.row_token, p.offsets + E, 0,
                                                   reinterpret_cast<const __nv_bfloat16*>(h), static_cast<int>(I),
                                                   hq_codes, hq_scales);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(p.mark());
  }
  // (a7) down projection + sum-of-squares partials
  {
    TmaMaps maps;
    Fp4Args q4{};
    if (q4a) {
      // W4A4: its maps are built at the launch below
    } else if (fp4) {
      const muse_nvfp4_weight* wd = static_cast<const muse_nvfp4_weight*>(W_down);
      std::memset(&maps, 0, sizeof(maps));
      if (!make_code_map(&maps.a, wd->codes, E * L, I) || !make_code_map(&maps.a2, wd->codes, E * L, I)) return MUSE_ERR_CUDA;
      for (int i = 0; i < 5; ++i)
        if (!make_map(&maps.b[i], h, bf, I, R, 16 << i)) return MUSE_ERR_CUDA;
      q4 = Fp4Args{static_cast<const uint8_t*>(wd->block_scales), static_cast<const uint8_t*>(wd->block_scales),
                   wd->matrix_scale, wd->matrix_scale, static_cast<int>(I / 16)};
    } else if (!make_maps(&maps, W_down, nullptr, E * L, h, R, I, bf)) {
      return MUSE_ERR_CUDA;
    }
    GemmArgs g = base_args(p.status);
    g.tiles = p.template ptr<int4>(lay.tiles_dn);
    g.num_tiles_dev = p.ntiles + 1;
    g.tile_counter = p.ntiles + 5;
    g.rows_per_group = static_cast<int>(L);
    g.m_valid = static_cast<int>(L);
    g.k_blocks = static_cast<int>(I * sizeof(T) / 128);
    g.out = y;
    g.ld_out = L;
    g.ss = ss;
    g.ss_ld = static_cast<int>(L / 32);
    if (c.norm_mode == MUSE_NORM_INPUT_SCALED) {
      g.ss_gain = gamma;
      g.ss_gain_group_stride = c.gamma_shared ? 0 : L;
    }
    if (pdn.pair && !make_out_map(&maps.out, y, R, L)) return MUSE_ERR_CUDA;
    if (q4a) {
      W4A4Maps wm;
      const muse_nvfp4_weight* wd = static_cast<const muse_nvfp4_weight*>(W_down);
      if (!make_w4a4_maps(&wm, wd, wd, E * L, hq_codes, hq_scales, R, I, bn_g)) return MUSE_ERR_CUDA;
      const W4A4Args wq{wd->matrix_scale, wd->matrix_scale};
      g.k_blocks = static_cast<int>(I / 256);
      MUSE_CK(launch_gemm_w4a4<EPI_STORE_SS>(bn_g, wm, g, wq, nsm, st));
    } else if (fp4_gemv(c)) {
      const muse_nvfp4_weight* wd = static_cast<const muse_nvfp4_weight*>(W_down);
      GemvMaps vm;
      if (!make_gemv_maps(&vm, wd, wd, E * L, h, R, I)) return MUSE_ERR_CUDA;
      GemvArgs v{};
      v.tiles = g.tiles;
      v.num_tiles = g.num_tiles_dev;
      v.mscale[0] = v.mscale[1] = wd->matrix_scale;
      v.rows_per_group = static_cast<int>(L);
      v.K = static_cast<int>(I);
      v.out = y;
      v.status = p.status;
      v.ld_out = L;
      v.ss = ss;
      v.ss_ld = static_cast<int>(L / 32);
      if (c.norm_mode == MUSE_NORM_INPUT_SCALED) {
        v.ss_gain = static_cast<const __nv_bfloat16*>(gamma);
        v.ss_gain_stride = c.gamma_shared ? 0 : L;
      }
      MUSE_CK(launch_gemv_fp4<EPI_STORE_SS>(vm, v, nsm, st));
    } else if (fp4) {
      MUSE_CK(launch_gemm_fp4<EPI_STORE_SS>(bn_g, pdn.mt, maps, g, q4, nsm, st));
    } else if (pdn.pair && pdn.mt == 2) {
      MUSE_CK((launch_gemm_2sm<T, EPI_STORE_SS, 2>(maps, g, nsm / 2, st)));
    } else if (pdn.pair) {
      MUSE_CK((launch_gemm_2sm<T, EPI_STORE_SS, 1>(maps, g, nsm / 2, st)));
    } else {
      MUSE_CK((launch_gemm_bn<T, T, EPI_STORE_SS>(bn_g, pdn.mt, maps, g, nsm, st)));
    }
    MUSE_CK(p.mark());
  }
  return MUSE_OK;
}

// (a8 + a9) per-expert RMSNorm and weighted combine of the expert outputs y (row inv[t*k+j]
// for token t's j-th expert) with their sum-of-squares partials ss, (a10) unpooler, and the
// feed-forward sublayer's post-norm and residual gate (optional)
template <typename T>
muse_status combine(Pass<T>& p, const T* y, const float* ss, const void* x, const void* gamma, const void* W_unpool,
                    void* out) {
  const muse_moe_config& c = p.c;
  const int64_t Tn = c.T, D = c.D, L = c.L, k = c.top_k;
  T* cbuf = p.template ptr<T>(p.lay.pub.c);
  {
    const int vec = 16 / static_cast<int>(sizeof(T));
    // a vector per thread up to 256 threads; one warp per selected row for the scales
    const int threads = static_cast<int>(
        std::max<int64_t>(32 * std::min<int64_t>(k, 8), std::min<int64_t>(256, align_up(static_cast<size_t>(L / vec), 32))));
    k_combine<T><<<static_cast<unsigned>(Tn), threads, 0, p.st>>>(
        p.topk_idx, p.topk_w, p.inv, ss, static_cast<int>(L / 32), y, reinterpret_cast<const T*>(gamma),
        c.gamma_shared ? 0 : L, static_cast<int>(L), static_cast<int>(k), c.eps, cbuf);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(p.mark());
  }
  // (a10) unpooler; with the sublayer post-norm its epilogue also writes the partial sums
  // of (f * (1 + w))^2
  const bool post = c.ffn_post_gain != nullptr;
  if (post) {
    DenseSS sq;
    sq.ss = p.template ptr<float>(p.lay.pub.ss_out);
    sq.ld = static_cast<int>(D / 32);
    sq.gain = c.ffn_post_gain;
    MUSE_TRY((dense_gemm<T, T, EPI_STORE_SS>(W_unpool, D, cbuf, Tn, L, out, dense_bn(c), p.status, p.ntiles + 7,
                                             p.st, sq)));
  } else {
    MUSE_TRY((dense_gemm<T, T>(W_unpool, D, cbuf, Tn, L, out, dense_bn(c), p.status, p.ntiles + 7, p.st, DenseSS{},
                               p.splitk())));
  }
  MUSE_CK(p.mark());
  // feed-forward sublayer post-norm and residual gate (optional), in place on out
  if (post || c.residual_gate != nullptr) {
    const int vec = 16 / static_cast<int>(sizeof(T));
    const dim3 grid(static_cast<unsigned>(cdiv(Tn, kFinishRows)),
                    static_cast<unsigned>(cdiv(D, static_cast<int64_t>(kFinishThreads) * vec)));
    k_ffn_finish<T><<<grid, kFinishThreads, 0, p.st>>>(
        reinterpret_cast<T*>(out), reinterpret_cast<const T*>(x), p.template ptr<const float>(p.lay.pub.ss_out),
        static_cast<int>(D / 32), reinterpret_cast<const T*>(c.ffn_post_gain), c.ffn_post_eps, c.residual_gate,
        1.0f / c.residual_gate_temperature, c.residual_gate_eps, static_cast<int>(D), static_cast<int>(Tn));
    MUSE_CK(cudaGetLastError());
    MUSE_CK(p.mark());
  }
  return MUSE_OK;
}

template <typename T>
muse_status forward_impl(const muse_moe_config& c, const Layout& lay, const void* x, const void* W_router,
                         const void* W_pool, const void* W_gate, const void* W_up, const void* W_down,
                         const void* gamma, const void* W_unpool, void* out, cudaStream_t st) {
  Pass<T> p(c, lay, st, c.stage_events);
  const int64_t assign = c.T * c.top_k;
  const void* xin = nullptr;
  MUSE_TRY(begin(p));
  MUSE_TRY(route(p, x, W_router, &xin));
  MUSE_TRY(hist(p, p.topk_idx, assign));
  MUSE_TRY(permute(p, p.topk_idx, assign, c.top_k));
  MUSE_TRY(pool(p, xin, W_pool));
  MUSE_TRY(experts(p, p.template ptr<const T>(lay.pub.z), c.T, W_gate, W_up, W_down, gamma));
  return combine(p, p.template ptr<const T>(lay.pub.y), p.template ptr<const float>(lay.pub.ss), x, gamma, W_unpool,
                 out);
}

// Expert parallelism, the token's own rank before the exchange: routing, the send plan,
// the pooler and the send buffer.
template <typename T>
muse_status ep_dispatch_impl(const muse_moe_config& c, const Layout& lay, int G, const void* x, const void* W_router,
                             const void* W_pool, void* send_z, int32_t* send_expert, int32_t* rank_counts,
                             cudaStream_t st) {
  Pass<T> p(c, lay, st, nullptr);
  const int64_t assign = c.T * c.top_k;
  const int E_loc = static_cast<int>(c.E / G);
  const void* xin = nullptr;
  MUSE_TRY(begin(p));
  MUSE_TRY(route(p, x, W_router, &xin));
  MUSE_TRY(hist(p, p.topk_idx, assign));
  const int threads = static_cast<int>(align_up(static_cast<size_t>(c.E), 32));
  k_ep_plan<<<1, threads, 0, st>>>(p.counts, static_cast<int>(c.E), E_loc, G, p.offsets, rank_counts, p.ntiles + 4);
  MUSE_CK(cudaGetLastError());
  k_assign_rows<<<static_cast<unsigned>(c.E), 1024, 0, st>>>(p.topk_idx, static_cast<int>(assign), c.top_k, p.counts,
                                                             p.offsets, p.inv, p.row_token);
  MUSE_CK(cudaGetLastError());
  MUSE_TRY(pool(p, xin, W_pool));
  const int vpr = static_cast<int>(c.L * sizeof(T) / 16);
  const int grid = static_cast<int>(std::min<int64_t>(assign, 16 * p.nsm));
  k_ep_pack<<<grid, 128, 0, st>>>(p.topk_idx, p.inv, static_cast<int>(assign), c.top_k, E_loc,
                                  p.template ptr<const uint4>(lay.pub.z), vpr, static_cast<uint4*>(send_z),
                                  send_expert);
  MUSE_CK(cudaGetLastError());
  return MUSE_OK;
}

// Expert parallelism, an expert shard: the received rows through this rank's experts
// (cl: the local configuration, cl.T = rows received, cl.top_k = 1, cl.E = E / G), the
// results put back in the order received.
template <typename T>
muse_status ep_experts_impl(const muse_moe_config& cl, const Layout& lay, const void* recv_z,
                            const int32_t* recv_expert, const void* W_gate, const void* W_up, const void* W_down,
                            const void* gamma, void* ret_y, float* ret_ss, cudaStream_t st) {
  Pass<T> p(cl, lay, st, nullptr);
  const int64_t R = cl.T;
  MUSE_TRY(begin(p));
  MUSE_CK(cudaMemsetAsync(p.inv, 0xFF, sizeof(int) * R, st));  // rows with no slot stay -1
  MUSE_TRY(hist(p, recv_expert, R));
  MUSE_TRY(permute(p, recv_expert, R, 1));
  MUSE_TRY(experts(p, static_cast<const T*>(recv_z), R, W_gate, W_up, W_down, gamma));
  const int grid = static_cast<int>(std::min<int64_t>(R, 16 * p.nsm));
  k_ep_unpermute<<<grid, 128, 0, st>>>(p.inv, static_cast<int>(R), p.template ptr<const uint4>(lay.pub.y),
                                       p.template ptr<const uint4>(lay.pub.ss),
                                       static_cast<int>(cl.L * sizeof(T) / 16), static_cast<int>(cl.L / 128),
                                       static_cast<uint4*>(ret_y), reinterpret_cast<uint4*>(ret_ss));
  MUSE_CK(cudaGetLastError());
  return MUSE_OK;
}

// weight operands of the expert GEMMs: dense (16-byte aligned) or NVFP4 descriptors
muse_status validate_experts(const muse_moe_config* cfg, const void* W_gate, const void* W_up, const void* W_down) {
  const void* experts[] = {W_gate, W_up, W_down};
  for (const void* p : experts) {
    if (cfg->expert_weights == MUSE_EXPERTS_NVFP4) {
      if (!valid_nvfp4(p)) return MUSE_ERR_INVALID_ARG;
    } else if (p == nullptr || !aligned16(p)) {
      return MUSE_ERR_INVALID_ARG;
    }
  }
  return MUSE_OK;
}

// the configuration's optional pointers and their parameters
muse_status validate_options(const muse_moe_config* cfg) {
  if (cfg->router_bias != nullptr && (reinterpret_cast<uintptr_t>(cfg->router_bias) & 3u)) return MUSE_ERR_INVALID_ARG;
  if (cfg->pre_norm_gain != nullptr && !aligned16(cfg->pre_norm_gain)) return MUSE_ERR_INVALID_ARG;
  if (cfg->pre_norm_gain != nullptr && !(cfg->pre_norm_eps >= 0.0f)) return MUSE_ERR_INVALID_ARG;
  if (cfg->ffn_pre_gain != nullptr && (!aligned16(cfg->ffn_pre_gain) || !(cfg->ffn_pre_eps >= 0.0f)))
    return MUSE_ERR_INVALID_ARG;
  if (cfg->ffn_post_gain != nullptr && (!aligned16(cfg->ffn_post_gain) || !(cfg->ffn_post_eps >= 0.0f)))
    return MUSE_ERR_INVALID_ARG;
  if (cfg->residual_gate != nullptr &&
      (!aligned16(cfg->residual_gate) || !(cfg->residual_gate_temperature > 0.0f) || !(cfg->residual_gate_eps >= 0.0f)))
    return MUSE_ERR_INVALID_ARG;
  return MUSE_OK;
}

// workspace present, aligned and large enough for the layout; the driver entry point
// the tensor maps need
muse_status check_workspace(const muse_moe_config* cfg, const Layout& lay) {
  if (cfg->workspace == nullptr || (reinterpret_cast<uintptr_t>(cfg->workspace) & (kAlign - 1)))
    return MUSE_ERR_WORKSPACE;
  if (cfg->workspace_bytes < lay.pub.total) return MUSE_ERR_WORKSPACE;
  if (encode_fn() == nullptr) return MUSE_ERR_CUDA;
  return MUSE_OK;
}

// model configuration valid and its experts divisible among ep_size ranks
muse_status validate_ep(const muse_moe_config* cfg, int32_t ep_size) {
  MUSE_TRY(validate_sizes(cfg));
  if (ep_size < 1 || cfg->E % ep_size != 0) return MUSE_ERR_INVALID_ARG;
  return MUSE_OK;
}

// An expert shard's configuration: its E / G experts, the rows it received as tokens with
// one expert each; the steps before and after the experts belong to the tokens' ranks.
muse_moe_config expert_shard_config(const muse_moe_config& c, int32_t G, int64_t rows) {
  muse_moe_config l = c;
  l.E = c.E / G;
  l.top_k = 1;
  l.T = rows;
  l.router_bias = nullptr;
  l.pre_norm_gain = nullptr;
  l.ffn_pre_gain = l.ffn_post_gain = nullptr;
  l.residual_gate = nullptr;
  l.topk_idx_out = nullptr;
  l.topk_w_out = nullptr;
  l.stage_events = nullptr;
  return l;
}

// ---------------------------------------------------------------------- shape checks
// A descriptor names a contiguous row-major tensor of element type `elem` and exactly the
// extents `dims` (n of them), on a 16-byte boundary.
bool tensor_is(const muse_tensor* t, int32_t elem, std::initializer_list<int64_t> dims) {
  if (t == nullptr || t->data == nullptr || !aligned16(t->data) || t->elem != elem) return false;
  if (t->ndim != static_cast<int32_t>(dims.size()) || t->ndim < 1 || t->ndim > 3) return false;
  int i = 0;
  for (int64_t d : dims)
    if (t->shape[i++] != d) return false;
  int64_t stride = 1;
  for (int k = t->ndim - 1; k >= 0; --k) {
    if (t->stride[k] != stride) return false;
    stride *= t->shape[k];
  }
  return true;
}

size_t tensor_bytes(const muse_tensor* t) {
  const size_t es = t->elem == MUSE_ELEM_F32 ? 4 : t->elem == MUSE_ELEM_BF16 ? 2 : 1;
  size_t n = es;
  for (int k = 0; k < t->ndim; ++k) n *= static_cast<size_t>(t->shape[k]);
  return n;
}

bool overlaps(const muse_tensor* a, const muse_tensor* b) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a->data), b0 = reinterpret_cast<uintptr_t>(b->data);
  return a0 < b0 + tensor_bytes(b) && b0 < a0 + tensor_bytes(a);
}

// An expert tensor [E, rows, cols]: one dense descriptor, or the three NVFP4 descriptors
// (codes, block scales, matrix scales); fills the weight the forward takes.
bool expert_tensor_is(const muse_moe_config& c, const muse_tensor* t, int64_t rows, int64_t cols,
                      muse_nvfp4_weight* q, const void** dense) {
  if (c.expert_weights == MUSE_EXPERTS_NVFP4) {
    if (t == nullptr || cols % 16 != 0) return false;
    if (!tensor_is(&t[0], MUSE_ELEM_U8, {c.E, rows, cols / 2}) || !tensor_is(&t[1], MUSE_ELEM_U8, {c.E, rows, cols / 16}))
      return false;
    // matrix scales: float [E], 4-byte aligned is enough for the kernels
    const muse_tensor* m = &t[2];
    if (m->data == nullptr || (reinterpret_cast<uintptr_t>(m->data) & 3u) || m->elem != MUSE_ELEM_F32 ||
        m->ndim != 1 || m->shape[0] != c.E || m->stride[0] != 1)
      return false;
    *q = muse_nvfp4_weight{t[0].data, t[1].data, static_cast<const float*>(m->data)};
    *dense = q;
    return true;
  }
  if (!tensor_is(t, c.dtype, {c.E, rows, cols})) return false;
  *dense = t->data;
  return true;
}

// Scratch for muse_latent_moe_forward_static_scratch: a fixed array in device global
// memory, so that entry point never allocates. In host code this name stands for the
// symbol, not a device address; the address comes from cudaGetSymbolAddress.
__device__ __align__(256) uint8_t g_static_scratch[MUSE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_scratch_mu;
void* g_static_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device. It is looked up again on every
// call made outside stream capture (a cheap lookup once the module is loaded), so that an
// address cached before a cudaDeviceReset -- which unloads the module and frees the array --
// is never used afterwards; during capture the address of the last uncaptured call on this
// device is used, so the first call on a device must come before any capture.
muse_status static_scratch_address(cudaStream_t st, void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MUSE_ERR_CUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return MUSE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return MUSE_ERR_CUDA;
    g_static_scratch_ptr[dev] = p;
  }
  if (g_static_scratch_ptr[dev] == nullptr) return MUSE_ERR_CUDA;  // first call made under capture
  *ptr = g_static_scratch_ptr[dev];
  return MUSE_OK;
}

}  // namespace

extern "C" {

void muse_moe_config_init(muse_moe_config* cfg) {
  if (cfg == nullptr) return;
  std::memset(cfg, 0, sizeof(*cfg));
  cfg->top_k = 1;
  cfg->dtype = MUSE_BF16;
  cfg->eps = 1e-6f;
  cfg->router_mode = MUSE_ROUTER_SOFTMAX;
  cfg->router_logit_scale = 1.0f;
  cfg->routed_scaling = 1.0f;
  cfg->norm_mode = MUSE_NORM_CENTRED;
  cfg->pre_norm_eps = 1e-5f;
  cfg->ffn_pre_eps = 1e-5f;
  cfg->ffn_post_eps = 1e-8f;
  cfg->residual_gate_temperature = 0.3f;
  cfg->residual_gate_eps = 1e-3f;
}

muse_status muse_latent_moe_workspace_size(const muse_moe_config* cfg, size_t* bytes) {
  if (bytes == nullptr) return MUSE_ERR_INVALID_ARG;
  const muse_status s = validate_sizes(cfg);
  if (s != MUSE_OK) return s;
  *bytes = make_layout(*cfg).pub.total;
  return MUSE_OK;
}

muse_status muse_latent_moe_workspace_layout(const muse_moe_config* cfg, muse_moe_workspace_layout* layout) {
  if (layout == nullptr) return MUSE_ERR_INVALID_ARG;
  const muse_status s = validate_sizes(cfg);
  if (s != MUSE_OK) return s;
  *layout = make_layout(*cfg).pub;
  return MUSE_OK;
}

muse_status muse_latent_moe_forward(const muse_moe_config* cfg, const void* x, const void* W_router,
                                    const void* W_pool, const void* W_gate, const void* W_up, const void* W_down,
                                    const void* gamma, const void* W_unpool, void* out, void* stream) {
  MUSE_TRY(validate_sizes(cfg));
  const void* ptrs[] = {x, W_router, W_pool, gamma, W_unpool, out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  MUSE_TRY(validate_experts(cfg, W_gate, W_up, W_down));
  MUSE_TRY(validate_options(cfg));
  const Layout lay = make_layout(*cfg);
  MUSE_TRY(check_workspace(cfg, lay));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == MUSE_BF16)
    return forward_impl<__nv_bfloat16>(*cfg, lay, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out, st);
  return forward_impl<float>(*cfg, lay, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out, st);
}

muse_status muse_latent_moe_forward_checked(const muse_moe_config* cfg, const muse_tensor* x,
                                            const muse_tensor* W_router, const muse_tensor* W_pool,
                                            const muse_tensor* W_gate, const muse_tensor* W_up,
                                            const muse_tensor* W_down, const muse_tensor* gamma,
                                            const muse_tensor* W_unpool, const muse_tensor* out, void* stream) {
  MUSE_TRY(validate_sizes(cfg));
  const muse_moe_config& c = *cfg;
  const int32_t a = c.dtype;  // MUSE_F32 / MUSE_BF16 equal MUSE_ELEM_F32 / MUSE_ELEM_BF16
  if (!tensor_is(x, a, {c.T, c.D}) || !tensor_is(W_router, a, {c.E, c.D}) || !tensor_is(W_pool, a, {c.L, c.D}) ||
      !tensor_is(W_unpool, a, {c.D, c.L}) || !tensor_is(out, a, {c.T, c.D}))
    return MUSE_ERR_INVALID_ARG;
  if (!(c.gamma_shared ? tensor_is(gamma, a, {c.L}) : tensor_is(gamma, a, {c.E, c.L}))) return MUSE_ERR_INVALID_ARG;
  muse_nvfp4_weight qg{}, qu{}, qd{};
  const void *wg = nullptr, *wu = nullptr, *wd = nullptr;
  if (!expert_tensor_is(c, W_gate, c.I, c.L, &qg, &wg) || !expert_tensor_is(c, W_up, c.I, c.L, &qu, &wu) ||
      !expert_tensor_is(c, W_down, c.L, c.I, &qd, &wd))
    return MUSE_ERR_INVALID_ARG;
  const muse_tensor* inputs[] = {x, W_router, W_pool, gamma, W_unpool};
  for (const muse_tensor* t : inputs)
    if (overlaps(out, t)) return MUSE_ERR_INVALID_ARG;
  const int n_exp = c.expert_weights == MUSE_EXPERTS_NVFP4 ? 3 : 1;
  const muse_tensor* experts[] = {W_gate, W_up, W_down};
  for (const muse_tensor* t : experts)
    for (int i = 0; i < n_exp; ++i)
      if (overlaps(out, &t[i])) return MUSE_ERR_INVALID_ARG;
  return muse_latent_moe_forward(cfg, x->data, W_router->data, W_pool->data, wg, wu, wd, gamma->data,
                                 W_unpool->data, const_cast<void*>(out->data), stream);
}

muse_status muse_ep_workspace_layout(const muse_moe_config* cfg, int32_t ep_size, int32_t role, int64_t rows,
                                     muse_moe_workspace_layout* layout) {
  if (layout == nullptr) return MUSE_ERR_INVALID_ARG;
  MUSE_TRY(validate_ep(cfg, ep_size));
  if (role == MUSE_EP_HOME) {
    *layout = make_layout(*cfg, Role::kHome).pub;
  } else if (role == MUSE_EP_EXPERTS) {
    if (rows < 0) return MUSE_ERR_INVALID_ARG;
    const muse_moe_config cl = expert_shard_config(*cfg, ep_size, std::max<int64_t>(rows, 1));
    MUSE_TRY(validate_sizes(&cl));
    *layout = make_layout(cl, Role::kExperts).pub;
  } else {
    return MUSE_ERR_INVALID_ARG;
  }
  return MUSE_OK;
}

muse_status muse_ep_dispatch(const muse_moe_config* cfg, int32_t ep_size, const void* x, const void* W_router,
                             const void* W_pool, void* send_z, int32_t* send_expert, int32_t* rank_counts,
                             void* stream) {
  MUSE_TRY(validate_ep(cfg, ep_size));
  const void* ptrs[] = {x, W_router, W_pool, send_z};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  if (send_expert == nullptr || rank_counts == nullptr || (reinterpret_cast<uintptr_t>(send_expert) & 3u) ||
      (reinterpret_cast<uintptr_t>(rank_counts) & 3u))
    return MUSE_ERR_INVALID_ARG;
  MUSE_TRY(validate_options(cfg));
  const Layout lay = make_layout(*cfg, Role::kHome);
  MUSE_TRY(check_workspace(cfg, lay));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == MUSE_BF16)
    return ep_dispatch_impl<__nv_bfloat16>(*cfg, lay, ep_size, x, W_router, W_pool, send_z, send_expert, rank_counts,
                                           st);
  return ep_dispatch_impl<float>(*cfg, lay, ep_size, x, W_router, W_pool, send_z, send_expert, rank_counts, st);
}

muse_status muse_ep_experts(const muse_moe_config* cfg, int32_t ep_size, int64_t rows, const void* recv_z,
                            const int32_t* recv_expert, const void* W_gate, const void* W_up, const void* W_down,
                            const void* gamma, void* ret_y, float* ret_ss, void* stream) {
  MUSE_TRY(validate_ep(cfg, ep_size));
  if (rows < 0) return MUSE_ERR_INVALID_ARG;
  if (rows == 0) return MUSE_OK;  // nothing received: nothing to launch
  const void* ptrs[] = {recv_z, gamma, ret_y, ret_ss};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  if (recv_expert == nullptr || (reinterpret_cast<uintptr_t>(recv_expert) & 3u)) return MUSE_ERR_INVALID_ARG;
  const muse_moe_config cl = expert_shard_config(*cfg, ep_size, rows);
  MUSE_TRY(validate_sizes(&cl));
  MUSE_TRY(validate_experts(&cl, W_gate, W_up, W_down));
  const Layout lay = make_layout(cl, Role::kExperts);
  MUSE_TRY(check_workspace(&cl, lay));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cl.dtype == MUSE_BF16)
    return ep_experts_impl<__nv_bfloat16>(cl, lay, recv_z, recv_expert, W_gate, W_up, W_down, gamma, ret_y, ret_ss,
                                          st);
  return ep_experts_impl<float>(cl, lay, recv_z, recv_expert, W_gate, W_up, W_down, gamma, ret_y, ret_ss, st);
}

muse_status muse_ep_combine(const muse_moe_config* cfg, int32_t ep_size, const void* x, const void* back_y,
                            const float* back_ss, const void* gamma, const void* W_unpool, void* out, void* stream) {
  MUSE_TRY(validate_ep(cfg, ep_size));
  const void* ptrs[] = {x, back_y, back_ss, gamma, W_unpool, out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  MUSE_TRY(validate_options(cfg));
  const Layout lay = make_layout(*cfg, Role::kHome);
  MUSE_TRY(check_workspace(cfg, lay));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == MUSE_BF16) {
    Pass<__nv_bfloat16> p(*cfg, lay, st, nullptr);
    return combine(p, static_cast<const __nv_bfloat16*>(back_y), back_ss, x, gamma, W_unpool, out);
  }
  Pass<float> p(*cfg, lay, st, nullptr);
  return combine(p, static_cast<const float*>(back_y), back_ss, x, gamma, W_unpool, out);
}

muse_status muse_latent_moe_forward_host_io(const muse_moe_config* cfg, const void* x_host, void* x_dev,
                                            const void* W_router, const void* W_pool, const void* W_gate,
                                            const void* W_up, const void* W_down, const void* gamma,
                                            const void* W_unpool, void* out_dev, void* out_host, void* stream) {
  muse_status s = validate_sizes(cfg);
  if (s != MUSE_OK) return s;
  if (x_host == nullptr || out_host == nullptr || x_dev == nullptr || out_dev == nullptr) return MUSE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(cfg->T) * cfg->D * act_size(*cfg);
  if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return MUSE_ERR_CUDA;
  s = muse_latent_moe_forward(cfg, x_dev, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out_dev, stream);
  if (s != MUSE_OK) return s;
  if (cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MUSE_ERR_CUDA;
  return MUSE_OK;
}

muse_status muse_latent_moe_forward_host_batches(const muse_moe_config* cfg, int64_t n_batches,
                                                 const void* const* x_host, void* const* out_host,
                                                 void* const* x_dev, void* const* out_dev, const void* W_router,
                                                 const void* W_pool, const void* W_gate, const void* W_up,
                                                 const void* W_down, const void* gamma, const void* W_unpool,
                                                 void* stream, void* h2d_stream, void* d2h_stream) {
  muse_status s = validate_sizes(cfg);
  if (s != MUSE_OK) return s;
  if (n_batches < 1 || x_host == nullptr || out_host == nullptr || x_dev == nullptr || out_dev == nullptr)
    return MUSE_ERR_INVALID_ARG;
  if (stream == h2d_stream || stream == d2h_stream || h2d_stream == d2h_stream) return MUSE_ERR_INVALID_ARG;
  for (int64_t b = 0; b < n_batches; ++b)
    if (x_host[b] == nullptr || out_host[b] == nullptr) return MUSE_ERR_INVALID_ARG;
  for (int i = 0; i < 2; ++i)
    if (x_dev[i] == nullptr || out_dev[i] == nullptr || !aligned16(x_dev[i]) || !aligned16(out_dev[i]))
      return MUSE_ERR_INVALID_ARG;
  cudaStream_t sc = static_cast<cudaStream_t>(stream), su = static_cast<cudaStream_t>(h2d_stream),
               sd = static_cast<cudaStream_t>(d2h_stream);
  const size_t bytes = static_cast<size_t>(cfg->T) * cfg->D * act_size(*cfg);
  // per device buffer: uploaded, computed, downloaded
  cudaEvent_t up[2] = {nullptr, nullptr}, comp[2] = {nullptr, nullptr}, down[2] = {nullptr, nullptr};
  muse_status rc = MUSE_OK;
  for (int i = 0; i < 2 && rc == MUSE_OK; ++i)
    if (cudaEventCreateWithFlags(&up[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&comp[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&down[i], cudaEventDisableTiming) != cudaSuccess)
      rc = MUSE_ERR_CUDA;
  for (int64_t b = 0; b < n_batches && rc == MUSE_OK; ++b) {
    const int i = static_cast<int>(b & 1);
    // upload batch b once the forward of batch b - 2 has read x_dev[i]
    if (b >= 2 && cudaStreamWaitEvent(su, comp[i], 0) != cudaSuccess) rc = MUSE_ERR_CUDA;
    if (rc == MUSE_OK && (cudaMemcpyAsync(x_dev[i], x_host[b], bytes, cudaMemcpyHostToDevice, su) != cudaSuccess ||
                          cudaEventRecord(up[i], su) != cudaSuccess))
      rc = MUSE_ERR_CUDA;
    // compute once uploaded and once batch b - 2's output has left out_dev[i]
    if (rc == MUSE_OK && cudaStreamWaitEvent(sc, up[i], 0) != cudaSuccess) rc = MUSE_ERR_CUDA;
    if (rc == MUSE_OK && b >= 2 && cudaStreamWaitEvent(sc, down[i], 0) != cudaSuccess) rc = MUSE_ERR_CUDA;
    if (rc == MUSE_OK)
      rc = muse_latent_moe_forward(cfg, x_dev[i], W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool,
                                   out_dev[i], stream);
    if (rc == MUSE_OK && cudaEventRecord(comp[i], sc) != cudaSuccess) rc = MUSE_ERR_CUDA;
    // download once computed
    if (rc == MUSE_OK && (cudaStreamWaitEvent(sd, comp[i], 0) != cudaSuccess ||
                          cudaMemcpyAsync(out_host[b], out_dev[i], bytes, cudaMemcpyDeviceToHost, sd) != cudaSuccess ||
                          cudaEventRecord(down[i], sd) != cudaSuccess))
      rc = MUSE_ERR_CUDA;
  }
  for (int i = 0; i < 2; ++i) {  // released once the work recorded on them completes
    if (up[i]) cudaEventDestroy(up[i]);
    if (comp[i]) cudaEventDestroy(comp[i]);
    if (down[i]) cudaEventDestroy(down[i]);
  }
  return rc;
}

muse_status muse_latent_moe_forward_static_scratch(const muse_moe_config* cfg, const void* x, const void* W_router,
                                                  const void* W_pool, const void* W_gate, const void* W_up,
                                                  const void* W_down, const void* gamma, const void* W_unpool,
                                                  void* out, void* stream) {
  const muse_status s = validate_sizes(cfg);
  if (s != MUSE_OK) return s;
  if (make_layout(*cfg).pub.total > MUSE_STATIC_SCRATCH_BYTES) return MUSE_ERR_WORKSPACE;
  void* scratch = nullptr;
  const muse_status a = static_scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (a != MUSE_OK) return a;
  muse_moe_config c = *cfg;
  c.workspace = scratch;
  c.workspace_bytes = MUSE_STATIC_SCRATCH_BYTES;
  return muse_latent_moe_forward(&c, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out, stream);
}

muse_status muse_latent_moe_last_device_status(const muse_moe_config* cfg, void* stream, uint32_t* detail) {
  muse_status s = validate_sizes(cfg);
  if (s != MUSE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // no workspace: the word of the built-in scratch array (muse_latent_moe_forward_static_scratch)
  void* ws = cfg->workspace;
  if (ws == nullptr && static_scratch_address(st, &ws) != MUSE_OK) return MUSE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MUSE_ERR_CUDA;
  uint32_t word[2] = {0, 0};
  const Layout lay = make_layout(*cfg);
  if (cudaMemcpy(word, static_cast<uint8_t*>(ws) + lay.pub.status, sizeof(word), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return MUSE_ERR_CUDA;
  if (detail != nullptr) *detail = word[1];
  return static_cast<muse_status>(word[0]);
}

muse_status muse_quantize_nvfp4_rows(const void* src, int64_t rows, int64_t K, void* codes, void* scales,
                                     void* stream) {
  if (src == nullptr || codes == nullptr || scales == nullptr || !aligned16(src) || !aligned16(codes)) return MUSE_ERR_INVALID_ARG;
  if (rows < 1 || K < 16 || K % 16 != 0 || rows > (int64_t(1) << 30) || K > (int64_t(1) << 20)) return MUSE_ERR_INVALID_ARG;
  const int grid = static_cast<int>(std::min<int64_t>(rows, 16 * sm_count()));
  k_quant_rows_nvfp4<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      nullptr, nullptr, static_cast<int>(rows), static_cast<const __nv_bfloat16*>(src), static_cast<int>(K),
      static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales));
  return cudaGetLastError() == cudaSuccess ? MUSE_OK : MUSE_ERR_CUDA;
}

muse_status muse_selftest_bounded_wait(uint64_t limit_ns, uint32_t* status_dev, void* stream) {
  if (status_dev == nullptr || limit_ns < 1 || limit_ns > 10000000000ull) return MUSE_ERR_INVALID_ARG;
  k_selftest_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, status_dev);
  return cudaGetLastError() == cudaSuccess ? MUSE_OK : MUSE_ERR_CUDA;
}

const char* muse_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

const char* muse_status_string(muse_status s) {
  switch (s) {
    case MUSE_OK: return "ok";
    case MUSE_ERR_INVALID_ARG: return "invalid argument";
    case MUSE_ERR_UNSUPPORTED: return "unsupported shape or mode";
    case MUSE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MUSE_ERR_CUDA: return "CUDA call failed";
    case MUSE_ERR_TIMEOUT: return "device-side wait timed out";
    case MUSE_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

int32_t muse_latent_moe_launch_count(const muse_moe_config* cfg) {
  if (validate_sizes(cfg) != MUSE_OK) return -1;
  int32_t n = 0;
  while (muse_latent_moe_stage_name(cfg, n) != nullptr) ++n;
  return n;
}

const char* muse_latent_moe_stage_name(const muse_moe_config* cfg, int32_t i) {
  if (validate_sizes(cfg) != MUSE_OK || i < 0) return nullptr;
  const muse_moe_config& c = *cfg;
  const char* names[20];
  int n = 0;
  if (c.ffn_pre_gain != nullptr) names[n++] = "ffn_pre_norm";
  names[n++] = "router";
  names[n++] = "topk";
  names[n++] = "expert_hist";
  names[n++] = "tiles";
  names[n++] = "assign_rows";
  names[n++] = "pooler";
  if (c.pre_norm_gain != nullptr) names[n++] = "pre_expert_norm";
  if (w4a4(c)) {
    names[n++] = "quant_z";
    names[n++] = "gather_codes";
  } else {
    names[n++] = "gather";
  }
  names[n++] = "gate_up_swiglu";
  if (w4a4(c)) names[n++] = "quant_h";
  names[n++] = "down_sumsq";
  names[n++] = "norm_combine";
  names[n++] = "unpooler";
  if (c.ffn_post_gain != nullptr || c.residual_gate != nullptr) names[n++] = "ffn_post_norm_gate";
  return i < n ? names[i] : nullptr;
}

}  // extern "C"
