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

#include <cstdint>
#include <cstring>
#include <mutex>

#include "muse_moe.h"
#include "gemm_umma.cuh"
#include "gemm_umma_2sm.cuh"
#include "gemm_umma_fp4.cuh"
#include "gemm_umma_w4a4.cuh"
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
int grouped_bn(const muse_moe_config& c) {
  if ((c.T * c.top_k) <= 32 * c.E) return 32;
  if (w4a4(c)) return 128;                                    // W4A4: accumulators leave TMEM room for scales
  return c.expert_weights == MUSE_EXPERTS_NVFP4 ? 192 : 256;  // NVFP4: accumulators leave TMEM room for weights
}
int dense_bn(const muse_moe_config& c) { return c.T <= 32 ? 32 : 256; }

struct Layout {
  muse_moe_workspace_layout pub;
  size_t tiles_gu, tiles_dn, ntiles;  // int4 lists; int[8]: tile counts [0..1], tile counters [4..7]
  size_t zt_codes, zt_scales;         // W4A4: the latent quantised in token order [T, L/2], [T, L/16]
  int64_t max_tiles_gu, max_tiles_dn;
};

size_t act_size(const muse_moe_config& c) { return c.dtype == MUSE_BF16 ? 2 : 4; }

Layout make_layout(const muse_moe_config& c) {
  Layout l{};
  const int64_t T = c.T, E = c.E, k = c.top_k;
  const int64_t assign = T * k;
  const int64_t rows = align_up(static_cast<size_t>(assign + 15 * std::min<int64_t>(E, assign)), 16);
  const int bn = grouped_bn(c);
  const int64_t chunks = cdiv(assign, bn) + std::min<int64_t>(E, assign);
  l.max_tiles_gu = chunks * (c.I / 128);
  l.max_tiles_dn = chunks * (c.L / 128);
  const size_t as = act_size(c);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, kAlign);
    return at;
  };
  l.pub.status = take(16);
  l.pub.expert_count = take(sizeof(int32_t) * E);
  l.pub.expert_offset = take(sizeof(int32_t) * (E + 1));
  l.ntiles = take(sizeof(int32_t) * 8);
  l.pub.logits = take(sizeof(float) * T * E);
  l.pub.topk_idx = take(sizeof(int32_t) * assign);
  l.pub.topk_w = take(sizeof(float) * assign);
  l.pub.inv = take(sizeof(int32_t) * assign);
  l.pub.row_token = take(sizeof(int32_t) * rows);
  l.tiles_gu = take(sizeof(int4) * l.max_tiles_gu);
  l.tiles_dn = take(sizeof(int4) * l.max_tiles_dn);
  l.pub.z = take(as * T * c.L);
  l.pub.zp = take(as * rows * c.L);
  l.pub.h = take(as * rows * c.I);
  l.pub.y = take(as * rows * c.L);
  l.pub.ss = take(sizeof(float) * rows * (c.L / 32));
  l.pub.c = take(as * T * c.L);
  l.pub.xn = c.ffn_pre_gain != nullptr ? take(as * T * c.D) : 0;
  l.pub.ss_out = c.ffn_post_gain != nullptr ? take(sizeof(float) * T * (c.D / 32)) : 0;
  l.zt_codes = l.zt_scales = 0;
  if (w4a4(c)) {
    l.zt_codes = take(T * (c.L / 2));
    l.zt_scales = take(T * (c.L / 16));
    l.pub.zq_codes = take(rows * (c.L / 2));
    l.pub.zq_scales = take(rows * (c.L / 16));
    l.pub.hq_codes = take(rows * (c.I / 2));
    l.pub.hq_scales = take(rows * (c.I / 16));
  }
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

template <int EPI>
cudaError_t launch_gemm_fp4(int bn, int mt, const TmaMaps& maps, const GemmArgs& args, const Fp4Args& q4, int grid,
                            cudaStream_t st) {
  if constexpr (EPI == EPI_SWIGLU) {
    return bn == 32 ? launch_gemm_fp4_t<32, EPI, 2>(maps, args, q4, grid, st)
                    : launch_gemm_fp4_t<192, EPI, 2>(maps, args, q4, grid, st);
  } else {
    if (bn == 32) return mt == 2 ? launch_gemm_fp4_t<32, EPI, 2>(maps, args, q4, grid, st)
                                 : launch_gemm_fp4_t<32, EPI, 1>(maps, args, q4, grid, st);
    return mt == 2 ? launch_gemm_fp4_t<192, EPI, 2>(maps, args, q4, grid, st)
                   : launch_gemm_fp4_t<192, EPI, 1>(maps, args, q4, grid, st);
  }
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

// dense C[T, M] = X[T, K] W[M, K]^T
template <typename TIn, typename TOut, int EPI = EPI_STORE>
muse_status dense_gemm(const void* W, int64_t M, const void* X, int64_t T, int64_t K, void* out, int bn,
                       uint32_t* status, int* tile_counter, cudaStream_t st, DenseSS sq = DenseSS{}) {
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
  // a CTA pair per 256 features x 256 tokens when that fills at least one wave of pairs
  if (bf && bn == 256 && cdiv(M, 256) * cdiv(T, 256) >= nsm / 2) {
    if (sizeof(TOut) == 2 && !make_out_map(&maps.out, out, T, M)) return MUSE_ERR_CUDA;
    g.m_step = 256;
    g.m_tiles = static_cast<int>(cdiv(M, 256));
    g.num_tiles = static_cast<int>(g.m_tiles * cdiv(T, 256));
    g.tile_counter = tile_counter;
    const int pairs = std::min(g.num_tiles, nsm / 2);
    return launch_gemm_2sm<TOut, EPI, 1>(maps, g, pairs, st) == cudaSuccess ? MUSE_OK : MUSE_ERR_CUDA;
  }
  // two 128-row weight tiles per CTA when that still leaves at least a full wave of tiles
  const int mt = (cdiv(M, 256) * cdiv(T, bn) >= nsm) ? 2 : 1;
  g.m_step = 128 * mt;
  g.m_tiles = static_cast<int>(cdiv(M, g.m_step));
  g.num_tiles = static_cast<int>(g.m_tiles * cdiv(T, bn));
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
  if (c.expert_weights == MUSE_EXPERTS_NVFP4) return c.L % 256 == 0 ? GemmPlan{false, 2, 256} : GemmPlan{false, 1, 128};
  if (c.dtype == MUSE_BF16 && bn_g == 256 && c.L % 512 == 0) return {true, 2, 512};
  if (c.dtype == MUSE_BF16 && bn_g == 256 && c.L % 256 == 0) return {true, 1, 256};
  if (bn_g == 256 && c.L % 256 == 0) return {false, 2, 256};
  return {false, 1, 128};
}

#define MUSE_CK(x)                                 \
  do {                                             \
    if ((x) != cudaSuccess) return MUSE_ERR_CUDA;  \
  } while (0)

template <typename T>
muse_status forward_impl(const muse_moe_config& c, const Layout& lay, const void* x, const void* W_router,
                         const void* W_pool, const void* W_gate, const void* W_up, const void* W_down,
                         const void* gamma, const void* W_unpool, void* out, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(c.workspace);
  auto at = [&](size_t off) { return ws + off; };
  uint32_t* status = reinterpret_cast<uint32_t*>(at(lay.pub.status));
  int* counts = reinterpret_cast<int*>(at(lay.pub.expert_count));
  int* offsets = reinterpret_cast<int*>(at(lay.pub.expert_offset));
  int* ntiles = reinterpret_cast<int*>(at(lay.ntiles));
  float* logits = reinterpret_cast<float*>(at(lay.pub.logits));
  int* topk_idx = reinterpret_cast<int*>(at(lay.pub.topk_idx));
  float* topk_w = reinterpret_cast<float*>(at(lay.pub.topk_w));
  int* inv = reinterpret_cast<int*>(at(lay.pub.inv));
  int* row_token = reinterpret_cast<int*>(at(lay.pub.row_token));
  int4* tiles_gu = reinterpret_cast<int4*>(at(lay.tiles_gu));
  int4* tiles_dn = reinterpret_cast<int4*>(at(lay.tiles_dn));
  T* z = reinterpret_cast<T*>(at(lay.pub.z));
  T* zp = reinterpret_cast<T*>(at(lay.pub.zp));
  T* h = reinterpret_cast<T*>(at(lay.pub.h));
  T* y = reinterpret_cast<T*>(at(lay.pub.y));
  float* ss = reinterpret_cast<float*>(at(lay.pub.ss));
  T* cbuf = reinterpret_cast<T*>(at(lay.pub.c));
  const bool bf = sizeof(T) == 2;
  const int64_t Tn = c.T, D = c.D, L = c.L, I = c.I, E = c.E, k = c.top_k;
  const int64_t assign = Tn * k;
  const int nsm = sm_count();
  const int bn_d = dense_bn(c), bn_g = grouped_bn(c);
  const GemmPlan pgu = plan_gate_up(c, bn_g), pdn = plan_down(c, bn_g);

  MUSE_CK(cudaMemsetAsync(status, 0, 16, st));
  MUSE_CK(cudaMemsetAsync(counts, 0, sizeof(int) * E, st));
  int stage = 0;
  auto mark = [&]() -> cudaError_t {
    if (c.stage_events == nullptr) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(c.stage_events[stage++]), st);
  };
  MUSE_CK(mark());

  // feed-forward sublayer pre-norm (optional): the router and the pooler read xn
  const void* xin = x;
  if (c.ffn_pre_gain != nullptr) {
    T* xn = reinterpret_cast<T*>(at(lay.pub.xn));
    k_rmsnorm_rows<T><<<static_cast<unsigned>(Tn), 256, 0, st>>>(reinterpret_cast<const T*>(x), xn,
                                                                 reinterpret_cast<const T*>(c.ffn_pre_gain),
                                                                 static_cast<int>(D), c.ffn_pre_eps);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
    xin = xn;
  }
  // (a1) router logits
  if (bf) {
    muse_status s = dense_gemm<T, float>(W_router, E, xin, Tn, D, logits, bn_d, status, nullptr, st);
    if (s != MUSE_OK) return s;
  } else {
    k_router_logits_f32<<<static_cast<unsigned>(Tn), 256, 0, st>>>(reinterpret_cast<const float*>(xin),
                                                                  reinterpret_cast<const float*>(W_router),
                                                                  static_cast<int>(D), static_cast<int>(E), logits);
    MUSE_CK(cudaGetLastError());
  }
  MUSE_CK(mark());
  // (a2) top-k and weights
  k_topk<<<static_cast<unsigned>(cdiv(Tn * 32, 256)), 256, 0, st>>>(
      logits, static_cast<int>(Tn), static_cast<int>(E), static_cast<int>(k), c.router_bias, c.router_mode,
      c.router_logit_scale, c.routed_scaling, topk_idx, topk_w, c.topk_idx_out, c.topk_w_out);
  MUSE_CK(cudaGetLastError());
  MUSE_CK(mark());
  // (a3) permutation
  {
    const int grid = static_cast<int>(std::min<int64_t>(cdiv(assign, 256), 4 * nsm));
    k_expert_hist<<<grid, 256, sizeof(int) * E, st>>>(topk_idx, static_cast<int>(assign), static_cast<int>(E),
                                                      counts, status);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
    const int threads = static_cast<int>(align_up(static_cast<size_t>(E), 32));
    k_build_tiles<<<1, threads, 0, st>>>(counts, static_cast<int>(E), bn_g, static_cast<int>(I / pgu.step), pgu.step,
                                         static_cast<int>(L / pdn.step), pdn.step, offsets, tiles_gu, ntiles,
                                         tiles_dn, ntiles + 1, ntiles + 4, row_token);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
    k_assign_rows<<<static_cast<unsigned>(E), 1024, 0, st>>>(topk_idx, static_cast<int>(assign), static_cast<int>(k),
                                                            counts, offsets, inv, row_token);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
  }
  // (a4) pooler
  {
    muse_status s = dense_gemm<T, T>(W_pool, L, xin, Tn, D, z, bn_d, status, ntiles + 6, st);
    if (s != MUSE_OK) return s;
    MUSE_CK(mark());
  }
  // pages' pre_expert_norm on z (optional)
  if (c.pre_norm_gain != nullptr) {
    k_rmsnorm_rows<T><<<static_cast<unsigned>(Tn), 256, 0, st>>>(z, z, reinterpret_cast<const T*>(c.pre_norm_gain),
                                                                 static_cast<int>(L), c.pre_norm_eps);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
  }
  // (a5) gather into expert order (W4A4: gather and quantise to NVFP4 in one pass)
  const bool q4a = w4a4(c);
  uint8_t* zq_codes = at(lay.pub.zq_codes);
  uint8_t* zq_scales = at(lay.pub.zq_scales);
  uint8_t* hq_codes = at(lay.pub.hq_codes);
  uint8_t* hq_scales = at(lay.pub.hq_scales);
  const int quant_grid = static_cast<int>(std::min<int64_t>(lay.pub.rows, 16 * nsm));
  if (q4a) {
    uint8_t* zt_codes = at(lay.zt_codes);
    uint8_t* zt_scales = at(lay.zt_scales);
    k_quant_rows_nvfp4<<<static_cast<unsigned>(std::min<int64_t>(Tn, 16 * nsm)), 256, 0, st>>>(
        nullptr, nullptr, static_cast<int>(Tn), reinterpret_cast<const __nv_bfloat16*>(z), static_cast<int>(L),
        zt_codes, zt_scales);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
    k_gather_nvfp4_rows<<<quant_grid, 128, 0, st>>>(row_token, offsets + E, reinterpret_cast<const uint4*>(zt_codes),
                                                    reinterpret_cast<const uint4*>(zt_scales),
                                                    reinterpret_cast<uint4*>(zq_codes),
                                                    reinterpret_cast<uint4*>(zq_scales), static_cast<int>(L));
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
  } else {
    const int vpr = static_cast<int>(L * sizeof(T) / 16);
    const int rows_grid = static_cast<int>(std::min<int64_t>(lay.pub.rows, 16 * nsm));
    k_gather_rows<<<rows_grid, 128, 0, st>>>(row_token, offsets + E, reinterpret_cast<const uint4*>(z),
                                            reinterpret_cast<uint4*>(zp), vpr);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
  }
  const int64_t R = lay.pub.rows;
  // (a6) gate/up + SwiGLU
  {
    const bool fp4 = c.expert_weights == MUSE_EXPERTS_NVFP4;
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
    GemmArgs g = base_args(status);
    g.tiles = tiles_gu;
    g.num_tiles_dev = ntiles;
    g.tile_counter = ntiles + 4;
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
      g.tile_counter = ntiles + 4;
      MUSE_CK(launch_gemm_w4a4<EPI_SWIGLU>(bn_g, wm, g, wq, nsm, st));
    } else if (fp4) {
      MUSE_CK(launch_gemm_fp4<EPI_SWIGLU>(bn_g, 2, maps, g, q4, nsm, st));
    } else if (pgu.pair) {
      if (!make_out_map(&maps.out, h, R, I)) return MUSE_ERR_CUDA;
      MUSE_CK((launch_gemm_2sm<T, EPI_SWIGLU, 2>(maps, g, nsm / 2, st)));
    } else {
      MUSE_CK((launch_gemm_bn<T, T, EPI_SWIGLU>(bn_g, 2, maps, g, nsm, st)));
    }
    MUSE_CK(mark());
  }
  // W4A4: quantise h (already in expert order) for the down projection
  if (q4a) {
    k_quant_rows_nvfp4<<<quant_grid, 256, 0, st>>>(row_token, offsets + E, 0, reinterpret_cast<const __nv_bfloat16*>(h),
                                                   static_cast<int>(I), hq_codes, hq_scales);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
  }
  // (a7) down projection + sum-of-squares partials
  {
    const bool fp4 = c.expert_weights == MUSE_EXPERTS_NVFP4;
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
    GemmArgs g = base_args(status);
    g.tiles = tiles_dn;
    g.num_tiles_dev = ntiles + 1;
    g.tile_counter = ntiles + 5;
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
      g.tile_counter = ntiles + 5;
      MUSE_CK(launch_gemm_w4a4<EPI_STORE_SS>(bn_g, wm, g, wq, nsm, st));
    } else if (fp4) {
      MUSE_CK(launch_gemm_fp4<EPI_STORE_SS>(bn_g, pdn.mt, maps, g, q4, nsm, st));
    } else if (pdn.pair && pdn.mt == 2) {
      MUSE_CK((launch_gemm_2sm<T, EPI_STORE_SS, 2>(maps, g, nsm / 2, st)));
    } else if (pdn.pair) {
      MUSE_CK((launch_gemm_2sm<T, EPI_STORE_SS, 1>(maps, g, nsm / 2, st)));
    } else {
      MUSE_CK((launch_gemm_bn<T, T, EPI_STORE_SS>(bn_g, pdn.mt, maps, g, nsm, st)));
    }
    MUSE_CK(mark());
  }
  // (a8 + a9) per-expert RMSNorm and weighted combine
  {
    const int vec = 16 / static_cast<int>(sizeof(T));
    // a vector per thread up to 256 threads; one warp per selected row for the scales
    const int threads = static_cast<int>(
        std::max<int64_t>(32 * std::min<int64_t>(k, 8), std::min<int64_t>(256, align_up(static_cast<size_t>(L / vec), 32))));
    k_combine<T><<<static_cast<unsigned>(Tn), threads, 0, st>>>(
        topk_idx, topk_w, inv, ss, static_cast<int>(L / 32), y, reinterpret_cast<const T*>(gamma),
        c.gamma_shared ? 0 : L, static_cast<int>(L), static_cast<int>(k), c.eps, cbuf);
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
  }
  // (a10) unpooler; with the sublayer post-norm its epilogue also writes the partial sums
  // of (f * (1 + w))^2
  const bool post = c.ffn_post_gain != nullptr;
  {
    muse_status s;
    if (post) {
      DenseSS sq;
      sq.ss = reinterpret_cast<float*>(at(lay.pub.ss_out));
      sq.ld = static_cast<int>(D / 32);
      sq.gain = c.ffn_post_gain;
      s = dense_gemm<T, T, EPI_STORE_SS>(W_unpool, D, cbuf, Tn, L, out, bn_d, status, ntiles + 7, st, sq);
    } else {
      s = dense_gemm<T, T>(W_unpool, D, cbuf, Tn, L, out, bn_d, status, ntiles + 7, st);
    }
    if (s != MUSE_OK) return s;
  }
  MUSE_CK(mark());
  // feed-forward sublayer post-norm and residual gate (optional), in place on out
  if (post || c.residual_gate != nullptr) {
    const int vec = 16 / static_cast<int>(sizeof(T));
    const dim3 grid(static_cast<unsigned>(cdiv(Tn, kFinishRows)),
                    static_cast<unsigned>(cdiv(D, static_cast<int64_t>(kFinishThreads) * vec)));
    k_ffn_finish<T><<<grid, kFinishThreads, 0, st>>>(
        reinterpret_cast<T*>(out), reinterpret_cast<const T*>(x), reinterpret_cast<const float*>(at(lay.pub.ss_out)),
        static_cast<int>(D / 32), reinterpret_cast<const T*>(c.ffn_post_gain), c.ffn_post_eps, c.residual_gate,
        1.0f / c.residual_gate_temperature, c.residual_gate_eps, static_cast<int>(D), static_cast<int>(Tn));
    MUSE_CK(cudaGetLastError());
    MUSE_CK(mark());
  }
  return MUSE_OK;
}

// Scratch for muse_latent_moe_forward_static_scratch: a fixed array in device global
// memory, so that entry point never allocates. In host code this name stands for the
// symbol, not a device address; the address comes from cudaGetSymbolAddress.
__device__ __align__(256) uint8_t g_static_scratch[MUSE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_scratch_mu;
void* g_static_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once per device.
muse_status static_scratch_address(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MUSE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (g_static_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return MUSE_ERR_CUDA;
    g_static_scratch_ptr[dev] = p;
  }
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
  muse_status s = validate_sizes(cfg);
  if (s != MUSE_OK) return s;
  const void* ptrs[] = {x, W_router, W_pool, gamma, W_unpool, out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  const void* experts[] = {W_gate, W_up, W_down};
  for (const void* p : experts) {
    if (cfg->expert_weights == MUSE_EXPERTS_NVFP4) {
      if (!valid_nvfp4(p)) return MUSE_ERR_INVALID_ARG;
    } else if (p == nullptr || !aligned16(p)) {
      return MUSE_ERR_INVALID_ARG;
    }
  }
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
  const Layout lay = make_layout(*cfg);
  if (cfg->workspace == nullptr || (reinterpret_cast<uintptr_t>(cfg->workspace) & (kAlign - 1)))
    return MUSE_ERR_WORKSPACE;
  if (cfg->workspace_bytes < lay.pub.total) return MUSE_ERR_WORKSPACE;
  if (encode_fn() == nullptr) return MUSE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == MUSE_BF16)
    return forward_impl<__nv_bfloat16>(*cfg, lay, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out, st);
  return forward_impl<float>(*cfg, lay, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out, st);
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
  const muse_status a = static_scratch_address(&scratch);
  if (a != MUSE_OK) return a;
  muse_moe_config c = *cfg;
  c.workspace = scratch;
  c.workspace_bytes = MUSE_STATIC_SCRATCH_BYTES;
  return muse_latent_moe_forward(&c, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out, stream);
}

muse_status muse_latent_moe_last_device_status(const muse_moe_config* cfg, void* stream, uint32_t* detail) {
  muse_status s = validate_sizes(cfg);
  if (s != MUSE_OK) return s;
  if (cfg->workspace == nullptr) return MUSE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MUSE_ERR_CUDA;
  uint32_t word[2] = {0, 0};
  const Layout lay = make_layout(*cfg);
  if (cudaMemcpy(word, static_cast<uint8_t*>(cfg->workspace) + lay.pub.status, sizeof(word),
                 cudaMemcpyDeviceToHost) != cudaSuccess)
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
  // router, top-k, hist, tiles, rows, pooler, gather, gate/up, down, combine, unpooler,
  // and the optional sublayer pre-norm (first), pre-expert norm (between pooler and
  // gather) and sublayer post-norm / residual gate (last)
  return 11 + (cfg->pre_norm_gain != nullptr) + (cfg->ffn_pre_gain != nullptr) +
         (cfg->ffn_post_gain != nullptr || cfg->residual_gate != nullptr) + 2 * (cfg->act_format == MUSE_ACT_NVFP4);
}

}  // extern "C"
