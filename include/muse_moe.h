/*
 * muse_moe.h -- C ABI of the latent mixture-of-experts block (forward pass) on one
 * NVIDIA B200 (sm_100a).
 *
 * The block (Muse Spark Open deep dive, §4.3, block equation; §4.2 router):
 *
 *   l   = W_router x                     router logits over E experts, full width D
 *   S,g = top-k of l (+ bias), weights    softmax over the E logits renormalised on S
 *   z   = W_pool x                        shared pooler D -> L
 *   y_j = W_down[e] (SiLU(W_gate[e] z) * W_up[e] z),   e = S_j   (SwiGLU L -> I -> L)
 *   n_j = y_j / sqrt(mean(y_j^2) + eps) * (1 + gamma[e])          per-expert RMSNorm
 *   c   = sum_j g_j n_j                   weighted combine, after each norm
 *   out = W_unpool c                      shared unpooler L -> D
 *
 * Readings fixed by this library where the pages leave a step open: softmax router
 * (the released model's sigmoid router is MUSE_ROUTER_SIGMOID), top-k ordered by key
 * descending with ties to the lower expert index, per-expert centred gain (the released
 * model's single input-scaled gain is MUSE_NORM_INPUT_SCALED with gamma_shared = 1).
 *
 * Layouts (row-major, every weight stored [out, in], the K dimension contiguous):
 *   x        [T, D]        W_router [E, D]       W_pool   [L, D]
 *   W_gate   [E, I, L]     W_up     [E, I, L]    W_down   [E, L, I]
 *   gamma    [E, L] (or [L] when gamma_shared)    W_unpool [D, L]     out [T, D]
 * Every tensor has the dtype cfg->dtype (float32 or bfloat16). Accumulation is FP32.
 *
 * Ownership: the caller owns every buffer, including the device workspace. The library
 * allocates no device memory, keeps no per-call state, and enqueues all work on the
 * given stream without synchronising (except muse_latent_moe_last_device_status).
 * Errors: every function returns a muse_status. Arguments are validated before any
 * launch; a failed validation launches nothing. Device-side waits are bounded: a wait
 * that runs out records MUSE_ERR_TIMEOUT in the workspace's status word instead of
 * hanging, readable with muse_latent_moe_last_device_status.
 */
#ifndef MUSE_MOE_H_
#define MUSE_MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MUSE_API __attribute__((visibility("default")))
#else
#define MUSE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum muse_status {
  MUSE_OK = 0,
  MUSE_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, inconsistent sizes */
  MUSE_ERR_UNSUPPORTED = 2,   /* shape or mode the library does not implement   */
  MUSE_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  MUSE_ERR_CUDA = 4,          /* a CUDA runtime / driver call failed */
  MUSE_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out */
  MUSE_ERR_DEVICE = 6         /* a device-side check failed (e.g. a bad index) */
} muse_status;

typedef enum muse_dtype { MUSE_F32 = 0, MUSE_BF16 = 1 } muse_dtype;

typedef enum muse_router_mode {
  MUSE_ROUTER_SOFTMAX = 0,    /* key = l + b; g = softmax(l) renormalised on S        */
  MUSE_ROUTER_SIGMOID = 1     /* released router (deep dive §4.2): s = sigmoid(scale*l),
                                 key = s + b, g = rsf * s / (sum_S s + 1e-15)          */
} muse_router_mode;

typedef enum muse_expert_weights {
  MUSE_EXPERTS_DENSE = 0,     /* W_gate / W_up / W_down are dense tensors of cfg->dtype   */
  MUSE_EXPERTS_NVFP4 = 1      /* each points to a muse_nvfp4_weight (below); bf16 only    */
} muse_expert_weights;

/* One NVFP4 expert weight tensor [E, out, in] (deep dive §7.3-7.4: 4-bit values, one FP8
 * E4M3 scale per 16 weights; 0.5625 bytes per weight): element (e, o, i) is
 *   e2m1(nibble) * e4m3(block_scales[e, o, i / 16]) * matrix_scale[e],
 * the nibble being the low half of codes[e, o, i / 2] for even i, the high half for odd i.
 * E2M1 and E4M3 are the OCP MX v1.0 FP4 and FP8 formats. The struct lives in host memory;
 * its pointers are device memory, 16-byte aligned. */
typedef struct muse_nvfp4_weight {
  const void* codes;          /* uint8 [E, out, in/2]                                 */
  const void* block_scales;   /* uint8 (E4M3) [E, out, in/16]                          */
  const float* matrix_scale;  /* float [E]                                            */
} muse_nvfp4_weight;

/* Format of the expert GEMMs' activation operands (with NVFP4 expert weights). */
typedef enum muse_act_format {
  MUSE_ACT_BF16 = 0,          /* W4A16: activations stay 16-bit: the expert GEMMs
                                 multiply f16 operands -- the decoded weights (exact) and
                                 the latent rows converted bf16 -> f16 (exact for
                                 magnitudes 2^-14 .. 65504; smaller ones round to f16's
                                 subnormal grid, larger ones saturate); h is kept as f16;
                                 FP32 accumulation                                       */
  MUSE_ACT_NVFP4 = 1          /* W4A4 (deep dive §7.4): the latent rows and the SwiGLU
                                 output are quantised per 16 values: scale E4M3(amax / 6),
                                 codes the E2M1 values nearest to value / scale (ties to
                                 even, no tensor scale); the tensor core reads both
                                 operands as 4-bit codes; requires NVFP4 experts and
                                 L, I multiples of 256                                   */
} muse_act_format;

typedef enum muse_norm_mode {
  MUSE_NORM_CENTRED = 0,      /* y / sqrt(mean(y^2)+eps) * (1+gamma)                   */
  MUSE_NORM_INPUT_SCALED = 1  /* u / sqrt(mean(u^2)+eps), u = y * (1+gamma)           */
} muse_norm_mode;

/* Block configuration. Zero-initialise, then set the sizes; muse_moe_config_init
 * fills the defaults (softmax router, centred per-expert norm, eps 1e-6). */
typedef struct muse_moe_config {
  int64_t T;                  /* tokens, >= 1                                         */
  int64_t D;                  /* hidden width; multiple of 128                        */
  int64_t L;                  /* latent width; multiple of 128                        */
  int64_t I;                  /* expert intermediate width; multiple of 128           */
  int64_t E;                  /* experts, 1..1024                                     */
  int32_t top_k;              /* 1..min(E, 32)                                        */
  int32_t dtype;              /* muse_dtype of x, weights, gamma, out                 */
  float eps;                  /* per-expert RMSNorm epsilon                           */
  int32_t router_mode;        /* muse_router_mode                                     */
  float router_logit_scale;   /* multiplies l before the sigmoid (sigmoid mode only)  */
  float routed_scaling;       /* multiplies g (sigmoid mode only)                     */
  const float* router_bias;   /* device [E] float32 selection-only bias, or NULL      */
  int32_t norm_mode;          /* muse_norm_mode                                       */
  int32_t gamma_shared;       /* 0: gamma is [E, L]; 1: one [L] gain for all experts  */
  const void* pre_norm_gain;  /* optional device [L] gain offsets of a centred RMSNorm
                                 on z before dispatch (pages' pre_expert_norm), or NULL */
  float pre_norm_eps;         /* epsilon of that norm (pages: 1e-5)                   */
  void* workspace;            /* device, 256-byte aligned, caller-owned               */
  size_t workspace_bytes;
  int32_t* topk_idx_out;      /* optional device [T, k] int32: selected experts       */
  float* topk_w_out;          /* optional device [T, k] float32: their weights        */
  void* const* stage_events;  /* optional: launch_count + 1 cudaEvent_t handles; event i
                                 is recorded on the stream before launch i and the last
                                 after the final launch (per-kernel device timing)     */
  int32_t expert_weights;     /* muse_expert_weights                                  */
  /* The feed-forward sublayer around the block (deep dive §2.1 steps 6-7, §5.2 residual
   * gate, §5.3 norm table); each step is off when its pointer is NULL. With all three,
   * x is the decoder layer's residual stream and out its next value:
   *   xn  = x / sqrt(mean(x^2) + ffn_pre_eps) * (1 + ffn_pre_gain)   (centred RMSNorm;
   *         the router and the pooler read xn instead of x)
   *   f   = the block applied to xn
   *   v   = f * (1 + ffn_post_gain);  fn = v / sqrt(mean(v^2) + ffn_post_eps)
   *   out = alpha * x + beta * fn, beta = sigmoid(g / T),
   *         alpha = sqrt(max(sigmoid(-g / T) * (1 + beta), residual_gate_eps)),
   *   with g = residual_gate, T = residual_gate_temperature; statistics and gate
   *   coefficients in FP32, out rounded once to cfg->dtype. Without the gate
   *   out = fn (or f); without the post norm the gate mixes x and f. */
  const void* ffn_pre_gain;   /* device [D] gain offsets in cfg->dtype, or NULL       */
  float ffn_pre_eps;          /* pages: 1e-5                                          */
  const void* ffn_post_gain;  /* device [D] gain offsets in cfg->dtype, or NULL       */
  float ffn_post_eps;         /* pages: 1e-8                                          */
  const float* residual_gate; /* device [D] float32 gate parameters g, or NULL        */
  float residual_gate_temperature; /* pages: 0.3                                      */
  float residual_gate_eps;    /* floor of alpha^2; pages: 1e-3                         */
  int32_t act_format;         /* muse_act_format of the expert GEMMs' activations      */
} muse_moe_config;

/* Byte offsets of the intermediates inside the workspace after a forward call, for
 * inspection by tests. Rows of the expert-ordered buffers are grouped by expert, each
 * expert's group padded to a multiple of 16 rows; inv maps assignment t*k+j to its row. */
typedef struct muse_moe_workspace_layout {
  size_t status;        /* uint32[2]: status code, detail                            */
  size_t expert_count;  /* int32 [E]     tokens routed to each expert                 */
  size_t expert_offset; /* int32 [E+1]   first padded row of each expert              */
  size_t logits;        /* float [T, E]  router logits                                */
  size_t topk_idx;      /* int32 [T, k]  selected experts, key descending            */
  size_t topk_w;        /* float [T, k]  routing weights                             */
  size_t inv;           /* int32 [T*k]   row of assignment t*k+j                      */
  size_t row_token;     /* int32 [R]     token of each row, -1 for padding            */
  size_t z;             /* act   [T, L]  pooler output                                */
  size_t zp;            /* act   [R, L]  z gathered into expert order                 */
  size_t h;             /* act   [R, I]  SiLU(gate) * up                              */
  size_t y;             /* act   [R, L]  expert outputs before the norm               */
  size_t ss;            /* float [R, L/32] partial sums of y^2 per 32 columns         */
  size_t c;             /* act   [T, L]  combined latent                              */
  size_t xn;            /* act   [T, D]  normalised input (with ffn_pre_gain; else 0)  */
  size_t ss_out;        /* float [T, D/32] partial sums of v^2 per 32 columns (with
                           ffn_post_gain; else 0)                                     */
  size_t zq_codes;      /* uint8 [R, L/2]  W4A4: quantised expert-ordered latent rows   */
  size_t zq_scales;     /* uint8 [R, L/16] their E4M3 block scales                     */
  size_t hq_codes;      /* uint8 [R, I/2]  W4A4: quantised SwiGLU output (else 0)      */
  size_t hq_scales;     /* uint8 [R, I/16]                                             */
  size_t total;         /* bytes required                                             */
  int64_t rows;         /* R: upper bound of padded rows                              */
} muse_moe_workspace_layout;

/* Fills defaults: router softmax, scale 1, rsf 1, norm centred per expert, eps 1e-6;
 * sublayer steps off, with the pages' epsilons (1e-5, 1e-8), temperature 0.3 and
 * alpha^2 floor 1e-3 ready for when their pointers are set. */
MUSE_API void muse_moe_config_init(muse_moe_config* cfg);

/* Workspace bytes for cfg's sizes (cfg->workspace is not read). */
MUSE_API muse_status muse_latent_moe_workspace_size(const muse_moe_config* cfg, size_t* bytes);

/* Offsets of each intermediate in the workspace for cfg's sizes. */
MUSE_API muse_status muse_latent_moe_workspace_layout(const muse_moe_config* cfg,
                                             muse_moe_workspace_layout* layout);

/* Forward pass of the block on device buffers (layouts above); enqueued on `stream`
 * (with cfg->expert_weights == MUSE_EXPERTS_NVFP4, W_gate / W_up / W_down are host
 * pointers to muse_nvfp4_weight descriptions of device tensors)
 * (a cudaStream_t, NULL = legacy default stream). Pointers must be device memory,
 * 16-byte aligned; `out` must not alias an input. Returns without synchronising. */
MUSE_API muse_status muse_latent_moe_forward(const muse_moe_config* cfg, const void* x,
                                    const void* W_router, const void* W_pool,
                                    const void* W_gate, const void* W_up, const void* W_down,
                                    const void* gamma, const void* W_unpool, void* out,
                                    void* stream);

/* A tensor as muse_latent_moe_forward_checked receives it: a device pointer with its element
 * type, rank, extents and strides (in elements, outermost first). The library reads
 * row-major contiguous tensors only: strides must be the contiguous ones
 * (stride[ndim-1] = 1, stride[i] = stride[i+1] * shape[i+1]). */
typedef enum muse_elem_type { MUSE_ELEM_F32 = 0, MUSE_ELEM_BF16 = 1, MUSE_ELEM_U8 = 2 } muse_elem_type;
typedef struct muse_tensor {
  const void* data;           /* device memory, 16-byte aligned                        */
  int32_t elem;               /* muse_elem_type (F32 / BF16 match muse_dtype)          */
  int32_t ndim;               /* 1..3                                                  */
  int64_t shape[3];
  int64_t stride[3];
} muse_tensor;

/* muse_latent_moe_forward with every tensor described by its shape (Muse Spark Open deep
 * dive, §4.3 implementation notes: the module's weights carry their shapes, e.g. the
 * experts' gate/up projection [256, 8192, 4096] in the released code's fused layout). Before
 * anything is launched, each tensor is checked against cfg:
 *   x [T, D], W_router [E, D], W_pool [L, D], W_gate [E, I, L], W_up [E, I, L],
 *   W_down [E, L, I], gamma [E, L] (or [L] with gamma_shared), W_unpool [D, L], out [T, D],
 * all of element type cfg->dtype, contiguous, 16-byte aligned; out may not overlap any
 * input. With cfg->expert_weights == MUSE_EXPERTS_NVFP4, W_gate / W_up / W_down each point
 * to THREE consecutive descriptors -- codes u8 [E, out, in/2], block scales u8 [E, out,
 * in/16], matrix scales f32 [E] -- and the forward receives them as muse_nvfp4_weight.
 * Any mismatch returns MUSE_ERR_INVALID_ARG with nothing launched; otherwise the result
 * is that of muse_latent_moe_forward on the same pointers. */
MUSE_API muse_status muse_latent_moe_forward_checked(const muse_moe_config* cfg, const muse_tensor* x,
                                                     const muse_tensor* W_router, const muse_tensor* W_pool,
                                                     const muse_tensor* W_gate, const muse_tensor* W_up,
                                                     const muse_tensor* W_down, const muse_tensor* gamma,
                                                     const muse_tensor* W_unpool, const muse_tensor* out,
                                                     void* stream);

/* Same, with x and out in HOST memory (pinned for asynchronous copies): copies x into
 * the device buffer x_dev, runs the forward into out_dev, copies out_dev back to
 * out_host, all on `stream`. x_dev / out_dev are caller-owned device buffers. The
 * caller synchronises the stream before reading out_host. */
MUSE_API muse_status muse_latent_moe_forward_host_io(const muse_moe_config* cfg, const void* x_host,
                                            void* x_dev, const void* W_router,
                                            const void* W_pool, const void* W_gate,
                                            const void* W_up, const void* W_down,
                                            const void* gamma, const void* W_unpool,
                                            void* out_dev, void* out_host, void* stream);

/* A sequence of batches through the forward with host buffers, the copies overlapped with
 * the compute. Batch b (of n_batches, each cfg->T tokens): x_host[b] (pinned host memory)
 * is copied into x_dev[b % 2] on h2d_stream, its forward runs on `stream` into
 * out_dev[b % 2], and out_dev[b % 2] is copied into out_host[b] on d2h_stream, so that while
 * batch b computes, batch b + 1 uploads and batch b - 1 downloads. Events (created and
 * released inside) order every reuse of the two device buffers; the batches' forwards share
 * cfg->workspace, serialised on `stream`. x_host / out_host: host arrays of n_batches
 * pointers; x_dev / out_dev: host arrays of 2 device pointers (16-byte aligned); the three
 * streams must differ. Returns after enqueueing; synchronise d2h_stream before reading the
 * last out_host. */
MUSE_API muse_status muse_latent_moe_forward_host_batches(const muse_moe_config* cfg, int64_t n_batches,
                                                 const void* const* x_host, void* const* out_host,
                                                 void* const* x_dev, void* const* out_dev,
                                                 const void* W_router, const void* W_pool,
                                                 const void* W_gate, const void* W_up,
                                                 const void* W_down, const void* gamma,
                                                 const void* W_unpool, void* stream,
                                                 void* h2d_stream, void* d2h_stream);

/* Synchronises `stream` and returns the status word the last forward on this
 * workspace recorded on the device (MUSE_OK, MUSE_ERR_TIMEOUT or MUSE_ERR_DEVICE);
 * *detail (may be NULL) receives the kernel-specific detail code. With cfg->workspace ==
 * NULL it reads the word of the built-in scratch array that
 * muse_latent_moe_forward_static_scratch uses on the current device. */
MUSE_API muse_status muse_latent_moe_last_device_status(const muse_moe_config* cfg, void* stream,
                                               uint32_t* detail);

/* Forward pass for callers that cannot allocate device memory at all: a plug-in whose
 * host application owns every allocation, code that runs where cudaMalloc is not
 * permitted or would stall the device, or a service with a fixed memory budget. It is
 * muse_latent_moe_forward with the workspace taken from a scratch array compiled into
 * this library (a file-scope __device__ array of MUSE_STATIC_SCRATCH_BYTES, held by
 * every GPU that loads the library until the process exits) instead of from
 * cfg->workspace, which is ignored. The pages describe nothing like it: it exists
 * for callers of this library only.
 *   - Sizes whose workspace (muse_latent_moe_workspace_size) exceeds
 *     MUSE_STATIC_SCRATCH_BYTES are rejected with MUSE_ERR_WORKSPACE before any launch.
 *   - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *   - Each call made outside stream capture looks up the array's device address on the
 *     current device (so an address from before a cudaDeviceReset, which frees the array,
 *     is never reused); a call made during capture uses the address of the last uncaptured
 *     call on that device, so make the first call on each device before any capture.
 *   - All calls share the one array and it keeps the last call's contents (each call
 *     clears what must start at zero). Calls whose work overlaps on the GPU -- on two
 *     streams, or on one device from two threads without ordering -- race on it: order
 *     them on one stream or serialise them.
 *   - The device-side status word (bounded-wait timeouts, index checks) lives in that
 *     shared array: muse_latent_moe_last_device_status with cfg->workspace == NULL reads
 *     it (the last call's word on the current device). */
#define MUSE_STATIC_SCRATCH_BYTES (16u << 20)
MUSE_API muse_status muse_latent_moe_forward_static_scratch(const muse_moe_config* cfg, const void* x,
                                                            const void* W_router, const void* W_pool,
                                                            const void* W_gate, const void* W_up,
                                                            const void* W_down, const void* gamma,
                                                            const void* W_unpool, void* out, void* stream);

/* Self-test of the device-side bounded waits every kernel of this library uses: launches
 * one small kernel whose single waiting thread waits on an mbarrier that nothing ever
 * completes, with a limit of limit_ns nanoseconds (1 .. 10^10), on `stream`. The wait
 * gives up, the kernel ends normally and status_dev (caller-owned device uint32[2],
 * zero it first) receives {MUSE_ERR_TIMEOUT, detail}; the context stays usable. Returns
 * MUSE_OK once launched, MUSE_ERR_INVALID_ARG for a null pointer or a limit out of range. */
MUSE_API muse_status muse_selftest_bounded_wait(uint64_t limit_ns, uint32_t* status_dev, void* stream);

/* The W4A4 activation quantiser on its own (the step the forward applies to the latent rows
 * and to h, muse_act_format): rows x K bf16 values (device, row-major, 16-byte aligned, K a
 * multiple of 16) -> codes uint8 [rows, K/2] (two E2M1 codes per byte, low nibble = even
 * element; 16-byte aligned) and scales uint8 [rows, K/16] (E4M3), per block of 16 values
 * scale = E4M3(amax / 6) (amax / 6 in float32), code = the E2M1 value nearest to the exact
 * quotient value / scale, ties to even. Enqueued on `stream`; INVALID_ARG for null /
 * misaligned pointers or sizes. */
MUSE_API muse_status muse_quantize_nvfp4_rows(const void* src, int64_t rows, int64_t K, void* codes,
                                              void* scales, void* stream);

/* ---------------------------------------------------------------------------------
 * Expert parallelism (EP) over G ranks (Muse Spark Open deep dive, §4.3: the two expert
 * tensors split along the expert dimension, the latent rows moved to the experts' ranks
 * and back, the norm weights replicated; on each rank the local experts see every row
 * with top-1 routing and unit weight, and the routing weights are applied after the
 * rows return, so the per-expert norm still precedes the weighting). Rank r owns the
 * experts [r * E / G, (r + 1) * E / G); E must be a multiple of G. One forward is three
 * calls around two exchanges that the caller performs (an all-to-all, e.g. NCCL):
 *
 *   1. muse_ep_dispatch on every rank, for its own cfg->T tokens: routing, pooler, and
 *      the send buffer of its T * k (token, expert) rows, grouped by destination rank
 *      (rank_counts[r] rows for rank r, in rank order).
 *   2. exchange: rank r receives the rows every rank sent to it, concatenated in source
 *      rank order, with their local expert indices.
 *   3. muse_ep_experts on every rank over the rows it received: gate/up + SwiGLU, down
 *      projection and the partial sums of squares, returned in the order received.
 *   4. exchange back: the inverse of step 2, so that each rank's results land in the
 *      rows of its own send buffer.
 *   5. muse_ep_combine on every rank: per-expert norm, weighted combine, unpooler (and
 *      the optional feed-forward sublayer steps), into out.
 *
 * cfg is the whole block's configuration (E = all experts) on every call. Calls 1 and 5
 * of one forward use the same cfg->workspace (the token rank's workspace, role
 * MUSE_EP_HOME); call 3 uses an expert workspace (role MUSE_EP_EXPERTS) in
 * cfg->workspace. The result equals muse_latent_moe_forward on the same tokens bit for
 * bit: the expert GEMMs see other row counts and may tile them differently, but every
 * output element is accumulated over K in the same order whatever the tiling. Calls are
 * enqueued on `stream` without synchronising; the host reads rank_counts (a device
 * array) to size the exchange. stage_events is ignored. Status word: calls 1 and 3 reset
 * their workspace's word, call 5 adds to the word of call 1.
 * --------------------------------------------------------------------------------- */
typedef enum muse_ep_role {
  MUSE_EP_HOME = 1,    /* routing, pooler, send plan, combine, unpooler of cfg->T tokens */
  MUSE_EP_EXPERTS = 2  /* grouped GEMMs over up to `rows` received rows                  */
} muse_ep_role;

/* Offsets of the buffers of a role's workspace (total = bytes to allocate, 256-byte
 * aligned base). For MUSE_EP_EXPERTS, rows = the most rows one call will receive (at
 * most the sum over ranks of T_rank * min(k, E / G)); buffers a role does not use have
 * offset 0 and no bytes. INVALID_ARG if E is not a multiple of ep_size or the role is
 * unknown. */
MUSE_API muse_status muse_ep_workspace_layout(const muse_moe_config* cfg, int32_t ep_size, int32_t role,
                                              int64_t rows, muse_moe_workspace_layout* layout);

/* EP step 1 on the tokens' rank. x [T, D] -> send_z [T * k, L] (dtype cfg->dtype): row
 * p is the latent z of the token of the p-th (token, expert) pair in destination order
 * -- experts ascending, then tokens ascending, then slot -- so the rows for rank r form
 * the contiguous block [sum_{q<r} rank_counts[q], + rank_counts[r]); send_expert
 * int32 [T * k]: each row's expert index on its owning rank (0 .. E/G - 1);
 * rank_counts int32 [ep_size]. All device memory (send_z 16-byte aligned). */
MUSE_API muse_status muse_ep_dispatch(const muse_moe_config* cfg, int32_t ep_size, const void* x,
                                      const void* W_router, const void* W_pool, void* send_z,
                                      int32_t* send_expert, int32_t* rank_counts, void* stream);

/* EP step 3 on an expert rank. recv_z [rows, L] and recv_expert int32 [rows] (local
 * expert indices) -> ret_y [rows, L] (dtype cfg->dtype), the expert outputs before the
 * norm, and ret_ss float [rows, L/32], their partial sums of squares per 32 columns,
 * both in the order received. W_gate / W_up / W_down: this rank's E/G experts, laid out
 * as in muse_latent_moe_forward with E/G in place of E (NVFP4: descriptors of them);
 * gamma: this rank's slice [E/G, L] (or the shared [L]), read only in
 * MUSE_NORM_INPUT_SCALED mode. rows = 0 launches nothing. A local index outside
 * 0 .. E/G - 1 is recorded as MUSE_ERR_DEVICE in the status word and its row returns
 * zeros. */
MUSE_API muse_status muse_ep_experts(const muse_moe_config* cfg, int32_t ep_size, int64_t rows,
                                     const void* recv_z, const int32_t* recv_expert, const void* W_gate,
                                     const void* W_up, const void* W_down, const void* gamma, void* ret_y,
                                     float* ret_ss, void* stream);

/* EP step 5 on the tokens' rank, after the exchange back: back_y [T * k, L] and back_ss
 * float [T * k, L/32] in the rows of this rank's send buffer -> out [T, D]. gamma: all
 * E experts' gains (replicated), x: this rank's input (read by the residual gate). */
MUSE_API muse_status muse_ep_combine(const muse_moe_config* cfg, int32_t ep_size, const void* x,
                                     const void* back_y, const float* back_ss, const void* gamma,
                                     const void* W_unpool, void* out, void* stream);

/* Static string for a status code. */
MUSE_API const char* muse_status_string(muse_status s);

/* The CUDA runtime's description (a static string) of the last CUDA error behind a
 * MUSE_ERR_CUDA that a call on the calling host thread returned -- e.g. a launch the device
 * cannot schedule, or an error left by an earlier kernel. "no error" when no CUDA call has
 * failed on this thread (a tensor-map encoding refused by the driver also returns
 * MUSE_ERR_CUDA without a CUDA error). */
MUSE_API const char* muse_last_cuda_error(void);

/* Number of stages one forward call runs for cfg -- the positions of stage_events -- and
 * the name of stage i (a static string; NULL past the last). In order: [ffn_pre_norm],
 * router, topk, expert_hist, tiles, assign_rows, pooler, [pre_expert_norm], gather (with
 * W4A4 activations: quant_z, gather_codes), gate_up_swiglu, [quant_h (W4A4)], down_sumsq,
 * norm_combine, unpooler, [ffn_post_norm_gate]. Each stage is
 * one kernel, except that a dense GEMM (router, pooler, unpooler) whose tiles would fill
 * less than half the SMs splits K and adds a partial-sum kernel inside its stage
 * (decode-sized token counts). stage_events must hold launch_count + 1 events. -1 / NULL
 * for an invalid cfg. */
MUSE_API const char* muse_latent_moe_stage_name(const muse_moe_config* cfg, int32_t i);
MUSE_API int32_t muse_latent_moe_launch_count(const muse_moe_config* cfg);

#ifdef __cplusplus
}
#endif
#endif /* MUSE_MOE_H_ */
