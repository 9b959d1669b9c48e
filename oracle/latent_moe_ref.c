/*
 * latent_moe_ref.c -- plain FP64 CPU reference of the latent-MoE block forward pass.
 * TEST INFRASTRUCTURE ONLY: the tests, smoke() and the benchmark's CPU baseline may call it;
 * the CUDA library never does, and the two share no code.
 *
 * One token at a time, the steps in the order of the block's definition ("Muse Spark Open
 * deep dive", §4.3 block equation; §4.2 routing equation), loops only, double throughout:
 *
 *   l_e   = sum_d W_router[e, d] x[d]                                   router logits
 *   key_e = l_e + b_e                     (softmax mode)
 *         = sigmoid(scale * l_e) + b_e    (sigmoid mode, the released router)
 *   S     = the k experts with the largest key, key descending, ties to the lower index
 *   g_j   = exp(l_Sj - m) / sum_j' exp(l_Sj' - m), m = max_j l_Sj      (softmax mode)
 *         = rsf * s_Sj / (sum_j' s_Sj' + 1e-15), s = sigmoid(scale * l) (sigmoid mode)
 *   z     = W_pool x;  optionally z <- z / sqrt(mean(z^2) + eps_pre) * (1 + w_pre)
 *   y_j   = W_down[e] (silu(W_gate[e] z) * (W_up[e] z)), e = S_j, silu(a) = a / (1 + e^-a)
 *   n_j   = y_j / sqrt(mean(y_j^2) + eps) * (1 + gamma_e)              (centred norm)
 *         = v / sqrt(mean(v^2) + eps), v = y_j * (1 + gamma_e)          (input-scaled norm)
 *   c     = sum_j g_j n_j   (j in routing order)
 *   out   = W_unpool c
 *
 * The bias only selects (deep dive §4.2: weights come from the unbiased scores). All
 * matrices are row-major [out, in]; W_gate / W_up are [E, I, L], W_down [E, L, I]; gamma is
 * [E, L], or [L] when gamma_shared.
 *
 * NVFP4 expert weights (deep dive §7.3 bytes bullet, §7.4 NVFP4 paragraph: 4-bit values,
 * one E4M3 scale per 16 consecutive weights of a row, one FP32 scale per matrix) are
 * decoded element by element from the bit fields of the OCP MX v1.0 formats:
 *   E2M1 code s.ee.m:  (-1)^s * (e == 0 ? m / 2 : 2^(e-1) * (1 + m / 2))
 *   E4M3 byte s.eeee.mmm: (-1)^s * (e == 0 ? m / 8 * 2^-6 : 2^(e-7) * (1 + m / 8)),
 *                         S.1111.111 is NaN
 *   w[o, i] = e2m1(nibble i of row o) * e4m3(scale byte i / 16 of row o) * matrix_scale,
 * the nibble of an even i being the low half of byte i / 2.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int T, D, L, I, E, k;
  double eps;
  int router_mode;         /* 0 softmax, 1 sigmoid */
  double logit_scale;      /* sigmoid mode */
  double routed_scaling;   /* sigmoid mode */
  const double* bias;      /* [E] or NULL */
  int norm_mode;           /* 0 centred, 1 input-scaled */
  int gamma_shared;        /* gamma is [L] */
  const double* pre_gain;  /* [L] gain offsets of a centred norm on z, or NULL */
  double pre_eps;
} ref_cfg;

static double sigmoid(double a) { return 1.0 / (1.0 + exp(-a)); }

/* y[r] = sum_c M[r, c] v[c] for an R x C row-major matrix */
static void matvec(const double* M, const double* v, int R, int C, double* y) {
  for (int r = 0; r < R; ++r) {
    double s = 0.0;
    for (int c = 0; c < C; ++c) s += M[(size_t)r * C + c] * v[c];
    y[r] = s;
  }
}

static double mean_square(const double* v, int n) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += v[i] * v[i];
  return s / n;
}

/* ---- NVFP4 expert weights ---------------------------------------------------------- */
typedef struct {
  const unsigned char* codes;   /* [E, out, in/2], low nibble = even element */
  const unsigned char* scales;  /* [E, out, in/16] E4M3 bytes                */
  const float* matrix_scale;    /* [E]                                       */
} ref_nvfp4;

double ref_e2m1_value(unsigned code) {
  const unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
  const double mag = e == 0 ? m * 0.5 : ldexp(1.0 + m * 0.5, (int)e - 1);
  return s ? -mag : mag;
}

double ref_e4m3_value(unsigned byte) {
  const unsigned s = (byte >> 7) & 1u, e = (byte >> 3) & 15u, m = byte & 7u;
  if (e == 15u && m == 7u) return NAN;
  const double mag = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, (int)e - 7);
  return s ? -mag : mag;
}

/* y[r] = sum_c W_e[r, c] v[c] for expert e's R x C NVFP4 matrix, decoded per element */
static void matvec_nvfp4(const ref_nvfp4* w, size_t e, int R, int C, const double* v, double* y) {
  const double ms = (double)w->matrix_scale[e];
  for (int r = 0; r < R; ++r) {
    const unsigned char* crow = w->codes + (e * (size_t)R + r) * (size_t)(C / 2);
    const unsigned char* srow = w->scales + (e * (size_t)R + r) * (size_t)(C / 16);
    double s = 0.0;
    for (int c = 0; c < C; ++c) {
      const unsigned byte = crow[c / 2];
      const unsigned code = (c % 2 == 0) ? (byte & 15u) : (byte >> 4);
      s += ref_e2m1_value(code) * ref_e4m3_value(srow[c / 16]) * ms * v[c];
    }
    y[r] = s;
  }
}

/* The expert weights of one forward: dense double matrices, or NVFP4 descriptions. */
typedef struct {
  const double *gate, *up, *down;
  const ref_nvfp4 *qgate, *qup, *qdown;
} ref_experts;

static void expert_matvec(const ref_experts* x, int which, size_t e, int R, int C, const double* v, double* y) {
  const double* dense = which == 0 ? x->gate : which == 1 ? x->up : x->down;
  const ref_nvfp4* q = which == 0 ? x->qgate : which == 1 ? x->qup : x->qdown;
  if (q != NULL)
    matvec_nvfp4(q, e, R, C, v, y);
  else
    matvec(dense + e * (size_t)R * C, v, R, C, y);
}

static int forward(const ref_cfg* c, const double* x, const double* W_router, const double* W_pool,
                   const ref_experts* ex, const double* gamma, const double* W_unpool, double* out, int* idx_out,
                   double* g_out);

/* Returns 0, or -1 for an invalid configuration or a failed allocation. idx_out [T, k] and
 * g_out [T, k] may be NULL. */
int ref_latent_moe_forward(const ref_cfg* c, const double* x, const double* W_router, const double* W_pool,
                           const double* W_gate, const double* W_up, const double* W_down, const double* gamma,
                           const double* W_unpool, double* out, int* idx_out, double* g_out) {
  const ref_experts ex = {W_gate, W_up, W_down, NULL, NULL, NULL};
  return forward(c, x, W_router, W_pool, &ex, gamma, W_unpool, out, idx_out, g_out);
}

/* The same block with NVFP4 expert weights (in must be a multiple of 16 for every matrix:
 * L for gate / up, I for down). */
int ref_latent_moe_forward_nvfp4(const ref_cfg* c, const double* x, const double* W_router, const double* W_pool,
                                 const ref_nvfp4* W_gate, const ref_nvfp4* W_up, const ref_nvfp4* W_down,
                                 const double* gamma, const double* W_unpool, double* out, int* idx_out,
                                 double* g_out) {
  if (c == NULL || W_gate == NULL || W_up == NULL || W_down == NULL || c->L % 16 || c->I % 16) return -1;
  const ref_experts ex = {NULL, NULL, NULL, W_gate, W_up, W_down};
  return forward(c, x, W_router, W_pool, &ex, gamma, W_unpool, out, idx_out, g_out);
}

static int forward(const ref_cfg* c, const double* x, const double* W_router, const double* W_pool,
                   const ref_experts* ex, const double* gamma, const double* W_unpool, double* out, int* idx_out,
                   double* g_out) {
  if (c == NULL || c->T < 0 || c->D < 1 || c->L < 1 || c->I < 1 || c->E < 1 || c->k < 1 || c->k > c->E) return -1;
  const int D = c->D, L = c->L, I = c->I, E = c->E, k = c->k;
  double* l = malloc(sizeof(double) * E);
  double* key = malloc(sizeof(double) * E);
  char* taken = malloc((size_t)E);
  int* sel = malloc(sizeof(int) * k);
  double* g = malloc(sizeof(double) * k);
  double* z = malloc(sizeof(double) * L);
  double* a = malloc(sizeof(double) * I);
  double* u = malloc(sizeof(double) * I);
  double* y = malloc(sizeof(double) * L);
  double* cc = malloc(sizeof(double) * L);
  int rc = 0;
  if (!l || !key || !taken || !sel || !g || !z || !a || !u || !y || !cc) {
    rc = -1;
    goto done;
  }
  for (int t = 0; t < c->T; ++t) {
    const double* xt = x + (size_t)t * D;
    /* router logits and selection keys */
    matvec(W_router, xt, E, D, l);
    for (int e = 0; e < E; ++e) {
      const double score = c->router_mode == 1 ? sigmoid(c->logit_scale * l[e]) : l[e];
      key[e] = score + (c->bias ? c->bias[e] : 0.0);
    }
    /* top-k: k passes, each taking the largest remaining key; scanning upwards with a
     * strict comparison keeps the lower index on ties */
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || key[e] > key[best])) best = e;
      taken[best] = 1;
      sel[j] = best;
    }
    /* routing weights from the unbiased scores of the selected experts */
    if (c->router_mode == 1) {
      double sum = 0.0;
      for (int j = 0; j < k; ++j) sum += sigmoid(c->logit_scale * l[sel[j]]);
      for (int j = 0; j < k; ++j) g[j] = c->routed_scaling * sigmoid(c->logit_scale * l[sel[j]]) / (sum + 1e-15);
    } else {
      double m = l[sel[0]];
      for (int j = 1; j < k; ++j) m = l[sel[j]] > m ? l[sel[j]] : m;
      double sum = 0.0;
      for (int j = 0; j < k; ++j) sum += exp(l[sel[j]] - m);
      for (int j = 0; j < k; ++j) g[j] = exp(l[sel[j]] - m) / sum;
    }
    /* pooler (and the optional centred norm on the latent) */
    matvec(W_pool, xt, L, D, z);
    if (c->pre_gain) {
      const double r = sqrt(mean_square(z, L) + c->pre_eps);
      for (int i = 0; i < L; ++i) z[i] = z[i] / r * (1.0 + c->pre_gain[i]);
    }
    /* experts, each output normalised with its expert's gain, then the weighted sum */
    for (int i = 0; i < L; ++i) cc[i] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int e = sel[j];
      expert_matvec(ex, 0, (size_t)e, I, L, z, a);
      expert_matvec(ex, 1, (size_t)e, I, L, z, u);
      for (int i = 0; i < I; ++i) a[i] = a[i] * sigmoid(a[i]) * u[i];
      expert_matvec(ex, 2, (size_t)e, L, I, a, y);
      const double* gm = c->gamma_shared ? gamma : gamma + (size_t)e * L;
      if (c->norm_mode == 1) {
        for (int i = 0; i < L; ++i) y[i] *= 1.0 + gm[i];
        const double r = sqrt(mean_square(y, L) + c->eps);
        for (int i = 0; i < L; ++i) cc[i] += g[j] * (y[i] / r);
      } else {
        const double r = sqrt(mean_square(y, L) + c->eps);
        for (int i = 0; i < L; ++i) cc[i] += g[j] * (y[i] / r * (1.0 + gm[i]));
      }
    }
    /* unpooler */
    matvec(W_unpool, cc, D, L, out + (size_t)t * D);
    for (int j = 0; j < k; ++j) {
      if (idx_out) idx_out[(size_t)t * k + j] = sel[j];
      if (g_out) g_out[(size_t)t * k + j] = g[j];
    }
  }
done:
  free(l);
  free(key);
  free(taken);
  free(sel);
  free(g);
  free(z);
  free(a);
  free(u);
  free(y);
  free(cc);
  return rc;
}
