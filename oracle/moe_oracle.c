/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of the top-k mixture-of-experts
 * FFN layer of DiffusionGemma 26B-A4B.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table
 * or helper with the CUDA path, and the CUDA path never calls it.
 *
 * Sources (page title, section):
 *  [QT]  Quant-Tuner pull request "Add DiffusionGemma (Gemma-4 MoE
 *        block-diffusion) support": Summary (128 experts, 8 active);
 *        "Answers to the motivating questions" (the router reads the raw
 *        residual through its own internal norm; the fused 3-D
 *        experts.gate_up_proj; Gemma's (1+gamma) RMSNorm convention).
 *  [AR]  auto-round pull request "Add quantization support for DiffusionGemma":
 *        Description (fused gate_up_proj / down_proj), transformers backend
 *        test log (act_fn GELUTanh; gate_proj 2816->704, up_proj 2816->704,
 *        down_proj 704->2816; quantization_config bits 4, group_size 128,
 *        sym True, data_type int).
 *  [RF]  Hugging Face card "kingjones777/DiffusionGemma-26B-A4B-it-ROCmFP4-GGUF":
 *        header (128 experts / top-8; FP4 / FP8 builds of the weights) and its
 *        finding that at a 256-token canvas the 8-bit build steps faster.
 *  [OCP] OCP 8-bit Floating Point Specification (OFP8), E4M3 encoding: the
 *        8-bit float format of the fp8 weight storage (the pages name FP8
 *        builds but do not define the encoding).
 *  [MX]  OCP Microscaling Formats (MX) Specification, FP4 E2M1 element
 *        encoding: the 4-bit float of the fp4 weight storage (the pages name
 *        FP4 builds but do not define them).
 *
 * Where the pages are silent this file follows the readings adopted by the
 * library (they are listed once, here):
 *  - routing: p = softmax over all E logits; S = the k largest logits, the
 *    lower expert index winning ties, ordered by (logit desc, index asc);
 *    w_j = p[S_j] / sum_{j'} p[S_j'];  gap = z_(k) - z_(k+1);
 *  - gated form: out = down(gelu_tanh(gate(x)) * up(x)), gate = rows [0,f)
 *    of the fused gate_up weight, up = rows [f,2f);
 *  - the experts read x as given, or, with an expert gamma, the expert-side
 *    (1+gamma2) RMSNorm of x ([QT] Answers: pre_feedforward_layernorm_2 is
 *    the only consumer of the fused gate_up; the router does not see it);
 *  - RMSNorm: u_i = x_i / sqrt(mean_i x_i^2 + eps) * (1 + gamma_i);
 *  - router bias (optional) is added to the logits before the softmax;
 *  - int4: element i of a row sits in byte i/2, low nibble for even i, 4-bit
 *    two's complement; w = code * scale[i / 128] with fp16 scales, exact here;
 *  - fp8: element i of a row is byte i, an E4M3 value [OCP]; w = value *
 *    scale[row] with one fp32 scale per weight row (output channel), exact;
 *  - fp4: element i of a row is the nibble of byte i/2 (low nibble for even
 *    i), an E2M1 value [MX]; w = value * e4m3(block[i/16][row]) * s[row]:
 *    an E4M3 scale per 16 consecutive elements and an fp32 scale per row.
 *    The scales of expert e form one record {fp32 s[R]; uint8 block[NB][R]}
 *    (NB = ceil(C/16); each block's rows contiguous), records back to back;
 *  - out = residual + sum_j w_j y_j, summed in j order (residual optional).
 *
 * Everything is computed in double precision from the exact bf16 / fp16 /
 * int4 / fp8 values the GPU receives; nothing is rounded in between.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_W_BF16 0
#define ORACLE_W_INT4 1
#define ORACLE_W_FP8 2
#define ORACLE_W_FP4 3
#define ORACLE_GROUP 128

/* ---- scalar decoders (IEEE definitions) -------------------------------- */

/* bfloat16: the upper 16 bits of an IEEE binary32. */
static double bf16_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 mantissa bits. */
static double fp16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int ex = (h >> 10) & 0x1f;
  int man = h & 0x3ff;
  double v;
  if (ex == 0)
    v = ldexp((double)man, -24); /* subnormal: man * 2^-14 * 2^-10 */
  else if (ex == 31)
    v = man ? NAN : INFINITY;
  else
    v = ldexp(1.0 + man / 1024.0, ex - 15);
  return sign ? -v : v;
}

/* OFP8 E4M3 [OCP]: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
 * exponent 0 is subnormal (m/8 * 2^-6); exponent 15 with mantissa 7 is NaN
 * (the format has no infinities, so 15 with mantissa 0..6 is an ordinary
 * binade: the largest value is 1.75 * 2^8 = 448). */
static double e4m3_to_double(uint8_t b) {
  int sign = (b >> 7) & 1;
  int ex = (b >> 3) & 0xf;
  int man = b & 0x7;
  double v;
  if (ex == 0xf && man == 0x7)
    v = NAN;
  else if (ex == 0)
    v = ldexp((double)man, -9); /* man/8 * 2^-6 */
  else
    v = ldexp(1.0 + man / 8.0, ex - 7);
  return sign ? -v : v;
}

/* MX FP4 E2M1 [MX]: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit;
 * exponent 0 is subnormal (m * 0.5); no infinities or NaN.  The magnitudes
 * are 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static double e2m1_to_double(int nib) {
  int sign = (nib >> 3) & 1;
  int ex = (nib >> 1) & 0x3;
  int man = nib & 0x1;
  double v = (ex == 0) ? 0.5 * man : ldexp(1.0 + 0.5 * man, ex - 1);
  return sign ? -v : v;
}

/* 4-bit two's complement code of element i of a packed row. */
static int int4_code(const uint8_t* row, int i) {
  int byte = row[i / 2];
  int nib = (i % 2 == 0) ? (byte & 0xf) : ((byte >> 4) & 0xf);
  return nib >= 8 ? nib - 16 : nib;
}

/* One expert-weight element W[e][r][i] of a [E, R, C] weight in any of the
 * storage formats.  int4: code * fp16 scale of group i/128 ([AR] w4g128);
 * fp8: E4M3 value * fp32 scale of the row. */
static double weight_elem(int wdtype, const void* w, const void* scales, int R, int C, int e,
                          int r, int i) {
  size_t row = (size_t)e * R + r;
  if (wdtype == ORACLE_W_BF16) {
    const uint16_t* wb = (const uint16_t*)w;
    return bf16_to_double(wb[row * C + i]);
  }
  if (wdtype == ORACLE_W_FP8) {
    const uint8_t* wp = (const uint8_t*)w + row * (size_t)C;
    return e4m3_to_double(wp[i]) * (double)((const float*)scales)[row];
  }
  if (wdtype == ORACLE_W_FP4) {
    const uint8_t* wp = (const uint8_t*)w + row * (size_t)(C / 2);
    int byte = wp[i / 2];
    int nib = (i % 2 == 0) ? (byte & 0xf) : ((byte >> 4) & 0xf);
    const size_t NB = (size_t)(C + 15) / 16;
    const uint8_t* rec = (const uint8_t*)scales + (size_t)e * ((size_t)R * 4 + NB * R);
    float srow;
    memcpy(&srow, rec + (size_t)r * 4, sizeof srow);
    const uint8_t blk = rec[(size_t)R * 4 + (size_t)(i / 16) * R + r];
    return e2m1_to_double(nib) * e4m3_to_double(blk) * (double)srow;
  }
  const uint8_t* wp = (const uint8_t*)w + row * (size_t)(C / 2);
  int ng = (C + ORACLE_GROUP - 1) / ORACLE_GROUP;
  double s = fp16_to_double(((const uint16_t*)scales)[row * ng + i / ORACLE_GROUP]);
  return (double)int4_code(wp, i) * s;
}

/* ---- the layer, step by step -------------------------------------------- */

/* GELU, tanh form ([AR] act_fn GELUTanh):
 * 0.5 a (1 + tanh( sqrt(2/pi) (a + 0.044715 a^3) )). */
double oracle_gelu_tanh(double a) {
  const double c = sqrt(2.0 / M_PI);
  return 0.5 * a * (1.0 + tanh(c * (a + 0.044715 * a * a * a)));
}

/* The router's own norm on the raw residual, Gemma (1+gamma) form ([QT]). */
void oracle_rmsnorm_plus_one(int d, const double* x, const float* gamma, double eps,
                             double* u) {
  double ss = 0.0;
  for (int i = 0; i < d; i++) ss += x[i] * x[i];
  double r = sqrt(ss / d + eps);
  for (int i = 0; i < d; i++) u[i] = x[i] / r * (1.0 + (double)gamma[i]);
}

/* Router logits z_e = sum_i W_r[e][i] u_i (+ b_e) ([QT]; fp32 weights). */
void oracle_router_logits(int E, int d, const double* u, const float* router_w,
                          const float* bias, double* z) {
  for (int e = 0; e < E; e++) {
    double acc = 0.0;
    for (int i = 0; i < d; i++) acc += (double)router_w[(size_t)e * d + i] * u[i];
    z[e] = acc + (bias ? (double)bias[e] : 0.0);
  }
}

/* Top-k of E ([QT] Summary, [RF]: 8 of 128): k rounds, each taking the
 * largest remaining logit; a strict '>' while scanning e upward keeps the
 * lower index on ties.  gap = z_(k) - z_(k+1) (+inf when k == E). */
void oracle_select_topk(int E, int k, const double* z, int32_t* idx, double* gap) {
  char* taken = (char*)calloc((size_t)E, 1);
  for (int j = 0; j < k; j++) {
    int best = -1;
    for (int e = 0; e < E; e++)
      if (!taken[e] && (best < 0 || z[e] > z[best])) best = e;
    idx[j] = best;
    taken[best] = 1;
  }
  if (gap) {
    int next = -1;
    for (int e = 0; e < E; e++)
      if (!taken[e] && (next < 0 || z[e] > z[next])) next = e;
    *gap = (next < 0) ? INFINITY : z[idx[k - 1]] - z[next];
  }
  free(taken);
}

/* Routing weights: softmax over all E logits, restricted to S and
 * renormalised so that the k weights sum to one. */
void oracle_route_weights(int E, int k, const double* z, const int32_t* idx, double* w) {
  double m = z[0];
  for (int e = 1; e < E; e++)
    if (z[e] > m) m = z[e];
  double den = 0.0;
  for (int e = 0; e < E; e++) den += exp(z[e] - m);
  double sel = 0.0;
  for (int j = 0; j < k; j++) {
    w[j] = exp(z[idx[j]] - m) / den; /* p[S_j] */
    sel += w[j];
  }
  for (int j = 0; j < k; j++) w[j] /= sel;
}

/* One expert e on one token ([QT] fused 3-D gate_up; [AR] gate/up 2816->704,
 * down 704->2816, GELUTanh):
 *   g_r = sum_i Wgu[e][r][i] x_i,  v_r = sum_i Wgu[e][f+r][i] x_i   (r < f)
 *   h_r = gelu_tanh(g_r) * v_r
 *   y_m = sum_r Wd[e][m][r] h_r                                    (m < d) */
void oracle_expert_ffn(int d, int f, int wdtype, const void* w_gu, const void* w_d,
                       const void* s_gu, const void* s_d, int e, const double* x,
                       double* y, double* h_out) {
  double* h = (double*)malloc(sizeof(double) * (size_t)f);
  for (int r = 0; r < f; r++) {
    double g = 0.0, v = 0.0;
    for (int i = 0; i < d; i++) {
      g += weight_elem(wdtype, w_gu, s_gu, 2 * f, d, e, r, i) * x[i];
      v += weight_elem(wdtype, w_gu, s_gu, 2 * f, d, e, f + r, i) * x[i];
    }
    h[r] = oracle_gelu_tanh(g) * v;
  }
  for (int m = 0; m < d; m++) {
    double acc = 0.0;
    for (int r = 0; r < f; r++) acc += weight_elem(wdtype, w_d, s_d, d, f, e, m, r) * h[r];
    y[m] = acc;
  }
  if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)f);
  free(h);
}

/* Dequantised (or widened) row r of expert e of a [E, R, C] weight. */
void oracle_weight_row(int wdtype, const void* w, const void* scales, int R, int C, int e,
                       int r, double* out) {
  for (int i = 0; i < C; i++) out[i] = weight_elem(wdtype, w, scales, R, C, e, r, i);
}

/* Routing of one token: norm -> logits -> top-k -> weights. */
static void route_token(int E, int k, int d, const uint16_t* x_row, const float* router_w,
                        const float* gamma, const float* bias, double eps,
                        const int32_t* forced_idx, double* xs, double* u, double* z,
                        int32_t* idx, double* w, double* gap) {
  for (int i = 0; i < d; i++) xs[i] = bf16_to_double(x_row[i]);
  oracle_rmsnorm_plus_one(d, xs, gamma, eps, u);
  oracle_router_logits(E, d, u, router_w, bias, z);
  double g = 0.0;
  oracle_select_topk(E, k, z, idx, &g);
  if (gap) *gap = g;
  if (forced_idx)
    for (int j = 0; j < k; j++) idx[j] = forced_idx[j];
  oracle_route_weights(E, k, z, idx, w);
}

static int n_threads_wanted = 0;

void oracle_set_threads(int n) { n_threads_wanted = n; }

int oracle_get_threads(void) {
#ifdef _OPENMP
  return n_threads_wanted > 0 ? n_threads_wanted : omp_get_max_threads();
#else
  return 1;
#endif
}

/* Routing only, for T tokens.  Outputs: idx [T,k], w [T,k], gap [T],
 * z [T,E] (any output may be NULL except idx and w). */
void oracle_route(int T, int E, int k, int d, const uint16_t* x, const float* router_w,
                  const float* gamma, const float* bias, double eps, int32_t* idx, double* w,
                  double* gap, double* z_out) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_get_threads())
  for (int t = 0; t < T; t++) {
    double* xs = (double*)malloc(sizeof(double) * (size_t)d);
    double* u = (double*)malloc(sizeof(double) * (size_t)d);
    double* z = (double*)malloc(sizeof(double) * (size_t)E);
    route_token(E, k, d, x + (size_t)t * d, router_w, gamma, bias, eps, NULL, xs, u, z,
                idx + (size_t)t * k, w + (size_t)t * k, gap ? gap + t : NULL);
    if (z_out) memcpy(z_out + (size_t)t * E, z, sizeof(double) * (size_t)E);
    free(xs);
    free(u);
    free(z);
  }
}

/* The whole layer for T tokens, one token at a time over its k selected
 * experts.  forced_idx [T,k] (or NULL) replaces the selected set S (the j
 * order is then the given order); residual [T,d] bf16 (or NULL) is added;
 * expert_gamma [d] (or NULL) applies the expert-side (1+gamma2) RMSNorm to
 * the experts' input (the residual is still the raw x).
 * Outputs: out [T,d] (double), idx [T,k], w [T,k], gap [T] (NULL allowed
 * for w and gap). */
void oracle_moe_forward(int T, int E, int k, int d, int f, int wdtype, const uint16_t* x,
                        const float* router_w, const float* gamma, const float* bias,
                        const float* expert_gamma, double eps, const void* w_gu,
                        const void* w_d, const void* s_gu, const void* s_d,
                        const uint16_t* residual, const int32_t* forced_idx, double* out,
                        int32_t* idx_out, double* w_out, double* gap_out) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_get_threads())
  for (int t = 0; t < T; t++) {
    double* xs = (double*)malloc(sizeof(double) * (size_t)d);
    double* u = (double*)malloc(sizeof(double) * (size_t)d);
    double* z = (double*)malloc(sizeof(double) * (size_t)E);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* w = (double*)malloc(sizeof(double) * (size_t)k);
    double gap = 0.0;
    route_token(E, k, d, x + (size_t)t * d, router_w, gamma, bias, eps,
                forced_idx ? forced_idx + (size_t)t * k : NULL, xs, u, z, idx, w, &gap);
    /* the experts' input: x itself, or its expert-side (1+gamma2) RMSNorm */
    if (expert_gamma) {
      oracle_rmsnorm_plus_one(d, xs, expert_gamma, eps, u);
      memcpy(xs, u, sizeof(double) * (size_t)d);
    }
    double* o = out + (size_t)t * d;
    for (int m = 0; m < d; m++)
      o[m] = residual ? bf16_to_double(residual[(size_t)t * d + m]) : 0.0;
    for (int j = 0; j < k; j++) {
      oracle_expert_ffn(d, f, wdtype, w_gu, w_d, s_gu, s_d, idx[j], xs, y, NULL);
      for (int m = 0; m < d; m++) o[m] += w[j] * y[m];
    }
    if (idx_out) memcpy(idx_out + (size_t)t * k, idx, sizeof(int32_t) * (size_t)k);
    if (w_out) memcpy(w_out + (size_t)t * k, w, sizeof(double) * (size_t)k);
    if (gap_out) gap_out[t] = gap;
    free(xs);
    free(u);
    free(z);
    free(y);
    free(idx);
    free(w);
  }
}

/* Vector helpers for the pins: GELU-tanh and the (1+gamma) norm on rows. */
void oracle_gelu_tanh_vec(int n, const double* a, double* out) {
  for (int i = 0; i < n; i++) out[i] = oracle_gelu_tanh(a[i]);
}

void oracle_rmsnorm_rows(int T, int d, const double* x, const float* gamma, double eps,
                         double* u) {
  for (int t = 0; t < T; t++)
    oracle_rmsnorm_plus_one(d, x + (size_t)t * d, gamma, eps, u + (size_t)t * d);
}

void oracle_decode_bf16(int n, const uint16_t* in, double* out) {
  for (int i = 0; i < n; i++) out[i] = bf16_to_double(in[i]);
}

void oracle_decode_fp16(int n, const uint16_t* in, double* out) {
  for (int i = 0; i < n; i++) out[i] = fp16_to_double(in[i]);
}

void oracle_decode_e2m1(int n, const uint8_t* in, double* out) {
  for (int i = 0; i < n; i++) out[i] = e2m1_to_double(in[i] & 0xf);
}

void oracle_decode_e4m3(int n, const uint8_t* in, double* out) {
  for (int i = 0; i < n; i++) out[i] = e4m3_to_double(in[i]);
}

/* ---- the step after the layer stack: lm_head over the canvas ------------
 *
 * Sources (page title, section):
 *  [FU]  fucina docs "DiffusionGemma 26B-A4B -- block text-diffusion": the
 *        runner denoises 256-token canvases with the entropy-bound sampler
 *        (defaults from the model: <= 48 steps, temperature 0.8 -> 0.4,
 *        bound 0.1); the mean canvas entropy is what the status line shows.
 *  [AR]  auto-round pull request: EntropyBoundSamplerConfig, entropy_bound 0.1.
 *  [QT]  Quant-Tuner pull request, Testing: the entropy-bound acceptance rule
 *        is unit-tested there (its text is not on the pages).
 * Readings (the pages fix none of these):
 *  - logits z_v = h . W[v] over the whole vocabulary (W the lm_head / tied
 *    embedding matrix, bf16), optionally soft-capped c * tanh(z / c);
 *  - the sampler's distribution is p = softmax(z / temperature); a token's
 *    entropy is H = -sum_v p_v log p_v = logZ - sum_v p_v u_v with
 *    u = z / temperature and logZ = log sum_v exp(u_v);
 *  - the proposed token is the argmax of z (lowest vocabulary index on ties);
 *  - acceptance, over the still-masked positions: sort them by entropy
 *    (ties by position) and accept the longest prefix whose entropies, all
 *    but the largest, sum to at most the bound; the lowest-entropy position
 *    is therefore always accepted (the entropy-bounded unmasking rule of
 *    Ben-Hamu et al., "Accelerated Sampling from Masked Diffusion Models via
 *    Entropy Bounded Unmasking", which the pages name only as the
 *    entropy-bound sampler).  PARITY UNPINNED against the pages: they print
 *    neither the rule nor an example; the pins check the definitions. */

/* Statistics of token rows `rows[0..n)` of h [T, d] against W [V, d]:
 * logZ, entropy H, argmax index and the gap between the two largest u. */
void oracle_lmhead_stats(int V, int d, const uint16_t* h, const uint16_t* W, double inv_temp,
                         double softcap, const int32_t* rows, int n, double* logz, double* H,
                         int32_t* argmax, double* gap) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_get_threads())
  for (int j = 0; j < n; j++) {
    const uint16_t* hr = h + (size_t)rows[j] * d;
    double* u = (double*)malloc(sizeof(double) * (size_t)V);
    double* hx = (double*)malloc(sizeof(double) * (size_t)d);
    for (int i = 0; i < d; i++) hx[i] = bf16_to_double(hr[i]);
    int best = 0;
    for (int v = 0; v < V; v++) {
      const uint16_t* wr = W + (size_t)v * d;
      double z = 0.0;
      for (int i = 0; i < d; i++) z += hx[i] * bf16_to_double(wr[i]);
      if (softcap > 0.0) z = softcap * tanh(z / softcap);
      u[v] = z * inv_temp;
      if (u[v] > u[best]) best = v;
    }
    double second = -INFINITY;
    for (int v = 0; v < V; v++)
      if (v != best && u[v] > second) second = u[v];
    double s = 0.0;
    for (int v = 0; v < V; v++) s += exp(u[v] - u[best]);
    const double lz = u[best] + log(s);
    double eu = 0.0;
    for (int v = 0; v < V; v++) eu += exp(u[v] - lz) * u[v];
    logz[j] = lz;
    H[j] = lz - eu;
    argmax[j] = best;
    gap[j] = u[best] - second;
    free(u);
    free(hx);
  }
}

/* Entropy-bounded acceptance over the masked positions (reading above). */
void oracle_eb_accept(int T, const double* H, const uint8_t* masked, double bound,
                      uint8_t* accept) {
  int* order = (int*)malloc(sizeof(int) * (size_t)(T > 0 ? T : 1));
  int n = 0;
  for (int t = 0; t < T; t++) {
    accept[t] = 0;
    if (!masked || masked[t]) order[n++] = t;
  }
  /* insertion sort by (H, position): plain and obviously stable */
  for (int i = 1; i < n; i++) {
    int t = order[i], j = i - 1;
    while (j >= 0 && (H[order[j]] > H[t])) {
      order[j + 1] = order[j];
      j--;
    }
    order[j + 1] = t;
  }
  double below = 0.0; /* sum of the entropies before position i in the order */
  for (int i = 0; i < n; i++) {
    if (below > bound) break;
    accept[order[i]] = 1;
    below += H[order[i]];
  }
  free(order);
}
