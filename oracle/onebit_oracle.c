/*
 * onebit_oracle.c -- TEST INFRASTRUCTURE, not the product.
 *
 * A plain, slow, single-threaded CPU statement of what the 1-bit Adam
 * compressed-phase step computes.  It is the oracle the CUDA path is checked
 * against.  Only tests/, __graft_entry__.smoke() and the CPU-baseline leg of
 * bench.py may load it; the library under bit_adam_error_b200/ never does, and
 * the two share no code, header, table or constant.
 *
 * Sources followed (page title, section):
 *  - "DeepSpeed Communication Compression and Hiding", section "1-bit Adam:
 *    预热、冻结方差、误差反馈 / 机制": the structure of the step -- full Adam moments
 *    on the averaged gradient during warmup (step < freeze_step); afterwards each
 *    worker's gradient plus its error buffer is reduced to signs and a scale,
 *    the workers' messages are combined by a compressed allreduce and expanded
 *    into the direction g_hat, the error buffer keeps what quantisation lost,
 *    m follows g_hat with v frozen, and p moves by lr m / (sqrt(v) + eps).
 *  - same page, section "基线：Adam 为什么难压缩": the Adam moment equations.
 *  - same page, section "1-bit LAMB": r_l = ||w_l|| / ||u_l||,
 *    w_l <- w_l - eta r_l u_l, computed from the reconstructed global direction.
 *  - the CANN 1-bit Adam article (intelliparadigm.com), section 3.2
 *    "核心算法实现细节": clipping of extreme gradient
 *    values before quantisation (threshold 5.0) and a NaN check after the
 *    error update.
 *  - where the pages name a step but give no formula, this oracle fixes it as:
 *    scale s = ||c||_2 / sqrt(n) per chunk, sign(0) = +1, signs packed into
 *    uint32 words, err = c - s * sign(c) per worker, and a server stage that
 *    unpacks the W workers, averages their scaled signs and re-compresses the
 *    average with its own server error buffer.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - bit = (c >= 0.0f): +0 and -0 give +1; NaN gives -1 and raises
 *    ORC_STATUS_NONFINITE.
 *  - element i of a chunk -> bit (i % 32) of word (i / 32) of that chunk;
 *    every chunk starts on a fresh word; padding bits are 0.
 *  - norms are accumulated in double, in ascending element order; the scale is
 *    (float)(sqrt(S) / sqrt((double)n_k)); an empty chunk has scale 0.
 *  - the server average is sum over w = 0..W-1 (ascending) of +-s_w in float,
 *    then divided by (float)W.
 *  - no bias correction; warmup averages the W gradients in float, ascending w.
 *  - clip (when > 0) clamps the raw gradient before the error is added; a NaN
 *    gradient passes through unchanged.
 *  - LAMB: layer = chunk; u = m / (sqrtf(v) + eps); r = ||p|| / ||u|| with the
 *    pre-update p, and r = 1 when either norm is 0; no weight decay.
 *  - error buffers may be stored in bfloat16 (half the bytes; the gradient-
 *    compression survey page suggests half-precision error storage): each
 *    stored error is the float32 result rounded to nearest-even bfloat16.
 *
 * Two more compression rules follow the main one, each under its own heading
 * with its passages and readings: the CANN article's momentum-error rule
 * (int8 ternary codes) and 2-bit Adam (two residual sign planes).
 *
 * Parity pins: every function here is checked by tests/test_oracle_pins.py
 * against hand-worked cases, closed forms, invariants and brute force.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (no FMA contraction, plain
 * IEEE float/double).  All arrays are host memory, caller-owned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_ADAM 0
#define ORC_LAMB 1
#define ORC_STATUS_NONFINITE 1u

/* ---- small helpers -------------------------------------------------------- */

static int64_t words_of(int64_t n) { return (n + 31) / 32; }

/* First word of every chunk: chunks start on a fresh word. */
static void word_offsets(int32_t C, const int64_t* off, int64_t* wo) {
  wo[0] = 0;
  for (int32_t k = 0; k < C; ++k) wo[k + 1] = wo[k] + words_of(off[k + 1] - off[k]);
}

/* bf16 -> float is exact: the 16 bits are the top half of the float32. */
static float grad_at(const void* grads, int32_t dtype, int64_t idx) {
  if (dtype == ORC_BF16) {
    uint32_t u = (uint32_t)((const uint16_t*)grads)[idx] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
  }
  return ((const float*)grads)[idx];
}

/* Error buffers are stored as float32, or as bfloat16 (the top 16 bits of the
 * float32, rounded to nearest with ties to even; NaN stays NaN) and widened
 * exactly on load; all arithmetic stays float32. */
static uint16_t to_bf16_rne(float x) {
  uint32_t u;
  memcpy(&u, &x, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
  uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

static float err_get(const void* e, int32_t dtype, int64_t i) {
  if (dtype == ORC_BF16) return grad_at(e, ORC_BF16, i);
  return ((const float*)e)[i];
}

static void err_set(void* e, int32_t dtype, int64_t i, float x) {
  if (dtype == ORC_BF16) ((uint16_t*)e)[i] = to_bf16_rne(x);
  else ((float*)e)[i] = x;
}

static float clip_grad(float g, float clip) {
  if (!(clip > 0.0f)) return g;
  if (g > clip) return clip;
  if (g < -clip) return -clip;
  return g; /* NaN falls through */
}

static int is_nonfinite(float x) { return !isfinite(x); }

/* one_bit_quantize, scale part: s = ||c||_2 / sqrt(n). */
static float quantize_scale(const float* c, int64_t n) {
  if (n == 0) return 0.0f;
  double S = 0.0;
  for (int64_t i = 0; i < n; ++i) S += (double)c[i] * (double)c[i];
  return (float)(sqrt(S) / sqrt((double)n));
}

/* one_bit_quantize, sign part: bit i = (c_i >= 0), LSB-first in uint32 words. */
static void quantize_signs(const float* c, int64_t n, uint32_t* words) {
  int64_t nw = words_of(n);
  for (int64_t j = 0; j < nw; ++j) words[j] = 0u;
  for (int64_t i = 0; i < n; ++i)
    if (c[i] >= 0.0f) words[i / 32] |= 1u << (i % 32);
}

static int sign_bit(const uint32_t* words, int64_t i) {
  return (int)((words[i / 32] >> (i % 32)) & 1u);
}

/* dequantize: +scale for a set bit, -scale otherwise. */
static float dequantize(const uint32_t* words, float scale, int64_t i) {
  return sign_bit(words, i) ? scale : -scale;
}

/* ---- exported --------------------------------------------------------------- */

int64_t orc_words_total(int32_t C, const int64_t* off) {
  int64_t t = 0;
  for (int32_t k = 0; k < C; ++k) t += words_of(off[k + 1] - off[k]);
  return t;
}

/*
 * Worker stage, every worker w and chunk k:
 *   compensated c = clip(g_w) + err_w
 *   (q, s_wk)     = one_bit_quantize(c)
 *   err_w         = c - dequantize(q, s_wk)
 * grads: [W][n] (float32 or bf16 bits); err: [W][n] in/out;
 * bits_w: [W][words_total] out; s_w: [W][C] out.  Returns status flags.
 */
uint32_t orc_compress(int32_t W, int64_t n, int32_t C, const int64_t* off,
                      const void* grads, int32_t dtype, float clip, void* err,
                      int32_t err_dtype, uint32_t* bits_w, float* s_w) {
  uint32_t flags = 0;
  int64_t* wo = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  word_offsets(C, off, wo);
  int64_t words_total = wo[C];
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k];
    float* c = (float*)malloc(sizeof(float) * (size_t)(nk > 0 ? nk : 1));
    for (int32_t w = 0; w < W; ++w) {
      const int64_t e0 = (int64_t)w * n + o;
      uint32_t* q = bits_w + (int64_t)w * words_total + wo[k];
      for (int64_t i = 0; i < nk; ++i) {
        c[i] = clip_grad(grad_at(grads, dtype, e0 + i), clip) + err_get(err, err_dtype, e0 + i);
        if (is_nonfinite(c[i])) flags |= ORC_STATUS_NONFINITE;
      }
      float s = quantize_scale(c, nk);
      quantize_signs(c, nk, q);
      s_w[(int64_t)w * C + k] = s;
      for (int64_t i = 0; i < nk; ++i) err_set(err, err_dtype, e0 + i, c[i] - dequantize(q, s, i));
    }
    free(c);
  }
  free(wo);
  return flags;
}

/*
 * Server stage (the compressed allreduce), every chunk k:
 *   avg_i  = (sum_{w=0..W-1} dequantize(q_w, s_wk)_i) / W
 *   c_srv  = avg + srv_err
 *   (q', s_srv_k) = one_bit_quantize(c_srv)
 *   srv_err = c_srv - dequantize(q', s_srv_k)
 * bits_w: [W][words_total]; s_w: [W][C]; srv_err: [n] in/out;
 * bits_srv: [words_total] out; s_srv: [C] out.  Returns status flags.
 */
uint32_t orc_server_reduce(int32_t W, int64_t n, int32_t C, const int64_t* off,
                           const uint32_t* bits_w, const float* s_w, void* srv_err,
                           int32_t err_dtype, uint32_t* bits_srv, float* s_srv) {
  (void)n;
  uint32_t flags = 0;
  int64_t* wo = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  word_offsets(C, off, wo);
  int64_t words_total = wo[C];
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k];
    float* c = (float*)malloc(sizeof(float) * (size_t)(nk > 0 ? nk : 1));
    for (int64_t i = 0; i < nk; ++i) {
      float acc = 0.0f;
      for (int32_t w = 0; w < W; ++w)
        acc += dequantize(bits_w + (int64_t)w * words_total + wo[k], s_w[(int64_t)w * C + k], i);
      float avg = acc / (float)W;
      c[i] = avg + err_get(srv_err, err_dtype, o + i);
      if (is_nonfinite(c[i])) flags |= ORC_STATUS_NONFINITE;
    }
    float s = quantize_scale(c, nk);
    uint32_t* q = bits_srv + wo[k];
    quantize_signs(c, nk, q);
    s_srv[k] = s;
    for (int64_t i = 0; i < nk; ++i) err_set(srv_err, err_dtype, o + i, c[i] - dequantize(q, s, i));
    free(c);
  }
  free(wo);
  return flags;
}

/*
 * Compressed-phase Adam update with frozen v:
 *   g_hat = dequantize(q', s_srv)
 *   m = beta1 m + (1 - beta1) g_hat
 *   p = p - lr m / (sqrtf(v) + eps)
 */
uint32_t orc_adam_apply(int64_t n, int32_t C, const int64_t* off,
                        const uint32_t* bits_srv, const float* s_srv, float beta1,
                        float lr, float eps, float* m, const float* v, float* p) {
  (void)n;
  uint32_t flags = 0;
  int64_t* wo = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  word_offsets(C, off, wo);
  const float one_minus_b1 = 1.0f - beta1;
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k];
    for (int64_t i = 0; i < nk; ++i) {
      float g_hat = dequantize(bits_srv + wo[k], s_srv[k], i);
      float mi = beta1 * m[o + i] + one_minus_b1 * g_hat;
      m[o + i] = mi;
      float pi = p[o + i] - lr * mi / (sqrtf(v[o + i]) + eps);
      if (is_nonfinite(pi)) flags |= ORC_STATUS_NONFINITE;
      p[o + i] = pi;
    }
  }
  free(wo);
  return flags;
}

/* Per-layer trust ratio r = ||p|| / ||u|| (pre-update p), 1 if either is 0. */
static float trust_ratio(const float* p, const float* m, const float* v, float eps, int64_t nk) {
  double P = 0.0, U = 0.0;
  for (int64_t i = 0; i < nk; ++i) {
    float u = m[i] / (sqrtf(v[i]) + eps);
    P += (double)p[i] * (double)p[i];
    U += (double)u * (double)u;
  }
  if (P > 0.0 && U > 0.0) return (float)(sqrt(P) / sqrt(U));
  return 1.0f;
}

static uint32_t lamb_update_layer(float* p, const float* m, const float* v, float lr,
                                  float eps, int64_t nk) {
  uint32_t flags = 0;
  float r = trust_ratio(p, m, v, eps, nk);
  for (int64_t i = 0; i < nk; ++i) {
    float u = m[i] / (sqrtf(v[i]) + eps);
    float pi = p[i] - lr * r * u;
    if (is_nonfinite(pi)) flags |= ORC_STATUS_NONFINITE;
    p[i] = pi;
  }
  return flags;
}

/*
 * Compressed-phase 1-bit LAMB update (layer = chunk), v frozen:
 *   m = beta1 m + (1 - beta1) g_hat;  u = m / (sqrtf(v) + eps)
 *   r_l = ||p_l|| / ||u_l||;          p -= lr r_l u
 * r_out (may be NULL): [C] trust ratios used.
 */
uint32_t orc_lamb_apply(int64_t n, int32_t C, const int64_t* off,
                        const uint32_t* bits_srv, const float* s_srv, float beta1,
                        float lr, float eps, float* m, const float* v, float* p,
                        float* r_out) {
  (void)n;
  uint32_t flags = 0;
  int64_t* wo = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  word_offsets(C, off, wo);
  const float one_minus_b1 = 1.0f - beta1;
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k];
    for (int64_t i = 0; i < nk; ++i) {
      float g_hat = dequantize(bits_srv + wo[k], s_srv[k], i);
      m[o + i] = beta1 * m[o + i] + one_minus_b1 * g_hat;
    }
    if (r_out) r_out[k] = trust_ratio(p + o, m + o, v + o, eps, nk);
    flags |= lamb_update_layer(p + o, m + o, v + o, lr, eps, nk);
  }
  free(wo);
  return flags;
}

/*
 * Full-precision warmup step (step < freeze_step):
 *   g = (sum_{w=0..W-1} g_w) / W
 *   m = beta1 m + (1 - beta1) g;  v = beta2 v + (1 - beta2) g^2
 *   Adam: p -= lr m / (sqrtf(v) + eps);  LAMB: trust-ratio update as above.
 * Error buffers are not touched.
 */
uint32_t orc_warmup(int32_t W, int64_t n, int32_t C, const int64_t* off,
                    const void* grads, int32_t dtype, int32_t optimizer, float beta1,
                    float beta2, float lr, float eps, float* m, float* v, float* p) {
  uint32_t flags = 0;
  const float one_minus_b1 = 1.0f - beta1;
  const float one_minus_b2 = 1.0f - beta2;
  for (int64_t i = 0; i < n; ++i) {
    float acc = 0.0f;
    for (int32_t w = 0; w < W; ++w) acc += grad_at(grads, dtype, (int64_t)w * n + i);
    float g = acc / (float)W;
    if (is_nonfinite(g)) flags |= ORC_STATUS_NONFINITE;
    m[i] = beta1 * m[i] + one_minus_b1 * g;
    v[i] = beta2 * v[i] + one_minus_b2 * (g * g);
    if (optimizer == ORC_ADAM) {
      float pi = p[i] - lr * m[i] / (sqrtf(v[i]) + eps);
      if (is_nonfinite(pi)) flags |= ORC_STATUS_NONFINITE;
      p[i] = pi;
    }
  }
  if (optimizer == ORC_LAMB)
    for (int32_t k = 0; k < C; ++k) {
      int64_t o = off[k], nk = off[k + 1] - off[k];
      flags |= lamb_update_layer(p + o, m + o, v + o, lr, eps, nk);
    }
  return flags;
}

/* One whole compressed-phase step: worker stage, server stage, update. */
uint32_t orc_step(int32_t W, int64_t n, int32_t C, const int64_t* off,
                  const void* grads, int32_t dtype, int32_t optimizer, float clip,
                  float beta1, float lr, float eps, float* p, float* m, const float* v,
                  void* err, void* srv_err, int32_t err_dtype, uint32_t* bits_w, float* s_w,
                  uint32_t* bits_srv, float* s_srv) {
  uint32_t flags = orc_compress(W, n, C, off, grads, dtype, clip, err, err_dtype, bits_w, s_w);
  flags |= orc_server_reduce(W, n, C, off, bits_w, s_w, srv_err, err_dtype, bits_srv, s_srv);
  if (optimizer == ORC_LAMB)
    flags |= orc_lamb_apply(n, C, off, bits_srv, s_srv, beta1, lr, eps, m, v, p, NULL);
  else
    flags |= orc_adam_apply(n, C, off, bits_srv, s_srv, beta1, lr, eps, m, v, p);
  return flags;
}

/* ---- the momentum-error rule ------------------------------------------------------
 *
 * The CANN 1-bit Adam article, section 2.1 "量化与误差补偿机制" (sign quantisation,
 * error, momentum-form error compensation), section 2.2 "动量修正策略" (m follows
 * the compressed gradient) and section 3.2 (clip before quantisation, NaN check
 * after the error update, int8 storage of the compressed gradient).  Per worker
 * w and element, with eps_w the worker's error buffer:
 *   c      = clip(g_w) + eps_w
 *   q      = sign(c)                        in {-1, 0, +1}, no scale
 *   Delta  = c - q
 *   eps_w  = beta1 eps_w + (1 - beta1) Delta
 * The article's snippet is one worker.  Readings for W workers and the rest:
 *  - q travels as an int8 code; the W codes of an element are combined by
 *    their sum (exact in int8 for W <= 127), and the direction is their mean
 *    g_hat = (float)sum / (float)W (the compressed allreduce of the DeepSpeed
 *    page, section "机制", averaging the workers' messages);
 *  - m = beta1 m + (1 - beta1) g_hat and the parameter step are the ones of
 *    orc_adam_apply / orc_lamb_apply, v frozen;
 *  - sign(+0) = sign(-0) = 0, and a NaN c gives code 0 (its error is NaN);
 *  - the check after the error update flags any non-finite error (NaN or
 *    +-inf), and a non-finite parameter as elsewhere;
 *  - codes of chunk k occupy bytes [4 cw_k, 4 cw_k + n_k) of a row, where
 *    every chunk starts on a fresh 32-bit word and takes ceil(n_k / 4) words;
 *    padding bytes are 0.
 */

static int64_t code_words_of(int64_t n) { return (n + 3) / 4; }

static void code_word_offsets(int32_t C, const int64_t* off, int64_t* cw) {
  cw[0] = 0;
  for (int32_t k = 0; k < C; ++k) cw[k + 1] = cw[k] + code_words_of(off[k + 1] - off[k]);
}

int64_t orc_code_words_total(int32_t C, const int64_t* off) {
  int64_t t = 0;
  for (int32_t k = 0; k < C; ++k) t += code_words_of(off[k + 1] - off[k]);
  return t;
}

/* sign() with sign(0) = 0; NaN compares false both ways and gives 0. */
static int8_t ternary_sign(float c) {
  if (c > 0.0f) return 1;
  if (c < 0.0f) return -1;
  return 0;
}

/*
 * Worker stage of the momentum-error rule.  grads: [W][n]; err: [W][n] in/out;
 * codes_w: [W][4 * code_words_total] int8 out.  Returns status flags.
 */
uint32_t orc_ternary_compress(int32_t W, int64_t n, int32_t C, const int64_t* off,
                              const void* grads, int32_t dtype, float clip, float beta1,
                              void* err, int32_t err_dtype, int8_t* codes_w) {
  uint32_t flags = 0;
  const float one_minus_b1 = 1.0f - beta1;
  int64_t* cw = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  code_word_offsets(C, off, cw);
  const int64_t row_bytes = 4 * cw[C];
  for (int32_t w = 0; w < W; ++w) {
    int8_t* row = codes_w + (int64_t)w * row_bytes;
    memset(row, 0, (size_t)row_bytes);
    for (int32_t k = 0; k < C; ++k) {
      int64_t o = off[k], nk = off[k + 1] - off[k];
      for (int64_t i = 0; i < nk; ++i) {
        const int64_t e = (int64_t)w * n + o + i;
        float eps_old = err_get(err, err_dtype, e);
        float c = clip_grad(grad_at(grads, dtype, e), clip) + eps_old;
        int8_t q = ternary_sign(c);
        float delta = c - (float)q;
        float eps_new = beta1 * eps_old + one_minus_b1 * delta;
        if (is_nonfinite(eps_new)) flags |= ORC_STATUS_NONFINITE;
        err_set(err, err_dtype, e, eps_new);
        row[4 * cw[k] + i] = q;
      }
    }
  }
  free(cw);
  return flags;
}

/*
 * Server stage of the momentum-error rule: codes_srv = sum over w = 0..W-1 of
 * codes_w, per element (the caller keeps W <= 127).  codes_w: [W][row bytes];
 * codes_srv: [row bytes] out, padding bytes 0.
 */
uint32_t orc_ternary_server(int32_t W, int32_t C, const int64_t* off, const int8_t* codes_w,
                            int8_t* codes_srv) {
  int64_t* cw = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  code_word_offsets(C, off, cw);
  const int64_t row_bytes = 4 * cw[C];
  memset(codes_srv, 0, (size_t)row_bytes);
  for (int32_t k = 0; k < C; ++k) {
    int64_t nk = off[k + 1] - off[k];
    for (int64_t i = 0; i < nk; ++i) {
      const int64_t b = 4 * cw[k] + i;
      int sum = 0;
      for (int32_t w = 0; w < W; ++w) sum += codes_w[(int64_t)w * row_bytes + b];
      codes_srv[b] = (int8_t)sum;
    }
  }
  free(cw);
  return 0u;
}

/*
 * Update of the momentum-error rule: g_hat = (float)codes_srv / (float)W, then
 * m and p as orc_adam_apply (optimizer ORC_ADAM) or orc_lamb_apply (ORC_LAMB;
 * r_out, may be NULL, receives the [C] trust ratios).
 */
uint32_t orc_ternary_apply(int64_t n, int32_t C, const int64_t* off, int32_t W,
                           const int8_t* codes_srv, int32_t optimizer, float beta1, float lr,
                           float eps, float* m, const float* v, float* p, float* r_out) {
  (void)n;
  uint32_t flags = 0;
  int64_t* cw = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  code_word_offsets(C, off, cw);
  const float one_minus_b1 = 1.0f - beta1;
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k];
    for (int64_t i = 0; i < nk; ++i) {
      float g_hat = (float)codes_srv[4 * cw[k] + i] / (float)W;
      float mi = beta1 * m[o + i] + one_minus_b1 * g_hat;
      m[o + i] = mi;
      if (optimizer == ORC_ADAM) {
        float pi = p[o + i] - lr * mi / (sqrtf(v[o + i]) + eps);
        if (is_nonfinite(pi)) flags |= ORC_STATUS_NONFINITE;
        p[o + i] = pi;
      }
    }
    if (optimizer == ORC_LAMB) {
      if (r_out) r_out[k] = trust_ratio(p + o, m + o, v + o, eps, nk);
      flags |= lamb_update_layer(p + o, m + o, v + o, lr, eps, nk);
    }
  }
  free(cw);
  return flags;
}

/* One whole compressed-phase step of the momentum-error rule. */
uint32_t orc_ternary_step(int32_t W, int64_t n, int32_t C, const int64_t* off,
                          const void* grads, int32_t dtype, int32_t optimizer, float clip,
                          float beta1, float lr, float eps, float* p, float* m, const float* v,
                          void* err, int32_t err_dtype, int8_t* codes_w, int8_t* codes_srv) {
  uint32_t flags = orc_ternary_compress(W, n, C, off, grads, dtype, clip, beta1, err, err_dtype,
                                        codes_w);
  flags |= orc_ternary_server(W, C, off, codes_w, codes_srv);
  flags |= orc_ternary_apply(n, C, off, W, codes_srv, optimizer, beta1, lr, eps, m, v, p, NULL);
  return flags;
}

/* ---- 2-bit Adam ----------------------------------------------------------------------
 *
 * The CANN 1-bit Adam article names 2-bit Adam (section 5.1, table: 6.25% of the
 * traffic; section 8: weaker compression for embedding layers) but gives no
 * quantiser.  Reading: the 1-bit quantiser of this file applied twice, the
 * second time to what the first left over -- two sign planes with one scale
 * each, 2 bits per element plus 2 scales per chunk:
 *   (q1, s1) = one_bit_quantize(c),        r   = c - dequantize(q1, s1)
 *   (q2, s2) = one_bit_quantize(r),        err = r - dequantize(q2, s2)
 *   dequantized value = dequantize(q1, s1) + dequantize(q2, s2)   (float add)
 * Workers and server use it in place of one_bit_quantize; everything else
 * (error feedback, server average and error, update) is unchanged.
 * Layout: chunk k owns 2 ceil(n_k / 32) words of a row -- plane 1, then plane
 * 2 -- starting on a fresh word; scales are [..][C][2] (plane 1, plane 2).
 */

static int64_t words2_of(int64_t n) { return 2 * words_of(n); }

int64_t orc_words2_total(int32_t C, const int64_t* off) {
  int64_t t = 0;
  for (int32_t k = 0; k < C; ++k) t += words2_of(off[k + 1] - off[k]);
  return t;
}

/* Two planes of c: words[0 .. 2 nw), s[0..1]; resid (may alias nothing) gets
 * the final residual r - dequantize(q2, s2). */
static void two_bit_quantize(const float* c, int64_t nk, uint32_t* words, float* s, float* r,
                             float* resid) {
  const int64_t nw = words_of(nk);
  s[0] = quantize_scale(c, nk);
  quantize_signs(c, nk, words);
  for (int64_t i = 0; i < nk; ++i) r[i] = c[i] - dequantize(words, s[0], i);
  s[1] = quantize_scale(r, nk);
  quantize_signs(r, nk, words + nw);
  for (int64_t i = 0; i < nk; ++i) resid[i] = r[i] - dequantize(words + nw, s[1], i);
}

static float dequantize2(const uint32_t* words, int64_t nw, const float* s, int64_t i) {
  return dequantize(words, s[0], i) + dequantize(words + nw, s[1], i);
}

/* Worker stage of 2-bit Adam.  bits_w: [W][words2_total]; s_w: [W][C][2]. */
uint32_t orc_twobit_compress(int32_t W, int64_t n, int32_t C, const int64_t* off,
                             const void* grads, int32_t dtype, float clip, void* err,
                             int32_t err_dtype, uint32_t* bits_w, float* s_w) {
  uint32_t flags = 0;
  int64_t* wo = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  wo[0] = 0;
  for (int32_t k = 0; k < C; ++k) wo[k + 1] = wo[k] + words2_of(off[k + 1] - off[k]);
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k];
    size_t bytes = sizeof(float) * (size_t)(nk > 0 ? nk : 1);
    float *c = (float*)malloc(bytes), *r = (float*)malloc(bytes), *e = (float*)malloc(bytes);
    for (int32_t w = 0; w < W; ++w) {
      const int64_t e0 = (int64_t)w * n + o;
      for (int64_t i = 0; i < nk; ++i) {
        c[i] = clip_grad(grad_at(grads, dtype, e0 + i), clip) + err_get(err, err_dtype, e0 + i);
        if (is_nonfinite(c[i])) flags |= ORC_STATUS_NONFINITE;
      }
      two_bit_quantize(c, nk, bits_w + (int64_t)w * wo[C] + wo[k], s_w + ((int64_t)w * C + k) * 2, r, e);
      for (int64_t i = 0; i < nk; ++i) err_set(err, err_dtype, e0 + i, e[i]);
    }
    free(c); free(r); free(e);
  }
  free(wo);
  return flags;
}

/* Server stage of 2-bit Adam: c_srv = mean_w(dequantized worker w) + srv_err,
 * quantised to two planes; srv_err keeps the residual. */
uint32_t orc_twobit_server(int32_t W, int64_t n, int32_t C, const int64_t* off,
                           const uint32_t* bits_w, const float* s_w, void* srv_err,
                           int32_t err_dtype, uint32_t* bits_srv, float* s_srv) {
  (void)n;
  uint32_t flags = 0;
  int64_t* wo = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  wo[0] = 0;
  for (int32_t k = 0; k < C; ++k) wo[k + 1] = wo[k] + words2_of(off[k + 1] - off[k]);
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k], nw = words_of(nk);
    size_t bytes = sizeof(float) * (size_t)(nk > 0 ? nk : 1);
    float *c = (float*)malloc(bytes), *r = (float*)malloc(bytes), *e = (float*)malloc(bytes);
    for (int64_t i = 0; i < nk; ++i) {
      float acc = 0.0f;
      for (int32_t w = 0; w < W; ++w)
        acc += dequantize2(bits_w + (int64_t)w * wo[C] + wo[k], nw, s_w + ((int64_t)w * C + k) * 2, i);
      float avg = acc / (float)W;
      c[i] = avg + err_get(srv_err, err_dtype, o + i);
      if (is_nonfinite(c[i])) flags |= ORC_STATUS_NONFINITE;
    }
    two_bit_quantize(c, nk, bits_srv + wo[k], s_srv + 2 * k, r, e);
    for (int64_t i = 0; i < nk; ++i) err_set(srv_err, err_dtype, o + i, e[i]);
    free(c); free(r); free(e);
  }
  free(wo);
  return flags;
}

/* Update of 2-bit Adam: g_hat = dequantized server planes; m and p as
 * orc_adam_apply (ORC_ADAM) or orc_lamb_apply (ORC_LAMB; r_out may be NULL). */
uint32_t orc_twobit_apply(int64_t n, int32_t C, const int64_t* off, const uint32_t* bits_srv,
                          const float* s_srv, int32_t optimizer, float beta1, float lr, float eps,
                          float* m, const float* v, float* p, float* r_out) {
  (void)n;
  uint32_t flags = 0;
  const float one_minus_b1 = 1.0f - beta1;
  int64_t wo = 0;
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k], nw = words_of(nk);
    for (int64_t i = 0; i < nk; ++i) {
      float g_hat = dequantize2(bits_srv + wo, nw, s_srv + 2 * k, i);
      float mi = beta1 * m[o + i] + one_minus_b1 * g_hat;
      m[o + i] = mi;
      if (optimizer == ORC_ADAM) {
        float pi = p[o + i] - lr * mi / (sqrtf(v[o + i]) + eps);
        if (is_nonfinite(pi)) flags |= ORC_STATUS_NONFINITE;
        p[o + i] = pi;
      }
    }
    if (optimizer == ORC_LAMB) {
      if (r_out) r_out[k] = trust_ratio(p + o, m + o, v + o, eps, nk);
      flags |= lamb_update_layer(p + o, m + o, v + o, lr, eps, nk);
    }
    wo += 2 * nw;
  }
  return flags;
}

/* One whole compressed-phase step of 2-bit Adam. */
uint32_t orc_twobit_step(int32_t W, int64_t n, int32_t C, const int64_t* off,
                         const void* grads, int32_t dtype, int32_t optimizer, float clip,
                         float beta1, float lr, float eps, float* p, float* m, const float* v,
                         void* err, void* srv_err, int32_t err_dtype, uint32_t* bits_w, float* s_w,
                         uint32_t* bits_srv, float* s_srv) {
  uint32_t flags = orc_twobit_compress(W, n, C, off, grads, dtype, clip, err, err_dtype, bits_w, s_w);
  flags |= orc_twobit_server(W, n, C, off, bits_w, s_w, srv_err, err_dtype, bits_srv, s_srv);
  flags |= orc_twobit_apply(n, C, off, bits_srv, s_srv, optimizer, beta1, lr, eps, m, v, p, NULL);
  return flags;
}

/* ---- monitoring: the quantisation rate ---------------------------------------------
 *
 * The CANN 1-bit Adam article, section 8 ("监控指标"), watches the gradient
 * quantisation rate ("梯度量化率") next to the error-buffer L2 norm and expects it
 * near its theoretical value.  The article gives no formula.  Reading: the
 * rate of a chunk is the fraction of its n_k elements sent as +1, i.e. whose
 * sign bit is set; for a message symmetric about zero its theoretical value is
 * 1/2.  A rate far from 1/2 means the error feedback is carrying a bias.
 *
 * rows: packed rows, each laid out as the sign words are: chunk k starts at
 * word planes * sum_{j<k} ceil(n_j / 32), its `planes` planes follow one
 * another, ceil(n_k / 32) words each (planes = 2 for 2-bit Adam, else 1).
 * rates[(r * C + k) * planes + p] = (float)((double)count / (double)n_k), the
 * count taken over the n_k real bits only (padding bits never count); an
 * empty chunk has rate 0.
 */
void orc_sign_rates(int32_t rows, int32_t C, const int64_t* off, int32_t planes,
                    const uint32_t* bits, float* rates) {
  int64_t row_words = 0;
  for (int32_t k = 0; k < C; ++k) row_words += planes * words_of(off[k + 1] - off[k]);
  for (int32_t r = 0; r < rows; ++r) {
    int64_t base = (int64_t)r * row_words;
    for (int32_t k = 0; k < C; ++k) {
      int64_t nk = off[k + 1] - off[k], nw = words_of(nk);
      for (int32_t pl = 0; pl < planes; ++pl) {
        const uint32_t* q = bits + base + pl * nw;
        int64_t count = 0;
        for (int64_t i = 0; i < nk; ++i) count += sign_bit(q, i);
        rates[((int64_t)r * C + k) * planes + pl] = nk > 0 ? (float)((double)count / (double)nk) : 0.0f;
      }
      base += planes * nw;
    }
  }
}

/* ---- 0/1 Adam: the local step ------------------------------------------------------
 *
 * "DeepSpeed Communication Compression and Hiding", section "0/1 Adam": 0/1
 * Adam alternates full-precision variance refreshes with 1-bit synchronised
 * steps, and adds local updates that lower the synchronisation frequency: its
 * listing updates m only from a synchronised g_hat, applies
 * param = adam_update(param, m, v) on every step, and lets local steps run
 * between one global synchronisation and the next.  The page gives no formula
 * for a local step.  Reading:
 *   - a local step sends nothing;
 *   - the parameters take the update of the listing's last line with the
 *     current m and v, which stay as they are:
 *       p = p - lr m / (sqrtf(v) + eps)
 *     (1-bit LAMB: u = m / (sqrtf(v) + eps), r_l = ||p_l|| / ||u_l||,
 *     p -= lr r_l u, as orc_lamb_apply);
 *   - the gradient was not sent, so, as error feedback keeps whatever a step
 *     did not transmit, each worker adds it to its error buffer and it reaches
 *     the next synchronised step inside the compensated value:
 *       err_w = clip(g_w) + err_w
 *     (the same float addition the worker stage makes).
 * Rules with additive error feedback only (the scaled-sign rule and 2-bit Adam).
 * grads: [W][n]; err: [W][n] in/out.  Returns status flags (non-finite error or
 * parameter).
 */
uint32_t orc_local_step(int32_t W, int64_t n, int32_t C, const int64_t* off, const void* grads,
                        int32_t dtype, int32_t optimizer, float clip, float lr, float eps, float* p,
                        const float* m, const float* v, void* err, int32_t err_dtype) {
  uint32_t flags = 0;
  for (int32_t w = 0; w < W; ++w)
    for (int64_t i = 0; i < n; ++i) {
      const int64_t e = (int64_t)w * n + i;
      float kept = clip_grad(grad_at(grads, dtype, e), clip) + err_get(err, err_dtype, e);
      if (is_nonfinite(kept)) flags |= ORC_STATUS_NONFINITE;
      err_set(err, err_dtype, e, kept);
    }
  for (int32_t k = 0; k < C; ++k) {
    int64_t o = off[k], nk = off[k + 1] - off[k];
    if (optimizer == ORC_LAMB) {
      flags |= lamb_update_layer(p + o, m + o, v + o, lr, eps, nk);
      continue;
    }
    for (int64_t i = 0; i < nk; ++i) {
      float pi = p[o + i] - lr * m[o + i] / (sqrtf(v[o + i]) + eps);
      if (is_nonfinite(pi)) flags |= ORC_STATUS_NONFINITE;
      p[o + i] = pi;
    }
  }
  return flags;
}
