/*
 * onebit_oracle_mt.c -- TEST INFRASTRUCTURE, not the product.
 *
 * The oracle's compressed-phase step (the scaled-sign rule of onebit_oracle.c)
 * on several host threads.  It exists for two test-side uses:
 *   - timing the CPU baseline on all host cores next to the single-thread
 *     figure;
 *   - long chained parity runs at full chunk sizes (100 steps of 2^26-element
 *     chunks), which the single-thread oracle takes minutes for.
 *
 * It compiles onebit_oracle.c into the same unit and uses its helpers
 * (clip_grad, grad_at, err_get/err_set, quantize_scale, quantize_signs,
 * dequantize, trust_ratio).  The step is the sequence of onebit_oracle.c's
 * orc_step, cut into phases at its reductions:
 *   1  c = clip(g_w) + err_w                       element ranges, every (k, w)
 *   2  s_wk = quantize_scale(c of chunk k)         one task per (k, w)
 *   3  sign words, err_w = c - dequantize(q, s_wk)  element ranges
 *   4  c_srv = (sum_w dequantize(q_w, s_wk)) / W + srv_err   element ranges
 *   5  s_srv_k = quantize_scale(c_srv of chunk k)  one task per k
 *   6  server words, srv_err, then m (and p for Adam)   element ranges
 *   7  LAMB: r_k = trust_ratio(layer k)            one task per k
 *   8  LAMB: p -= lr r_k u                          element ranges
 * Every per-element statement is the single-thread oracle's, and every
 * reduction (a chunk's sum of squares, a layer's trust-ratio sums) is still one
 * ascending loop run by one thread.  So the results are bit for bit those of
 * orc_step, whatever the thread count; a CPU test checks that on ragged
 * multi-chunk inputs.  Element ranges start on multiples of 32, so two threads
 * never write the same packed word.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared -pthread (the flags of the
 * single-thread oracle plus -pthread).
 */
#include "onebit_oracle.c"

#include <pthread.h>

/* Elements per range task: a multiple of 32 (whole packed words). */
#define ORC_MT_RANGE ((int64_t)1 << 16)

typedef struct {
  int32_t k, w;     /* chunk, worker (w unused by the server and update phases) */
  int64_t i0, i1;   /* chunk-relative element range [i0, i1) */
} orc_task;

typedef struct orc_mt orc_mt;
typedef void (*orc_phase_fn)(orc_mt* s, const orc_task* t, uint32_t* flags);

struct orc_mt {
  /* problem */
  int32_t W, C, dtype, err_dtype, optimizer;
  int64_t n, words;
  const int64_t* off;
  int64_t* wo;
  const void* grads;
  float clip, beta1, one_minus_b1, lr, eps;
  float *p, *m;
  const float* v;
  void *err, *srv_err;
  uint32_t *bits_w, *bits_srv;
  float *s_w, *s_srv;
  float* cw;     /* [W][n] compensated values */
  float* csrv;   /* [n] server values */
  float* r;      /* [C] LAMB trust ratios */
  /* current phase */
  orc_phase_fn fn;
  const orc_task* tasks;
  int64_t ntasks;
  int64_t next;  /* atomic task counter */
  uint32_t flags; /* atomic OR of the tasks' flags */
};

static void* orc_mt_worker(void* arg) {
  orc_mt* s = (orc_mt*)arg;
  uint32_t flags = 0;
  for (;;) {
    int64_t i = __atomic_fetch_add(&s->next, 1, __ATOMIC_RELAXED);
    if (i >= s->ntasks) break;
    s->fn(s, &s->tasks[i], &flags);
  }
  __atomic_fetch_or(&s->flags, flags, __ATOMIC_RELAXED);
  return NULL;
}

/* Run fn over the tasks on nthreads threads (the caller is one of them). */
static void orc_mt_run(orc_mt* s, int32_t nthreads, orc_phase_fn fn, const orc_task* tasks,
                       int64_t ntasks) {
  s->fn = fn;
  s->tasks = tasks;
  s->ntasks = ntasks;
  s->next = 0;
  int32_t extra = nthreads - 1;
  if (extra > ntasks - 1) extra = ntasks > 0 ? (int32_t)(ntasks - 1) : 0;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)(extra > 0 ? extra : 1));
  int32_t started = 0;
  for (int32_t j = 0; j < extra; ++j)
    if (pthread_create(&th[started], NULL, orc_mt_worker, s) == 0) ++started;
  orc_mt_worker(s); /* a failed pthread_create only means fewer threads */
  for (int32_t j = 0; j < started; ++j) pthread_join(th[j], NULL);
  free(th);
}

/* Task lists: element ranges of every (chunk, worker) with rows > 1, or one task
 * per (chunk, worker) with ranges = 0.  Returns the count (tasks may be NULL). */
static int64_t orc_mt_tasks(const orc_mt* s, int32_t rows, int ranges, orc_task* tasks) {
  int64_t t = 0;
  for (int32_t k = 0; k < s->C; ++k) {
    const int64_t nk = s->off[k + 1] - s->off[k];
    for (int32_t w = 0; w < rows; ++w) {
      if (!ranges) {
        if (tasks) { tasks[t].k = k; tasks[t].w = w; tasks[t].i0 = 0; tasks[t].i1 = nk; }
        ++t;
        continue;
      }
      for (int64_t i0 = 0; i0 < nk; i0 += ORC_MT_RANGE) {
        if (tasks) {
          tasks[t].k = k; tasks[t].w = w; tasks[t].i0 = i0;
          tasks[t].i1 = i0 + ORC_MT_RANGE < nk ? i0 + ORC_MT_RANGE : nk;
        }
        ++t;
      }
    }
  }
  return t;
}

/* 1: compensated values of worker w, as orc_compress forms them. */
static void ph_compensate(orc_mt* s, const orc_task* t, uint32_t* flags) {
  const int64_t o = s->off[t->k], e0 = (int64_t)t->w * s->n + o;
  float* c = s->cw + e0;
  for (int64_t i = t->i0; i < t->i1; ++i) {
    c[i] = clip_grad(grad_at(s->grads, s->dtype, e0 + i), s->clip) + err_get(s->err, s->err_dtype, e0 + i);
    if (is_nonfinite(c[i])) *flags |= ORC_STATUS_NONFINITE;
  }
}

/* 2: the worker scale of (k, w): one ascending sum. */
static void ph_worker_scale(orc_mt* s, const orc_task* t, uint32_t* flags) {
  (void)flags;
  const int64_t o = s->off[t->k], nk = s->off[t->k + 1] - o;
  s->s_w[(int64_t)t->w * s->C + t->k] = quantize_scale(s->cw + (int64_t)t->w * s->n + o, nk);
}

/* 3: sign words of the range (it starts on a word) and the worker error. */
static void ph_worker_pack(orc_mt* s, const orc_task* t, uint32_t* flags) {
  (void)flags;
  const int64_t o = s->off[t->k], e0 = (int64_t)t->w * s->n + o;
  const float* c = s->cw + e0;
  uint32_t* q = s->bits_w + (int64_t)t->w * s->words + s->wo[t->k];
  const float sc = s->s_w[(int64_t)t->w * s->C + t->k];
  quantize_signs(c + t->i0, t->i1 - t->i0, q + t->i0 / 32);
  for (int64_t i = t->i0; i < t->i1; ++i) err_set(s->err, s->err_dtype, e0 + i, c[i] - dequantize(q, sc, i));
}

/* 4: the server value, as orc_server_reduce forms it. */
static void ph_server_value(orc_mt* s, const orc_task* t, uint32_t* flags) {
  const int32_t k = t->k;
  const int64_t o = s->off[k];
  for (int64_t i = t->i0; i < t->i1; ++i) {
    float acc = 0.0f;
    for (int32_t w = 0; w < s->W; ++w)
      acc += dequantize(s->bits_w + (int64_t)w * s->words + s->wo[k], s->s_w[(int64_t)w * s->C + k], i);
    float avg = acc / (float)s->W;
    s->csrv[o + i] = avg + err_get(s->srv_err, s->err_dtype, o + i);
    if (is_nonfinite(s->csrv[o + i])) *flags |= ORC_STATUS_NONFINITE;
  }
}

/* 5: the server scale of chunk k: one ascending sum. */
static void ph_server_scale(orc_mt* s, const orc_task* t, uint32_t* flags) {
  (void)flags;
  const int64_t o = s->off[t->k], nk = s->off[t->k + 1] - o;
  s->s_srv[t->k] = quantize_scale(s->csrv + o, nk);
}

/* 6: server words and error, then the update of m (and p for Adam), as
 * orc_server_reduce and orc_adam_apply / orc_lamb_apply write them. */
static void ph_server_pack_update(orc_mt* s, const orc_task* t, uint32_t* flags) {
  const int32_t k = t->k;
  const int64_t o = s->off[k];
  const float* c = s->csrv + o;
  uint32_t* q = s->bits_srv + s->wo[k];
  const float sc = s->s_srv[k];
  quantize_signs(c + t->i0, t->i1 - t->i0, q + t->i0 / 32);
  for (int64_t i = t->i0; i < t->i1; ++i) err_set(s->srv_err, s->err_dtype, o + i, c[i] - dequantize(q, sc, i));
  for (int64_t i = t->i0; i < t->i1; ++i) {
    float g_hat = dequantize(q, sc, i);
    float mi = s->beta1 * s->m[o + i] + s->one_minus_b1 * g_hat;
    s->m[o + i] = mi;
    if (s->optimizer == ORC_ADAM) {
      float pi = s->p[o + i] - s->lr * mi / (sqrtf(s->v[o + i]) + s->eps);
      if (is_nonfinite(pi)) *flags |= ORC_STATUS_NONFINITE;
      s->p[o + i] = pi;
    }
  }
}

/* 7: LAMB trust ratio of layer k (pre-update p): one pair of ascending sums. */
static void ph_lamb_ratio(orc_mt* s, const orc_task* t, uint32_t* flags) {
  (void)flags;
  const int64_t o = s->off[t->k], nk = s->off[t->k + 1] - o;
  s->r[t->k] = trust_ratio(s->p + o, s->m + o, s->v + o, s->eps, nk);
}

/* 8: LAMB parameter step, as lamb_update_layer takes it. */
static void ph_lamb_param(orc_mt* s, const orc_task* t, uint32_t* flags) {
  const int64_t o = s->off[t->k];
  const float r = s->r[t->k];
  for (int64_t i = t->i0; i < t->i1; ++i) {
    float u = s->m[o + i] / (sqrtf(s->v[o + i]) + s->eps);
    float pi = s->p[o + i] - s->lr * r * u;
    if (is_nonfinite(pi)) *flags |= ORC_STATUS_NONFINITE;
    s->p[o + i] = pi;
  }
}

/*
 * One whole compressed-phase step on nthreads threads: the arguments and
 * results of orc_step, bit for bit.  Returns the status flags, or
 * ORC_STATUS_NONFINITE | 0x80000000u if a scratch allocation failed (nothing is
 * then written).
 */
uint32_t orc_step_mt(int32_t nthreads, int32_t W, int64_t n, int32_t C, const int64_t* off,
                     const void* grads, int32_t dtype, int32_t optimizer, float clip, float beta1,
                     float lr, float eps, float* p, float* m, const float* v, void* err,
                     void* srv_err, int32_t err_dtype, uint32_t* bits_w, float* s_w,
                     uint32_t* bits_srv, float* s_srv) {
  orc_mt s;
  memset(&s, 0, sizeof s);
  s.W = W; s.C = C; s.n = n; s.off = off; s.dtype = dtype; s.err_dtype = err_dtype;
  s.optimizer = optimizer; s.grads = grads; s.clip = clip; s.beta1 = beta1;
  s.one_minus_b1 = 1.0f - beta1; s.lr = lr; s.eps = eps;
  s.p = p; s.m = m; s.v = v; s.err = err; s.srv_err = srv_err;
  s.bits_w = bits_w; s.bits_srv = bits_srv; s.s_w = s_w; s.s_srv = s_srv;
  if (nthreads < 1) nthreads = 1;
  s.wo = (int64_t*)malloc(sizeof(int64_t) * (size_t)(C + 1));
  s.cw = (float*)malloc(sizeof(float) * (size_t)((int64_t)W * n > 0 ? (int64_t)W * n : 1));
  s.csrv = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
  s.r = (float*)malloc(sizeof(float) * (size_t)C);
  const int64_t n_wr = orc_mt_tasks(&s, W, 1, NULL), n_w1 = orc_mt_tasks(&s, W, 0, NULL);
  const int64_t n_sr = orc_mt_tasks(&s, 1, 1, NULL), n_s1 = orc_mt_tasks(&s, 1, 0, NULL);
  orc_task* t_wr = (orc_task*)malloc(sizeof(orc_task) * (size_t)(n_wr > 0 ? n_wr : 1));
  orc_task* t_w1 = (orc_task*)malloc(sizeof(orc_task) * (size_t)(n_w1 > 0 ? n_w1 : 1));
  orc_task* t_sr = (orc_task*)malloc(sizeof(orc_task) * (size_t)(n_sr > 0 ? n_sr : 1));
  orc_task* t_s1 = (orc_task*)malloc(sizeof(orc_task) * (size_t)(n_s1 > 0 ? n_s1 : 1));
  uint32_t result;
  if (!s.wo || !s.cw || !s.csrv || !s.r || !t_wr || !t_w1 || !t_sr || !t_s1) {
    result = ORC_STATUS_NONFINITE | 0x80000000u;
  } else {
    word_offsets(C, off, s.wo);
    s.words = s.wo[C];
    orc_mt_tasks(&s, W, 1, t_wr);
    orc_mt_tasks(&s, W, 0, t_w1);
    orc_mt_tasks(&s, 1, 1, t_sr);
    orc_mt_tasks(&s, 1, 0, t_s1);
    orc_mt_run(&s, nthreads, ph_compensate, t_wr, n_wr);
    orc_mt_run(&s, nthreads, ph_worker_scale, t_w1, n_w1);
    orc_mt_run(&s, nthreads, ph_worker_pack, t_wr, n_wr);
    orc_mt_run(&s, nthreads, ph_server_value, t_sr, n_sr);
    orc_mt_run(&s, nthreads, ph_server_scale, t_s1, n_s1);
    orc_mt_run(&s, nthreads, ph_server_pack_update, t_sr, n_sr);
    if (optimizer == ORC_LAMB) {
      orc_mt_run(&s, nthreads, ph_lamb_ratio, t_s1, n_s1);
      orc_mt_run(&s, nthreads, ph_lamb_param, t_sr, n_sr);
    }
    result = s.flags;
  }
  free(s.wo); free(s.cw); free(s.csrv); free(s.r);
  free(t_wr); free(t_w1); free(t_sr); free(t_s1);
  return result;
}
