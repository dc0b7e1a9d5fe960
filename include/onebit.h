/*
 * onebit.h -- C ABI of the B200 (sm_100a) 1-bit Adam compressed-phase library.
 *
 * The calls follow the step described in "DeepSpeed Communication Compression
 * and Hiding", section "1-bit Adam: 预热、冻结方差、误差反馈" (机制).  Before freeze_step
 * the averaged gradient drives ordinary Adam moments (m and v).  From then on
 * each worker adds its error buffer to its gradient, sends the sum as one sign
 * bit per element plus a scale, the workers' messages are combined by a
 * compressed allreduce and expanded back into a direction g_hat, the error
 * buffer keeps what quantisation dropped, m follows g_hat while v stays
 * frozen, and the parameters move by lr * m / (sqrt(v) + eps) --
 * with W data-parallel workers held in one GPU's memory.  Where the page gives
 * no formula the library fixes it as follows:
 *   - the gradient is cut into chunks (one per parameter tensor or per flat
 *     slice); each chunk has its own scale s = ||c||_2 / sqrt(n_k);
 *   - sign(c) is the bit (c >= 0.0f): +0 and -0 send +1, NaN sends -1;
 *   - element i of chunk k -> bit (i % 32) of word (i / 32) of that chunk's
 *     words; every chunk starts on a fresh uint32 word; padding bits are 0;
 *   - the worker error is local, err_w = c - s_wk * sign(c);
 *   - the compressed allreduce unpacks the W workers, averages the scaled signs
 *     (sum over w = 0..W-1 in float, then / W), adds a server error buffer,
 *     re-quantises that sum with its own per-chunk scale, and keeps
 *     srv_err = c_srv - s_srv * sign(c_srv); g_hat = s_srv * sign(c_srv);
 *   - norms are accumulated in double and rounded once to float;
 *   - no bias correction; the warmup averages the W gradients in float.
 * The 1-bit LAMB variant ("DeepSpeed Communication Compression and Hiding",
 * section "1-bit LAMB") replaces the last line by u = m / (sqrt(v) + eps),
 * r_l = ||p_l|| / ||u_l|| per layer (layer = chunk, pre-update p, r = 1 if
 * either norm is 0), p -= lr r_l u.  Clipping before quantisation (CANN 1-bit
 * Adam article, section 3.2) clamps the raw gradient to [-clip, clip].
 *
 * A second compression rule, the momentum-error rule of the CANN 1-bit Adam
 * article (sections 2.1, 2.2 and 3.2), is selected by ob_config.rule =
 * OB_RULE_MOMENTUM_ERROR.  Per worker and element:
 *   c = clip(g_w) + err_w;  q = sign(c) in {-1, 0, +1} (sign(+-0) = 0, no scale);
 *   err_w = beta1 err_w + (1 - beta1) (c - q)
 * q travels as an int8 code; the W codes of an element are summed (exact in
 * int8, so W <= 127), g_hat = sum / W, and m, p move as above (v frozen).
 * There is no server error and no scale under this rule.
 *
 * A third rule, 2-bit Adam (named by the CANN article, section 5.1, without a
 * quantiser), is selected by OB_RULE_TWO_BIT: the 1-bit quantiser applied twice,
 * the second time to what the first left over --
 *   s1 = ||c|| / sqrt(n_k), q1 = sign(c), r = c - s1 q1,
 *   s2 = ||r|| / sqrt(n_k), q2 = sign(r), err = r - s2 q2,
 * dequantised as s1 q1 + s2 q2 -- for the workers and, on their average plus
 * the server error, for the server.  ||r||^2 is formed from per-tile sums of
 * |c| and of its squared deviations (sum (|c| - s1)^2, an identity), so it
 * equals the sum of the squared float residuals to within their rounding
 * (2^-23 relative at most); the planes depend on s1 and c only.
 *
 * Conventions for every call:
 *   - Device buffers are caller-owned and must stay valid for the ctx's life.
 *     The ctx stores their pointers and owns only its own scratch (per-tile
 *     partial norms, chunk tables, status word), allocated in ob_create.
 *   - Element arrays (gradients, p, m, v, err, srv_err, staging) must be 32-byte
 *     aligned (cudaMalloc and the PyTorch caching allocator give 256 or more);
 *     packed words and scales (bits_w, bits_srv, s_w, s_srv, norm outputs) 4-byte
 *     aligned; otherwise OB_EINVAL.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work on it and return; none synchronises except
 *     ob_get_status and ob_create.
 *   - Calls return ob_err and never abort or trap.  On failure
 *     ob_last_error() returns a message (thread-local, valid until the next
 *     call on the same thread).
 *   - Calls on one ctx must be ordered (same stream, or synchronised); ctxs
 *     that share a state buffer must order their calls the same way.
 *   - The step counter advances in ob_warmup_step, ob_step and ob_step_host,
 *     never in the stage calls.
 */
#ifndef ONEBIT_H_
#define ONEBIT_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ob_ctx ob_ctx; /* opaque */

typedef enum {
  OB_OK = 0,
  OB_EINVAL = -1, /* bad argument: null/misaligned pointer, bad size or layout */
  OB_ECUDA = -2,  /* a CUDA runtime call or kernel launch failed */
  OB_EPHASE = -3, /* call not allowed in the current phase (warmup vs compressed) */
  OB_ENOMEM = -4  /* scratch allocation failed */
} ob_err;

enum { OB_F32 = 0, OB_BF16 = 1 };  /* gradient element type */
enum { OB_ADAM = 0, OB_LAMB = 1 }; /* update rule after the compressed allreduce */
enum {                             /* compression rule (ob_config.rule) */
  OB_RULE_SCALED_SIGN = 0,         /* sign bits + per-chunk scale, worker and server error */
  OB_RULE_MOMENTUM_ERROR = 1,      /* int8 ternary codes, momentum-form worker error */
  OB_RULE_TWO_BIT = 2              /* two residual sign planes, two scales per chunk */
};

#define OB_STATUS_NONFINITE 1u /* a compensated value, server value or parameter was NaN/Inf */

typedef struct {
  int64_t n;                    /* total elements (parameters); >= 0 */
  int32_t num_chunks;           /* C >= 1 */
  const int64_t* chunk_offsets; /* HOST array of C+1 entries: [0] = 0, non-decreasing, [C] = n;
                                   copied in ob_create.  Empty chunks are allowed (scale 0). */
  int32_t W;                    /* virtual workers, 1 <= W <= 1024 */
  int32_t grad_dtype;           /* OB_F32 or OB_BF16 */
  int32_t optimizer;            /* OB_ADAM or OB_LAMB (LAMB layers = chunks) */
  float lr, beta1, beta2, eps;
  float clip;                   /* <= 0: off; else clamp the raw gradient to [-clip, clip] */
  int32_t freeze_step;          /* steps 0..freeze_step-1 are full-precision warmup */
  int32_t err_dtype;            /* OB_F32, or OB_BF16: err and srv_err stored as bfloat16
                                   (rounded to nearest even; arithmetic stays float32) --
                                   half the error-buffer bytes, different rounding */
  int32_t rule;                 /* OB_RULE_SCALED_SIGN (default 0), OB_RULE_MOMENTUM_ERROR
                                   (then W <= 127) or OB_RULE_TWO_BIT */
} ob_config;

/* Number of uint32 words one packed row holds.  OB_RULE_SCALED_SIGN: sign bits,
 * sum_k ceil(n_k / 32).  OB_RULE_MOMENTUM_ERROR: int8 codes, sum_k ceil(n_k / 4);
 * element i of chunk k is byte i of the chunk's words (byte b of a word is bits
 * 8b..8b+7), every chunk starts on a fresh word, padding bytes are 0.
 * OB_RULE_TWO_BIT: sum_k 2 ceil(n_k / 32) -- chunk k's words hold plane 1 then
 * plane 2, each laid out like the sign bits.
 * Host-only; validates the config.  words_total must be non-NULL. */
ob_err ob_layout(const ob_config* cfg, int64_t* words_total);

/* Create a ctx: the optimizer state of the CANN 1-bit Adam article, section 3.1
 * (OneBitAdamState: an error-feedback buffer of the parameters' shape, the
 * first and second moments, beta1/beta2/eps and the step count), here with one
 * error buffer per worker, the server error buffer, the packed messages and
 * their scales, all caller-owned.
 * Create it over caller-owned DEVICE buffers (float32 unless stated):
 *   p, m, v: [n];  err: [W][n] (worker-major), srv_err: [n], both of err_dtype;
 *   bits_w: uint32 [W][words_total];  s_w: [W][C];
 *   bits_srv: uint32 [words_total];  s_srv: [C].
 * Does not initialise them (the caller sets p, m, v; err and srv_err start at 0).
 * A buffer may be NULL when the ctx never makes a call that touches it; calls
 * return OB_EINVAL when one of theirs is missing:
 *   ob_warmup_step: p, m, v          ob_compress: err, bits_w, s_w
 *   ob_server_reduce: srv_err, bits_w, s_w, bits_srv, s_srv
 *   ob_step(NULL): p, m, v, bits_srv, s_srv    ob_step(grads), ob_step_host: all
 * (e.g. a rank that owns some chunks in a multi-GPU step keeps a server-only
 * ctx).  Several ctxs may share a buffer if their calls are ordered.
 * Under OB_RULE_MOMENTUM_ERROR: bits_w holds the workers' int8 codes and
 * bits_srv their per-element sums (int8), both in the ob_layout words; srv_err,
 * s_w and s_srv are never used (pass NULL); ob_compress needs err and bits_w,
 * ob_server_reduce bits_w and bits_srv, ob_step(NULL) p, m, v and bits_srv, and
 * ob_step(grads) p, m, v and err only.
 * Under OB_RULE_TWO_BIT: bits_w / bits_srv hold both planes (ob_layout words),
 * and s_w is [W][C][2], s_srv [C][2] (plane 1, plane 2 of each chunk).
 * Allocates the ctx scratch with cudaMalloc on the current device and
 * synchronises once.  The scratch holds the chunk tables and per-tile partial
 * sums; with W >= 4 and every buffer of the fused step given (scaled-sign and
 * 2-bit rules) it also holds one float per element for the fused step's server
 * value.  *out receives the ctx (NULL on failure). */
ob_err ob_create(const ob_config* cfg, float* p, float* m, float* v, void* err,
                 void* srv_err, uint32_t* bits_w, float* s_w, uint32_t* bits_srv,
                 float* s_srv, ob_ctx** out);

/* One full-precision warmup step ("DeepSpeed Communication Compression and
 * Hiding": the `step < freeze_step` branch of the listing in section "1-bit
 * Adam" 机制 -- average the workers' gradients, then the Adam moments of section
 * "基线：Adam 为什么难压缩" -- and the listing's last line, the parameter update);
 * step < freeze_step, else OB_EPHASE:
 *   g = (sum_w g_w) / W;  m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;
 *   Adam: p -= lr m / (sqrt(v) + eps);  LAMB: per-layer trust-ratio update.
 * grads: DEVICE [W][n] of grad_dtype.  Error buffers are not touched. */
ob_err ob_warmup_step(ob_ctx* ctx, const void* grads, void* stream);

/* Variance refresh of 0/1 Adam ("DeepSpeed Communication Compression and
 * Hiding", section "0/1 Adam"): the same full-precision step as
 * ob_warmup_step -- Adam (or LAMB) moments m AND v from the averaged gradient,
 * then the parameter update -- allowed in any phase, so the frozen variance is
 * refreshed between compressed steps.  Error buffers are not touched.  The
 * pages give no refresh schedule; the caller chooses the steps.  Advances the
 * step counter. */
ob_err ob_refresh_step(ob_ctx* ctx, const void* grads, void* stream);

/* The warmup's synchronisation alone ("DeepSpeed Communication Compression and
 * Hiding", section "1-bit Adam" 机制: the listing's `g = allreduce(local_grad)`
 * line before freeze_step, read as the float32 mean of the workers'
 * gradients): mean[i] = (sum_{w=0..W-1} g_w[i]) / W, float additions in
 * ascending w and one division, as ob_warmup_step forms it.  grads: DEVICE
 * [W][n] of grad_dtype; mean: DEVICE float32 [n], 32-byte aligned.  An
 * ob_warmup_step on a one-worker float32 ctx over `mean` then leaves p, m and v
 * as ob_warmup_step on the W gradients does, so a data-parallel driver can
 * average each owner's slice of the gradients instead of gathering every
 * worker's whole gradient.  Any phase; the step counter is unchanged; a
 * non-finite mean raises OB_STATUS_NONFINITE. */
ob_err ob_mean_grads(ob_ctx* ctx, const void* grads, float* mean, void* stream);

/* Worker stage only ("DeepSpeed Communication Compression and Hiding", section
 * "1-bit Adam" 机制, the listing's `compensated = local_grad + error`,
 * `q, scale = one_bit_quantize(compensated)` and -- for the worker's own part of
 * the residual -- `error = compensated - g_hat` lines; compressed phase): for
 * every worker and chunk,
 * c = clip(g_w) + err_w, s_w = ||c|| / sqrt(n_k), bits_w = sign(c),
 * err_w = c - s_w sign(c).  grads: DEVICE [W][n].  Step counter unchanged.
 * OB_RULE_MOMENTUM_ERROR: bits_w = int8 codes sign(c), err_w = beta1 err_w +
 * (1 - beta1)(c - sign(c)). */
ob_err ob_compress(ob_ctx* ctx, const void* grads, void* stream);

/* Server stage only ("DeepSpeed Communication Compression and Hiding", section
 * "1-bit Adam" 机制, the listing's `q_global = compressed_allreduce(q, scale)`
 * line: average the workers' messages and re-compress them with a server error
 * buffer) from bits_w / s_w:
 * c_srv = mean_w(s_w sign_w) + srv_err, s_srv = ||c_srv|| / sqrt(n_k),
 * bits_srv = sign(c_srv), srv_err = c_srv - s_srv sign(c_srv).
 * OB_RULE_MOMENTUM_ERROR: bits_srv = per-element sum of the W int8 codes. */
ob_err ob_server_reduce(ob_ctx* ctx, void* stream);

/* The compressed-phase step ("DeepSpeed Communication Compression and Hiding",
 * section "1-bit Adam" 机制: the listing's `else` branch, then
 * `g_hat = dequantize(q_global)`, `m = beta1 * m + (1 - beta1) * g_hat` with v
 * frozen, and `param -= lr * m / (sqrt(v_frozen) + eps)`; section "1-bit LAMB"
 * for the trust-ratio update under OB_LAMB).
 * grads != NULL: the whole fused compressed step (worker stage, server stage,
 * update) on DEVICE grads [W][n].  grads == NULL: the update alone from
 * bits_srv / s_srv (g_hat = s_srv sign), after ob_compress + ob_server_reduce.
 * Advances the step counter.  OB_EPHASE while step < freeze_step.
 * OB_RULE_MOMENTUM_ERROR: g_hat = (int8 sum in bits_srv) / W; the fused step is
 * one pass over the elements that keeps the codes in registers, so it writes
 * neither bits_w nor bits_srv. */
ob_err ob_step(ob_ctx* ctx, const void* grads, void* stream);

/* The same passage as ob_step ("DeepSpeed Communication Compression and
 * Hiding", section "1-bit Adam" 机制, the compressed-phase branch and update),
 * with the gradients in HOST memory:
 * copies [W][n] grad_dtype elements from host_grads into dev_staging (a
 * caller-owned DEVICE buffer of that size, 32-byte aligned), then runs the
 * fused step on `stream`.  The copy runs on an internal copy stream (created on
 * the first call, with a few events) and waits only for the kernels that last
 * read the same dev_staging buffer; `stream` waits for the copy.  Passing two
 * staging buffers alternately therefore overlaps the upload of one step's
 * gradients with the previous step's compute.  host_grads should be page-
 * locked, and must stay unchanged until `stream` has passed this step.
 * Advances the step counter. */
ob_err ob_step_host(ob_ctx* ctx, const void* host_grads, void* dev_staging, void* stream);

/* Destroy a ctx and free its scratch (not the caller's buffers).  NULL is OK. */
ob_err ob_destroy(ob_ctx* ctx);

/* Copy the status flags (OB_STATUS_*) accumulated since the last clear into
 * *flags (HOST); synchronises `stream`.  If clear != 0 the flags are reset. */
ob_err ob_get_status(ob_ctx* ctx, uint32_t* flags, int32_t clear, void* stream);

/* Step counter (number of completed warmup + compressed steps) for
 * checkpoint/resume.  ob_get_step returns -1 for a NULL ctx. */
int64_t ob_get_step(const ob_ctx* ctx);
ob_err ob_set_step(ob_ctx* ctx, int64_t step);

/* Error-feedback monitoring (CANN 1-bit Adam article, sections 6.2 and 8:
 * watch the L2 norm of the error buffers; a norm that collapses towards 0
 * signals vanishing updates): writes ||err_w restricted to chunk k||_2 to
 * worker_norms[w * C + k] and ||srv_err on chunk k||_2 to server_norms[k]
 * (DEVICE float arrays; either may be NULL; server_norms must be NULL under
 * OB_RULE_MOMENTUM_ERROR).  Norms are summed in double in a fixed order.  Uses the ctx scratch, so it must be ordered with the ctx's
 * steps (same stream); it does not change any state. */
ob_err ob_error_norms(ob_ctx* ctx, float* worker_norms, float* server_norms, void* stream);

/* Quantisation-rate monitoring (CANN 1-bit Adam article, section 8, "监控指标":
 * watch the gradient quantisation rate, which should stay near its theoretical
 * value).  The article gives no formula; here the rate of a chunk is the
 * fraction of its n_k elements sent as +1 (sign bit set), whose theoretical
 * value is 1/2 for a message symmetric about zero.  Writes, from the sign words
 * the last step or stage call left in bits_w / bits_srv,
 *   worker_rates[(w * C + k) * planes + p]  and  server_rates[k * planes + p]
 * (DEVICE float arrays, 4-byte aligned; either may be NULL; planes = 2 under
 * OB_RULE_TWO_BIT -- plane 1 the signs of c, plane 2 the signs of its residual --
 * else 1) as (float)(count / n_k), the count taken over the n_k real bits only;
 * an empty chunk gives 0.  OB_EINVAL under OB_RULE_MOMENTUM_ERROR (ternary codes,
 * no sign bits).  Uses the ctx scratch, so it must be ordered with the ctx's
 * steps (same stream); it changes no state. */
ob_err ob_quant_rates(ob_ctx* ctx, float* worker_rates, float* server_rates, void* stream);

/* 0/1 Adam local step ("DeepSpeed Communication Compression and Hiding",
 * section "0/1 Adam": local updates lower the synchronisation frequency; the
 * listing moves param with the current m and v on every step and updates m only
 * from a synchronised g_hat).  The page gives no formula for a local step; here
 * it sends nothing, keeps each worker's gradient for the next synchronised
 * step in its error buffer, and moves the parameters with the current m and v:
 *   err_w = clip(g_w) + err_w   (every worker; the worker stage's addition)
 *   Adam: p = p - lr m / (sqrt(v) + eps)
 *   LAMB: u = m / (sqrt(v) + eps), r_l = ||p_l|| / ||u_l||, p -= lr r_l u
 * m, v, srv_err and the packed words are untouched.  grads: DEVICE [W][n] of
 * grad_dtype.  Compressed phase only (OB_EPHASE while step < freeze_step); the
 * caller chooses which steps are local (the page gives no schedule).  OB_EINVAL
 * under OB_RULE_MOMENTUM_ERROR, whose error buffer is a momentum, not a sum.
 * Advances the step counter. */
ob_err ob_local_step(ob_ctx* ctx, const void* grads, void* stream);

/* ---- profiling (not part of the method) ----------------------------------
 * Kernel kinds the library launches, for per-kernel timing: */
enum {
  OB_K_WORKER_NORM = 0,    /* pass 1: per-tile sums of c^2, every worker */
  OB_K_FINALIZE_SCALE = 1, /* per-chunk scale from tile partials */
  OB_K_WORKER_PACK = 2,    /* pass 2: signs, worker error (+ server sums when fused) */
  OB_K_SERVER_NORM = 3,    /* server sums alone (stage call) */
  OB_K_SERVER_UPDATE = 4,  /* pass 3: server signs + error, and/or the update */
  OB_K_LAMB_PARAM = 5,     /* LAMB parameter step */
  OB_K_WARMUP = 6,         /* full-precision warmup step */
  OB_K_FINALIZE_RATIO = 7, /* LAMB trust ratio per layer */
  OB_K_TERNARY_STEP = 8,     /* momentum-error rule: the fused one-pass step */
  OB_K_TERNARY_COMPRESS = 9, /* momentum-error rule: codes + worker error (stage call) */
  OB_K_TERNARY_SERVER = 10,  /* momentum-error rule: sum of the workers' codes */
  OB_K_TERNARY_UPDATE = 11,  /* momentum-error rule: update from the code sums */
  OB_K_TB_WORKER_NORM = 12,  /* 2-bit pass 1: per-tile sums of c^2 and moments of |c|, every worker */
  OB_K_TB_PACK = 13,         /* 2-bit: both planes, worker error (+ server sums) */
  OB_K_TB_SERVER_NORM = 14,  /* 2-bit: server sums from the planes (stage call) */
  OB_K_TB_SERVER_UPDATE = 15,/* 2-bit: server planes + error, and/or the update */
  /* The fused step with W >= 4 workers: pass 2 also stores the server value
   * c_srv (one float per element, in the ctx scratch) and pass 3 reads it
   * instead of rebuilding it from the W workers' words. */
  OB_K_WORKER_PACK_CACHED = 16,
  OB_K_SERVER_UPDATE_CACHED = 17,
  OB_K_TB_PACK_CACHED = 18,
  OB_K_TB_FINALIZE = 19,     /* 2-bit: both scales of every chunk from the tile sums */
  OB_K_TB_SERVER_UPDATE_CACHED = 20,
  OB_K_LOCAL_STEP = 21,      /* 0/1 Adam local step */
  OB_K_SIGN_COUNT = 22,      /* quantisation rate: per-tile counts of set sign bits */
  OB_K_GRAD_MEAN = 23,       /* full-precision average of the workers' gradients */
  OB_K_KINDS = 24
};

/* Start recording a CUDA event pair around each of the next `capacity`
 * kernel launches of this ctx, on the stream each is launched on.  Creates
 * 2*capacity events (a set-up call: do it outside any timed region).
 * capacity must be in [1, 1<<20]. */
ob_err ob_profile_start(ob_ctx* ctx, int32_t capacity);

/* Stop recording, wait for the recorded events, and write per kind the total
 * elapsed milliseconds ms[OB_K_KINDS] and the number of timed launches
 * launches[OB_K_KINDS] (both HOST arrays).  Destroys the events. */
ob_err ob_profile_stop(ob_ctx* ctx, double* ms, int64_t* launches);

/* Name of a kernel kind ("" if out of range). */
const char* ob_kernel_name(int32_t kind);

/* Kernel launches this ctx has enqueued since ob_create (-1 for NULL). */
int64_t ob_launch_count(const ob_ctx* ctx);

/* ---- worker stage for callers that cannot allocate --------------------------
 * The paper has no counterpart to this call; it exists for integration.
 * Some callers must not allocate device memory at all: code whose GPU memory is
 * owned by another allocator (a framework's caching pool that has reserved the
 * device up front, where a raw cudaMalloc could fail or fragment the pool) and
 * code on a latency-critical path (a gradient hook inside a training step),
 * where cudaMalloc/cudaFree may synchronise the device.  Such callers cannot
 * use ob_create, which allocates the ctx scratch.
 *
 * ob_compress_noalloc is the worker stage of ob_compress without a ctx and
 * without any allocation: for every worker w and chunk k,
 *   c = clip(g_w) + err_w,  s_w[w][k] = ||c|| / sqrt(n_k),  bits_w = sign(c),
 *   err_w = c - s_w sign(c)
 * with results identical to ob_compress on the same inputs.  The caller passes
 * the config and DEVICE buffers as for ob_create/ob_compress: grads [W][n]
 * (grad_dtype), err [W][n] (float32, in/out; err_dtype must be OB_F32 and
 * rule OB_RULE_SCALED_SIGN),
 * bits_w [W][words_total], s_w [W][C]; 32-byte aligned.  lr, betas, eps and
 * freeze_step are ignored.
 *
 * Scratch: a fixed 8 MiB array in the library's device memory (every GPU that
 * loads the library holds it until the process exits), used for the chunk
 * tables and one double per (worker, 512-element tile).  Calls needing more --
 * about W*n above 5.3e8 elements, or more than 4096 chunks -- return
 * OB_EINVAL with a message, before any work is enqueued.  All calls share the
 * array: two calls whose work overlaps on the GPU (different streams, or
 * different host threads without ordering) race and give wrong results;
 * order them on one stream.  Each call rewrites the tables and clears the
 * status word it uses.  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current.  The chunk
 * tables are copied from a host buffer that every call rewrites, so the call
 * returns OB_EINVAL while `stream` is being captured into a CUDA graph.
 * Non-finite input: there is no status word to read back; instead a NaN or
 * infinite compensated value c in chunk k of worker w makes s_w[w][k] NaN or
 * infinite (the scale of a chunk of finite values is always finite), so a
 * caller checks the scales. */
ob_err ob_compress_noalloc(const ob_config* cfg, const void* grads, float* err,
                           uint32_t* bits_w, float* s_w, void* stream);

/* Message of the last failed call on this thread ("" if none). */
const char* ob_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ONEBIT_H_ */
