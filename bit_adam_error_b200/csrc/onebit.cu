// onebit.cu -- host side of the C ABI declared in include/onebit.h.
//
// Validates arguments, owns the per-ctx scratch (chunk tables, per-tile partial
// norms, LAMB ratios, status word, and for W >= 4 the fused step's server values)
// and enqueues the kernels of the ctx's rule on the caller's stream: kernels.cuh
// (scaled sign bits), ternary.cuh (the momentum-error rule's int8 codes),
// twobit.cuh (2-bit Adam's two planes).  After ob_create no call allocates device memory; the step
// calls only enqueue work.  ob_get_status synchronises the stream (one 4-byte
// read-back); ob_step_host creates its copy stream and events on first use;
// ob_profile_start/stop create, wait for and destroy CUDA events; ob_destroy
// waits for the copy stream.  ob_compress_noalloc (end of file) uses a fixed
// static scratch array instead of a ctx.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>
#include <type_traits>
#include <vector>

#include <cuda_runtime.h>

#include "onebit.h"
#include "kernels.cuh"
#include "ternary.cuh"
#include "twobit.cuh"

namespace {

thread_local char g_last_error[512] = "";

ob_err fail(ob_err code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return code;
}

ob_err cuda_fail(cudaError_t e, const char* what) {
  return fail(OB_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Element arrays need 32 bytes: the kernels move 8 fp32 elements per lane in one
// 256-bit access.  Packed words and scales are read and written one 4-byte word
// at a time, so 4 bytes suffice (slices of them can start on any word).
constexpr uintptr_t kAlignElems = 32, kAlignWords = 4;

// From this many workers on, the fused step's pass 2 stores c_srv (4 bytes per
// element) and pass 3 reads it back instead of rebuilding the server sum from
// the W workers' words, which is bound by per-element work at large W.
constexpr int32_t kCacheMinW = 4;

int64_t words_of(int64_t n) { return (n + 31) / 32; }

bool momentum_rule(const ob_config* c) { return c->rule == OB_RULE_MOMENTUM_ERROR; }
bool two_bit_rule(const ob_config* c) { return c->rule == OB_RULE_TWO_BIT; }

// Scales per chunk: one, or two for the two planes of the 2-bit rule.
int64_t scale_planes(const ob_config* c) { return two_bit_rule(c) ? 2 : 1; }

// Words of one chunk in a packed row: sign bits, int8 codes four to a word, or
// two sign planes.
int64_t row_words_of(const ob_config* c, int64_t nk) {
  if (momentum_rule(c)) return (nk + 3) / 4;
  return scale_planes(c) * words_of(nk);
}

// The int8 sum of W codes in {-1, 0, 1} is exact up to this many workers.
constexpr int32_t kMaxMomentumWorkers = 127;

// Checks everything about a config that needs no device.
ob_err check_config(const ob_config* c) {
  if (!c) return fail(OB_EINVAL, "config is NULL");
  if (c->n < 0) return fail(OB_EINVAL, "n = %lld < 0", (long long)c->n);
  if (c->num_chunks < 1) return fail(OB_EINVAL, "num_chunks = %d < 1", c->num_chunks);
  if (!c->chunk_offsets) return fail(OB_EINVAL, "chunk_offsets is NULL");
  if (c->chunk_offsets[0] != 0) return fail(OB_EINVAL, "chunk_offsets[0] must be 0");
  for (int32_t k = 0; k < c->num_chunks; ++k)
    if (c->chunk_offsets[k + 1] < c->chunk_offsets[k])
      return fail(OB_EINVAL, "chunk_offsets decrease at chunk %d", k);
  if (c->chunk_offsets[c->num_chunks] != c->n)
    return fail(OB_EINVAL, "chunk_offsets[C] = %lld != n = %lld",
                (long long)c->chunk_offsets[c->num_chunks], (long long)c->n);
  if (c->W < 1 || c->W > 1024) return fail(OB_EINVAL, "W = %d outside [1, 1024]", c->W);
  if (c->grad_dtype != OB_F32 && c->grad_dtype != OB_BF16)
    return fail(OB_EINVAL, "grad_dtype = %d is neither OB_F32 nor OB_BF16", c->grad_dtype);
  if (c->optimizer != OB_ADAM && c->optimizer != OB_LAMB)
    return fail(OB_EINVAL, "optimizer = %d is neither OB_ADAM nor OB_LAMB", c->optimizer);
  const float hp[] = {c->lr, c->beta1, c->beta2, c->eps, c->clip};
  for (float x : hp)
    if (!std::isfinite(x)) return fail(OB_EINVAL, "hyper-parameters must be finite");
  if (c->freeze_step < 0) return fail(OB_EINVAL, "freeze_step = %d < 0", c->freeze_step);
  if (c->err_dtype != OB_F32 && c->err_dtype != OB_BF16)
    return fail(OB_EINVAL, "err_dtype = %d is neither OB_F32 nor OB_BF16", c->err_dtype);
  if (c->rule != OB_RULE_SCALED_SIGN && c->rule != OB_RULE_MOMENTUM_ERROR && c->rule != OB_RULE_TWO_BIT)
    return fail(OB_EINVAL, "rule = %d is not OB_RULE_SCALED_SIGN, OB_RULE_MOMENTUM_ERROR or OB_RULE_TWO_BIT",
                c->rule);
  if (momentum_rule(c) && c->W > kMaxMomentumWorkers)
    return fail(OB_EINVAL, "W = %d > %d: the int8 sum of the codes could overflow", c->W, kMaxMomentumWorkers);
  // Element and word indices of [W][n] rows must fit in int64 comfortably.
  if (c->n > (int64_t(1) << 50) / c->W) return fail(OB_EINVAL, "W * n too large");
  return OB_OK;
}

// A device buffer argument: NULL only when it holds no element; aligned to
// `align` bytes; device (or managed) memory of the current device.
ob_err check_dev(const void* p, int64_t count, const char* name, int device,
                 uintptr_t align = kAlignElems) {
  if (count == 0) return OB_OK;
  if (!p) return fail(OB_EINVAL, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % align != 0)
    return fail(OB_EINVAL, "%s is not %d-byte aligned", name, int(align));
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, name);
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(OB_EINVAL, "%s is not device memory", name);
  if (a.type == cudaMemoryTypeDevice && a.device != device)
    return fail(OB_EINVAL, "%s lives on device %d, ctx on device %d", name, a.device, device);
  return OB_OK;
}

}  // namespace

struct ob_ctx {
  ob_config cfg;
  std::vector<int64_t> off;       // host copy of the chunk offsets
  int64_t words = 0, T = 0;
  int device = 0, num_sms = 0;
  int64_t step = 0;
  float *p, *m, *v, *s_w, *s_srv;
  void *err, *srv_err;              // float32 or bfloat16 (cfg.err_dtype)
  uint32_t *bits_w, *bits_srv;
  // scratch (one cudaMalloc)
  void* scratch = nullptr;
  ob::Layout L{};
  double *part_w = nullptr, *part_srv = nullptr, *partP = nullptr, *partU = nullptr;
  float* csrv = nullptr;            // c_srv of the fused step's pass 2 (W >= kCacheMinW), else NULL
  float* ratio = nullptr;
  uint32_t* status = nullptr;
  unsigned* ticket = nullptr;       // the fused finaliser's CTA counter (zero between launches)
  ob::Hyper h{};
  const void* grads_checked = nullptr;   // last grads pointer that passed check_dev
  std::vector<std::pair<const void*, int>> occ;  // kernel -> resident CTAs per SM
  // ob_step_host: internal copy stream, "copied" event, and per staging buffer
  // an event recorded after the last kernels that read it.
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t copied = nullptr;
  struct Staging { const void* ptr = nullptr; cudaEvent_t free_ev = nullptr; bool used = false; };
  Staging staging[4];
  int staging_next = 0;
  // profiling: event pairs around launches
  int64_t launches = 0;
  bool prof_on = false;
  int32_t prof_cap = 0, prof_used = 0;
  std::vector<cudaEvent_t> prof_ev;
  std::vector<int32_t> prof_kind;
};

namespace {

// Persistent grid: enough CTAs to cover `warps` warp-items, at most one full
// wave of resident CTAs (num_sms x occupancy).
template <typename K>
int grid_for(ob_ctx* c, K kernel, int64_t warps) {
  const void* key = reinterpret_cast<const void*>(kernel);
  int per_sm = 0;
  for (auto& kv : c->occ)
    if (kv.first == key) per_sm = kv.second;
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, ob::kBlock, 0) != cudaSuccess ||
        per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
    c->occ.emplace_back(key, per_sm);
  }
  const int64_t need = (warps + ob::kWarpsPerBlock - 1) / ob::kWarpsPerBlock;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(need, int64_t(c->num_sms) * per_sm)));
}

// Run fn with the ctx's device current; restore the caller's device after.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the stream's previous kernel finishes, and waits for it (every kernel
// starts with pdl_enter) before touching memory.  Should a stream refuse the
// attribute, the same kernel is launched plainly (same results, no overlap).
// Launch errors surface through cudaGetLastError like those of <<<>>> launches.
template <typename... P, typename... A>
void pdl(void (*kernel)(P...), dim3 grid, unsigned block, cudaStream_t st, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess) return;
  cudaGetLastError();
  cfg.numAttrs = 0;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

// Enqueue one kernel launch (fn), with an event pair around it while profiling.
template <typename Fn>
void launch(ob_ctx* c, int kind, cudaStream_t st, Fn&& fn) {
  const bool rec = c->prof_on && c->prof_used < c->prof_cap;
  if (rec) cudaEventRecord(c->prof_ev[2 * c->prof_used], st);
  fn();
  if (rec) {
    cudaEventRecord(c->prof_ev[2 * c->prof_used + 1], st);
    c->prof_kind[c->prof_used++] = kind;
  }
  ++c->launches;
}

ob_err check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return OB_OK;
}

ob_err check_grads(ob_ctx* c, const void* grads) {
  if (grads == c->grads_checked && grads) return OB_OK;
  const int64_t count = int64_t(c->cfg.W) * c->cfg.n;
  ob_err r = check_dev(grads, count, "grads", c->device);
  if (r == OB_OK) c->grads_checked = grads;
  return r;
}

// ---- enqueue helpers (no validation) ----------------------------------------------

// Per-chunk scales from the tile partials of each row (rows of row_stride slots).
void enqueue_finalize_scale(ob_ctx* c, const double* part, float* out, int rows, int64_t row_stride,
                            cudaStream_t st) {
  launch(c, OB_K_FINALIZE_SCALE, st, [&] {
    pdl(ob::k_finalize_scale<true>, dim3(c->cfg.num_chunks, rows), ob::kFinalizeThreads, st, c->L, part,
        row_stride, out);
  });
}

// W a power of two: the server mean is an exact multiply (see ob::Mean).
bool pow2_workers(const ob_ctx* c) { return (c->cfg.W & (c->cfg.W - 1)) == 0; }

// Pass 2 issues one group of a tile at a time (3 CTAs per SM) up to this many
// workers, two groups at a time (2 CTAs per SM) above it -- measured on B200:
// W = 1 bf16 3.19 vs 3.47 ms per 1.5e9 elements, W = 16 fp32 10.30 vs 10.05 ms.
// With bf16 error buffers two groups win at W = 1 too (3.13 vs 2.80 ms).
constexpr int kPackOneGroupMaxW = 2;

// Problems this small take the fused finaliser (the pass's last CTA computes the
// scales, see ob::fused_finalize) instead of a separate finaliser launch: at most
// this many tile partials and (row, chunk) pairs, so the last CTA's share stays
// a few microseconds.  The stage calls decide the same way, so on a given
// problem the fused step and the stages compute every scale alike.
constexpr int64_t kFinMaxPartials = int64_t(1) << 15;
constexpr int64_t kFinMaxTasks = 64;

bool fused_fin(const ob_ctx* c, int64_t rows) {
  return c->T > 0 && rows * c->T <= kFinMaxPartials && rows * c->cfg.num_chunks <= kFinMaxTasks;
}

template <typename GT, typename ET, bool CLIP, bool POW2>
void enqueue_worker_t(ob_ctx* c, const GT* grads, bool with_server, cudaStream_t st) {
  const int W = c->cfg.W;
  ET* err = static_cast<ET*>(c->err);
  const ET* srv_err = static_cast<const ET*>(c->srv_err);
  const bool fin1 = fused_fin(c, W), fin2 = with_server && fused_fin(c, 1);
  if (c->T > 0 && fin1) {
    auto k1 = ob::k_worker_norm_fin<GT, ET, CLIP>;
    const int g1 = grid_for(c, k1, W * c->T);
    const ob::Fin f{c->ticket, c->part_w, c->T, W, c->s_w};
    launch(c, OB_K_WORKER_NORM, st, [&] {
      pdl(k1, g1, ob::kBlock, st, c->L, W, grads, err, c->h.clip, c->part_w, c->status, f);
    });
  } else if (c->T > 0) {
    auto k1 = ob::k_worker_norm<GT, ET, CLIP>;
    const int g1 = grid_for(c, k1, W * c->T);
    launch(c, OB_K_WORKER_NORM, st, [&] {
      pdl(k1, g1, ob::kBlock, st, c->L, W, grads, err, c->h.clip, c->part_w, c->status);
    });
  }
  if (!fin1) enqueue_finalize_scale(c, c->part_w, c->s_w, W, c->T, st);
  if (c->T > 0) {
    // The stage call (no server part) never uses the mean: one instantiation each.
    // Many workers: the fused step also stores c_srv for pass 3 (CACHE).
    const bool one = W <= kPackOneGroupMaxW && !std::is_same<ET, uint16_t>::value;
    const bool cache = with_server && c->csrv;
    const int kind = cache ? OB_K_WORKER_PACK_CACHED : OB_K_WORKER_PACK;
    if (fin2) {
      auto k2 = cache ? (one ? ob::k_worker_pack_fin<GT, ET, true, CLIP, POW2, 1, true>
                             : ob::k_worker_pack_fin<GT, ET, true, CLIP, POW2, 2, true>)
                      : (one ? ob::k_worker_pack_fin<GT, ET, true, CLIP, POW2, 1, false>
                             : ob::k_worker_pack_fin<GT, ET, true, CLIP, POW2, 2, false>);
      const int g2 = grid_for(c, k2, c->T);
      const ob::Fin f{c->ticket, c->part_srv, 0, 1, c->s_srv};
      launch(c, kind, st, [&] {
        pdl(k2, g2, ob::kBlock, st, c->L, W, grads, err, c->s_w, c->bits_w, srv_err, c->part_srv, c->csrv,
            c->h.clip, c->status, f);
      });
    } else {
      auto k2 = with_server ? (cache ? (one ? ob::k_worker_pack<GT, ET, true, CLIP, POW2, 1, true>
                                            : ob::k_worker_pack<GT, ET, true, CLIP, POW2, 2, true>)
                                     : (one ? ob::k_worker_pack<GT, ET, true, CLIP, POW2, 1, false>
                                            : ob::k_worker_pack<GT, ET, true, CLIP, POW2, 2, false>))
                            : (one ? ob::k_worker_pack<GT, ET, false, CLIP, false, 1, false>
                                   : ob::k_worker_pack<GT, ET, false, CLIP, false, 2, false>);
      const int g2 = grid_for(c, k2, c->T);
      launch(c, kind, st, [&] {
        pdl(k2, g2, ob::kBlock, st, c->L, W, grads, err, c->s_w, c->bits_w, srv_err, c->part_srv, c->csrv,
            c->h.clip, c->status);
      });
    }
  }
  if (with_server && !fin2) enqueue_finalize_scale(c, c->part_srv, c->s_srv, 1, 0, st);
}

template <typename GT, typename ET>
void enqueue_worker_e(ob_ctx* c, const GT* grads, bool with_server, cudaStream_t st) {
  const bool clip = c->h.clip > 0.0f, p2 = pow2_workers(c);
  if (clip && p2) enqueue_worker_t<GT, ET, true, true>(c, grads, with_server, st);
  else if (clip) enqueue_worker_t<GT, ET, true, false>(c, grads, with_server, st);
  else if (p2) enqueue_worker_t<GT, ET, false, true>(c, grads, with_server, st);
  else enqueue_worker_t<GT, ET, false, false>(c, grads, with_server, st);
}

template <typename GT>
void enqueue_worker(ob_ctx* c, const GT* grads, bool with_server, cudaStream_t st) {
  if (c->cfg.err_dtype == OB_BF16) enqueue_worker_e<GT, uint16_t>(c, grads, with_server, st);
  else enqueue_worker_e<GT, float>(c, grads, with_server, st);
}

// CACHED: c_srv comes from c->csrv (the fused step's pass 2 stored it).
// One worker (rebuilding the server value from the words): the W1 instance.
template <ob::Upd U, bool FROM_WORKERS, typename ET, bool CACHED>
void launch_server_update(ob_ctx* c, cudaStream_t st) {
  constexpr bool kRebuild = FROM_WORKERS && !CACHED;
  auto k3 = (kRebuild && c->cfg.W == 1) ? ob::k_server_update<U, FROM_WORKERS, true, ET, CACHED, kRebuild>
            : pow2_workers(c)           ? ob::k_server_update<U, FROM_WORKERS, true, ET, CACHED, false>
                                        : ob::k_server_update<U, FROM_WORKERS, false, ET, CACHED, false>;
  const int g3 = grid_for(c, k3, c->T);
  ET* srv_err = static_cast<ET*>(c->srv_err);
  launch(c, CACHED ? OB_K_SERVER_UPDATE_CACHED : OB_K_SERVER_UPDATE, st, [&] {
    pdl(k3, g3, ob::kBlock, st, c->L, c->cfg.W, c->bits_w, c->s_w, c->csrv, c->s_srv, srv_err,
                                  c->bits_srv, c->m, c->v, c->p, c->h, c->partP, c->partU,
                                  c->status);
  });
}

template <ob::Upd U, bool FROM_WORKERS, typename ET>
void enqueue_server_update_e(ob_ctx* c, bool cached, cudaStream_t st) {
  if constexpr (FROM_WORKERS) {
    if (cached) launch_server_update<U, true, ET, true>(c, st);
    else launch_server_update<U, true, ET, false>(c, st);
  } else {
    launch_server_update<U, false, ET, false>(c, st);
  }
}

template <ob::Upd U, bool FROM_WORKERS>
void enqueue_server_update(ob_ctx* c, cudaStream_t st, bool cached = false) {
  if (c->T == 0) return;
  // The update-only call never reads the server error: one instantiation.
  if (FROM_WORKERS && c->cfg.err_dtype == OB_BF16) enqueue_server_update_e<U, FROM_WORKERS, uint16_t>(c, cached, st);
  else enqueue_server_update_e<U, FROM_WORKERS, float>(c, cached, st);
}

// LAMB: trust ratio per layer from the tile partials, then the parameter step.
void enqueue_lamb_param(ob_ctx* c, cudaStream_t st) {
  launch(c, OB_K_FINALIZE_RATIO, st, [&] {
    pdl(ob::k_finalize_ratio, c->cfg.num_chunks, ob::kFinalizeThreads, st, c->L, c->partP, c->partU,
        c->ratio);
  });
  if (c->T == 0) return;
  auto k = ob::k_lamb_param;
  const int g = grid_for(c, k, c->T);
  launch(c, OB_K_LAMB_PARAM, st, [&] {
    pdl(k, g, ob::kBlock, st, c->L, c->m, c->v, c->p, c->ratio, c->h, c->status);
  });
}

// Update from the packed worker signs (fused) or from bits_srv (stage call).
// from_workers is the fused step: its pass 2 stored c_srv when the ctx has csrv.
void enqueue_update(ob_ctx* c, bool from_workers, cudaStream_t st) {
  const bool lamb = c->cfg.optimizer == OB_LAMB, cached = from_workers && c->csrv;
  if (from_workers) {
    if (lamb) enqueue_server_update<ob::Upd::kLambM, true>(c, st, cached);
    else enqueue_server_update<ob::Upd::kAdam, true>(c, st, cached);
  } else {
    if (lamb) enqueue_server_update<ob::Upd::kLambM, false>(c, st);
    else enqueue_server_update<ob::Upd::kAdam, false>(c, st);
  }
  if (lamb) enqueue_lamb_param(c, st);
}

template <typename GT>
void enqueue_warmup(ob_ctx* c, const GT* grads, cudaStream_t st) {
  const bool lamb = c->cfg.optimizer == OB_LAMB, p2 = pow2_workers(c);
  if (c->T > 0) {
    auto k = lamb ? (p2 ? ob::k_warmup<GT, true, true> : ob::k_warmup<GT, true, false>)
                  : (p2 ? ob::k_warmup<GT, false, true> : ob::k_warmup<GT, false, false>);
    const int g = grid_for(c, k, c->T);
    launch(c, OB_K_WARMUP, st, [&] {
      pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, grads, c->m, c->v, c->p, c->h, c->partP,
                                  c->partU, c->status);
    });
  }
  if (lamb) enqueue_lamb_param(c, st);
}

// fin: the fused finaliser writes s_srv (small problems, as in the fused step).
template <typename ET>
void enqueue_server_norm(ob_ctx* c, bool fin, cudaStream_t st) {
  const ET* srv_err = static_cast<const ET*>(c->srv_err);
  const bool one = c->cfg.W == 1;
  if (fin) {
    auto k = one ? ob::k_server_norm_fin<ET, true, true>
                 : pow2_workers(c) ? ob::k_server_norm_fin<ET, true, false> : ob::k_server_norm_fin<ET, false, false>;
    const int g = grid_for(c, k, c->T);
    const ob::Fin f{c->ticket, c->part_srv, 0, 1, c->s_srv};
    launch(c, OB_K_SERVER_NORM, st, [&] {
      pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, c->bits_w, c->s_w, srv_err, c->part_srv, c->status, f);
    });
    return;
  }
  auto k = one ? ob::k_server_norm<ET, true, true>
               : pow2_workers(c) ? ob::k_server_norm<ET, true, false> : ob::k_server_norm<ET, false, false>;
  const int g = grid_for(c, k, c->T);
  launch(c, OB_K_SERVER_NORM, st, [&] {
    pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, c->bits_w, c->s_w, srv_err, c->part_srv, c->status);
  });
}

void enqueue_server_stage(ob_ctx* c, cudaStream_t st) {
  const bool fin = fused_fin(c, 1);
  if (c->T > 0) {
    if (c->cfg.err_dtype == OB_BF16) enqueue_server_norm<uint16_t>(c, fin, st);
    else enqueue_server_norm<float>(c, fin, st);
  }
  if (!fin) enqueue_finalize_scale(c, c->part_srv, c->s_srv, 1, 0, st);
  enqueue_server_update<ob::Upd::kNone, true>(c, st);
}

// ---- the momentum-error rule ---------------------------------------------------------

template <typename GT, typename ET, bool CLIP, bool POW2>
void enqueue_ternary_step_t(ob_ctx* c, const GT* grads, cudaStream_t st) {
  if (c->T == 0) return;
  auto k = c->cfg.optimizer == OB_LAMB ? ob::k_ternary_step<GT, ET, CLIP, POW2, ob::Upd::kLambM>
                                       : ob::k_ternary_step<GT, ET, CLIP, POW2, ob::Upd::kAdam>;
  const int g = grid_for(c, k, c->T);
  launch(c, OB_K_TERNARY_STEP, st, [&] {
    pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, grads, static_cast<ET*>(c->err), c->m, c->v, c->p,
                                c->h, c->partP, c->partU, c->status);
  });
}

template <typename GT, typename ET, bool CLIP>
void enqueue_ternary_compress_t(ob_ctx* c, const GT* grads, cudaStream_t st) {
  if (c->T == 0) return;
  auto k = ob::k_ternary_compress<GT, ET, CLIP>;
  const int g = grid_for(c, k, c->cfg.W * c->T);
  launch(c, OB_K_TERNARY_COMPRESS, st, [&] {
    pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, grads, static_cast<ET*>(c->err), c->bits_w, c->h,
                                c->status);
  });
}

// Worker stage (fused = false) or the whole one-pass step (fused = true).
template <typename GT, typename ET>
void enqueue_ternary_e(ob_ctx* c, const GT* grads, bool fused, cudaStream_t st) {
  const bool clip = c->h.clip > 0.0f, p2 = pow2_workers(c);
  if (!fused) {
    if (clip) enqueue_ternary_compress_t<GT, ET, true>(c, grads, st);
    else enqueue_ternary_compress_t<GT, ET, false>(c, grads, st);
    return;
  }
  if (clip && p2) enqueue_ternary_step_t<GT, ET, true, true>(c, grads, st);
  else if (clip) enqueue_ternary_step_t<GT, ET, true, false>(c, grads, st);
  else if (p2) enqueue_ternary_step_t<GT, ET, false, true>(c, grads, st);
  else enqueue_ternary_step_t<GT, ET, false, false>(c, grads, st);
  if (c->cfg.optimizer == OB_LAMB) enqueue_lamb_param(c, st);
}

void enqueue_ternary(ob_ctx* c, const void* grads, bool fused, cudaStream_t st) {
  const bool bf16_err = c->cfg.err_dtype == OB_BF16;
  if (c->cfg.grad_dtype == OB_BF16) {
    const uint16_t* g = static_cast<const uint16_t*>(grads);
    if (bf16_err) enqueue_ternary_e<uint16_t, uint16_t>(c, g, fused, st);
    else enqueue_ternary_e<uint16_t, float>(c, g, fused, st);
  } else {
    const float* g = static_cast<const float*>(grads);
    if (bf16_err) enqueue_ternary_e<float, uint16_t>(c, g, fused, st);
    else enqueue_ternary_e<float, float>(c, g, fused, st);
  }
}

void enqueue_ternary_server(ob_ctx* c, cudaStream_t st) {
  if (c->words == 0) return;
  auto k = ob::k_ternary_server;
  const int g = grid_for(c, k, (c->words + 31) / 32);
  launch(c, OB_K_TERNARY_SERVER, st, [&] {
    pdl(k, g, ob::kBlock, st, c->cfg.W, c->words, c->bits_w, c->bits_srv);
  });
}

void enqueue_ternary_update(ob_ctx* c, cudaStream_t st) {
  const bool lamb = c->cfg.optimizer == OB_LAMB, p2 = pow2_workers(c);
  if (c->T > 0) {
    auto k = lamb ? (p2 ? ob::k_ternary_update<ob::Upd::kLambM, true> : ob::k_ternary_update<ob::Upd::kLambM, false>)
                  : (p2 ? ob::k_ternary_update<ob::Upd::kAdam, true> : ob::k_ternary_update<ob::Upd::kAdam, false>);
    const int g = grid_for(c, k, c->T);
    launch(c, OB_K_TERNARY_UPDATE, st, [&] {
      pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, c->bits_srv, c->m, c->v, c->p, c->h, c->partP,
                                  c->partU, c->status);
    });
  }
  if (lamb) enqueue_lamb_param(c, st);
}

// ---- the 2-bit rule (two residual sign planes) ------------------------------------------

// Both scales of every (row, chunk) from the tile sums of a 2-bit pass (grid C x rows).
void enqueue_tb_finalize(ob_ctx* c, const double* part, int rows, float* out, cudaStream_t st) {
  launch(c, OB_K_TB_FINALIZE, st, [&] {
    pdl(ob::k_tb_finalize, dim3(c->cfg.num_chunks, rows), ob::kFinalizeThreads, st, c->L, part, rows, out);
  });
}

// Worker stage (passes 1 and 2, each followed by its scales) and, when
// with_server, the server scales from pass 2's sums.  (A fused finaliser in the
// pass's last CTA, as the 1-bit rule has for small problems, measured slower
// here: one CTA finishing both sweeps of every (row, chunk) has less
// parallelism than k_tb_finalize's one block per (row, chunk).)
template <typename GT, typename ET, bool CLIP, bool POW2>
void enqueue_tb_worker_t(ob_ctx* c, const GT* grads, bool with_server, cudaStream_t st) {
  const int W = c->cfg.W;
  ET* err = static_cast<ET*>(c->err);
  const ET* srv_err = static_cast<const ET*>(c->srv_err);
  if (c->T > 0) {
    auto k1 = ob::k_tb_worker_norm<GT, ET, CLIP>;
    const int g1 = grid_for(c, k1, W * c->T);
    launch(c, OB_K_TB_WORKER_NORM, st, [&] {
      pdl(k1, g1, ob::kBlock, st, c->L, W, grads, err, c->h.clip, c->part_w, c->status);
    });
  }
  enqueue_tb_finalize(c, c->part_w, W, c->s_w, st);
  const bool cache = with_server && c->csrv;       // many workers: keep c_srv for pass 3
  if (c->T > 0) {
    auto k2 = !with_server ? ob::k_tb_pack<GT, ET, false, CLIP, false, false>
              : cache      ? ob::k_tb_pack<GT, ET, true, CLIP, POW2, true>
                           : ob::k_tb_pack<GT, ET, true, CLIP, POW2, false>;
    const int g2 = grid_for(c, k2, c->T);
    launch(c, cache ? OB_K_TB_PACK_CACHED : OB_K_TB_PACK, st, [&] {
      pdl(k2, g2, ob::kBlock, st, c->L, W, grads, err, c->s_w, c->bits_w, srv_err, c->part_srv,
                                    c->csrv, c->h.clip, c->status);
    });
  }
  if (with_server) enqueue_tb_finalize(c, c->part_srv, 1, c->s_srv, st);
}

template <typename GT, typename ET>
void enqueue_tb_worker_e(ob_ctx* c, const GT* grads, bool with_server, cudaStream_t st) {
  const bool clip = c->h.clip > 0.0f, p2 = pow2_workers(c);
  if (clip && p2) enqueue_tb_worker_t<GT, ET, true, true>(c, grads, with_server, st);
  else if (clip) enqueue_tb_worker_t<GT, ET, true, false>(c, grads, with_server, st);
  else if (p2) enqueue_tb_worker_t<GT, ET, false, true>(c, grads, with_server, st);
  else enqueue_tb_worker_t<GT, ET, false, false>(c, grads, with_server, st);
}

void enqueue_tb_worker(ob_ctx* c, const void* grads, bool with_server, cudaStream_t st) {
  const bool bf16_err = c->cfg.err_dtype == OB_BF16;
  if (c->cfg.grad_dtype == OB_BF16) {
    const uint16_t* g = static_cast<const uint16_t*>(grads);
    if (bf16_err) enqueue_tb_worker_e<uint16_t, uint16_t>(c, g, with_server, st);
    else enqueue_tb_worker_e<uint16_t, float>(c, g, with_server, st);
  } else {
    const float* g = static_cast<const float*>(grads);
    if (bf16_err) enqueue_tb_worker_e<float, uint16_t>(c, g, with_server, st);
    else enqueue_tb_worker_e<float, float>(c, g, with_server, st);
  }
}

template <ob::Upd U, bool FROM_WORKERS, typename ET, bool CACHED>
void launch_tb_server_update(ob_ctx* c, cudaStream_t st) {
  if (c->T == 0) return;
  constexpr bool kRebuild = FROM_WORKERS && !CACHED;
  auto k = (kRebuild && c->cfg.W == 1) ? ob::k_tb_server_update<U, FROM_WORKERS, true, ET, CACHED, kRebuild>
           : pow2_workers(c)           ? ob::k_tb_server_update<U, FROM_WORKERS, true, ET, CACHED, false>
                                       : ob::k_tb_server_update<U, FROM_WORKERS, false, ET, CACHED, false>;
  const int g = grid_for(c, k, c->T);
  launch(c, CACHED ? OB_K_TB_SERVER_UPDATE_CACHED : OB_K_TB_SERVER_UPDATE, st, [&] {
    pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, c->bits_w, c->s_w, c->csrv, c->s_srv,
                                static_cast<ET*>(c->srv_err), c->bits_srv, c->m, c->v, c->p, c->h,
                                c->partP, c->partU, c->status);
  });
}

// cached: the fused step's pass 2 stored c_srv in c->csrv.
template <ob::Upd U, bool FROM_WORKERS>
void enqueue_tb_server_update(ob_ctx* c, cudaStream_t st, bool cached = false) {
  const bool bf = FROM_WORKERS && c->cfg.err_dtype == OB_BF16;
  if constexpr (FROM_WORKERS) {
    if (cached) {
      if (bf) launch_tb_server_update<U, true, uint16_t, true>(c, st);
      else launch_tb_server_update<U, true, float, true>(c, st);
      return;
    }
  }
  if (bf) launch_tb_server_update<U, FROM_WORKERS, uint16_t, false>(c, st);
  else launch_tb_server_update<U, FROM_WORKERS, float, false>(c, st);
}

// Update from the worker planes (fused step) or from bits_srv (stage call).
void enqueue_tb_update(ob_ctx* c, bool from_workers, cudaStream_t st) {
  const bool lamb = c->cfg.optimizer == OB_LAMB, cached = from_workers && c->csrv;
  if (from_workers) {
    if (lamb) enqueue_tb_server_update<ob::Upd::kLambM, true>(c, st, cached);
    else enqueue_tb_server_update<ob::Upd::kAdam, true>(c, st, cached);
  } else {
    if (lamb) enqueue_tb_server_update<ob::Upd::kLambM, false>(c, st);
    else enqueue_tb_server_update<ob::Upd::kAdam, false>(c, st);
  }
  if (lamb) enqueue_lamb_param(c, st);
}

// Server stage alone: the server sums (one pass over the planes), both server
// scales, then the server planes and error.
template <typename ET, bool POW2>
void enqueue_tb_server_stage_t(ob_ctx* c, cudaStream_t st) {
  const ET* srv_err = static_cast<const ET*>(c->srv_err);
  if (c->T > 0) {
    auto k = c->cfg.W == 1 ? ob::k_tb_server_norm<ET, true, true> : ob::k_tb_server_norm<ET, POW2, false>;
    const int g = grid_for(c, k, c->T);
    launch(c, OB_K_TB_SERVER_NORM, st, [&] {
      pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, c->bits_w, c->s_w, srv_err, c->part_srv, c->status);
    });
  }
  enqueue_tb_finalize(c, c->part_srv, 1, c->s_srv, st);
  enqueue_tb_server_update<ob::Upd::kNone, true>(c, st);
}

void enqueue_tb_server_stage(ob_ctx* c, cudaStream_t st) {
  const bool p2 = pow2_workers(c);
  if (c->cfg.err_dtype == OB_BF16) {
    if (p2) enqueue_tb_server_stage_t<uint16_t, true>(c, st); else enqueue_tb_server_stage_t<uint16_t, false>(c, st);
  } else {
    if (p2) enqueue_tb_server_stage_t<float, true>(c, st); else enqueue_tb_server_stage_t<float, false>(c, st);
  }
}

// ---- 0/1 Adam local step ------------------------------------------------------------------

template <typename GT, typename ET, bool CLIP>
void enqueue_local_t(ob_ctx* c, const GT* grads, cudaStream_t st) {
  const bool lamb = c->cfg.optimizer == OB_LAMB;
  if (c->T > 0) {
    auto k = lamb ? ob::k_local_step<GT, ET, CLIP, ob::Upd::kLambM> : ob::k_local_step<GT, ET, CLIP, ob::Upd::kAdam>;
    const int g = grid_for(c, k, c->T);
    launch(c, OB_K_LOCAL_STEP, st, [&] {
      pdl(k, g, ob::kBlock, st, c->L, c->cfg.W, grads, static_cast<ET*>(c->err), c->m, c->v, c->p, c->h,
                                  c->partP, c->partU, c->status);
    });
  }
  if (lamb) enqueue_lamb_param(c, st);
}

template <typename GT, typename ET>
void enqueue_local_e(ob_ctx* c, const void* grads, cudaStream_t st) {
  const GT* g = static_cast<const GT*>(grads);
  if (c->h.clip > 0.0f) enqueue_local_t<GT, ET, true>(c, g, st);
  else enqueue_local_t<GT, ET, false>(c, g, st);
}

void enqueue_local(ob_ctx* c, const void* grads, cudaStream_t st) {
  const bool bf16_err = c->cfg.err_dtype == OB_BF16;
  if (c->cfg.grad_dtype == OB_BF16) {
    if (bf16_err) enqueue_local_e<uint16_t, uint16_t>(c, grads, st);
    else enqueue_local_e<uint16_t, float>(c, grads, st);
  } else {
    if (bf16_err) enqueue_local_e<float, uint16_t>(c, grads, st);
    else enqueue_local_e<float, float>(c, grads, st);
  }
}

ob_err fused_step(ob_ctx* c, const void* grads, cudaStream_t st) {
  if (two_bit_rule(&c->cfg)) {
    enqueue_tb_worker(c, grads, true, st);
    enqueue_tb_update(c, true, st);
    ob_err r = check_launch("ob_step");
    if (r == OB_OK) ++c->step;
    return r;
  }
  if (momentum_rule(&c->cfg)) {
    enqueue_ternary(c, grads, true, st);
    ob_err r = check_launch("ob_step");
    if (r == OB_OK) ++c->step;
    return r;
  }
  if (c->cfg.grad_dtype == OB_BF16)
    enqueue_worker<uint16_t>(c, static_cast<const uint16_t*>(grads), true, st);
  else
    enqueue_worker<float>(c, static_cast<const float*>(grads), true, st);
  enqueue_update(c, true, st);
  ob_err r = check_launch("ob_step");
  if (r == OB_OK) ++c->step;
  return r;
}

ob_err check_ctx(const ob_ctx* c) {
  if (!c) return fail(OB_EINVAL, "ctx is NULL");
  return OB_OK;
}

// The buffers each call touches; a ctx may be created without the others
// (e.g. a server-only ctx on the rank that owns some chunks).
enum Need : unsigned {
  kNeedUpdate = 1u,  // p, m, v, bits_srv, s_srv
  kNeedWarm = 2u,    // p, m, v
  kNeedWorker = 4u,  // err, bits_w, s_w
  kNeedServer = 8u,  // srv_err, bits_w, s_w, bits_srv, s_srv
  kNeedErr = 16u,    // err alone (the one-pass step of the momentum-error rule)
};

ob_err require_buffers(const ob_ctx* c, unsigned need, const char* call) {
  const int64_t n = c->cfg.n, W = c->cfg.W, C = c->cfg.num_chunks;
  // The momentum-error rule has no scales and no server error.
  const unsigned scaled = momentum_rule(&c->cfg) ? 0u : ~0u;
  const struct { unsigned mask; const void* p; int64_t count; const char* name; } list[] = {
      {kNeedUpdate | kNeedWarm, c->p, n, "p"},
      {kNeedUpdate | kNeedWarm, c->m, n, "m"},
      {kNeedUpdate | kNeedWarm, c->v, n, "v"},
      {kNeedWorker | kNeedErr, c->err, W * n, "err"},
      {kNeedServer & scaled, c->srv_err, n, "srv_err"},
      {kNeedWorker | kNeedServer, c->bits_w, W * c->words, "bits_w"},
      {(kNeedWorker | kNeedServer) & scaled, c->s_w, W * C * scale_planes(&c->cfg), "s_w"},
      {kNeedUpdate | kNeedServer, c->bits_srv, c->words, "bits_srv"},
      {(kNeedUpdate | kNeedServer) & scaled, c->s_srv, C * scale_planes(&c->cfg), "s_srv"}};
  for (const auto& b : list)
    if ((b.mask & need) && b.count > 0 && !b.p)
      return fail(OB_EINVAL, "%s: the ctx was created without %s", call, b.name);
  return OB_OK;
}

ob_err require_compressed(const ob_ctx* c, const char* call) {
  if (c->step < c->cfg.freeze_step)
    return fail(OB_EPHASE, "%s: step %lld is in the warmup phase (freeze_step = %d)", call,
                (long long)c->step, c->cfg.freeze_step);
  return OB_OK;
}

}  // namespace

extern "C" {

ob_err ob_layout(const ob_config* cfg, int64_t* words_total) {
  ob_err r = check_config(cfg);
  if (r != OB_OK) return r;
  if (!words_total) return fail(OB_EINVAL, "words_total is NULL");
  int64_t t = 0;
  for (int32_t k = 0; k < cfg->num_chunks; ++k)
    t += row_words_of(cfg, cfg->chunk_offsets[k + 1] - cfg->chunk_offsets[k]);
  *words_total = t;
  return OB_OK;
}

ob_err ob_create(const ob_config* cfg, float* p, float* m, float* v, void* err, void* srv_err,
                 uint32_t* bits_w, float* s_w, uint32_t* bits_srv, float* s_srv, ob_ctx** out) {
  if (!out) return fail(OB_EINVAL, "out is NULL");
  *out = nullptr;
  int64_t words = 0;
  ob_err r = ob_layout(cfg, &words);
  if (r != OB_OK) return r;
  const int64_t n = cfg->n, W = cfg->W, C = cfg->num_chunks;

  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  struct { const void* p; int64_t count; const char* name; uintptr_t align; } bufs[] = {
      {p, n, "p", kAlignElems}, {m, n, "m", kAlignElems}, {v, n, "v", kAlignElems},
      {err, W * n, "err", kAlignElems}, {srv_err, n, "srv_err", kAlignElems},
      {bits_w, W * words, "bits_w", kAlignWords}, {s_w, W * C * scale_planes(cfg), "s_w", kAlignWords},
      {bits_srv, words, "bits_srv", kAlignWords}, {s_srv, C * scale_planes(cfg), "s_srv", kAlignWords}};
  for (auto& b : bufs)  // NULL: the ctx is created without that buffer (see require_buffers)
    if (b.p && (r = check_dev(b.p, b.count, b.name, device, b.align)) != OB_OK) return r;

  ob_ctx* c = new (std::nothrow) ob_ctx();
  if (!c) return fail(OB_ENOMEM, "ctx allocation failed");
  c->cfg = *cfg;
  c->off.assign(cfg->chunk_offsets, cfg->chunk_offsets + C + 1);
  c->cfg.chunk_offsets = c->off.data();
  c->device = device;
  c->words = words;
  c->p = p; c->m = m; c->v = v; c->err = err; c->srv_err = srv_err;
  c->bits_w = bits_w; c->s_w = s_w; c->bits_srv = bits_srv; c->s_srv = s_srv;
  c->h.lr = cfg->lr;
  c->h.b1 = cfg->beta1;
  c->h.omb1 = 1.0f - cfg->beta1;
  c->h.b2 = cfg->beta2;
  c->h.omb2 = 1.0f - cfg->beta2;
  c->h.eps = cfg->eps;
  c->h.clip = cfg->clip;
  if ((e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, device)) != cudaSuccess) {
    delete c;
    return cuda_fail(e, "cudaDeviceGetAttribute");
  }

  // Chunk tables.
  std::vector<int64_t> wo(C + 1), tp(C + 1);
  std::vector<uint8_t> vec(C);
  wo[0] = tp[0] = 0;
  for (int64_t k = 0; k < C; ++k) {
    const int64_t o = c->off[k], nk = c->off[k + 1] - o;
    wo[k + 1] = wo[k] + row_words_of(cfg, nk);
    tp[k + 1] = tp[k] + (nk + ob::kTile - 1) / ob::kTile;
    // 8-wide path: chunk start and length multiples of 8, and every worker row
    // starts on a multiple of 8 elements (16 bytes of bf16, 32 bytes of fp32).
    vec[k] = (o % 8 == 0) && (nk % 8 == 0) && (W == 1 || n % 8 == 0);
  }
  c->T = tp[C];

  // Scratch layout: tables, then partials, every piece 256-byte aligned.
  auto up256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t sz_tab = up256(sizeof(int64_t) * (C + 1));
  const size_t sz_vec = up256(size_t(C));
  // The 2-bit rule keeps three sums per tile: c^2, |c| and the squared
  // deviations of |c| (twobit.cuh).
  const size_t sums = two_bit_rule(cfg) ? 3 : 1;
  const size_t sz_pw = up256(sizeof(double) * sums * size_t(W) * size_t(c->T));
  const size_t sz_ps = up256(sizeof(double) * sums * size_t(c->T));
  const size_t sz_pt = up256(sizeof(double) * size_t(c->T));
  const size_t sz_ratio = up256(sizeof(float) * size_t(C));
  // c_srv cache of the fused step: scaled-sign rules with many workers, on a ctx
  // that holds every buffer the fused step needs.
  const bool fused_capable = p && m && v && err && srv_err && bits_w && s_w && bits_srv && s_srv;
  const bool cache = !momentum_rule(cfg) && W >= kCacheMinW && fused_capable && n > 0;
  const size_t sz_cs = cache ? up256(sizeof(float) * size_t(n)) : 0;
  const size_t total = 3 * sz_tab + sz_vec + sz_pw + sz_ps + 2 * sz_pt + sz_ratio + sz_cs + 512;
  if ((e = cudaMalloc(&c->scratch, total)) != cudaSuccess) {
    cudaGetLastError();
    delete c;
    return fail(OB_ENOMEM, "cudaMalloc of %zu scratch bytes failed: %s", total, cudaGetErrorString(e));
  }
  char* base = static_cast<char*>(c->scratch);
  int64_t* d_off = reinterpret_cast<int64_t*>(base); base += sz_tab;
  int64_t* d_wo = reinterpret_cast<int64_t*>(base); base += sz_tab;
  int64_t* d_tp = reinterpret_cast<int64_t*>(base); base += sz_tab;
  uint8_t* d_vec = reinterpret_cast<uint8_t*>(base); base += sz_vec;
  c->part_w = reinterpret_cast<double*>(base); base += sz_pw;
  c->part_srv = reinterpret_cast<double*>(base); base += sz_ps;
  c->partP = reinterpret_cast<double*>(base); base += sz_pt;
  c->partU = reinterpret_cast<double*>(base); base += sz_pt;
  c->ratio = reinterpret_cast<float*>(base); base += sz_ratio;
  c->csrv = cache ? reinterpret_cast<float*>(base) : nullptr; base += sz_cs;
  c->status = reinterpret_cast<uint32_t*>(base);
  c->ticket = reinterpret_cast<unsigned*>(base + 256);

  const struct { void* dst; const void* src; size_t bytes; } copies[] = {
      {d_off, c->off.data(), sizeof(int64_t) * (C + 1)},
      {d_wo, wo.data(), sizeof(int64_t) * (C + 1)},
      {d_tp, tp.data(), sizeof(int64_t) * (C + 1)},
      {d_vec, vec.data(), size_t(C)}};
  for (auto& cp : copies)
    if ((e = cudaMemcpy(cp.dst, cp.src, cp.bytes, cudaMemcpyHostToDevice)) != cudaSuccess) {
      cudaFree(c->scratch);
      delete c;
      return cuda_fail(e, "cudaMemcpy of chunk tables");
    }
  if ((e = cudaMemset(c->status, 0, 512)) != cudaSuccess ||
      (e = cudaDeviceSynchronize()) != cudaSuccess) {
    cudaFree(c->scratch);
    delete c;
    return cuda_fail(e, "scratch initialisation");
  }
  c->L.off = d_off;
  c->L.wo = d_wo;
  c->L.tp = d_tp;
  c->L.vec = d_vec;
  c->L.n = n;
  c->L.T = c->T;
  c->L.words = words;
  c->L.C = static_cast<int32_t>(C);
  *out = c;
  return OB_OK;
}

namespace {

// Full-precision step (warmup, or a 0/1 Adam variance refresh): no phase check.
ob_err full_precision_step(ob_ctx* c, const void* grads, void* stream, const char* call) {
  ob_err r = require_buffers(c, kNeedWarm, call);
  if (r != OB_OK) return r;
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  if ((r = check_grads(c, grads)) != OB_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c->cfg.grad_dtype == OB_BF16) enqueue_warmup<uint16_t>(c, static_cast<const uint16_t*>(grads), st);
  else enqueue_warmup<float>(c, static_cast<const float*>(grads), st);
  if ((r = check_launch(call)) != OB_OK) return r;
  ++c->step;
  return OB_OK;
}

}  // namespace

ob_err ob_warmup_step(ob_ctx* c, const void* grads, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if (c->step >= c->cfg.freeze_step)
    return fail(OB_EPHASE, "ob_warmup_step: step %lld >= freeze_step %d", (long long)c->step,
                c->cfg.freeze_step);
  return full_precision_step(c, grads, stream, "ob_warmup_step");
}

ob_err ob_refresh_step(ob_ctx* c, const void* grads, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  return full_precision_step(c, grads, stream, "ob_refresh_step");
}

ob_err ob_local_step(ob_ctx* c, const void* grads, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if (momentum_rule(&c->cfg))
    return fail(OB_EINVAL, "ob_local_step: the momentum-error rule's error buffer is not additive");
  if ((r = require_compressed(c, "ob_local_step")) != OB_OK) return r;
  if ((r = require_buffers(c, kNeedWarm | kNeedErr, "ob_local_step")) != OB_OK) return r;
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  if ((r = check_grads(c, grads)) != OB_OK) return r;
  enqueue_local(c, grads, static_cast<cudaStream_t>(stream));
  if ((r = check_launch("ob_local_step")) != OB_OK) return r;
  ++c->step;
  return OB_OK;
}

ob_err ob_mean_grads(ob_ctx* c, const void* grads, float* mean, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  if ((r = check_grads(c, grads)) != OB_OK) return r;
  if ((r = check_dev(mean, c->cfg.n, "mean", c->device)) != OB_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c->T > 0) {
    const bool p2 = pow2_workers(c), bf = c->cfg.grad_dtype == OB_BF16;
    auto launch_mean = [&](auto k, const auto* g) {
      const int grid = grid_for(c, k, c->T);
      launch(c, OB_K_GRAD_MEAN, st, [&] { pdl(k, grid, ob::kBlock, st, c->L, c->cfg.W, g, mean, c->status); });
    };
    const uint16_t* gh = static_cast<const uint16_t*>(grads);
    const float* gf = static_cast<const float*>(grads);
    if (bf && p2) launch_mean(ob::k_grad_mean<uint16_t, true>, gh);
    else if (bf) launch_mean(ob::k_grad_mean<uint16_t, false>, gh);
    else if (p2) launch_mean(ob::k_grad_mean<float, true>, gf);
    else launch_mean(ob::k_grad_mean<float, false>, gf);
  }
  return check_launch("ob_mean_grads");
}

ob_err ob_compress(ob_ctx* c, const void* grads, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if ((r = require_compressed(c, "ob_compress")) != OB_OK) return r;
  if ((r = require_buffers(c, kNeedWorker, "ob_compress")) != OB_OK) return r;
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  if ((r = check_grads(c, grads)) != OB_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (momentum_rule(&c->cfg)) enqueue_ternary(c, grads, false, st);
  else if (two_bit_rule(&c->cfg)) enqueue_tb_worker(c, grads, false, st);
  else if (c->cfg.grad_dtype == OB_BF16) enqueue_worker<uint16_t>(c, static_cast<const uint16_t*>(grads), false, st);
  else enqueue_worker<float>(c, static_cast<const float*>(grads), false, st);
  return check_launch("ob_compress");
}

ob_err ob_server_reduce(ob_ctx* c, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if ((r = require_compressed(c, "ob_server_reduce")) != OB_OK) return r;
  if ((r = require_buffers(c, kNeedServer, "ob_server_reduce")) != OB_OK) return r;
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  if (momentum_rule(&c->cfg)) enqueue_ternary_server(c, static_cast<cudaStream_t>(stream));
  else if (two_bit_rule(&c->cfg)) enqueue_tb_server_stage(c, static_cast<cudaStream_t>(stream));
  else enqueue_server_stage(c, static_cast<cudaStream_t>(stream));
  return check_launch("ob_server_reduce");
}

ob_err ob_step(ob_ctx* c, const void* grads, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if ((r = require_compressed(c, "ob_step")) != OB_OK) return r;
  // The fused step of the momentum-error rule touches p, m, v and err only.
  const unsigned need = !grads ? kNeedUpdate
                        : momentum_rule(&c->cfg) ? (kNeedWarm | kNeedErr)
                                                 : (kNeedWorker | kNeedServer | kNeedUpdate);
  if ((r = require_buffers(c, need, "ob_step")) != OB_OK) return r;
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (grads) {
    if ((r = check_grads(c, grads)) != OB_OK) return r;
    return fused_step(c, grads, st);
  }
  if (momentum_rule(&c->cfg)) enqueue_ternary_update(c, st);
  else if (two_bit_rule(&c->cfg)) enqueue_tb_update(c, false, st);
  else enqueue_update(c, false, st);
  if ((r = check_launch("ob_step")) != OB_OK) return r;
  ++c->step;
  return OB_OK;
}

namespace {

// The staging slot of `ptr`, created (with its event) on first use; with more
// than 4 distinct buffers the oldest slot is recycled after its event completes.
ob_err staging_slot(ob_ctx* c, const void* ptr, ob_ctx::Staging** out) {
  for (auto& s : c->staging)
    if (s.ptr == ptr && s.free_ev) { *out = &s; return OB_OK; }
  ob_ctx::Staging& s = c->staging[c->staging_next];
  c->staging_next = (c->staging_next + 1) % 4;
  cudaError_t e = cudaSuccess;
  if (s.free_ev && s.used) e = cudaEventSynchronize(s.free_ev);
  if (e == cudaSuccess && !s.free_ev) e = cudaEventCreateWithFlags(&s.free_ev, cudaEventDisableTiming);
  if (e != cudaSuccess) return cuda_fail(e, "ob_step_host: staging event");
  s.ptr = ptr;
  s.used = false;
  *out = &s;
  return OB_OK;
}

}  // namespace

ob_err ob_step_host(ob_ctx* c, const void* host_grads, void* dev_staging, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if ((r = require_compressed(c, "ob_step_host")) != OB_OK) return r;
  const unsigned need = momentum_rule(&c->cfg) ? (kNeedWarm | kNeedErr) : (kNeedWorker | kNeedServer | kNeedUpdate);
  if ((r = require_buffers(c, need, "ob_step_host")) != OB_OK) return r;
  const int64_t count = int64_t(c->cfg.W) * c->cfg.n;
  if (count > 0 && !host_grads) return fail(OB_EINVAL, "host_grads is NULL");
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  if ((r = check_grads(c, dev_staging)) != OB_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = size_t(count) * (c->cfg.grad_dtype == OB_BF16 ? 2 : 4);
  ob_ctx::Staging* slot = nullptr;
  if (bytes > 0) {
    cudaError_t e = cudaSuccess;
    if (!c->copy_stream) e = cudaStreamCreateWithFlags(&c->copy_stream, cudaStreamNonBlocking);
    if (e == cudaSuccess && !c->copied) e = cudaEventCreateWithFlags(&c->copied, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "ob_step_host: copy stream");
    if ((r = staging_slot(c, dev_staging, &slot)) != OB_OK) return r;
    // The upload waits only for the kernels that last read this staging buffer,
    // so it overlaps the compute of the step before when buffers alternate.
    if (slot->used) e = cudaStreamWaitEvent(c->copy_stream, slot->free_ev, 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dev_staging, host_grads, bytes, cudaMemcpyHostToDevice, c->copy_stream);
    if (e == cudaSuccess) e = cudaEventRecord(c->copied, c->copy_stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, c->copied, 0);
    if (e != cudaSuccess) return cuda_fail(e, "ob_step_host: host-to-device copy");
  }
  if ((r = fused_step(c, dev_staging, st)) != OB_OK) return r;
  if (slot) {
    cudaError_t e = cudaEventRecord(slot->free_ev, st);
    if (e != cudaSuccess) return cuda_fail(e, "ob_step_host: staging event");
    slot->used = true;
  }
  return OB_OK;
}

ob_err ob_destroy(ob_ctx* c) {
  if (!c) return OB_OK;
  ob_err r = OB_OK;
  for (auto& ev : c->prof_ev) cudaEventDestroy(ev);
  if (c->copy_stream) {
    cudaStreamSynchronize(c->copy_stream);
    cudaStreamDestroy(c->copy_stream);
  }
  if (c->copied) cudaEventDestroy(c->copied);
  for (auto& s : c->staging)
    if (s.free_ev) cudaEventDestroy(s.free_ev);
  if (c->scratch) {
    DeviceGuard dg(c->device);
    cudaError_t e = cudaFree(c->scratch);
    if (e != cudaSuccess) r = cuda_fail(e, "cudaFree");
  }
  delete c;
  return r;
}

ob_err ob_get_status(ob_ctx* c, uint32_t* flags, int32_t clear, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if (!flags) return fail(OB_EINVAL, "flags is NULL");
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, c->status, sizeof h, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(c->status, 0, sizeof(uint32_t), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "ob_get_status");
  *flags = h;
  return OB_OK;
}

int64_t ob_get_step(const ob_ctx* c) { return c ? c->step : -1; }

ob_err ob_set_step(ob_ctx* c, int64_t step) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if (step < 0) return fail(OB_EINVAL, "step = %lld < 0", (long long)step);
  c->step = step;
  return OB_OK;
}

ob_err ob_error_norms(ob_ctx* c, float* worker_norms, float* server_norms, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  const int64_t W = c->cfg.W, C = c->cfg.num_chunks;
  if (!worker_norms && !server_norms) return fail(OB_EINVAL, "ob_error_norms: no output");
  if (worker_norms && !c->err && c->cfg.n > 0) return fail(OB_EINVAL, "ob_error_norms: the ctx has no err");
  if (server_norms && momentum_rule(&c->cfg))
    return fail(OB_EINVAL, "ob_error_norms: the momentum-error rule has no server error");
  if (server_norms && !c->srv_err && c->cfg.n > 0) return fail(OB_EINVAL, "ob_error_norms: the ctx has no srv_err");
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  if (worker_norms && (r = check_dev(worker_norms, W * C, "worker_norms", c->device, kAlignWords)) != OB_OK)
    return r;
  if (server_norms && (r = check_dev(server_norms, C, "server_norms", c->device, kAlignWords)) != OB_OK)
    return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Reuses the partial-sum scratch of the step: call it between steps on the same stream.
  auto norms = [&](const void* x, int rows, double* part, float* out) {
    if (c->T > 0) {
      if (c->cfg.err_dtype == OB_BF16) {
        auto k = ob::k_rows_sumsq<uint16_t>;
        const int g = grid_for(c, k, rows * c->T);
        launch(c, OB_K_WORKER_NORM, st, [&] {
          pdl(k, g, ob::kBlock, st, c->L, rows, static_cast<const uint16_t*>(x), part);
        });
      } else {
        auto k = ob::k_rows_sumsq<float>;
        const int g = grid_for(c, k, rows * c->T);
        launch(c, OB_K_WORKER_NORM, st, [&] {
          pdl(k, g, ob::kBlock, st, c->L, rows, static_cast<const float*>(x), part);
        });
      }
    }
    launch(c, OB_K_FINALIZE_SCALE, st, [&] {
      pdl(ob::k_finalize_scale<false>, dim3(unsigned(C), unsigned(rows)), ob::kFinalizeThreads, st,
          c->L, part, c->T, out);
    });
  };
  if (worker_norms) norms(c->err, int(W), c->part_w, worker_norms);
  if (server_norms) norms(c->srv_err, 1, c->part_srv, server_norms);
  return check_launch("ob_error_norms");
}

ob_err ob_quant_rates(ob_ctx* c, float* worker_rates, float* server_rates, void* stream) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if (momentum_rule(&c->cfg))
    return fail(OB_EINVAL, "ob_quant_rates: the momentum-error rule sends ternary codes, not sign bits");
  const int64_t W = c->cfg.W, C = c->cfg.num_chunks, planes = scale_planes(&c->cfg);
  if (!worker_rates && !server_rates) return fail(OB_EINVAL, "ob_quant_rates: no output");
  if (worker_rates && !c->bits_w && c->words > 0) return fail(OB_EINVAL, "ob_quant_rates: the ctx has no bits_w");
  if (server_rates && !c->bits_srv && c->words > 0) return fail(OB_EINVAL, "ob_quant_rates: the ctx has no bits_srv");
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  if (worker_rates && (r = check_dev(worker_rates, W * C * planes, "worker_rates", c->device, kAlignWords)) != OB_OK)
    return r;
  if (server_rates && (r = check_dev(server_rates, C * planes, "server_rates", c->device, kAlignWords)) != OB_OK)
    return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Reuses the partial-sum scratch of the step: call it between steps on the same stream.
  auto rates = [&](const uint32_t* bits, int rows, double* part, float* out) {
    for (int pl = 0; pl < int(planes); ++pl) {
      if (c->T > 0) {
        auto k = ob::k_sign_count;
        const int g = grid_for(c, k, (rows * c->T + ob::kWarp - 1) / ob::kWarp);   // a thread per tile
        launch(c, OB_K_SIGN_COUNT, st, [&] { pdl(k, g, ob::kBlock, st, c->L, rows, bits, pl, part); });
      }
      launch(c, OB_K_FINALIZE_SCALE, st, [&] {
        pdl(ob::k_finalize_rate, dim3(unsigned(C), unsigned(rows)), ob::kFinalizeThreads, st,
            c->L, part, c->T, out, int(planes), pl);
      });
    }
  };
  if (worker_rates) rates(c->bits_w, int(W), c->part_w, worker_rates);
  if (server_rates) rates(c->bits_srv, 1, c->part_srv, server_rates);
  return check_launch("ob_quant_rates");
}

ob_err ob_profile_start(ob_ctx* c, int32_t capacity) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if (capacity < 1 || capacity > (1 << 20)) return fail(OB_EINVAL, "capacity = %d outside [1, 2^20]", capacity);
  if (c->prof_on) return fail(OB_EINVAL, "profiling already started");
  DeviceGuard dg(c->device);
  if (!dg.ok) return fail(OB_ECUDA, "cannot select device %d", c->device);
  c->prof_ev.assign(2 * size_t(capacity), nullptr);
  for (auto& ev : c->prof_ev) {
    cudaError_t e = cudaEventCreate(&ev);
    if (e != cudaSuccess) {
      for (auto& x : c->prof_ev) if (x) cudaEventDestroy(x);
      c->prof_ev.clear();
      return cuda_fail(e, "cudaEventCreate");
    }
  }
  c->prof_kind.assign(size_t(capacity), 0);
  c->prof_cap = capacity;
  c->prof_used = 0;
  c->prof_on = true;
  return OB_OK;
}

ob_err ob_profile_stop(ob_ctx* c, double* ms, int64_t* launches) {
  ob_err r = check_ctx(c);
  if (r != OB_OK) return r;
  if (!ms || !launches) return fail(OB_EINVAL, "ms / launches is NULL");
  if (!c->prof_on) return fail(OB_EINVAL, "profiling not started");
  DeviceGuard dg(c->device);
  for (int k = 0; k < OB_K_KINDS; ++k) { ms[k] = 0.0; launches[k] = 0; }
  cudaError_t first = cudaSuccess;
  for (int32_t i = 0; i < c->prof_used; ++i) {
    float t = 0.0f;
    cudaError_t e = cudaEventSynchronize(c->prof_ev[2 * i + 1]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, c->prof_ev[2 * i], c->prof_ev[2 * i + 1]);
    if (e != cudaSuccess) { if (first == cudaSuccess) first = e; continue; }
    ms[c->prof_kind[i]] += t;
    launches[c->prof_kind[i]] += 1;
  }
  for (auto& ev : c->prof_ev) cudaEventDestroy(ev);
  c->prof_ev.clear();
  c->prof_kind.clear();
  c->prof_on = false;
  c->prof_cap = c->prof_used = 0;
  if (first != cudaSuccess) return cuda_fail(first, "ob_profile_stop");
  return OB_OK;
}

const char* ob_kernel_name(int32_t kind) {
  static const char* names[OB_K_KINDS] = {
      "k_worker_norm", "k_finalize_scale", "k_worker_pack", "k_server_norm",
      "k_server_update", "k_lamb_param", "k_warmup", "k_finalize_ratio",
      "k_ternary_step", "k_ternary_compress", "k_ternary_server", "k_ternary_update",
      "k_tb_worker_norm", "k_tb_pack", "k_tb_server_norm", "k_tb_server_update",
      "k_worker_pack_cached", "k_server_update_cached", "k_tb_pack_cached", "k_tb_finalize",
      "k_tb_server_update_cached", "k_local_step", "k_sign_count", "k_grad_mean"};
  return (kind >= 0 && kind < OB_K_KINDS) ? names[kind] : "";
}

int64_t ob_launch_count(const ob_ctx* c) { return c ? c->launches : -1; }

const char* ob_last_error(void) { return g_last_error; }

}  // extern "C"

// ---- worker stage without allocation -------------------------------------------------
// ob_compress_noalloc (declared in onebit.h) serves callers that must not allocate
// device memory.  Its scratch is one fixed file-scope device array; host code here
// only ever passes the array's device address, obtained once per device with
// cudaGetSymbolAddress (the symbol itself is a host-side stand-in, not an address).
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB on every device

// Every GPU that loads this library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int32_t kNoAllocMaxChunks = 4096;
constexpr int kNoAllocMaxDevices = 64;
constexpr size_t kNoAllocTableBytes = 3 * sizeof(int64_t) * (kNoAllocMaxChunks + 1) + kNoAllocMaxChunks;

struct NoAllocDevice {
  bool ready = false;
  char* scratch = nullptr;   // device address of g_noalloc_scratch on this device
  int num_sms = 0;
  int occ_norm[2][2] = {{1, 1}, {1, 1}};  // resident CTAs per SM: [bf16 grads][clip]
  int occ_pack[2][2] = {{1, 1}, {1, 1}};
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];
// Host image of the scratch header (chunk tables + zeroed status word), rebuilt
// under the mutex and copied with one cudaMemcpyAsync per call.
alignas(256) unsigned char g_noalloc_header[kNoAllocTableBytes + 512];

int occupancy(const void* fn) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, ob::kBlock, 0) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  return per_sm;
}

// Once per device, with that device current: look up the array's device address.
ob_err noalloc_setup(int device, NoAllocDevice** out) {
  if (device < 0 || device >= kNoAllocMaxDevices) return fail(OB_EINVAL, "device %d out of range", device);
  NoAllocDevice& d = g_noalloc_dev[device];
  if (!d.ready) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    if ((e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, device)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    // Every instance that a call may launch, so each grid is sized for its own kernel.
    d.occ_norm[0][0] = occupancy(reinterpret_cast<const void*>(ob::k_worker_norm<float, float, false>));
    d.occ_norm[0][1] = occupancy(reinterpret_cast<const void*>(ob::k_worker_norm<float, float, true>));
    d.occ_norm[1][0] = occupancy(reinterpret_cast<const void*>(ob::k_worker_norm<uint16_t, float, false>));
    d.occ_norm[1][1] = occupancy(reinterpret_cast<const void*>(ob::k_worker_norm<uint16_t, float, true>));
    d.occ_pack[0][0] = occupancy(reinterpret_cast<const void*>(ob::k_worker_pack<float, float, false, false, false, 2, false>));
    d.occ_pack[0][1] = occupancy(reinterpret_cast<const void*>(ob::k_worker_pack<float, float, false, true, false, 2, false>));
    d.occ_pack[1][0] = occupancy(reinterpret_cast<const void*>(ob::k_worker_pack<uint16_t, float, false, false, false, 2, false>));
    d.occ_pack[1][1] = occupancy(reinterpret_cast<const void*>(ob::k_worker_pack<uint16_t, float, false, true, false, 2, false>));
    d.scratch = static_cast<char*>(ptr);
    d.ready = true;
  }
  *out = &d;
  return OB_OK;
}

int noalloc_grid(int num_sms, int per_sm, int64_t warps) {
  const int64_t need = (warps + ob::kWarpsPerBlock - 1) / ob::kWarpsPerBlock;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(need, int64_t(num_sms) * per_sm)));
}

}  // namespace

extern "C" ob_err ob_compress_noalloc(const ob_config* cfg, const void* grads, float* err,
                                      uint32_t* bits_w, float* s_w, void* stream) {
  int64_t words = 0;
  ob_err r = ob_layout(cfg, &words);
  if (r != OB_OK) return r;
  const int64_t n = cfg->n, W = cfg->W, C = cfg->num_chunks;
  if (cfg->err_dtype != OB_F32)
    return fail(OB_EINVAL, "ob_compress_noalloc: float32 error buffers only");
  if (cfg->rule != OB_RULE_SCALED_SIGN)
    return fail(OB_EINVAL, "ob_compress_noalloc: the scaled-sign rule only");
  if (C > kNoAllocMaxChunks)
    return fail(OB_EINVAL, "ob_compress_noalloc: %lld chunks, at most %d", (long long)C, kNoAllocMaxChunks);
  // Scratch needed: header (tables, status) + one double per (worker, warp tile).
  int64_t T = 0;
  for (int64_t k = 0; k < C; ++k) T += (cfg->chunk_offsets[k + 1] - cfg->chunk_offsets[k] + ob::kTile - 1) / ob::kTile;
  const size_t header = (kNoAllocTableBytes + 256 + 255) & ~size_t(255);
  const size_t need = header + sizeof(double) * size_t(W) * size_t(T);
  if (need > kNoAllocScratchBytes)
    return fail(OB_EINVAL,
                "ob_compress_noalloc: W=%lld, n=%lld needs %zu bytes of scratch; the fixed array holds %zu "
                "(about W*n <= %lld elements); use ob_create/ob_compress instead",
                (long long)W, (long long)n, need, kNoAllocScratchBytes,
                (long long)((kNoAllocScratchBytes - header) / sizeof(double) * ob::kTile));
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The chunk tables travel from a host buffer that the next call rewrites; a
  // copy recorded into a graph would read whatever that buffer holds at replay.
  // (Checked before any other runtime call, so a refused call leaves the
  // capture untouched.)
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if ((e = cudaStreamIsCapturing(st, &cap)) != cudaSuccess) return cuda_fail(e, "ob_compress_noalloc: cudaStreamIsCapturing");
  if (cap != cudaStreamCaptureStatusNone)
    return fail(OB_EINVAL, "ob_compress_noalloc: the stream is being captured into a graph; "
                           "this call copies its chunk tables from a host buffer that every call rewrites");
  struct { const void* p; int64_t count; const char* name; uintptr_t align; } bufs[] = {
      {grads, W * n, "grads", kAlignElems}, {err, W * n, "err", kAlignElems},
      {bits_w, W * words, "bits_w", kAlignWords}, {s_w, W * C, "s_w", kAlignWords}};
  for (auto& b : bufs)
    if ((r = check_dev(b.p, b.count, b.name, device, b.align)) != OB_OK) return r;

  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice* d = nullptr;
  if ((r = noalloc_setup(device, &d)) != OB_OK) return r;

  // Header image: off | wo | tp (int64, C+1 each) | vec (C bytes) | status (zeroed).
  std::memset(g_noalloc_header, 0, sizeof g_noalloc_header);
  int64_t* h_off = reinterpret_cast<int64_t*>(g_noalloc_header);
  int64_t* h_wo = h_off + (C + 1);
  int64_t* h_tp = h_wo + (C + 1);
  uint8_t* h_vec = reinterpret_cast<uint8_t*>(h_tp + (C + 1));
  const size_t status_at = (reinterpret_cast<unsigned char*>(h_vec + C) - g_noalloc_header + 255) & ~size_t(255);
  h_off[0] = h_wo[0] = h_tp[0] = 0;
  for (int64_t k = 0; k < C; ++k) {
    const int64_t o = cfg->chunk_offsets[k], nk = cfg->chunk_offsets[k + 1] - o;
    h_off[k + 1] = cfg->chunk_offsets[k + 1];
    h_wo[k + 1] = h_wo[k] + words_of(nk);
    h_tp[k + 1] = h_tp[k] + (nk + ob::kTile - 1) / ob::kTile;
    h_vec[k] = (o % 8 == 0) && (nk % 8 == 0) && (W == 1 || n % 8 == 0);
  }
  if ((e = cudaMemcpyAsync(d->scratch, g_noalloc_header, status_at + sizeof(uint32_t),
                           cudaMemcpyHostToDevice, st)) != cudaSuccess)
    return cuda_fail(e, "ob_compress_noalloc: header copy");

  ob::Layout L{};
  L.off = reinterpret_cast<const int64_t*>(d->scratch);
  L.wo = L.off + (C + 1);
  L.tp = L.wo + (C + 1);
  L.vec = reinterpret_cast<const uint8_t*>(L.tp + (C + 1));
  L.n = n;
  L.T = T;
  L.words = words;
  L.C = static_cast<int32_t>(C);
  uint32_t* status = reinterpret_cast<uint32_t*>(d->scratch + status_at);
  double* part = reinterpret_cast<double*>(d->scratch + header);
  const int bf = cfg->grad_dtype == OB_BF16 ? 1 : 0;
  const float clip = cfg->clip;
  const bool cl = clip > 0.0f;
  if (T > 0) {
    const int g1 = noalloc_grid(d->num_sms, d->occ_norm[bf][cl ? 1 : 0], W * T);
    const uint16_t* gh = static_cast<const uint16_t*>(grads);
    const float* gf = static_cast<const float*>(grads);
    if (bf && cl) ob::k_worker_norm<uint16_t, float, true><<<g1, ob::kBlock, 0, st>>>(L, int(W), gh, err, clip, part, status);
    else if (bf) ob::k_worker_norm<uint16_t, float, false><<<g1, ob::kBlock, 0, st>>>(L, int(W), gh, err, clip, part, status);
    else if (cl) ob::k_worker_norm<float, float, true><<<g1, ob::kBlock, 0, st>>>(L, int(W), gf, err, clip, part, status);
    else ob::k_worker_norm<float, float, false><<<g1, ob::kBlock, 0, st>>>(L, int(W), gf, err, clip, part, status);
  }
  ob::k_finalize_scale<true><<<dim3(unsigned(C), unsigned(W)), ob::kFinalizeThreads, 0, st>>>(L, part, T, s_w);
  if (T > 0) {
    const int g2 = noalloc_grid(d->num_sms, d->occ_pack[bf][cl ? 1 : 0], T);
    const uint16_t* gh = static_cast<const uint16_t*>(grads);
    const float* gf = static_cast<const float*>(grads);
    if (bf && cl) ob::k_worker_pack<uint16_t, float, false, true, false, 2, false><<<g2, ob::kBlock, 0, st>>>(L, int(W), gh, err, s_w, bits_w, nullptr, nullptr, nullptr, clip, status);
    else if (bf) ob::k_worker_pack<uint16_t, float, false, false, false, 2, false><<<g2, ob::kBlock, 0, st>>>(L, int(W), gh, err, s_w, bits_w, nullptr, nullptr, nullptr, clip, status);
    else if (cl) ob::k_worker_pack<float, float, false, true, false, 2, false><<<g2, ob::kBlock, 0, st>>>(L, int(W), gf, err, s_w, bits_w, nullptr, nullptr, nullptr, clip, status);
    else ob::k_worker_pack<float, float, false, false, false, 2, false><<<g2, ob::kBlock, 0, st>>>(L, int(W), gf, err, s_w, bits_w, nullptr, nullptr, nullptr, clip, status);
  }
  return check_launch("ob_compress_noalloc");
}
