// kernels.cuh -- sm_100a streaming kernels of the 1-bit Adam compressed-phase step.
//
// Method ("DeepSpeed Communication Compression and Hiding", section "1-bit Adam",
// 机制; "1-bit LAMB" for the trust ratio; CANN 1-bit Adam article section 3.2 for
// the clip and the NaN check):
//   worker w, chunk k:  c = clip(g_w) + err_w,  s_wk = ||c||_2 / sqrt(n_k),
//                       bit = (c >= 0),  err_w = c - s_wk * sign
//   server:             c_srv = (sum_w s_wk sign_w) / W + srv_err,
//                       s_srv = ||c_srv|| / sqrt(n_k),  srv_err = c_srv - s_srv sign'
//   update:             g_hat = s_srv sign';  m = b1 m + (1-b1) g_hat;
//                       p -= lr m / (sqrt(v) + eps)     (v frozen)
//
// Everything here is HBM streaming: no contraction, so no tensor cores.  The
// step is three element passes because two per-chunk norms gate the writes:
//   pass 1  k_worker_norm      reads g, err               -> per-tile sum c^2
//   pass 2  k_worker_pack      reads g, err, srv_err      -> err, bits_w, per-tile sum c_srv^2
//   pass 3  k_server_update    reads bits_w, srv_err, m, v, p -> bits_srv, srv_err, m, p
// with a tiny deterministic finalize (per-chunk fp64 sum of the tile partials,
// fixed order) between passes.
//
// Work unit: a warp tile of kTile = 512 consecutive elements of ONE chunk (a
// chunk is cut into ceil(n_k / 512) tiles; tiles never straddle chunks).  Warps
// stride over tiles (persistent grid), so chunks of any size mix freely and the
// per-tile partial norm lands at a fixed index: sums are reproducible run to run.
//
// Vector path (chunk start and length multiples of 8 elements, and the worker
// row stride a multiple of 8): lane L of a 256-element group holds elements
// 8L..8L+7 (one 32-byte v8.f32 access, or one 16-byte load of 8 bf16), so its 8 sign bits
// form byte (L % 4) of word (L / 4) of the group; two xor-shuffles assemble the
// eight 32-bit words, LSB-first.  Any other chunk takes the scalar path: lane L
// holds element 32j + L and one ballot is one word.
//
// Floating point: fp32 arithmetic in the order written, built with -fmad=false,
// IEEE division and square root, so every per-element value is the one the
// plain C statement of the method gives for the same scales.  Norms are summed
// in double with an explicit fma (c*c is exact in double, so fma(c, c, acc)
// equals acc + c*c rounded once).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ob {

constexpr int kWarp = 32;
constexpr int kVec = 8;                          // elements per lane per group
constexpr int kGroupElems = kWarp * kVec;        // 256 elements = 8 words
constexpr int kGroups = 2;                       // groups per warp tile
constexpr int kTile = kGroupElems * kGroups;     // 512 elements per warp tile
constexpr int kTileWords = kTile / 32;
constexpr int kBlock = 256;                      // threads per CTA (8 warps)
constexpr int kWarpsPerBlock = kBlock / kWarp;
constexpr int kFinalizeThreads = 1024;
constexpr bool kWide = true;                     // 256-bit (v8.f32) global accesses for fp32 arrays
constexpr int kUpdateMinBlocks = 2;              // pass 3: resident CTAs per SM asked of ptxas
constexpr unsigned kFull = 0xffffffffu;
constexpr uint32_t kStatusNonfinite = 1u;

// Chunk tables in device memory (owned by the ctx scratch).
struct Layout {
  const int64_t* off;   // [C+1] first element of every chunk
  const int64_t* wo;    // [C+1] first word of every chunk within a packed row
  const int64_t* tp;    // [C+1] first warp tile (kTile elements) of every chunk
  const uint8_t* vec;   // [C]   1: 8-wide vector path, 0: scalar path
  int64_t n;            // elements per row
  int64_t T;            // warp tiles per row
  int64_t words;        // packed words per row
  int32_t C;
};

struct Hyper {
  float lr, b1, omb1, b2, omb2, eps, clip;   // omb = 1 - b, computed in float on the host
};

struct Tile {
  int k;
  int64_t ck0;   // element index of the chunk start
  int64_t nk;    // chunk length
  int64_t rel;   // chunk-relative index of the tile's first element
  int64_t w0;    // word index of the chunk's first word
  bool vec;
};

// Largest k with tp[k] <= t (tp non-decreasing, tp[C] = T > t): the chunk that
// owns tile t; empty chunks are skipped automatically.
__device__ __forceinline__ int find_chunk(const Layout& L, int64_t t, int hint) {
  if (L.tp[hint] <= t && t < L.tp[hint + 1]) return hint;
  int lo = 0, hi = L.C;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (L.tp[mid] <= t) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ Tile tile_at(const Layout& L, int64_t t, int& hint) {
  const int k = find_chunk(L, t, hint);
  hint = k;
  Tile r;
  r.k = k;
  r.ck0 = L.off[k];
  r.nk = L.off[k + 1] - r.ck0;
  r.rel = (t - L.tp[k]) * kTile;
  r.w0 = L.wo[k];
  r.vec = L.vec[k] != 0;
  return r;
}

// ---- element access ------------------------------------------------------------

__device__ __forceinline__ void ld8_ro(const float* p, float (&x)[8]) {
  if constexpr (kWide) {
    asm("ld.global.nc.L1::no_allocate.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3]), "=f"(x[4]), "=f"(x[5]), "=f"(x[6]), "=f"(x[7])
        : "l"(p));
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

// bf16 -> fp32 is exact: the 16 bits are the top half of the float.
__device__ __forceinline__ void ld8_ro(const uint16_t* p, float (&x)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
  x[4] = __uint_as_float(u.z << 16); x[5] = __uint_as_float(u.z & 0xffff0000u);
  x[6] = __uint_as_float(u.w << 16); x[7] = __uint_as_float(u.w & 0xffff0000u);
}

// Read-write buffers: plain (coherent) loads; each element is read once, then
// written once by the same thread, so no load is ever moved past its store.
__device__ __forceinline__ void ld8(const float* p, float (&x)[8]) {
  if constexpr (kWide) {
    asm("ld.global.L1::no_allocate.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3]), "=f"(x[4]), "=f"(x[5]), "=f"(x[6]), "=f"(x[7])
        : "l"(p));
  } else {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

__device__ __forceinline__ void st8(float* p, const float (&x)[8]) {
  if constexpr (kWide) {
    asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(x[0]), "f"(x[1]),
                 "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7])
                 : "memory");
  } else {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
}

__device__ __forceinline__ float ld1_ro(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld1_ro(const uint16_t* p) {
  return __uint_as_float(static_cast<uint32_t>(__ldg(p)) << 16);
}

__device__ __forceinline__ void zero8(float (&x)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = 0.0f;
}

// Error buffers: float32, or bfloat16 (uint16 patterns, rounded to nearest even on
// store, widened exactly on load).  Arithmetic is float32 either way.
__device__ __forceinline__ uint16_t bf16_rne(float x) {
  const uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return static_cast<uint16_t>((u >> 16) | 0x0040u);  // quiet NaN
  return static_cast<uint16_t>((u + 0x7fffu + ((u >> 16) & 1u)) >> 16);
}

__device__ __forceinline__ void ld8(const uint16_t* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
  x[4] = __uint_as_float(u.z << 16); x[5] = __uint_as_float(u.z & 0xffff0000u);
  x[6] = __uint_as_float(u.w << 16); x[7] = __uint_as_float(u.w & 0xffff0000u);
}

// Two floats -> two bfloat16 (round to nearest even) packed low|high, in one
// conversion instruction; equal to bf16_rne for every non-NaN input (a NaN
// stays a NaN, possibly with another payload).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void st8(uint16_t* p, const float (&x)[8]) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

__device__ __forceinline__ float ld1(const float* p) { return *p; }
__device__ __forceinline__ float ld1(const uint16_t* p) { return __uint_as_float(static_cast<uint32_t>(*p) << 16); }
__device__ __forceinline__ void st1(float* p, float x) { *p = x; }
__device__ __forceinline__ void st1(uint16_t* p, float x) { *p = bf16_rne(x); }

// ---- method pieces -------------------------------------------------------------

// Clamp the raw gradient to [-clip, clip] when clip > 0; NaN passes through.
__device__ __forceinline__ float clip_grad(float g, float clip) {
  if (!(clip > 0.0f)) return g;
  if (g > clip) return clip;
  if (g < -clip) return -clip;
  return g;
}

__device__ __forceinline__ float signed_scale(bool bit, float s) { return bit ? s : -s; }

// The mean of W scaled signs, acc / W: IEEE division, or the product with 1/W when
// W is a power of two -- x / 2^k and x * 2^-k round the same exact value, so the
// result is identical and the division's instruction sequence is saved.
// POW2 is a template parameter of the kernels (chosen on the host from W), so the
// choice is never a branch inside an element loop.
template <bool POW2>
struct Mean {
  float Wf, invW;
  __device__ __forceinline__ float operator()(float acc) const {
    if constexpr (POW2) return acc * invW;
    else return __fdiv_rn(acc, Wf);
  }
};

template <bool POW2>
__device__ __forceinline__ Mean<POW2> make_mean(int W) {
  Mean<POW2> m;
  m.Wf = static_cast<float>(W);
  m.invW = __fdiv_rn(1.0f, m.Wf);
  return m;
}

// The mean of kernels specialised for one worker (W1): the multiply by 1, known
// at compile time, so it costs nothing (x * 1 is x exactly).
template <bool POW2, bool W1>
__device__ __forceinline__ Mean<POW2> make_mean_w(int W) {
  if constexpr (W1) {
    static_assert(POW2, "one worker is a power of two");
    return Mean<POW2>{1.0f, 1.0f};
  }
  return make_mean<POW2>(W);
}

// A sum of squares of finite floats cannot overflow a double, so a non-finite
// tile sum means a non-finite value in the tile: one check per tile replaces a
// check per element.
__device__ __forceinline__ void flag_tile_sum(double sum, uint32_t* status) {
  if (!isfinite(sum)) atomicOr(status, kStatusNonfinite);
}

// Lanes 4q..4q+3 each hold one byte of word q (LSB-first); returns the whole
// word in every lane of the quad (lane 4q writes it).
__device__ __forceinline__ uint32_t quad_word(uint32_t byte, int lane) {
  uint32_t v = byte << (8 * (lane & 3));
  v |= __shfl_xor_sync(kFull, v, 1);
  v |= __shfl_xor_sync(kFull, v, 2);
  return v;
}

__device__ __forceinline__ uint32_t lane_byte(uint32_t word, int lane) {
  return (word >> (8 * (lane & 3))) & 0xffu;
}

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
  return x;
}

__device__ __forceinline__ void flag_nonfinite(bool bad, uint32_t* status) {
  if (__any_sync(kFull, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kStatusNonfinite);
}

// Programmatic dependent launch: every kernel first waits until the kernels
// before it in the stream have completed and their writes are visible (a no-op
// when it was launched without the programmatic-serialization attribute), then
// lets the next kernel's launch begin, so its set-up overlaps this kernel's
// tail.  Nothing is read or written before the wait.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ int64_t warp_id() {
  return (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
}
__device__ __forceinline__ int64_t warp_count() {
  return (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
}

// Grid-stride loop over items it = r * T + t (rows x tiles) without a 64-bit
// division per item: the warp's first item is split once, then t advances by the
// stride and carries into r -- the same items, in the same order, as it += stride.
struct RowTile {
  int r;
  int64_t t;
};

__device__ __forceinline__ RowTile first_item(int64_t T) {   // T > 0
  const int64_t it = warp_id();
  const int r = static_cast<int>(it / T);
  return RowTile{r, it - static_cast<int64_t>(r) * T};
}

__device__ __forceinline__ void next_item(RowTile& x, int64_t T, int rows) {
  x.t += warp_count();
  while (x.t >= T && x.r < rows) {
    x.t -= T;
    ++x.r;
  }
}

// ---- fused finaliser (small problems) ---------------------------------------------
// On small problems a separate finaliser launch costs as much as a pass, so the
// pass's last CTA computes the scales itself.  Every thread fences its partial
// stores; one thread per CTA then takes a ticket; the CTA that draws the last
// ticket has every partial visible and turns each (row, chunk)'s tile partials
// into its scale, one warp per (row, chunk): lane l sums slots tp[k] + l,
// tp[k] + l + 32, ... in order, then the fixed xor butterfly of warp_sum, so
// the scale is the same on every launch.  It resets the ticket for the next
// launch.  No thread waits on another CTA.  The stage calls use the same
// finaliser on the same problems, so the fused step and the stages agree bit
// for bit.
struct Fin {
  unsigned* ticket;    // zero at the start of the launch (ctx scratch)
  const double* part;  // [rows][row_stride] tile partials
  int64_t row_stride;
  int rows;
  float* out;          // [rows][C]: ||.|| / sqrt(n_k)
};

__device__ __forceinline__ void fused_finalize(const Layout& L, const Fin& f) {
  __shared__ unsigned s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(f.ticket, 1u) == gridDim.x - 1 ? 1u : 0u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // rows * T <= 2^15 on this path: 32-bit slot indices.  With few (row, chunk)
  // pairs, wpt warps share one: warp `share` sums the share-th contiguous part
  // of its slots, each lane keeping kFinLanes running sums (slot a + 32 i + l
  // goes to sum i % kFinLanes) so that kFinLanes loads are in flight; the sums
  // are added in index order, across lanes by the butterfly, and across the
  // shares in warp order -- a fixed order for a given problem.
  constexpr int kFinLanes = 8;
  __shared__ double s_share[kWarpsPerBlock];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tasks = f.rows * L.C;
  const int wpt = tasks >= kWarpsPerBlock ? 1 : tasks >= kWarpsPerBlock / 2 ? 2 : tasks >= 2 ? 4 : 8;
  const int per_round = kWarpsPerBlock / wpt;
  const int rounds = (tasks + per_round - 1) / per_round;
  for (int rd = 0; rd < rounds; ++rd) {
    const int task = rd * per_round + warp / wpt, share = warp % wpt;
    double acc = 0.0;
    if (task < tasks) {
      const int r = task / L.C, k = task - r * L.C;
      const double* pr = f.part + r * static_cast<int>(f.row_stride);
      const int t0 = static_cast<int>(L.tp[k]), t1 = static_cast<int>(L.tp[k + 1]);
      const int len = (t1 - t0 + wpt - 1) / wpt;
      const int a = t0 + share * len, b = min(t1, a + len);
      double part[kFinLanes];
#pragma unroll
      for (int u = 0; u < kFinLanes; ++u) part[u] = 0.0;
      for (int t = a + lane; t < b; t += kWarp * kFinLanes) {
        double x[kFinLanes];
#pragma unroll
        for (int u = 0; u < kFinLanes; ++u) {
          const int tu = t + u * kWarp;
          x[u] = tu < b ? __ldcg(pr + tu) : 0.0;
        }
#pragma unroll
        for (int u = 0; u < kFinLanes; ++u) part[u] += x[u];
      }
#pragma unroll
      for (int u = 0; u < kFinLanes; ++u) acc += part[u];
      acc = warp_sum(acc);
    }
    if (lane == 0) s_share[warp] = acc;
    __syncthreads();
    if (threadIdx.x < per_round) {
      const int tk = rd * per_round + threadIdx.x;
      if (tk < tasks) {
        double S = 0.0;
        for (int i = 0; i < wpt; ++i) S += s_share[threadIdx.x * wpt + i];
        const int r = tk / L.C, k = tk - r * L.C;
        const int64_t nk = L.off[k + 1] - L.off[k];
        f.out[r * L.C + k] =
            nk > 0 ? __double2float_rn(__ddiv_rn(__dsqrt_rn(S), __dsqrt_rn(static_cast<double>(nk)))) : 0.0f;
      }
    }
    __syncthreads();
  }
  __syncthreads();
  if (threadIdx.x == 0) *f.ticket = 0u;
}

// ---- pass 1: per-tile sum of c^2 for every worker ----------------------------------
// part[w * T + t] = sum over tile t of (clip(g_w) + err_w)^2; a non-finite sum
// (some c is NaN/Inf) raises the status flag.
template <typename GT, typename ET, bool CLIP>
__device__ __forceinline__ void worker_norm_tiles(Layout L, int W, const GT* __restrict__ grads, const ET* __restrict__ err,
              float clip, double* __restrict__ part, uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t items = static_cast<int64_t>(W) * L.T;
  int hint = 0;
  for (int64_t it = warp_id(); it < items; it += warp_count()) {
    const int w = static_cast<int>(it / L.T);
    const int64_t t = it - static_cast<int64_t>(w) * L.T;
    const Tile tl = tile_at(L, t, hint);
    const GT* g = grads + static_cast<int64_t>(w) * L.n + tl.ck0;
    const ET* e = err + static_cast<int64_t>(w) * L.n + tl.ck0;
    double acc = 0.0;
    if (tl.vec) {
      float gv[kGroups][8], ev[kGroups][8];
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        if (i0 < tl.nk) { ld8_ro(g + i0, gv[q]); ld8_ro(e + i0, ev[q]); }
        else { zero8(gv[q]); zero8(ev[q]); }
      }
#pragma unroll
      for (int q = 0; q < kGroups; ++q)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float c = (CLIP ? clip_grad(gv[q][j], clip) : gv[q][j]) + ev[q][j];
          acc = fma(static_cast<double>(c), static_cast<double>(c), acc);
        }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          const float c = (CLIP ? clip_grad(ld1_ro(g + i), clip) : ld1_ro(g + i)) + ld1_ro(e + i);
          acc = fma(static_cast<double>(c), static_cast<double>(c), acc);
        }
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) {
      part[it] = acc;
      flag_tile_sum(acc, status);
    }
  }
}

template <typename GT, typename ET, bool CLIP>
__global__ void __launch_bounds__(kBlock)
k_worker_norm(Layout L, int W, const GT* __restrict__ grads, const ET* __restrict__ err,
              float clip, double* __restrict__ part, uint32_t* __restrict__ status) {
  pdl_enter();
  worker_norm_tiles<GT, ET, CLIP>(L, W, grads, err, clip, part, status);
}

// Small problems: pass 1 and the worker scales (fin: rows = W, part, s_w) in one launch.
template <typename GT, typename ET, bool CLIP>
__global__ void __launch_bounds__(kBlock)
k_worker_norm_fin(Layout L, int W, const GT* __restrict__ grads, const ET* __restrict__ err,
              float clip, double* __restrict__ part, uint32_t* __restrict__ status, Fin fin) {
  pdl_enter();
  worker_norm_tiles<GT, ET, CLIP>(L, W, grads, err, clip, part, status);
  fused_finalize(L, fin);
}


// ---- finalize: per-chunk scale from tile partials ----------------------------------
// The partials of chunk k are the slots [tp[k], tp[k+1]) of each row (one per
// warp tile).  out[r * C + k] = sqrt(sum of the slots, fixed order) / sqrt(n_k);
// 0 for an empty chunk.  grid = (C, R).
__device__ __forceinline__ double block_sum_fixed(double x, double* sm) {
  const int tid = threadIdx.x;
  sm[tid] = x;
  __syncthreads();
#pragma unroll
  for (int s = kFinalizeThreads / 2; s > 0; s >>= 1) {
    if (tid < s) sm[tid] += sm[tid + s];
    __syncthreads();
  }
  const double r = sm[0];
  __syncthreads();
  return r;
}

// The result of (row r, chunk k) goes to out[r * C + k].
template <bool RMS>
__global__ void __launch_bounds__(kFinalizeThreads)
k_finalize_scale(Layout L, const double* __restrict__ part, int64_t row_stride, float* __restrict__ out) {
  pdl_enter();
  __shared__ double sm[kFinalizeThreads];
  const int k = blockIdx.x, r = blockIdx.y;
  const double* pr = part + static_cast<int64_t>(r) * row_stride;
  double acc = 0.0;
  for (int64_t t = L.tp[k] + threadIdx.x; t < L.tp[k + 1]; t += kFinalizeThreads) acc += pr[t];
  const double S = block_sum_fixed(acc, sm);
  if (threadIdx.x == 0) {
    const int64_t nk = L.off[k + 1] - L.off[k];
    float o = 0.0f;
    if (!RMS) o = __double2float_rn(__dsqrt_rn(S));   // plain L2 norm (monitoring)
    else if (nk > 0) o = __double2float_rn(__ddiv_rn(__dsqrt_rn(S), __dsqrt_rn(static_cast<double>(nk))));
    out[static_cast<int64_t>(r) * L.C + k] = o;
  }
}

// LAMB trust ratio per layer (chunk): r = sqrt(P) / sqrt(U), 1 if either is 0.  grid = C.
__global__ void __launch_bounds__(kFinalizeThreads)
k_finalize_ratio(Layout L, const double* __restrict__ partP, const double* __restrict__ partU,
                 float* __restrict__ ratio) {
  pdl_enter();
  __shared__ double sm[kFinalizeThreads];
  const int k = blockIdx.x;
  double a = 0.0, b = 0.0;
  for (int64_t t = L.tp[k] + threadIdx.x; t < L.tp[k + 1]; t += kFinalizeThreads) {
    a += partP[t];
    b += partU[t];
  }
  const double P = block_sum_fixed(a, sm);
  const double U = block_sum_fixed(b, sm);
  if (threadIdx.x == 0)
    ratio[k] = (P > 0.0 && U > 0.0) ? __double2float_rn(__ddiv_rn(__dsqrt_rn(P), __dsqrt_rn(U)))
                                    : 1.0f;
}

// ---- pass 2: worker pack (+ server accumulation) -------------------------------------
// For every worker: c = clip(g) + err, bit = (c >= 0), err = c - s_w sign, bits_w.
// SERVER: also c_srv = (sum_w s_w sign_w) / W + srv_err and part_srv[t] = sum c_srv^2.
// Non-finite c were flagged by pass 1 (same values); non-finite c_srv by the tile sum.
// GP = groups of one tile whose loads are issued together: 1 keeps the kernel
// under 80 registers (3 CTAs per SM), best when W is small and a tile carries few
// bytes per instruction; 2 keeps more bytes in flight per warp, best for large W.
// CACHE (with SERVER): also store c_srv to csrv[n], so pass 3 reads one float
// per element instead of rebuilding the sum from the W workers' words.
template <typename GT, typename ET, bool SERVER, bool CLIP, bool POW2, int GP, bool CACHE>
__device__ __forceinline__ void worker_pack_tiles(Layout L, int W, const GT* __restrict__ grads, ET* __restrict__ err,
              const float* __restrict__ s_w, uint32_t* __restrict__ bits_w,
              const ET* __restrict__ srv_err, double* __restrict__ part_srv, float* __restrict__ csrv,
              float clip, uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean<POW2>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    double tsum = 0.0;
    if (tl.vec) {
#pragma unroll 1
      for (int q0 = 0; q0 < kGroups; q0 += GP) {
        float acc[GP][8], sv[GP][8];
        bool in[GP];
#pragma unroll
        for (int u = 0; u < GP; ++u) {
          const int64_t i0 = tl.rel + (q0 + u) * kGroupElems + lane * kVec;
          in[u] = i0 < tl.nk;
          zero8(acc[u]);
          if (SERVER) {
            if (in[u]) ld8_ro(srv_err + tl.ck0 + i0, sv[u]); else zero8(sv[u]);
          }
        }
        for (int w = 0; w < W; ++w) {
          const GT* g = grads + static_cast<int64_t>(w) * L.n + tl.ck0;
          ET* e = err + static_cast<int64_t>(w) * L.n + tl.ck0;
          const float s = __ldg(s_w + static_cast<int64_t>(w) * L.C + tl.k);
          float gv[GP][8], ev[GP][8];
#pragma unroll
          for (int u = 0; u < GP; ++u) {
            const int64_t i0 = tl.rel + (q0 + u) * kGroupElems + lane * kVec;
            if (in[u]) { ld8_ro(g + i0, gv[u]); ld8(e + i0, ev[u]); }
            else { zero8(gv[u]); zero8(ev[u]); }
          }
#pragma unroll
          for (int u = 0; u < GP; ++u) {
            const int64_t i0 = tl.rel + (q0 + u) * kGroupElems + lane * kVec;
            uint32_t byte = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float c = (CLIP ? clip_grad(gv[u][j], clip) : gv[u][j]) + ev[u][j];
              const bool b = c >= 0.0f;
              const float d = signed_scale(b, s);
              byte |= static_cast<uint32_t>(b) << j;
              ev[u][j] = c - d;
              acc[u][j] = acc[u][j] + d;
            }
            if (!in[u]) byte = 0;
            else st8(e + i0, ev[u]);
            const uint32_t word = quad_word(byte, lane);
            const int64_t wrel = (tl.rel + (q0 + u) * kGroupElems) / 32 + (lane >> 2);
            if ((lane & 3) == 0 && wrel * 32 < tl.nk)
              bits_w[static_cast<int64_t>(w) * L.words + tl.w0 + wrel] = word;
          }
        }
        if (SERVER) {
#pragma unroll
          for (int u = 0; u < GP; ++u)
            if (in[u]) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {        // c_srv in place of the sum
                acc[u][j] = mean(acc[u][j]) + sv[u][j];
                tsum = fma(static_cast<double>(acc[u][j]), static_cast<double>(acc[u][j]), tsum);
              }
              if (CACHE) st8(csrv + tl.ck0 + tl.rel + (q0 + u) * kGroupElems + lane * kVec, acc[u]);
            }
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        const bool inb = i < tl.nk;
        float acc = 0.0f;
        for (int w = 0; w < W; ++w) {
          const float s = __ldg(s_w + static_cast<int64_t>(w) * L.C + tl.k);
          ET* e = err + static_cast<int64_t>(w) * L.n + tl.ck0;
          bool b = false;
          if (inb) {
            const float g = ld1_ro(grads + static_cast<int64_t>(w) * L.n + tl.ck0 + i);
            const float c = (CLIP ? clip_grad(g, clip) : g) + ld1(e + i);
            b = c >= 0.0f;
            const float d = signed_scale(b, s);
            st1(e + i, c - d);
            acc = acc + d;
          }
          const uint32_t word = __ballot_sync(kFull, b);
          if (lane == 0 && (tl.rel + j * 32) < tl.nk)
            bits_w[static_cast<int64_t>(w) * L.words + tl.w0 + tl.rel / 32 + j] = word;
        }
        if (SERVER && inb) {
          const float cs = mean(acc) + ld1_ro(srv_err + tl.ck0 + i);
          tsum = fma(static_cast<double>(cs), static_cast<double>(cs), tsum);
          if (CACHE) csrv[tl.ck0 + i] = cs;
        }
      }
    }
    if (SERVER) {
      tsum = warp_sum(tsum);
      if (lane == 0) {
        part_srv[t] = tsum;
        flag_tile_sum(tsum, status);
      }
    }
  }
}

template <typename GT, typename ET, bool SERVER, bool CLIP, bool POW2, int GP, bool CACHE>
__global__ void __launch_bounds__(kBlock, GP == 1 ? 3 : 2)
k_worker_pack(Layout L, int W, const GT* __restrict__ grads, ET* __restrict__ err,
              const float* __restrict__ s_w, uint32_t* __restrict__ bits_w,
              const ET* __restrict__ srv_err, double* __restrict__ part_srv, float* __restrict__ csrv,
              float clip, uint32_t* __restrict__ status) {
  pdl_enter();
  worker_pack_tiles<GT, ET, SERVER, CLIP, POW2, GP, CACHE>(L, W, grads, err, s_w, bits_w, srv_err, part_srv, csrv, clip, status);
}

// Small problems (SERVER): pass 2 and the server scale (fin: rows = 1, part_srv, s_srv) in one launch.
template <typename GT, typename ET, bool SERVER, bool CLIP, bool POW2, int GP, bool CACHE>
__global__ void __launch_bounds__(kBlock, GP == 1 ? 3 : 2)
k_worker_pack_fin(Layout L, int W, const GT* __restrict__ grads, ET* __restrict__ err,
              const float* __restrict__ s_w, uint32_t* __restrict__ bits_w,
              const ET* __restrict__ srv_err, double* __restrict__ part_srv, float* __restrict__ csrv,
              float clip, uint32_t* __restrict__ status, Fin fin) {
  pdl_enter();
  worker_pack_tiles<GT, ET, SERVER, CLIP, POW2, GP, CACHE>(L, W, grads, err, s_w, bits_w, srv_err, part_srv, csrv, clip, status);
  fused_finalize(L, fin);
}


// ---- server average recomputed from the packed worker signs ---------------------------
// acc[j] = sum_w s_w[w][k] * sign_w(element), in ascending w (the same float
// additions pass 2 made), for the 8 elements of this lane in group (rel0).
// W1: exactly one worker, known at compile time -- the loop and its per-worker
// address arithmetic disappear (acc is still 0.0f + the one scaled sign, the
// same float operation), which is what lets pass 3 at W = 1 keep two groups of
// loads in flight under 96 registers.
template <bool W1>
__device__ __forceinline__ void server_sum8(const Layout& L, int W, const uint32_t* __restrict__ bits_w,
                                            const float* __restrict__ s_w, const Tile& tl,
                                            int64_t wrel, bool word_in, int lane, float (&acc)[8]) {
  zero8(acc);
  const int nw = W1 ? 1 : W;
  for (int w = 0; w < nw; ++w) {
    const float s = __ldg(s_w + static_cast<int64_t>(w) * L.C + tl.k);
    const uint32_t word =
        word_in ? __ldg(bits_w + static_cast<int64_t>(w) * L.words + tl.w0 + wrel) : 0u;
    const uint32_t byte = lane_byte(word, lane);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = acc[j] + signed_scale((byte >> j) & 1u, s);
  }
}

// Server norm only (stage-wise call): part_srv[t] = sum over the tile of c_srv^2,
// the values and the order of the fused pass 2.  The server errors of both groups
// are loaded before the sums; W1 (with POW2): one worker (see server_sum8).
template <typename ET, bool POW2, bool W1>
__device__ __forceinline__ void server_norm_tiles(Layout L, int W, const uint32_t* __restrict__ bits_w, const float* __restrict__ s_w,
              const ET* __restrict__ srv_err, double* __restrict__ part_srv,
              uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean_w<POW2, W1>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    double tsum = 0.0;
    if (tl.vec) {
      float sv[kGroups][8];
      bool in[kGroups];
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        in[q] = i0 < tl.nk;
        if (in[q]) ld8_ro(srv_err + tl.ck0 + i0, sv[q]); else zero8(sv[q]);
      }
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t wrel = (tl.rel + q * kGroupElems) / 32 + (lane >> 2);
        float acc[8];
        server_sum8<W1>(L, W, bits_w, s_w, tl, wrel, wrel * 32 < tl.nk, lane, acc);
        if (in[q]) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float cs = mean(acc[j]) + sv[q][j];
            tsum = fma(static_cast<double>(cs), static_cast<double>(cs), tsum);
          }
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          float acc = 0.0f;
          for (int w = 0; w < (W1 ? 1 : W); ++w) {
            const float s = __ldg(s_w + static_cast<int64_t>(w) * L.C + tl.k);
            const uint32_t word = __ldg(bits_w + static_cast<int64_t>(w) * L.words + tl.w0 + tl.rel / 32 + j);
            acc = acc + signed_scale((word >> lane) & 1u, s);
          }
          const float cs = mean(acc) + ld1_ro(srv_err + tl.ck0 + i);
          tsum = fma(static_cast<double>(cs), static_cast<double>(cs), tsum);
        }
      }
    }
    tsum = warp_sum(tsum);
    if (lane == 0) {
      part_srv[t] = tsum;
      flag_tile_sum(tsum, status);
    }
  }
}

template <typename ET, bool POW2, bool W1>
__global__ void __launch_bounds__(kBlock)
k_server_norm(Layout L, int W, const uint32_t* __restrict__ bits_w, const float* __restrict__ s_w,
              const ET* __restrict__ srv_err, double* __restrict__ part_srv,
              uint32_t* __restrict__ status) {
  pdl_enter();
  server_norm_tiles<ET, POW2, W1>(L, W, bits_w, s_w, srv_err, part_srv, status);
}

// Small problems: the server sums and the server scale in one launch (the stage
// call's counterpart of k_worker_pack_fin, so both give the same scale).
template <typename ET, bool POW2, bool W1>
__global__ void __launch_bounds__(kBlock)
k_server_norm_fin(Layout L, int W, const uint32_t* __restrict__ bits_w, const float* __restrict__ s_w,
              const ET* __restrict__ srv_err, double* __restrict__ part_srv,
              uint32_t* __restrict__ status, Fin fin) {
  pdl_enter();
  server_norm_tiles<ET, POW2, W1>(L, W, bits_w, s_w, srv_err, part_srv, status);
  fused_finalize(L, fin);
}


// ---- pass 3: server pack + update ------------------------------------------------------
enum class Upd : int {
  kNone = 0,   // server pack + server error only (stage-wise call)
  kAdam = 1,   // + m and p (frozen-v Adam)
  kLambM = 2,  // + m, and per-tile sums of p^2 and u^2 for the LAMB trust ratio
};

// Per element: the update given g_hat = d.
template <Upd U>
__device__ __forceinline__ void update_elem(float d, float& m, float v, float& p, const Hyper& h,
                                            double& P, double& Usum, bool& bad) {
  if (U == Upd::kAdam) {
    m = h.b1 * m + h.omb1 * d;
    p = p - __fdiv_rn(h.lr * m, __fsqrt_rn(v) + h.eps);
    bad |= !isfinite(p);
  } else if (U == Upd::kLambM) {
    m = h.b1 * m + h.omb1 * d;
    const float u = __fdiv_rn(m, __fsqrt_rn(v) + h.eps);
    P = fma(static_cast<double>(p), static_cast<double>(p), P);
    Usum = fma(static_cast<double>(u), static_cast<double>(u), Usum);
  }
}

// FROM_WORKERS: c_srv from bits_w/s_w/srv_err, quantised with s_srv, bits_srv and
// srv_err written (the compressed allreduce's second half).  Otherwise g_hat is
// read back from bits_srv/s_srv (the update-only stage call).  CACHED (with
// FROM_WORKERS): c_srv is read from csrv, where pass 2 stored it, and srv_err is
// only written.  W1 (with FROM_WORKERS, POW2): one worker (see server_sum8).
template <Upd U, bool FROM_WORKERS, bool POW2, typename ET, bool CACHED, bool W1>
__global__ void __launch_bounds__(kBlock, kUpdateMinBlocks)
k_server_update(Layout L, int W, const uint32_t* __restrict__ bits_w, const float* __restrict__ s_w,
                const float* __restrict__ csrv, const float* __restrict__ s_srv, ET* __restrict__ srv_err,
                uint32_t* __restrict__ bits_srv, float* __restrict__ m, const float* __restrict__ v,
                float* __restrict__ p, Hyper h, double* __restrict__ partP,
                double* __restrict__ partU, uint32_t* __restrict__ status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean_w<POW2, W1>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    const float s2 = __ldg(s_srv + tl.k);
    double Psum = 0.0, Usum = 0.0;
    bool bad = false;
    if (tl.vec) {
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        const int64_t wrel = (tl.rel + q * kGroupElems) / 32 + (lane >> 2);
        const bool word_in = wrel * 32 < tl.nk;
        const bool in = i0 < tl.nk;
        const int64_t gi = tl.ck0 + i0;
        float sv[8], mv[8], vv[8], pv[8];
        if (in) {
          if (FROM_WORKERS && !CACHED) ld8(srv_err + gi, sv);
          if (FROM_WORKERS && CACHED) ld8_ro(csrv + gi, sv);      // sv holds c_srv itself
          if (U != Upd::kNone) { ld8(m + gi, mv); ld8_ro(v + gi, vv); ld8(p + gi, pv); }
        }
        uint32_t byte = 0;
        if (FROM_WORKERS) {
          float acc[8];
          if (!CACHED) server_sum8<W1>(L, W, bits_w, s_w, tl, wrel, word_in, lane, acc);
          if (in) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float cs = CACHED ? sv[j] : mean(acc[j]) + sv[j];
              const bool b = cs >= 0.0f;
              const float d = signed_scale(b, s2);
              byte |= static_cast<uint32_t>(b) << j;
              sv[j] = cs - d;
              update_elem<U>(d, mv[j], vv[j], pv[j], h, Psum, Usum, bad);
            }
            st8(srv_err + gi, sv);
          }
          const uint32_t word = quad_word(byte, lane);
          if ((lane & 3) == 0 && word_in) bits_srv[tl.w0 + wrel] = word;
        } else {
          const uint32_t word = word_in ? __ldg(bits_srv + tl.w0 + wrel) : 0u;
          byte = lane_byte(word, lane);
          if (in) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              update_elem<U>(signed_scale((byte >> j) & 1u, s2), mv[j], vv[j], pv[j], h, Psum, Usum, bad);
          }
        }
        if (in && U != Upd::kNone) {
          st8(m + gi, mv);
          if (U == Upd::kAdam) st8(p + gi, pv);
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        const bool inb = i < tl.nk;
        const int64_t gi = tl.ck0 + i;
        const int64_t wi = tl.w0 + tl.rel / 32 + j;
        bool b = false;
        float d = 0.0f;
        if (FROM_WORKERS) {
          if (inb) {
            float acc = 0.0f;
            if (!CACHED)
              for (int w = 0; w < (W1 ? 1 : W); ++w) {
                const float s = __ldg(s_w + static_cast<int64_t>(w) * L.C + tl.k);
                const uint32_t word = __ldg(bits_w + static_cast<int64_t>(w) * L.words + wi);
                acc = acc + signed_scale((word >> lane) & 1u, s);
              }
            const float cs = CACHED ? __ldg(csrv + gi) : mean(acc) + ld1(srv_err + gi);
            b = cs >= 0.0f;
            d = signed_scale(b, s2);
            st1(srv_err + gi, cs - d);
          }
          const uint32_t word = __ballot_sync(kFull, b);
          if (lane == 0 && (tl.rel + j * 32) < tl.nk) bits_srv[wi] = word;
        } else if (inb) {
          d = signed_scale((__ldg(bits_srv + wi) >> lane) & 1u, s2);
        }
        if (inb && U != Upd::kNone) {
          float mv = m[gi], pv = p[gi];
          update_elem<U>(d, mv, __ldg(v + gi), pv, h, Psum, Usum, bad);
          m[gi] = mv;
          if (U == Upd::kAdam) p[gi] = pv;
        }
      }
    }
    if (U == Upd::kLambM) {
      Psum = warp_sum(Psum);
      Usum = warp_sum(Usum);
      if (lane == 0) { partP[t] = Psum; partU[t] = Usum; }
    }
    flag_nonfinite(bad, status);
  }
}

// ---- monitoring: per-tile sums of squares of R fp32 rows [R][n] --------------------------
template <typename ET>
__global__ void __launch_bounds__(kBlock)
k_rows_sumsq(Layout L, int R, const ET* __restrict__ x, double* __restrict__ part) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t items = static_cast<int64_t>(R) * L.T;
  int hint = 0;
  for (int64_t it = warp_id(); it < items; it += warp_count()) {
    const int r = static_cast<int>(it / L.T);
    const int64_t t = it - static_cast<int64_t>(r) * L.T;
    const Tile tl = tile_at(L, t, hint);
    const ET* row = x + static_cast<int64_t>(r) * L.n + tl.ck0;
    double acc = 0.0;
    if (tl.vec) {
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        if (i0 < tl.nk) {
          float v[8];
          ld8_ro(row + i0, v);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc = fma(static_cast<double>(v[j]), static_cast<double>(v[j]), acc);
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          const float v = ld1_ro(row + i);
          acc = fma(static_cast<double>(v), static_cast<double>(v), acc);
        }
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) part[it] = acc;
  }
}

// ---- monitoring: the quantisation rate ------------------------------------------------------
// The rate of a chunk is the fraction of its n_k elements sent as +1 (sign bit
// set); for a message symmetric about zero its theoretical value is 1/2.
// part[r * T + t] = set bits among the real elements of warp tile t in plane
// `plane` of packed row r (chunk k's plane p starts at word wo[k] + p ceil(n_k / 32)).
// Bits past n_k are masked off; a count is exact in a double.
__global__ void __launch_bounds__(kBlock)
k_sign_count(Layout L, int R, const uint32_t* __restrict__ bits, int plane, double* __restrict__ part) {
  pdl_enter();
  // One thread per (row, tile): a warp reads 32 consecutive tiles' words, 2 KB.
  const int64_t items = static_cast<int64_t>(R) * L.T;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int hint = 0;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < items; it += stride) {
    const int r = static_cast<int>(it / L.T);
    const int64_t t = it - static_cast<int64_t>(r) * L.T;
    const Tile tl = tile_at(L, t, hint);
    const int64_t nwk = (tl.nk + 31) / 32, wi0 = tl.rel / 32;
    const int nw = static_cast<int>(min(static_cast<int64_t>(kTileWords), nwk - wi0));
    const uint32_t* q = bits + static_cast<int64_t>(r) * L.words + tl.w0 + plane * nwk + wi0;
    unsigned cnt = 0;
    for (int j = 0; j < nw; ++j) {
      uint32_t word = __ldg(q + j);
      const int64_t left = tl.nk - (wi0 + j) * 32;   // real bits in this word
      if (left < 32) word &= (1u << left) - 1u;
      cnt += __popc(word);
    }
    part[it] = static_cast<double>(cnt);
  }
}

// out[(r * C + k) * planes + plane] = (float)(count / n_k) (double division, one
// rounding), 0 for an empty chunk.  grid = (C, R).
__global__ void __launch_bounds__(kFinalizeThreads)
k_finalize_rate(Layout L, const double* __restrict__ part, int64_t row_stride, float* __restrict__ out,
                int planes, int plane) {
  pdl_enter();
  __shared__ double sm[kFinalizeThreads];
  const int k = blockIdx.x, r = blockIdx.y;
  const double* pr = part + static_cast<int64_t>(r) * row_stride;
  double acc = 0.0;
  for (int64_t t = L.tp[k] + threadIdx.x; t < L.tp[k + 1]; t += kFinalizeThreads) acc += pr[t];
  const double S = block_sum_fixed(acc, sm);
  if (threadIdx.x == 0) {
    const int64_t nk = L.off[k + 1] - L.off[k];
    out[(static_cast<int64_t>(r) * L.C + k) * planes + plane] =
        nk > 0 ? __double2float_rn(__ddiv_rn(S, static_cast<double>(nk))) : 0.0f;
  }
}

// ---- 0/1 Adam local step ------------------------------------------------------------------
// A local step sends nothing: every worker keeps its gradient in its error
// buffer for the next synchronised step, err_w = clip(g_w) + err_w, and the
// parameters move with the current m and v, which stay as they are:
//   Adam: p -= lr m / (sqrt(v) + eps);
//   LAMB (kLambM): per-tile sums of p^2 and u^2, u = m / (sqrt(v) + eps), for the
//   trust ratio; the parameter step follows in k_lamb_param.
// A non-finite kept value or parameter raises the status flag.
template <Upd U>
__device__ __forceinline__ void local_elem(float m, float v, float& p, const Hyper& h, double& P,
                                           double& Usum, bool& bad) {
  if (U == Upd::kAdam) {
    p = p - __fdiv_rn(h.lr * m, __fsqrt_rn(v) + h.eps);
    bad |= !isfinite(p);
  } else {
    const float u = __fdiv_rn(m, __fsqrt_rn(v) + h.eps);
    P = fma(static_cast<double>(p), static_cast<double>(p), P);
    Usum = fma(static_cast<double>(u), static_cast<double>(u), Usum);
  }
}

template <typename GT, typename ET, bool CLIP, Upd U>
__global__ void __launch_bounds__(kBlock)
k_local_step(Layout L, int W, const GT* __restrict__ grads, ET* __restrict__ err,
             const float* __restrict__ m, const float* __restrict__ v, float* __restrict__ p, Hyper h,
             double* __restrict__ partP, double* __restrict__ partU, uint32_t* __restrict__ status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    double Psum = 0.0, Usum = 0.0;
    bool bad = false;
    if (tl.vec) {
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        if (i0 < tl.nk) {
          const int64_t gi = tl.ck0 + i0;
          float mv[8], vv[8], pv[8];
          ld8_ro(m + gi, mv);
          ld8_ro(v + gi, vv);
          ld8(p + gi, pv);
          for (int w = 0; w < W; ++w) {
            const int64_t e = static_cast<int64_t>(w) * L.n + gi;
            float gv[8], ev[8];
            ld8_ro(grads + e, gv);
            ld8(err + e, ev);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              ev[j] = (CLIP ? clip_grad(gv[j], h.clip) : gv[j]) + ev[j];
              bad |= !isfinite(ev[j]);
            }
            st8(err + e, ev);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) local_elem<U>(mv[j], vv[j], pv[j], h, Psum, Usum, bad);
          if (U == Upd::kAdam) st8(p + gi, pv);
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          const int64_t gi = tl.ck0 + i;
          for (int w = 0; w < W; ++w) {
            const int64_t e = static_cast<int64_t>(w) * L.n + gi;
            const float g = ld1_ro(grads + e);
            const float kept = (CLIP ? clip_grad(g, h.clip) : g) + ld1(err + e);
            bad |= !isfinite(kept);
            st1(err + e, kept);
          }
          float pv = p[gi];
          local_elem<U>(__ldg(m + gi), __ldg(v + gi), pv, h, Psum, Usum, bad);
          if (U == Upd::kAdam) p[gi] = pv;
        }
      }
    }
    if (U == Upd::kLambM) {
      Psum = warp_sum(Psum);
      Usum = warp_sum(Usum);
      if (lane == 0) { partP[t] = Psum; partU[t] = Usum; }
    }
    flag_nonfinite(bad, status);
  }
}

// ---- LAMB parameter step: p -= lr * r_k * m / (sqrt(v) + eps) ---------------------------
__global__ void __launch_bounds__(kBlock)
k_lamb_param(Layout L, const float* __restrict__ m, const float* __restrict__ v,
             float* __restrict__ p, const float* __restrict__ ratio, Hyper h,
             uint32_t* __restrict__ status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    const float lr_r = h.lr * __ldg(ratio + tl.k);
    bool bad = false;
    if (tl.vec) {
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        if (i0 < tl.nk) {
          const int64_t gi = tl.ck0 + i0;
          float mv[8], vv[8], pv[8];
          ld8_ro(m + gi, mv); ld8_ro(v + gi, vv); ld8(p + gi, pv);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float u = __fdiv_rn(mv[j], __fsqrt_rn(vv[j]) + h.eps);
            pv[j] = pv[j] - lr_r * u;
            bad |= !isfinite(pv[j]);
          }
          st8(p + gi, pv);
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          const int64_t gi = tl.ck0 + i;
          const float u = __fdiv_rn(__ldg(m + gi), __fsqrt_rn(__ldg(v + gi)) + h.eps);
          const float pn = p[gi] - lr_r * u;
          bad |= !isfinite(pn);
          p[gi] = pn;
        }
      }
    }
    flag_nonfinite(bad, status);
  }
}

// ---- the warmup's full-precision average ----------------------------------------------------
// mean[i] = (sum_{w=0..W-1} g_w[i]) / W: float additions in ascending w, one
// division (the average k_warmup forms before its moments).  A one-worker
// float32 warmup on `mean` then takes the same steps as the W-worker warmup.
// A non-finite mean raises the status flag.
template <typename GT, bool POW2>
__global__ void __launch_bounds__(kBlock)
k_grad_mean(Layout L, int W, const GT* __restrict__ grads, float* __restrict__ out,
            uint32_t* __restrict__ status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean<POW2>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    bool bad = false;
    if (tl.vec) {
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        if (i0 < tl.nk) {
          const int64_t gi = tl.ck0 + i0;
          float acc[8];
          zero8(acc);
          for (int w = 0; w < W; ++w) {
            float gv[8];
            ld8_ro(grads + static_cast<int64_t>(w) * L.n + gi, gv);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = acc[j] + gv[j];
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[j] = mean(acc[j]);
            bad |= !isfinite(acc[j]);
          }
          st8(out + gi, acc);
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          const int64_t gi = tl.ck0 + i;
          float acc = 0.0f;
          for (int w = 0; w < W; ++w) acc = acc + ld1_ro(grads + static_cast<int64_t>(w) * L.n + gi);
          acc = mean(acc);
          bad |= !isfinite(acc);
          out[gi] = acc;
        }
      }
    }
    flag_nonfinite(bad, status);
  }
}

// ---- full-precision warmup -------------------------------------------------------------
// g = (sum_w g_w) / W; m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
// Adam: p -= lr m / (sqrt(v) + eps).  LAMB: per-tile sums of p^2 and u^2 instead
// (the parameter step follows in k_lamb_param).
template <typename GT, bool LAMB, bool POW2>
__global__ void __launch_bounds__(kBlock)
k_warmup(Layout L, int W, const GT* __restrict__ grads, float* __restrict__ m,
         float* __restrict__ v, float* __restrict__ p, Hyper h, double* __restrict__ partP,
         double* __restrict__ partU, uint32_t* __restrict__ status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean<POW2>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    double Psum = 0.0, Usum = 0.0;
    bool bad = false;
    auto elem = [&](float gsum, float& mm, float& vv, float& pp) {
      const float g = mean(gsum);
      bad |= !isfinite(g);
      mm = h.b1 * mm + h.omb1 * g;
      vv = h.b2 * vv + h.omb2 * (g * g);
      if (LAMB) {
        const float u = __fdiv_rn(mm, __fsqrt_rn(vv) + h.eps);
        Psum = fma(static_cast<double>(pp), static_cast<double>(pp), Psum);
        Usum = fma(static_cast<double>(u), static_cast<double>(u), Usum);
      } else {
        pp = pp - __fdiv_rn(h.lr * mm, __fsqrt_rn(vv) + h.eps);
        bad |= !isfinite(pp);
      }
    };
    if (tl.vec) {
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        if (i0 < tl.nk) {
          const int64_t gi = tl.ck0 + i0;
          float acc[8], mv[8], vv[8], pv[8];
          zero8(acc);
          ld8(m + gi, mv); ld8(v + gi, vv); ld8(p + gi, pv);
          for (int w = 0; w < W; ++w) {
            float gv[8];
            ld8_ro(grads + static_cast<int64_t>(w) * L.n + gi, gv);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = acc[j] + gv[j];
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) elem(acc[j], mv[j], vv[j], pv[j]);
          st8(m + gi, mv);
          st8(v + gi, vv);
          if (!LAMB) st8(p + gi, pv);
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          const int64_t gi = tl.ck0 + i;
          float acc = 0.0f;
          for (int w = 0; w < W; ++w) acc = acc + ld1_ro(grads + static_cast<int64_t>(w) * L.n + gi);
          float mm = m[gi], vv = v[gi], pp = p[gi];
          elem(acc, mm, vv, pp);
          m[gi] = mm;
          v[gi] = vv;
          if (!LAMB) p[gi] = pp;
        }
      }
    }
    if (LAMB) {
      Psum = warp_sum(Psum);
      Usum = warp_sum(Usum);
      if (lane == 0) { partP[t] = Psum; partU[t] = Usum; }
    }
    flag_nonfinite(bad, status);
  }
}

}  // namespace ob
