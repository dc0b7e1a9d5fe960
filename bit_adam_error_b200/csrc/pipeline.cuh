// pipeline.cuh -- bulk-copy (1-D TMA) pipelined versions of the fused passes 2 and 3.
//
// Passes 2 and 3 of the step are latency-bound as plain warp-tile kernels: a warp
// loads its tile, then spends hundreds of instructions packing, reducing and
// storing it with nothing in flight.  Here memory and compute are decoupled:
//
//   CTA = 1 producer warp + kConsumers consumer warps, one CTA per SM, persistent
//   over block tiles of kBT = kConsumers * 256 elements of one chunk.
//   The producer streams the inputs of upcoming tiles into a ring of S shared-
//   memory stages with cp.async.bulk (global -> shared, completion counted in
//   bytes on the stage's "full" mbarrier); packed sign words, which need not be
//   16-byte aligned, come in with 4-byte cp.async whose completion also arrives
//   on the same mbarrier.  Consumer warp q computes the 256-element sub-tile q of
//   the stage, writes its outputs straight to global memory, and releases the
//   stage on its "empty" mbarrier.
//
// No multicast, no clusters, no tensor maps: plain bulk copies of 16-byte aligned
// contiguous ranges (vector-path chunks only; chunks off the 8-element grid are
// read by the consumers directly, as in the warp-tile kernels).
//
// Every mbarrier wait is bounded by a clock budget (about a second).  On expiry
// the waiter raises kStatusTimeout in the status word and the CTA winds down;
// before exiting, the producer waits (again bounded) for the copies it issued.
#pragma once

#include "kernels.cuh"

namespace ob {

constexpr int kConsumers = 8;
constexpr int kPipeCtasPerSm = 1;                        // resident CTAs per SM (shared-memory budget split)
constexpr int kPipeThreads = (kConsumers + 1) * kWarp;   // warp 0 = producer
constexpr int kBT = kConsumers * kGroupElems;            // 2048 elements per block tile
constexpr int kBTWords = kBT / 32;                       // 64 packed words
constexpr uint32_t kStatusTimeout = 2u;
constexpr long long kWaitBudget = 1ll << 31;             // clock cycles (~1 s at 1.9 GHz)

// ---- PTX wrappers -------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for the phase of `bar` with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitBudget) return false;
  return true;
}

// 1-D bulk copy global -> this CTA's shared memory; 16-byte aligned, size % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 4-byte asynchronous copy global -> shared.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies have landed (the
// barrier's expected count must include this arrival).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void ld8_smem(const float* p, float (&x)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void ld8_smem(const uint16_t* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
  x[4] = __uint_as_float(u.z << 16); x[5] = __uint_as_float(u.z & 0xffff0000u);
  x[6] = __uint_as_float(u.w << 16); x[7] = __uint_as_float(u.w & 0xffff0000u);
}

// Block tile tb of the layout (block-tile prefix L.tpb).
struct BTile {
  int k;
  int64_t ck0, nk, rel, len, w0;
  bool vec;
};

__device__ __forceinline__ int find_btile_chunk(const Layout& L, int64_t tb, int hint) {
  if (L.tpb[hint] <= tb && tb < L.tpb[hint + 1]) return hint;
  int lo = 0, hi = L.C;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (L.tpb[mid] <= tb) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ BTile btile_at(const Layout& L, int64_t tb, int& hint) {
  const int k = find_btile_chunk(L, tb, hint);
  hint = k;
  BTile b;
  b.k = k;
  b.ck0 = L.off[k];
  b.nk = L.off[k + 1] - b.ck0;
  b.rel = (tb - L.tpb[k]) * kBT;
  b.len = b.nk - b.rel < kBT ? b.nk - b.rel : kBT;
  b.w0 = L.wo[k];
  b.vec = L.vec[k] != 0;
  return b;
}

// avg = acc / W: IEEE division, or the exact product with 1/W when W is a power of two.
__device__ __forceinline__ float mean_of(float acc, float Wf, float invW, bool pow2) {
  return pow2 ? acc * invW : __fdiv_rn(acc, Wf);
}

// Shared ring bookkeeping common to both kernels.
struct Ring {
  uint64_t* full;
  uint64_t* empty;
  int* abort_flag;
};

__device__ __forceinline__ void raise_timeout(uint32_t* status, int* abort_flag) {
  atomicOr(status, kStatusTimeout);
  *reinterpret_cast<volatile int*>(abort_flag) = 1;
}

__device__ __forceinline__ bool aborted(const int* abort_flag) {
  return *reinterpret_cast<const volatile int*>(abort_flag) != 0;
}

// Producer epilogue: wait (bounded) until the copies of the last issued phase of
// every stage have landed, so none completes after the CTA exits.
__device__ __forceinline__ void drain_ring(const Ring& r, int S, long long issued) {
  for (int s = 0; s < S; ++s) {
    if (s >= issued) break;
    const long long last = issued - 1 - ((issued - 1 - s) % S);  // last item issued on stage s
    mbar_wait(&r.full[s], static_cast<uint32_t>((last / S) & 1));
  }
}

// ---- pass 2, pipelined: worker signs + error for every worker, server sums ----------
// Items are (block tile, worker) pairs, worker-inner, so a CTA sees all workers of
// a tile in a row and keeps the running sum of scaled signs in registers.
// Stage layout: g [kBT] (GT) | err [kBT] f32 | srv_err [kBT] f32 (last worker only).
template <typename GT>
__global__ void __launch_bounds__(kPipeThreads, kPipeCtasPerSm)
k_pack_server_pipe(Layout L, int W, const GT* __restrict__ grads, float* __restrict__ err,
                   const float* __restrict__ s_w, uint32_t* __restrict__ bits_w,
                   const float* __restrict__ srv_err, double* __restrict__ part_srv, float clip,
                   int S, uint32_t* __restrict__ status) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kStageBytes = kBT * (sizeof(GT) + 8);
  __shared__ uint64_t full_bar[16], empty_bar[16];
  __shared__ int abort_flag;
  const Ring ring{full_bar, empty_bar, &abort_flag};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumers);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t ntiles = L.Tb;
  const float Wf = static_cast<float>(W);
  const bool pow2 = (W & (W - 1)) == 0;
  const float invW = 1.0f / Wf;   // exact for powers of two
  const bool do_clip = clip > 0.0f;

  if (warp == 0) {
    // ---------------- producer ----------------
    long long it = 0;
    int hint = 0;
    for (int64_t tb = blockIdx.x; tb < ntiles; tb += gridDim.x) {
      if (__any_sync(kFull, aborted(&abort_flag))) break;
      const BTile bt = btile_at(L, tb, hint);
      for (int w = 0; w < W; ++w, ++it) {
        const int s = static_cast<int>(it % S);
        const bool free_ok = __all_sync(kFull, it < S || mbar_wait(&empty_bar[s], static_cast<uint32_t>(((it / S) - 1) & 1)));
        if (!free_ok) {
          if (lane == 0) raise_timeout(status, &abort_flag);
          break;
        }
        if (lane == 0) {
          unsigned char* st = smem + static_cast<size_t>(s) * kStageBytes;
          if (bt.vec) {
            const int64_t e0 = static_cast<int64_t>(w) * L.n + bt.ck0 + bt.rel;
            const bool last = w == W - 1;
            const uint32_t gbytes = static_cast<uint32_t>(bt.len * sizeof(GT));
            const uint32_t fbytes = static_cast<uint32_t>(bt.len * 4);
            mbar_arrive_expect_tx(&full_bar[s], gbytes + fbytes + (last ? fbytes : 0u));
            bulk_g2s(st, grads + e0, gbytes, &full_bar[s]);
            bulk_g2s(st + kBT * sizeof(GT), err + e0, fbytes, &full_bar[s]);
            if (last) bulk_g2s(st + kBT * (sizeof(GT) + 4), srv_err + bt.ck0 + bt.rel, fbytes, &full_bar[s]);
          } else {
            mbar_arrive(&full_bar[s]);   // scalar chunk: consumers read global memory
          }
        }
        __syncwarp();
      }
    }
    if (lane == 0) drain_ring(ring, S, it);
    return;
  }

  // ---------------- consumers ----------------
  const int q = warp - 1;
  long long it = 0;
  int hint = 0;
  for (int64_t tb = blockIdx.x; tb < ntiles; tb += gridDim.x) {
    const BTile bt = btile_at(L, tb, hint);
    const int64_t sub = bt.rel + q * kGroupElems;          // chunk-relative start of sub-tile q
    float acc[8];
    zero8(acc);
    double tsum = 0.0;
    bool ok = true;
    for (int w = 0; w < W; ++w, ++it) {
      const int s = static_cast<int>(it % S);
      if (!__all_sync(kFull, mbar_wait(&full_bar[s], static_cast<uint32_t>((it / S) & 1)))) {
        if (lane == 0) raise_timeout(status, &abort_flag);
        ok = false;
        break;
      }
      if (__any_sync(kFull, aborted(&abort_flag))) { ok = false; break; }
      const unsigned char* st = smem + static_cast<size_t>(s) * kStageBytes;
      const float s_wk = __ldg(s_w + static_cast<int64_t>(w) * L.C + bt.k);
      const bool last = w == W - 1;
      float* e_row = err + static_cast<int64_t>(w) * L.n + bt.ck0;
      if (bt.vec) {
        const int64_t i0 = sub + lane * kVec;
        const bool in = i0 < bt.nk;
        uint32_t byte = 0;
        if (in) {
          float gv[8], ev[8];
          ld8_smem(reinterpret_cast<const GT*>(st) + q * kGroupElems + lane * kVec, gv);
          ld8_smem(reinterpret_cast<const float*>(st + kBT * sizeof(GT)) + q * kGroupElems + lane * kVec, ev);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float g = do_clip ? clip_grad(gv[j], clip) : gv[j];
            const float c = g + ev[j];
            const bool b = c >= 0.0f;
            const float d = signed_scale(b, s_wk);
            byte |= static_cast<uint32_t>(b) << j;
            ev[j] = c - d;
            acc[j] = acc[j] + d;
          }
          st8(e_row + i0, ev);
          if (last) {
            float sv[8];
            ld8_smem(reinterpret_cast<const float*>(st + kBT * (sizeof(GT) + 4)) + q * kGroupElems + lane * kVec, sv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float cs = mean_of(acc[j], Wf, invW, pow2) + sv[j];
              tsum = fma(static_cast<double>(cs), static_cast<double>(cs), tsum);
            }
          }
        }
        const uint32_t word = quad_word(byte, lane);
        const int64_t wrel = sub / 32 + (lane >> 2);
        if ((lane & 3) == 0 && wrel * 32 < bt.nk)
          bits_w[static_cast<int64_t>(w) * L.words + bt.w0 + wrel] = word;
      } else {
        const GT* g_row = grads + static_cast<int64_t>(w) * L.n + bt.ck0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int64_t i = sub + j * 32 + lane;
          const bool inb = i < bt.nk;
          bool b = false;
          if (inb) {
            const float g = do_clip ? clip_grad(ld1_ro(g_row + i), clip) : ld1_ro(g_row + i);
            const float c = g + e_row[i];
            b = c >= 0.0f;
            const float d = signed_scale(b, s_wk);
            e_row[i] = c - d;
            acc[j] = acc[j] + d;
            if (last) {
              const float cs = mean_of(acc[j], Wf, invW, pow2) + __ldg(srv_err + bt.ck0 + i);
              tsum = fma(static_cast<double>(cs), static_cast<double>(cs), tsum);
            }
          }
          const uint32_t word = __ballot_sync(kFull, b);
          if (lane == 0 && sub + j * 32 < bt.nk)
            bits_w[static_cast<int64_t>(w) * L.words + bt.w0 + sub / 32 + j] = word;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }
    if (!ok) break;
    tsum = warp_sum(tsum);
    if (lane == 0) {
      part_srv[tb * kConsumers + q] = tsum;
      if (!isfinite(tsum)) atomicOr(status, kStatusNonfinite);
    }
  }
}

// ---- pass 3, pipelined: server signs + server error + update ------------------------
// Stage layout: srv_err | m | v | p  (f32 [kBT] each) | bits_w [W][64] words.
template <Upd U>
__global__ void __launch_bounds__(kPipeThreads, kPipeCtasPerSm)
k_server_update_pipe(Layout L, int W, const uint32_t* __restrict__ bits_w, const float* __restrict__ s_w,
                     const float* __restrict__ s_srv, float* __restrict__ srv_err,
                     uint32_t* __restrict__ bits_srv, float* __restrict__ m, const float* __restrict__ v,
                     float* __restrict__ p, Hyper h, double* __restrict__ partP,
                     double* __restrict__ partU, int S, uint32_t* __restrict__ status) {
  extern __shared__ __align__(128) unsigned char smem[];
  const size_t stage_bytes = static_cast<size_t>(kBT) * 16 + static_cast<size_t>(W) * kBTWords * 4;
  __shared__ uint64_t full_bar[16], empty_bar[16];
  __shared__ int abort_flag;
  const Ring ring{full_bar, empty_bar, &abort_flag};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1 + kWarp);    // expect_tx arrival + one cp.async arrival per producer lane
      mbar_init(&empty_bar[s], kConsumers);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t ntiles = L.Tb;
  const float Wf = static_cast<float>(W);
  const bool pow2 = (W & (W - 1)) == 0;
  const float invW = 1.0f / Wf;

  if (warp == 0) {
    // ---------------- producer ----------------
    long long it = 0;
    int hint = 0;
    for (int64_t tb = blockIdx.x; tb < ntiles; tb += gridDim.x, ++it) {
      if (__any_sync(kFull, aborted(&abort_flag))) break;
      const BTile bt = btile_at(L, tb, hint);
      const int s = static_cast<int>(it % S);
      if (!__all_sync(kFull, it < S || mbar_wait(&empty_bar[s], static_cast<uint32_t>(((it / S) - 1) & 1)))) {
        if (lane == 0) raise_timeout(status, &abort_flag);
        break;
      }
      unsigned char* st = smem + static_cast<size_t>(s) * stage_bytes;
      if (bt.vec) {
        if (lane == 0) {
          const int64_t e0 = bt.ck0 + bt.rel;
          const uint32_t fbytes = static_cast<uint32_t>(bt.len * 4);
          mbar_arrive_expect_tx(&full_bar[s], 4 * fbytes);
          bulk_g2s(st, srv_err + e0, fbytes, &full_bar[s]);
          bulk_g2s(st + kBT * 4, m + e0, fbytes, &full_bar[s]);
          bulk_g2s(st + kBT * 8, v + e0, fbytes, &full_bar[s]);
          bulk_g2s(st + kBT * 12, p + e0, fbytes, &full_bar[s]);
        }
        // packed worker signs of the tile: W x ceil(len/32) words, 4-byte async copies
        const int nwords = static_cast<int>((bt.len + 31) / 32);
        uint32_t* sb = reinterpret_cast<uint32_t*>(st + kBT * 16);
        for (int x = lane; x < W * nwords; x += kWarp) {
          const int w = x / nwords, j = x - w * nwords;
          cp_async4(sb + w * kBTWords + j, bits_w + static_cast<int64_t>(w) * L.words + bt.w0 + bt.rel / 32 + j);
        }
        cp_async_arrive(&full_bar[s]);
      } else {
        if (lane == 0) mbar_arrive(&full_bar[s]);
        cp_async_arrive(&full_bar[s]);      // no copies: arrives at once
      }
      __syncwarp();
    }
    if (lane == 0) drain_ring(ring, S, it);
    return;
  }

  // ---------------- consumers ----------------
  const int q = warp - 1;
  long long it = 0;
  int hint = 0;
  for (int64_t tb = blockIdx.x; tb < ntiles; tb += gridDim.x, ++it) {
    const BTile bt = btile_at(L, tb, hint);
    const int s = static_cast<int>(it % S);
    if (!__all_sync(kFull, mbar_wait(&full_bar[s], static_cast<uint32_t>((it / S) & 1)))) {
      if (lane == 0) raise_timeout(status, &abort_flag);
      break;
    }
    if (__any_sync(kFull, aborted(&abort_flag))) break;
    const unsigned char* st = smem + static_cast<size_t>(s) * stage_bytes;
    const float s2 = __ldg(s_srv + bt.k);
    const int64_t sub = bt.rel + q * kGroupElems;
    double Psum = 0.0, Usum = 0.0;
    bool bad = false;
    if (bt.vec) {
      const int64_t i0 = sub + lane * kVec;
      const bool in = i0 < bt.nk;
      const int wq = q * 8 + (lane >> 2);                    // word of this lane within the tile
      const bool word_in = (sub / 32 + (lane >> 2)) * 32 < bt.nk;
      float acc[8];
      zero8(acc);
      const uint32_t* sb = reinterpret_cast<const uint32_t*>(st + kBT * 16);
      for (int w = 0; w < W; ++w) {
        const float sw = __ldg(s_w + static_cast<int64_t>(w) * L.C + bt.k);
        const uint32_t byte = word_in ? lane_byte(sb[w * kBTWords + wq], lane) : 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = acc[j] + signed_scale((byte >> j) & 1u, sw);
      }
      uint32_t byte = 0;
      if (in) {
        const int64_t gi = bt.ck0 + i0;
        const int so = q * kGroupElems + lane * kVec;
        float sv[8], mv[8], vv[8], pv[8];
        ld8_smem(reinterpret_cast<const float*>(st) + so, sv);
        ld8_smem(reinterpret_cast<const float*>(st + kBT * 4) + so, mv);
        ld8_smem(reinterpret_cast<const float*>(st + kBT * 8) + so, vv);
        ld8_smem(reinterpret_cast<const float*>(st + kBT * 12) + so, pv);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float cs = mean_of(acc[j], Wf, invW, pow2) + sv[j];
          const bool b = cs >= 0.0f;
          const float d = signed_scale(b, s2);
          byte |= static_cast<uint32_t>(b) << j;
          sv[j] = cs - d;
          update_elem<U>(d, mv[j], vv[j], pv[j], h, Psum, Usum, bad);
        }
        st8(srv_err + gi, sv);
        st8(m + gi, mv);
        if (U == Upd::kAdam) st8(p + gi, pv);
      }
      const uint32_t word = quad_word(byte, lane);
      if ((lane & 3) == 0 && word_in) bits_srv[bt.w0 + sub / 32 + (lane >> 2)] = word;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t i = sub + j * 32 + lane;
        const bool inb = i < bt.nk;
        const int64_t gi = bt.ck0 + i;
        const int64_t wi = bt.w0 + sub / 32 + j;
        bool b = false;
        if (inb) {
          float acc = 0.0f;
          for (int w = 0; w < W; ++w) {
            const float sw = __ldg(s_w + static_cast<int64_t>(w) * L.C + bt.k);
            acc = acc + signed_scale((__ldg(bits_w + static_cast<int64_t>(w) * L.words + wi) >> lane) & 1u, sw);
          }
          const float cs = mean_of(acc, Wf, invW, pow2) + srv_err[gi];
          b = cs >= 0.0f;
          const float d = signed_scale(b, s2);
          srv_err[gi] = cs - d;
          float mv = m[gi], pv = p[gi];
          update_elem<U>(d, mv, __ldg(v + gi), pv, h, Psum, Usum, bad);
          m[gi] = mv;
          if (U == Upd::kAdam) p[gi] = pv;
        }
        const uint32_t word = __ballot_sync(kFull, b);
        if (lane == 0 && sub + j * 32 < bt.nk) bits_srv[wi] = word;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
    if (U == Upd::kLambM) {
      Psum = warp_sum(Psum);
      Usum = warp_sum(Usum);
      if (lane == 0) {
        partP[tb * kConsumers + q] = Psum;
        partU[tb * kConsumers + q] = Usum;
      }
    }
    flag_nonfinite(bad, status);
  }
}

}  // namespace ob
