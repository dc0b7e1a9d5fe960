// twobit.cuh -- sm_100a kernels of 2-bit Adam (two residual sign planes).
//
// 2-bit Adam is named by the CANN 1-bit Adam article (section 5.1 table: 6.25% of
// the traffic; section 8: weaker compression for embedding layers) without a
// quantiser.  Here it is the 1-bit quantiser of kernels.cuh applied twice:
//   s1 = ||c|| / sqrt(n_k),  q1 = (c >= 0),   r   = c - s1 sign(q1)
//   s2 = ||r|| / sqrt(n_k),  q2 = (r >= 0),   err = r - s2 sign(q2)
//   dequantised value = s1 sign(q1) + s2 sign(q2)
// for the workers and, on their average plus the server error, for the server.
//
// s2 needs s1, which is known only once the whole chunk has been read.  Since
// r_i^2 = (|c_i| - s1)^2, the sum over the chunk is, for any split of the chunk
// into tiles t of n_t elements with mean mu_t of |c|,
//   ||r||^2 = sum_t [ sum_{i in t} (|c_i| - mu_t)^2 + n_t (mu_t - s1)^2 ],
// an identity of real arithmetic whose terms are all >= 0 (no cancellation,
// even when every |c_i| is close to s1).  So the pass that reads c for ||c||
// also keeps, per warp tile, S = sum |c| and M2 = sum (|c| - S / n_t)^2, and
// the finaliser forms ||r||^2 from them once s1 is in hand: the fused step is
// three streaming passes, as for 1 bit.  ||r||^2 differs from the sum of the
// squared float residuals by their rounding only (at most 2^-23 relative).
//   1  k_tb_worker_norm     g, err            -> sum c^2, moments of |c|      -> s1, s2
//   2  k_tb_pack<SERVER>    g, err, srv_err   -> err, planes, the same of c_srv -> s1', s2'
//   3  k_tb_server_update   planes, srv_err, m, v, p -> server planes, srv_err, m, p
// Layout: chunk k owns 2 ceil(n_k / 32) words of a row, plane 1 then plane 2,
// from word wo[k]; scales are [row][C][2].  Tiling, vector/scalar paths and the
// floating-point order of the per-element values are those of kernels.cuh
// (every value equals the plain C statement of the rule for the same scales).
#pragma once

#include "kernels.cuh"

namespace ob {

__device__ __forceinline__ int64_t plane_words(int64_t nk) { return (nk + 31) / 32; }

// ---- tile sums of |c| for the second scale -------------------------------------------
// One sweep, shifted by K = |c| of the tile's first element (lane 0 holds it on
// both paths): every lane adds d = |c| - K and d^2 of its elements, and after the
// warp sums
//   S_t = n_t K + sum d,   M2_t = sum d^2 - (sum d)^2 / n_t   (>= 0, clamped).
// K is one of the values, so n_t (mean - K)^2 <= n_t M2_t and the subtraction
// loses at most about 2 n_t ulps of M2_t; equal magnitudes give M2_t = 0 exactly.
struct Shifted {
  double K, d1, d2;
};

__device__ __forceinline__ Shifted shifted_from(float first_lane0) {
  return Shifted{fabs(static_cast<double>(__shfl_sync(kFull, first_lane0, 0))), 0.0, 0.0};
}

__device__ __forceinline__ void shifted_add(Shifted& m, double c) {
  const double d = fabs(c) - m.K;
  m.d1 += d;
  m.d2 = fma(d, d, m.d2);
}

// Warp sums; lane 0 stores S_t at part[P + t] and M2_t at part[2P + t].
__device__ __forceinline__ void store_shifted(Shifted m, const Tile& tl, double* __restrict__ part, int64_t P,
                                              int64_t t, int lane) {
  const double d1 = warp_sum(m.d1), d2 = warp_sum(m.d2);
  if (lane == 0) {
    const int64_t left = tl.nk - tl.rel;
    const int nt = left < kTile ? static_cast<int>(left) : kTile;
    const double sq = nt == kTile ? d1 * d1 * (1.0 / kTile) : d1 * d1 / nt;
    part[P + t] = static_cast<double>(nt) * m.K + d1;
    part[2 * P + t] = fmax(d2 - sq, 0.0);
  }
}

// The four dequantised values (+-s1) + (+-s2) of one worker's chunk, d<b1><b2>,
// formed once per tile: the same float additions the per-element form makes.
struct Dq4 {
  float d00, d10, d01, d11;
};

__device__ __forceinline__ Dq4 dq4_of(const float* __restrict__ s_w, int k) {
  const float s1 = __ldg(s_w + static_cast<int64_t>(k) * 2), s2 = __ldg(s_w + static_cast<int64_t>(k) * 2 + 1);
  return Dq4{-s1 + -s2, s1 + -s2, -s1 + s2, s1 + s2};
}

// acc[j] += s1 sign1 + s2 sign2 of worker w, ascending w (the order of pass 2).
// W1: exactly one worker; each element selects one of the tile's four values dq.
template <bool W1>
__device__ __forceinline__ void tb_server_sum8(const Layout& L, int W, const uint32_t* __restrict__ bits_w,
                                               const float* __restrict__ s_w, const Tile& tl, int64_t wrel,
                                               int64_t nwk, bool word_in, int lane, float (&acc)[8],
                                               const Dq4& dq) {
  if constexpr (W1) {
    const uint32_t* row = bits_w + tl.w0;
    const uint32_t w1 = word_in ? __ldg(row + wrel) : 0u;
    const uint32_t w2 = word_in ? __ldg(row + nwk + wrel) : 0u;
    const uint32_t b1 = lane_byte(w1, lane), b2 = lane_byte(w2, lane);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool x1 = (b1 >> j) & 1u, x2 = (b2 >> j) & 1u;
      acc[j] = 0.0f + (x2 ? (x1 ? dq.d11 : dq.d01) : (x1 ? dq.d10 : dq.d00));
    }
    return;
  }
  zero8(acc);
  for (int w = 0; w < W; ++w) {
    const float* sc = s_w + (static_cast<int64_t>(w) * L.C + tl.k) * 2;
    const float s1 = __ldg(sc), s2 = __ldg(sc + 1);
    const uint32_t* row = bits_w + static_cast<int64_t>(w) * L.words + tl.w0;
    const uint32_t w1 = word_in ? __ldg(row + wrel) : 0u;
    const uint32_t w2 = word_in ? __ldg(row + nwk + wrel) : 0u;
    const uint32_t b1 = lane_byte(w1, lane), b2 = lane_byte(w2, lane);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      acc[j] = acc[j] + (signed_scale((b1 >> j) & 1u, s1) + signed_scale((b2 >> j) & 1u, s2));
  }
}

template <bool W1>
__device__ __forceinline__ float tb_server_sum1(const Layout& L, int W, const uint32_t* __restrict__ bits_w,
                                                const float* __restrict__ s_w, const Tile& tl, int64_t wi,
                                                int64_t nwk, int lane) {
  float acc = 0.0f;
  for (int w = 0; w < (W1 ? 1 : W); ++w) {
    const float* sc = s_w + (static_cast<int64_t>(w) * L.C + tl.k) * 2;
    const uint32_t* row = bits_w + static_cast<int64_t>(w) * L.words + tl.w0;
    const bool b1 = (__ldg(row + wi) >> lane) & 1u, b2 = (__ldg(row + nwk + wi) >> lane) & 1u;
    acc = acc + (signed_scale(b1, __ldg(sc)) + signed_scale(b2, __ldg(sc + 1)));
  }
  return acc;
}

// ---- pass 1: per tile, sum c^2 and the sums of |c| of every worker ---------------------
// Item it = w * T + t (P = W * T items): part[it] = sum c^2 (the order of the 1-bit
// pass 1), part[P + it] = S_t, part[2P + it] = M2_t (see Shifted).  A non-finite
// sum c^2 raises the status flag.
template <typename GT, typename ET, bool CLIP>
__device__ __forceinline__ void tb_worker_norm_tiles(Layout L, int W, const GT* __restrict__ grads,
                                                     const ET* __restrict__ err, float clip,
                                                     double* __restrict__ part, uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  if (L.T == 0) return;
  const int64_t items = static_cast<int64_t>(W) * L.T;
  int hint = 0;
  for (RowTile x = first_item(L.T); x.r < W; next_item(x, L.T, W)) {
    const int w = x.r;
    const int64_t t = x.t, it = static_cast<int64_t>(w) * L.T + t;
    const Tile tl = tile_at(L, t, hint);
    const GT* g = grads + static_cast<int64_t>(w) * L.n + tl.ck0;
    const ET* e = err + static_cast<int64_t>(w) * L.n + tl.ck0;
    double acc = 0.0;
    Shifted m;
    if (tl.vec) {
      float gv[kGroups][8], ev[kGroups][8];
      bool in[kGroups];
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        const int64_t i0 = tl.rel + q * kGroupElems + lane * kVec;
        in[q] = i0 < tl.nk;
        if (in[q]) { ld8_ro(g + i0, gv[q]); ld8_ro(e + i0, ev[q]); }
        else { zero8(gv[q]); zero8(ev[q]); }
      }
      m = shifted_from((CLIP ? clip_grad(gv[0][0], clip) : gv[0][0]) + ev[0][0]);
#pragma unroll
      for (int q = 0; q < kGroups; ++q)
        if (in[q]) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const double c = static_cast<double>((CLIP ? clip_grad(gv[q][j], clip) : gv[q][j]) + ev[q][j]);
            acc = fma(c, c, acc);
            shifted_add(m, c);
          }
        }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        float c = 0.0f;
        if (i < tl.nk) c = (CLIP ? clip_grad(ld1_ro(g + i), clip) : ld1_ro(g + i)) + ld1_ro(e + i);
        if (j == 0) m = shifted_from(c);
        if (i < tl.nk) {
          const double cd = static_cast<double>(c);
          acc = fma(cd, cd, acc);
          shifted_add(m, cd);
        }
      }
    }
    store_shifted(m, tl, part, items, it, lane);
    acc = warp_sum(acc);
    if (lane == 0) {
      part[it] = acc;
      flag_tile_sum(acc, status);
    }
  }
}

template <typename GT, typename ET, bool CLIP>
__global__ void __launch_bounds__(kBlock)
k_tb_worker_norm(Layout L, int W, const GT* __restrict__ grads, const ET* __restrict__ err,
                 float clip, double* __restrict__ part, uint32_t* __restrict__ status) {
  pdl_enter();
  tb_worker_norm_tiles<GT, ET, CLIP>(L, W, grads, err, clip, part, status);
}

// ---- pass 2: both planes, worker error (+ server sums) ---------------------------------
// SERVER: also c_srv = (sum_w dequantised_w) / W + srv_err, with part_srv[t] =
// sum c_srv^2, part_srv[T + t] = S_t and part_srv[2T + t] = M2_t of |c_srv| (see
// Shifted).  CACHE (with SERVER): c_srv also goes to csrv[n] for pass 3.
// Three CTAs per SM (at most 80 registers): the cached, clipped variant would
// otherwise take 92 and drop to two.
template <typename GT, typename ET, bool SERVER, bool CLIP, bool POW2, bool CACHE>
__device__ __forceinline__ void tb_pack_tiles(Layout L, int W, const GT* __restrict__ grads, ET* __restrict__ err,
          const float* __restrict__ s_w, uint32_t* __restrict__ bits_w, const ET* __restrict__ srv_err,
          double* __restrict__ part_srv, float* __restrict__ csrv, float clip, uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean<POW2>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    const int64_t nwk = plane_words(tl.nk);
    double tsum = 0.0;
    Shifted mo{0.0, 0.0, 0.0};
    if (tl.vec) {
#pragma unroll 1
      for (int gq = 0; gq < kGroups; ++gq) {
        const int64_t i0 = tl.rel + gq * kGroupElems + lane * kVec;
        const bool in = i0 < tl.nk;
        const int64_t wrel = (tl.rel + gq * kGroupElems) / 32 + (lane >> 2);
        float acc[8], sv[8];
        zero8(acc);
        if (SERVER) {
          if (in) ld8_ro(srv_err + tl.ck0 + i0, sv); else zero8(sv);
        }
        for (int w = 0; w < W; ++w) {
          const GT* g = grads + static_cast<int64_t>(w) * L.n + tl.ck0;
          ET* e = err + static_cast<int64_t>(w) * L.n + tl.ck0;
          const float* sc = s_w + (static_cast<int64_t>(w) * L.C + tl.k) * 2;
          const float s1 = __ldg(sc), s2 = __ldg(sc + 1);
          float gv[8], ev[8];
          if (in) { ld8_ro(g + i0, gv); ld8(e + i0, ev); }
          else { zero8(gv); zero8(ev); }
          uint32_t byte1 = 0, byte2 = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float c = (CLIP ? clip_grad(gv[j], clip) : gv[j]) + ev[j];
            const bool b1 = c >= 0.0f;
            const float d1 = signed_scale(b1, s1);
            const float r = c - d1;
            const bool b2 = r >= 0.0f;
            const float d2 = signed_scale(b2, s2);
            byte1 |= static_cast<uint32_t>(b1) << j;
            byte2 |= static_cast<uint32_t>(b2) << j;
            ev[j] = r - d2;
            acc[j] = acc[j] + (d1 + d2);
          }
          if (in) st8(e + i0, ev);
          else { byte1 = 0; byte2 = 0; }
          const uint32_t word1 = quad_word(byte1, lane), word2 = quad_word(byte2, lane);
          if ((lane & 3) == 0 && wrel * 32 < tl.nk) {
            uint32_t* row = bits_w + static_cast<int64_t>(w) * L.words + tl.w0;
            row[wrel] = word1;
            row[nwk + wrel] = word2;
          }
        }
        if constexpr (SERVER) {
          if (in) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {            // c_srv in place of the sum
              acc[j] = mean(acc[j]) + sv[j];
              tsum = fma(static_cast<double>(acc[j]), static_cast<double>(acc[j]), tsum);
            }
            if (CACHE) st8(csrv + tl.ck0 + i0, acc);
          }
          if (gq == 0) mo = shifted_from(acc[0]);
          if (in) {
#pragma unroll
            for (int j = 0; j < 8; ++j) shifted_add(mo, static_cast<double>(acc[j]));
          }
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        const bool inb = i < tl.nk;
        const int64_t wi = tl.rel / 32 + j;
        float acc = 0.0f;
        for (int w = 0; w < W; ++w) {
          const float* sc = s_w + (static_cast<int64_t>(w) * L.C + tl.k) * 2;
          ET* e = err + static_cast<int64_t>(w) * L.n + tl.ck0;
          bool b1 = false, b2 = false;
          if (inb) {
            const float g = ld1_ro(grads + static_cast<int64_t>(w) * L.n + tl.ck0 + i);
            const float c = (CLIP ? clip_grad(g, clip) : g) + ld1(e + i);
            b1 = c >= 0.0f;
            const float d1 = signed_scale(b1, __ldg(sc));
            const float r = c - d1;
            b2 = r >= 0.0f;
            const float d2 = signed_scale(b2, __ldg(sc + 1));
            st1(e + i, r - d2);
            acc = acc + (d1 + d2);
          }
          const uint32_t word1 = __ballot_sync(kFull, b1), word2 = __ballot_sync(kFull, b2);
          if (lane == 0 && (tl.rel + j * 32) < tl.nk) {
            uint32_t* row = bits_w + static_cast<int64_t>(w) * L.words + tl.w0;
            row[wi] = word1;
            row[nwk + wi] = word2;
          }
        }
        if constexpr (SERVER) {
          const float cs = inb ? mean(acc) + ld1_ro(srv_err + tl.ck0 + i) : 0.0f;
          if (j == 0) mo = shifted_from(cs);
          if (inb) {
            tsum = fma(static_cast<double>(cs), static_cast<double>(cs), tsum);
            if (CACHE) csrv[tl.ck0 + i] = cs;
            shifted_add(mo, static_cast<double>(cs));
          }
        }
      }
    }
    if constexpr (SERVER) {
      store_shifted(mo, tl, part_srv, L.T, t, lane);
      tsum = warp_sum(tsum);
      if (lane == 0) {
        part_srv[t] = tsum;
        flag_tile_sum(tsum, status);
      }
    }
  }
}

template <typename GT, typename ET, bool SERVER, bool CLIP, bool POW2, bool CACHE>
__global__ void __launch_bounds__(kBlock, 3)
k_tb_pack(Layout L, int W, const GT* __restrict__ grads, ET* __restrict__ err,
          const float* __restrict__ s_w, uint32_t* __restrict__ bits_w, const ET* __restrict__ srv_err,
          double* __restrict__ part_srv, float* __restrict__ csrv, float clip, uint32_t* __restrict__ status) {
  pdl_enter();
  tb_pack_tiles<GT, ET, SERVER, CLIP, POW2, CACHE>(L, W, grads, err, s_w, bits_w, srv_err, part_srv, csrv, clip,
                                                    status);
}

// ---- server sums from the worker planes (stage call) ----------------------------------
// part[t] = sum c_srv^2, part[T + t] = S_t, part[2T + t] = M2_t of |c_srv| (see
// Shifted; one row): the values and the order of the fused pass 2.  W1 (with
// POW2): one worker (see tb_server_sum8).
template <typename ET, bool POW2, bool W1>
__device__ __forceinline__ void tb_server_norm_tiles(Layout L, int W, const uint32_t* __restrict__ bits_w,
                                                     const float* __restrict__ s_w, const ET* __restrict__ srv_err,
                                                     double* __restrict__ part, uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean_w<POW2, W1>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    const int64_t nwk = plane_words(tl.nk);
    const Dq4 dq = W1 ? dq4_of(s_w, tl.k) : Dq4{};
    double tsum = 0.0;
    Shifted mo{0.0, 0.0, 0.0};
    if (tl.vec) {
#pragma unroll
      for (int gq = 0; gq < kGroups; ++gq) {
        const int64_t i0 = tl.rel + gq * kGroupElems + lane * kVec;
        const int64_t wrel = (tl.rel + gq * kGroupElems) / 32 + (lane >> 2);
        const bool in = i0 < tl.nk;
        float sv[8], acc[8];
        if (in) ld8_ro(srv_err + tl.ck0 + i0, sv); else zero8(sv);
        tb_server_sum8<W1>(L, W, bits_w, s_w, tl, wrel, nwk, wrel * 32 < tl.nk, lane, acc, dq);
        if (in) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[j] = mean(acc[j]) + sv[j];
            tsum = fma(static_cast<double>(acc[j]), static_cast<double>(acc[j]), tsum);
          }
        }
        if (gq == 0) mo = shifted_from(acc[0]);
        if (in) {
#pragma unroll
          for (int j = 0; j < 8; ++j) shifted_add(mo, static_cast<double>(acc[j]));
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        const bool inb = i < tl.nk;
        const float cs = inb ? mean(tb_server_sum1<W1>(L, W, bits_w, s_w, tl, tl.rel / 32 + j, nwk, lane)) +
                                   ld1_ro(srv_err + tl.ck0 + i)
                             : 0.0f;
        if (j == 0) mo = shifted_from(cs);
        if (inb) {
          tsum = fma(static_cast<double>(cs), static_cast<double>(cs), tsum);
          shifted_add(mo, static_cast<double>(cs));
        }
      }
    }
    store_shifted(mo, tl, part, L.T, t, lane);
    tsum = warp_sum(tsum);
    if (lane == 0) {
      part[t] = tsum;
      flag_tile_sum(tsum, status);
    }
  }
}

template <typename ET, bool POW2, bool W1>
__global__ void __launch_bounds__(kBlock)
k_tb_server_norm(Layout L, int W, const uint32_t* __restrict__ bits_w, const float* __restrict__ s_w,
                 const ET* __restrict__ srv_err, double* __restrict__ part, uint32_t* __restrict__ status) {
  pdl_enter();
  tb_server_norm_tiles<ET, POW2, W1>(L, W, bits_w, s_w, srv_err, part, status);
}

// ---- both scales of a chunk from the tile sums ----------------------------------------------
// Row r, chunk k (P = rows * T): A = sum_t part[r*T + t], s1 = sqrt(A) / sqrt(n_k);
// then, with S_t = part[P + r*T + t], M2_t = part[2P + r*T + t] and n_t the tile's
// element count,
//   R = sum_t [ M2_t + n_t (S_t / n_t - s1)^2 ],   s2 = sqrt(R) / sqrt(n_k);
// both 0 for an empty chunk.  Fixed-order sums (the order of k_finalize_scale);
// a full tile's mean is an exact multiply by 1/kTile.
// out[(r * C + k) * 2 + {0, 1}] = s1, s2.  grid = (C, rows).
__global__ void __launch_bounds__(kFinalizeThreads)
k_tb_finalize(Layout L, const double* __restrict__ part, int rows, float* __restrict__ out) {
  pdl_enter();
  __shared__ double sm[kFinalizeThreads];
  const int k = blockIdx.x, r = blockIdx.y;
  const int64_t P = static_cast<int64_t>(rows) * L.T;
  const double* pa = part + static_cast<int64_t>(r) * L.T;
  const double* ps = pa + P;
  const double* pm = pa + 2 * P;
  const int64_t t0 = L.tp[k], t1 = L.tp[k + 1], nk = L.off[k + 1] - L.off[k];
  double acc = 0.0;
  for (int64_t t = t0 + threadIdx.x; t < t1; t += kFinalizeThreads) acc += pa[t];
  const double A = block_sum_fixed(acc, sm);
  const double rn = __dsqrt_rn(static_cast<double>(nk));
  const float s1 = nk > 0 ? __double2float_rn(__ddiv_rn(__dsqrt_rn(A), rn)) : 0.0f;
  // Full tiles in the loop (no division, so loads pipeline); a ragged last tile
  // after it, by the thread whose stride reaches it.
  const int64_t tf = t0 + nk / kTile;
  const double s1d = static_cast<double>(s1);
  acc = 0.0;
  for (int64_t t = t0 + threadIdx.x; t < tf; t += kFinalizeThreads) {
    const double d = ps[t] * (1.0 / kTile) - s1d;
    acc += pm[t] + static_cast<double>(kTile) * d * d;
  }
  if (tf < t1 && (tf - t0) % kFinalizeThreads == threadIdx.x) {
    const double nt = static_cast<double>(nk - (tf - t0) * kTile);
    const double d = ps[tf] / nt - s1d;
    acc += pm[tf] + nt * d * d;
  }
  const double R = block_sum_fixed(acc, sm);
  if (threadIdx.x == 0) {
    float* o = out + (static_cast<int64_t>(r) * L.C + k) * 2;
    o[0] = s1;
    o[1] = nk > 0 ? __double2float_rn(__ddiv_rn(__dsqrt_rn(R), rn)) : 0.0f;
  }
}

// ---- pass 3: server planes + server error, and/or the update --------------------------
// FROM_WORKERS: c_srv from the worker planes and srv_err, quantised to two planes
// with s_srv (bits_srv and srv_err written).  Otherwise g_hat from bits_srv.
// CACHED (with FROM_WORKERS): c_srv read from csrv; srv_err only written.  W1
// (with FROM_WORKERS, POW2): one worker (see tb_server_sum8).
template <Upd U, bool FROM_WORKERS, bool POW2, typename ET, bool CACHED, bool W1>
__global__ void __launch_bounds__(kBlock, kUpdateMinBlocks)
k_tb_server_update(Layout L, int W, const uint32_t* __restrict__ bits_w, const float* __restrict__ s_w,
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
    const int64_t nwk = plane_words(tl.nk);
    const float s1 = __ldg(s_srv + 2 * tl.k), s2 = __ldg(s_srv + 2 * tl.k + 1);
    const Dq4 dq = (FROM_WORKERS && !CACHED && W1) ? dq4_of(s_w, tl.k) : Dq4{};
    uint32_t* srow = bits_srv + tl.w0;
    double Psum = 0.0, Usum = 0.0;
    bool bad = false;
    if (tl.vec) {
#pragma unroll 1
      for (int gq = 0; gq < kGroups; ++gq) {
        const int64_t i0 = tl.rel + gq * kGroupElems + lane * kVec;
        const int64_t wrel = (tl.rel + gq * kGroupElems) / 32 + (lane >> 2);
        const bool word_in = wrel * 32 < tl.nk;
        const bool in = i0 < tl.nk;
        const int64_t gi = tl.ck0 + i0;
        float sv[8], mv[8], vv[8], pv[8];
        if (in) {
          if (FROM_WORKERS && !CACHED) ld8(srv_err + gi, sv);
          if (FROM_WORKERS && CACHED) ld8_ro(csrv + gi, sv);      // sv holds c_srv itself
          if (U != Upd::kNone) { ld8(m + gi, mv); ld8_ro(v + gi, vv); ld8(p + gi, pv); }
        }
        if (FROM_WORKERS) {
          float acc[8];
          if (!CACHED) tb_server_sum8<W1>(L, W, bits_w, s_w, tl, wrel, nwk, word_in, lane, acc, dq);
          uint32_t byte1 = 0, byte2 = 0;
          if (in) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float cs = CACHED ? sv[j] : mean(acc[j]) + sv[j];
              const bool b1 = cs >= 0.0f;
              const float d1 = signed_scale(b1, s1);
              const float r = cs - d1;
              const bool b2 = r >= 0.0f;
              const float d2 = signed_scale(b2, s2);
              byte1 |= static_cast<uint32_t>(b1) << j;
              byte2 |= static_cast<uint32_t>(b2) << j;
              sv[j] = r - d2;
              update_elem<U>(d1 + d2, mv[j], vv[j], pv[j], h, Psum, Usum, bad);
            }
            st8(srv_err + gi, sv);
          }
          const uint32_t word1 = quad_word(byte1, lane), word2 = quad_word(byte2, lane);
          if ((lane & 3) == 0 && word_in) {
            srow[wrel] = word1;
            srow[nwk + wrel] = word2;
          }
        } else {
          const uint32_t w1 = word_in ? __ldg(srow + wrel) : 0u;
          const uint32_t w2 = word_in ? __ldg(srow + nwk + wrel) : 0u;
          const uint32_t byte1 = lane_byte(w1, lane), byte2 = lane_byte(w2, lane);
          if (in) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              update_elem<U>(signed_scale((byte1 >> j) & 1u, s1) + signed_scale((byte2 >> j) & 1u, s2),
                             mv[j], vv[j], pv[j], h, Psum, Usum, bad);
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
        const int64_t wi = tl.rel / 32 + j;
        float d = 0.0f;
        if (FROM_WORKERS) {
          bool b1 = false, b2 = false;
          if (inb) {
            const float cs = CACHED ? __ldg(csrv + gi)
                                    : mean(tb_server_sum1<W1>(L, W, bits_w, s_w, tl, wi, nwk, lane)) + ld1(srv_err + gi);
            b1 = cs >= 0.0f;
            const float d1 = signed_scale(b1, s1);
            const float r = cs - d1;
            b2 = r >= 0.0f;
            const float d2 = signed_scale(b2, s2);
            st1(srv_err + gi, r - d2);
            d = d1 + d2;
          }
          const uint32_t word1 = __ballot_sync(kFull, b1), word2 = __ballot_sync(kFull, b2);
          if (lane == 0 && (tl.rel + j * 32) < tl.nk) {
            srow[wi] = word1;
            srow[nwk + wi] = word2;
          }
        } else if (inb) {
          d = signed_scale((__ldg(srow + wi) >> lane) & 1u, s1) +
              signed_scale((__ldg(srow + nwk + wi) >> lane) & 1u, s2);
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

}  // namespace ob
