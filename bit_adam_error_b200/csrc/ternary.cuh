// ternary.cuh -- sm_100a kernels of the momentum-error rule.
//
// Method (CANN 1-bit Adam article, section 2.1 "量化与误差补偿机制", section 2.2
// "动量修正策略", section 3.2 for clipping, the NaN check and int8 codes), per
// worker w and element:
//   c = clip(g_w) + err_w,   q = sign(c) in {-1, 0, +1},
//   err_w = beta1 err_w + (1 - beta1)(c - q)
// and across the W workers:  g_hat = (sum_w q_w) / W,  then the frozen-v Adam
// (or LAMB) update of kernels.cuh.
//
// Nothing here is gated by a norm, so the fused step is ONE streaming pass:
// every element reads g_w and err_w of each worker and m, v, p once, and writes
// err_w, m and p once -- W (gb + 2 eb) + 20 bytes per element (gb, eb = gradient
// and error bytes).  The codes stay in registers; only the stage calls (one
// worker stage, the code sum, the update from the sums) put them in memory,
// as int8 bytes, four per uint32 word, every chunk starting on a fresh word.
//
// Tiling is the one of kernels.cuh: 512-element warp tiles inside a chunk, the
// 8-wide vector path where the chunk allows it, lane-per-element otherwise.
// Floating point follows the plain C statement of the rule (-fmad=false).
#pragma once

#include "kernels.cuh"

namespace ob {

// sign() with sign(+0) = sign(-0) = 0; a NaN compares false both ways: 0.
__device__ __forceinline__ int ternary_sign(float c) {
  return static_cast<int>(c > 0.0f) - static_cast<int>(c < 0.0f);
}

// One worker element: returns q and leaves the new error in e.  A non-finite
// new error raises `bad` (the check after the error update).
template <bool CLIP>
__device__ __forceinline__ int momentum_error_elem(float g, float& e, const Hyper& h, bool& bad) {
  const float c = (CLIP ? clip_grad(g, h.clip) : g) + e;
  const int q = ternary_sign(c);
  const float delta = c - static_cast<float>(q);
  e = h.b1 * e + h.omb1 * delta;
  bad |= !isfinite(e);
  return q;
}

// Eight int8 codes <-> two words (code j in byte j % 4 of word j / 4).
__device__ __forceinline__ uint2 pack_codes8(const int (&q)[8]) {
  uint2 r;
  r.x = (static_cast<uint32_t>(q[0]) & 0xffu) | ((static_cast<uint32_t>(q[1]) & 0xffu) << 8) |
        ((static_cast<uint32_t>(q[2]) & 0xffu) << 16) | (static_cast<uint32_t>(q[3]) << 24);
  r.y = (static_cast<uint32_t>(q[4]) & 0xffu) | ((static_cast<uint32_t>(q[5]) & 0xffu) << 8) |
        ((static_cast<uint32_t>(q[6]) & 0xffu) << 16) | (static_cast<uint32_t>(q[7]) << 24);
  return r;
}

__device__ __forceinline__ int code_of(uint32_t word, int b) {
  return static_cast<int>(static_cast<int8_t>(static_cast<uint8_t>(word >> (8 * b))));
}

// ---- fused step: worker stage, code sum and update in one pass --------------------
template <typename GT, typename ET, bool CLIP, bool POW2, Upd U>
__global__ void __launch_bounds__(kBlock)
k_ternary_step(Layout L, int W, const GT* __restrict__ grads, ET* __restrict__ err,
               float* __restrict__ m, const float* __restrict__ v, float* __restrict__ p, Hyper h,
               double* __restrict__ partP, double* __restrict__ partU, uint32_t* __restrict__ status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean<POW2>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    double Psum = 0.0, Usum = 0.0;
    bool bad = false;
    if (tl.vec) {
#pragma unroll
      for (int gq = 0; gq < kGroups; ++gq) {
        const int64_t i0 = tl.rel + gq * kGroupElems + lane * kVec;
        if (i0 < tl.nk) {
          const int64_t gi = tl.ck0 + i0;
          float mv[8], vv[8], pv[8];
          ld8(m + gi, mv);
          ld8_ro(v + gi, vv);
          ld8(p + gi, pv);
          int sum[8] = {0, 0, 0, 0, 0, 0, 0, 0};
          for (int w = 0; w < W; ++w) {
            const int64_t ri = static_cast<int64_t>(w) * L.n + gi;
            float gv[8], ev[8];
            ld8_ro(grads + ri, gv);
            ld8(err + ri, ev);
#pragma unroll
            for (int j = 0; j < 8; ++j) sum[j] += momentum_error_elem<CLIP>(gv[j], ev[j], h, bad);
            st8(err + ri, ev);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            update_elem<U>(mean(static_cast<float>(sum[j])), mv[j], vv[j], pv[j], h, Psum, Usum, bad);
          st8(m + gi, mv);
          if (U == Upd::kAdam) st8(p + gi, pv);
        }
      }
    } else {
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          const int64_t gi = tl.ck0 + i;
          int sum = 0;
          for (int w = 0; w < W; ++w) {
            const int64_t ri = static_cast<int64_t>(w) * L.n + gi;
            float e = ld1(err + ri);
            sum += momentum_error_elem<CLIP>(ld1_ro(grads + ri), e, h, bad);
            st1(err + ri, e);
          }
          float mm = m[gi], pp = p[gi];
          update_elem<U>(mean(static_cast<float>(sum)), mm, __ldg(v + gi), pp, h, Psum, Usum, bad);
          m[gi] = mm;
          if (U == Upd::kAdam) p[gi] = pp;
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

// ---- stage: worker codes and errors -----------------------------------------------
// codes: [W][L.words] words; chunk k's codes are bytes [4 wo[k], 4 wo[k] + n_k) of
// a row.  The scalar path also zeroes the padding bytes of a chunk's last word.
template <typename GT, typename ET, bool CLIP>
__global__ void __launch_bounds__(kBlock)
k_ternary_compress(Layout L, int W, const GT* __restrict__ grads, ET* __restrict__ err,
                   uint32_t* __restrict__ codes, Hyper h, uint32_t* __restrict__ status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  if (L.T == 0) return;
  int hint = 0;
  for (RowTile x = first_item(L.T); x.r < W; next_item(x, L.T, W)) {
    const int w = x.r;
    const int64_t t = x.t;
    const Tile tl = tile_at(L, t, hint);
    const GT* g = grads + static_cast<int64_t>(w) * L.n + tl.ck0;
    ET* e = err + static_cast<int64_t>(w) * L.n + tl.ck0;
    uint32_t* row = codes + static_cast<int64_t>(w) * L.words + tl.w0;
    bool bad = false;
    if (tl.vec) {
#pragma unroll
      for (int gq = 0; gq < kGroups; ++gq) {
        const int64_t i0 = tl.rel + gq * kGroupElems + lane * kVec;
        if (i0 < tl.nk) {
          float gv[8], ev[8];
          int q[8];
          ld8_ro(g + i0, gv);
          ld8(e + i0, ev);
#pragma unroll
          for (int j = 0; j < 8; ++j) q[j] = momentum_error_elem<CLIP>(gv[j], ev[j], h, bad);
          st8(e + i0, ev);
          const uint2 wd = pack_codes8(q);
          row[i0 / 4] = wd.x;          // i0 % 8 == 0: two whole words of this chunk
          row[i0 / 4 + 1] = wd.y;
        }
      }
    } else {
      int8_t* bytes = reinterpret_cast<int8_t*>(row);
      const int64_t padded = (tl.nk + 3) & ~int64_t(3);
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          float ev = ld1(e + i);
          const int q = momentum_error_elem<CLIP>(ld1_ro(g + i), ev, h, bad);
          st1(e + i, ev);
          bytes[i] = static_cast<int8_t>(q);
        } else if (i < padded) {
          bytes[i] = 0;
        }
      }
    }
    flag_nonfinite(bad, status);
  }
}

// ---- stage: per-element sum of the W workers' codes --------------------------------
// Byte-wise addition without carries between bytes (__vadd4): each byte is the
// sum mod 256, which is the exact int8 sum since |sum| <= W <= 127.  Padding
// bytes are 0 + ... + 0.
__global__ void __launch_bounds__(kBlock)
k_ternary_server(int W, int64_t words, const uint32_t* __restrict__ codes_w,
                 uint32_t* __restrict__ codes_srv) {
  pdl_enter();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride) {
    uint32_t acc = 0u;
    for (int w = 0; w < W; ++w) acc = __vadd4(acc, __ldg(codes_w + static_cast<int64_t>(w) * words + i));
    codes_srv[i] = acc;
  }
}

// ---- stage: update from the code sums -----------------------------------------------
template <Upd U, bool POW2>
__global__ void __launch_bounds__(kBlock)
k_ternary_update(Layout L, int W, const uint32_t* __restrict__ codes_srv, float* __restrict__ m,
                 const float* __restrict__ v, float* __restrict__ p, Hyper h,
                 double* __restrict__ partP, double* __restrict__ partU, uint32_t* __restrict__ status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const auto mean = make_mean<POW2>(W);
  int hint = 0;
  for (int64_t t = warp_id(); t < L.T; t += warp_count()) {
    const Tile tl = tile_at(L, t, hint);
    const uint32_t* row = codes_srv + tl.w0;
    double Psum = 0.0, Usum = 0.0;
    bool bad = false;
    if (tl.vec) {
#pragma unroll
      for (int gq = 0; gq < kGroups; ++gq) {
        const int64_t i0 = tl.rel + gq * kGroupElems + lane * kVec;
        if (i0 < tl.nk) {
          const int64_t gi = tl.ck0 + i0;
          float mv[8], vv[8], pv[8];
          ld8(m + gi, mv);
          ld8_ro(v + gi, vv);
          ld8(p + gi, pv);
          const uint32_t w0 = __ldg(row + i0 / 4), w1 = __ldg(row + i0 / 4 + 1);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int s = code_of(j < 4 ? w0 : w1, j & 3);
            update_elem<U>(mean(static_cast<float>(s)), mv[j], vv[j], pv[j], h, Psum, Usum, bad);
          }
          st8(m + gi, mv);
          if (U == Upd::kAdam) st8(p + gi, pv);
        }
      }
    } else {
      const int8_t* bytes = reinterpret_cast<const int8_t*>(row);
      for (int j = 0; j < kTileWords; ++j) {
        const int64_t i = tl.rel + j * 32 + lane;
        if (i < tl.nk) {
          const int64_t gi = tl.ck0 + i;
          float mm = m[gi], pp = p[gi];
          update_elem<U>(mean(static_cast<float>(bytes[i])), mm, __ldg(v + gi), pp, h, Psum, Usum, bad);
          m[gi] = mm;
          if (U == Upd::kAdam) p[gi] = pp;
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
