// Token-by-token update of one 16-token chunk on a 64x64 state held as m16n8 accumulator fragments
// by four warps (warp w: rows 16w..16w+15; acc[nt][e] = S[16w + g + 8(e>>1)][8nt + 2c + (e&1)],
// g = lane/4, c = lane%4), inputs read from global memory: the recurrence itself, used by the
// chunked forward kernels for chunks whose decay product leaves the range of the 1/L scaling and,
// in the split form, for a ragged last chunk.  Writes y of the chunk's len tokens -- to global memory,
// or, with `ys` given (a [16][ys_stride] tile of 16-bit y), into that tile for the caller to write out.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace wkv7 {

template <typename T>
__device__ __forceinline__ void state_chunk_tokens(const FwdArgs& p, unsigned mask, float (&acc)[8][4], int64_t b,
                                                   int64_t h, int64_t t0, int len, int warp, int lane,
                                                   uint16_t* ys = nullptr, int ys_stride = 0) {
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;
  const T* R = static_cast<const T*>(p.r);
  const T* Wd = static_cast<const T*>(p.w);
  const T* K = static_cast<const T*>(p.k);
  const T* V = static_cast<const T*>(p.v);
  const T* A = static_cast<const T*>(p.a);
  const T* Bb = static_cast<const T*>(p.b);
  T* y = static_cast<T*>(p.y);
  for (int tt = 0; tt < len; ++tt) {
    const int64_t o = tok_off(b, t0 + tt, h, p.T, p.H);
    if (!range_ok(o, kN, p.B * p.T * p.H * kN, p.status)) continue;   // (debug build)
    if ((mask >> tt) & 1u) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    }
    float s_lo = 0.f, s_hi = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float av = Elt<T>::to_f32(A[o + 8 * nt + 2 * c4 + (e & 1)]);
        if (e < 2) s_lo = fmaf(acc[nt][e], av, s_lo); else s_hi = fmaf(acc[nt][e], av, s_hi);
      }
    s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
    s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
    s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
    s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
    const float v_lo = Elt<T>::to_f32(V[o + row0 + g]);
    const float v_hi = Elt<T>::to_f32(V[o + row0 + g + 8]);
    float y_lo = 0.f, y_hi = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 8 * nt + 2 * c4 + (e & 1);
        const float wv = decay_of(Elt<T>::to_f32(Wd[o + col]), p.log_decay), bv = Elt<T>::to_f32(Bb[o + col]);
        const float kv = Elt<T>::to_f32(K[o + col]), rv = Elt<T>::to_f32(R[o + col]);
        const bool lo = e < 2;
        acc[nt][e] = fmaf(acc[nt][e], wv, fmaf(lo ? s_lo : s_hi, bv, (lo ? v_lo : v_hi) * kv));
        if (lo) y_lo = fmaf(acc[nt][e], rv, y_lo); else y_hi = fmaf(acc[nt][e], rv, y_hi);
      }
    y_lo += __shfl_xor_sync(0xffffffffu, y_lo, 1);
    y_lo += __shfl_xor_sync(0xffffffffu, y_lo, 2);
    y_hi += __shfl_xor_sync(0xffffffffu, y_hi, 1);
    y_hi += __shfl_xor_sync(0xffffffffu, y_hi, 2);
    if (c4 == 0) {
      if (ys) {   // 16-bit T: the tile holds its bits
        const T lo = Elt<T>::from_f32(y_lo), hi = Elt<T>::from_f32(y_hi);
        ys[tt * ys_stride + row0 + g] = *reinterpret_cast<const uint16_t*>(&lo);
        ys[tt * ys_stride + row0 + g + 8] = *reinterpret_cast<const uint16_t*>(&hi);
      } else {
        y[o + row0 + g] = Elt<T>::from_f32(y_lo);
        y[o + row0 + g + 8] = Elt<T>::from_f32(y_hi);
      }
    }
  }
}

}  // namespace wkv7
