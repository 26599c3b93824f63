// WKV-7 forward in 16-token chunks with the intra-chunk products on tensor
// cores (algo CHUNKED) -- the "chunk-parallel path" of the HF model card page,
// derived here from the recurrence.
//
// Inside a chunk of tokens t = 0..15 with entering state S0, let
// L_t = prod_{s<=t} w_s (per key channel j) and write the state relative to
// that decay, Sh_t = S_t diag(1/L_t).  The recurrence becomes additive:
//   Sh_t = Sh_{t-1} + sa_t bh_t^T + v_t kh_t^T,   sa_t = Sh_{t-1} at_t,  y_t = Sh_t rt_t
// with at_t = a_t L_{t-1}, rt_t = r_t L_t, bh_t = b_t / L_t, kh_t = k_t / L_t.
// Unrolling it gives, for the 16 x 64 blocks SA (rows sa_t) and Y (rows y_t),
//   (I - Lab) SA = At S0^T + Lak V,    Y = Rt S0^T + Mrb SA + Mrk V,
// where Lab[t,tau] = at_t . bh_tau, Lak[t,tau] = at_t . kh_tau (tau < t) and
// Mrb, Mrk are the same with rt_t (tau <= t).  Solving the unit lower
// triangular system by substitution (the triangular solve the rwkv-lab page
// names for chunked delta rules):
//   SA = W S0^T + X V,  Y = Q S0^T + Z V,
//   W = (I - Lab)^-1 At,  X = (I - Lab)^-1 Lak,  Q = Rt + Mrb W,  Z = Mrb X + Mrk,
//   S_16 = S0 diag(L_15) + (SA^T Bh + V^T Kh) diag(L_15).
// Reset flags inside a chunk become masks: pairs (t, tau) separated by a
// reset are dropped from Lab..Mrk, S0 only reaches tokens before the first
// reset (rows of At, Rt masked), only the last segment feeds S_16, and S0
// drops out of S_16 if the chunk holds any reset.
//
// Precision: every product with an fp32 operand uses the 3-term bf16 split
// (hi*hi + hi*lo + lo*hi, about 2^-16 relative); v enters exactly when the
// inputs are bf16.  A chunk whose decay product leaves [2^-40, 2^40] (e.g.
// w = 0) cannot use the 1/L scaling and is run token by token instead.
//
// Work split (one CTA of 8 warps per (b,h)):
//   warps 0-3 ("state"): warp w owns rows 16w..16w+15 of S as mma
//     accumulator fragments for the whole sequence; per chunk they do the
//     two state products above, write y and the chunk-end checkpoint;
//   warps 4-7 ("context"): meanwhile build everything the NEXT chunk's
//     state products need (decay-scaled operands, Gram, W, X, Q, Z) into the
//     other half of a double buffer, and stage the chunk after that with
//     cp.async.
// One CTA barrier per chunk hands the context over.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;
constexpr int kStr = 72;    // padded row stride (elements) of 64-wide tiles: conflict-free ldmatrix
constexpr int kStrS = 24;   // padded row stride of 16-wide tiles
constexpr int kIn = 6;      // staged inputs: r, w, k, v, a, b
using bf16 = __nv_bfloat16;

// Everything the state warps need for one chunk.
struct __align__(16) Ctx {
  bf16 Wh[kChunk][kStr], Wl[kChunk][kStr];   // W [t][j]
  bf16 Qh[kChunk][kStr], Ql[kChunk][kStr];   // Q [t][j]
  bf16 Bh[32][kStr], Bl[32][kStr];           // rows 0..15 bh_tau, 16..31 kh_tau  [tau][j]
  bf16 Vh[kChunk][kStr], Vl[kChunk][kStr];   // v [tau][i]  (Vl unused for bf16 inputs)
  bf16 Xh[kChunk][kStrS], Xl[kChunk][kStrS]; // X [t][tau]
  bf16 Zh[kChunk][kStrS], Zl[kChunk][kStrS]; // Z [t][tau]
  float lam15[kN];
  int mask;     // reset bits of the chunk
  int unsafe;   // decay product out of range: run this chunk token by token
};

template <typename T>
struct __align__(16) FwdSmem2 {
  Ctx ctx[2];
  T in[2][kIn][kChunk][kStr];                 // staged inputs of two chunks
  bf16 GAh[32][kStr], GAl[32][kStr];          // rows 0..15 at_t, 16..31 rt_t
  __align__(16) float LT[4][kChunk][20];      // masked Gram blocks, transposed [tau][t]: Lab, Lak, Mrb, Mrk
  bf16 Mrbh[kChunk][kStrS], Mrbl[kChunk][kStrS];
  float ybuf[kChunk][kN + 4];
  int kmask;
  int kbad[4];
};

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}

template <typename T>
__device__ __forceinline__ float2 ld2(const T* p);
template <>
__device__ __forceinline__ float2 ld2<bf16>(const bf16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
template <>
__device__ __forceinline__ float2 ld2<__half>(const __half* p) {
  return __half22float2(*reinterpret_cast<const __half2*>(p));
}
template <>
__device__ __forceinline__ float2 ld2<float>(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}

__device__ __forceinline__ void st_split2(bf16* hi, bf16* lo, float x0, float x1) {
  uint32_t h, l;
  split2(x0, x1, h, l);
  *reinterpret_cast<uint32_t*>(hi) = h;
  *reinterpret_cast<uint32_t*>(lo) = l;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Keep only the bf16 halves of an A fragment whose k index is set in `keep_bits`.
__device__ __forceinline__ void mask_a_k(uint32_t (&a)[4], int c4, unsigned keep_bits) {
  const int k0 = 2 * c4, k1 = 8 + 2 * c4;
  const uint32_t m0 = ((keep_bits >> k0) & 1u ? 0x0000ffffu : 0u) | ((keep_bits >> (k0 + 1)) & 1u ? 0xffff0000u : 0u);
  const uint32_t m1 = ((keep_bits >> k1) & 1u ? 0x0000ffffu : 0u) | ((keep_bits >> (k1 + 1)) & 1u ? 0xffff0000u : 0u);
  a[0] &= m0;
  a[1] &= m0;
  a[2] &= m1;
  a[3] &= m1;
}

template <typename T>
__device__ __forceinline__ void stage_chunk(const FwdArgs& p, T (*dst)[kChunk][kStr], int64_t b, int64_t h,
                                            int64_t t0, int len, int ktid) {
  constexpr int n = Vec16<T>::n;
  constexpr int VPT = kN / n;
  const T* src[kIn] = {static_cast<const T*>(p.r), static_cast<const T*>(p.w), static_cast<const T*>(p.k),
                       static_cast<const T*>(p.v), static_cast<const T*>(p.a), static_cast<const T*>(p.b)};
  for (int idx = ktid; idx < kIn * kChunk * VPT; idx += 128) {
    const int m = idx / (kChunk * VPT);
    const int rem = idx - m * kChunk * VPT;
    const int tt = rem / VPT, vec = rem - (rem / VPT) * VPT;
    T* s = &dst[m][tt][vec * n];
    if (tt < len) {
      cp_async16(s, src[m] + tok_off(b, t0 + tt, h, p.T, p.H) + vec * n);
    } else {   // padding token: w = 1, everything else 0 -> leaves the state unchanged
      const T fill = Elt<T>::from_f32(m == 1 ? 1.f : 0.f);
#pragma unroll
      for (int e = 0; e < n; ++e) s[e] = fill;
    }
  }
  cp_async_commit();
}

// ------------------------------------------------------------------ context warps
template <typename T>
__device__ __forceinline__ void build_context(FwdSmem2<T>& sm, Ctx& cx, const T (*X)[kChunk][kStr], unsigned mask,
                                              int ktid) {
  constexpr bool kVExact = std::is_same<T, bf16>::value;
  const int kw = ktid >> 5, lane = ktid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;

  // ---- K1: decay products and the decay-scaled operands (hi/lo bf16)
  bool bad = false;
  {
    const int j = 2 * lane;   // this thread's column pair
    float la[kChunk], lb[kChunk];
    float l0 = 1.f, l1 = 1.f;
#pragma unroll
    for (int t = 0; t < kChunk; ++t) {
      const float2 w2 = ld2<T>(&X[1][t][j]);
      l0 *= w2.x;
      l1 *= w2.y;
      la[t] = l0;
      lb[t] = l1;
      bad |= !(l0 >= 0x1p-40f && l0 <= 0x1p40f && l1 >= 0x1p-40f && l1 <= 0x1p40f);
    }
    if (kw == 0) {            // at_t = a_t L_{t-1}
      float p0 = 1.f, p1 = 1.f;
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        const float2 a2 = ld2<T>(&X[4][t][j]);
        st_split2(&sm.GAh[t][j], &sm.GAl[t][j], a2.x * p0, a2.y * p1);
        p0 = la[t];
        p1 = lb[t];
      }
    } else if (kw == 1) {     // rt_t = r_t L_t
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        const float2 r2 = ld2<T>(&X[0][t][j]);
        st_split2(&sm.GAh[16 + t][j], &sm.GAl[16 + t][j], r2.x * la[t], r2.y * lb[t]);
      }
    } else if (kw == 2) {     // bh_t = b_t / L_t ; L_15
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        const float2 b2 = ld2<T>(&X[5][t][j]);
        st_split2(&cx.Bh[t][j], &cx.Bl[t][j], b2.x * rcp_approx(la[t]), b2.y * rcp_approx(lb[t]));
      }
      cx.lam15[j] = la[kChunk - 1];
      cx.lam15[j + 1] = lb[kChunk - 1];
    } else {                  // kh_t = k_t / L_t ; v
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        const float2 k2 = ld2<T>(&X[2][t][j]);
        st_split2(&cx.Bh[16 + t][j], &cx.Bl[16 + t][j], k2.x * rcp_approx(la[t]), k2.y * rcp_approx(lb[t]));
        if constexpr (kVExact) {
          *reinterpret_cast<uint32_t*>(&cx.Vh[t][j]) = *reinterpret_cast<const uint32_t*>(&X[3][t][j]);
        } else {
          const float2 v2 = ld2<T>(&X[3][t][j]);
          st_split2(&cx.Vh[t][j], &cx.Vl[t][j], v2.x, v2.y);
        }
      }
    }
  }
  const unsigned any_bad = __ballot_sync(0xffffffffu, bad);
  if (lane == 0) sm.kbad[kw] = any_bad ? 1 : 0;
  named_bar(1, 128);
  const bool unsafe = (sm.kbad[0] | sm.kbad[1] | sm.kbad[2] | sm.kbad[3]) != 0;
  if (ktid == 0) {
    cx.mask = int(mask);
    cx.unsafe = unsafe ? 1 : 0;
  }
  if (unsafe) return;

  // ---- K2: 32x32 Gram of [at; rt] and [bh; kh] on tensor cores (3-term split), masked
  {
    const int m0 = (kw >> 1) * 16, n0 = (kw & 1) * 16;
    float gr[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t ah[4], al[4], bh[4], bl[4];
      ldsm_x4(ah, a_rowmajor_addr(&sm.GAh[0][0], kStr, m0, 16 * ks, lane));
      ldsm_x4(al, a_rowmajor_addr(&sm.GAl[0][0], kStr, m0, 16 * ks, lane));
      ldsm_x4(bh, b_nmajor_addr(&cx.Bh[0][0], kStr, n0, 16 * ks, lane));
      ldsm_x4(bl, b_nmajor_addr(&cx.Bl[0][0], kStr, n0, 16 * ks, lane));
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        mma16816(gr[nt], al, bh[2 * nt], bh[2 * nt + 1]);
        mma16816(gr[nt], ah, bl[2 * nt], bl[2 * nt + 1]);
        mma16816(gr[nt], ah, bh[2 * nt], bh[2 * nt + 1]);
      }
    }
    const bool strict = kw < 2;   // Lab, Lak strictly lower; Mrb, Mrk include the diagonal
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = g + (e >> 1) * 8;
        const int tau = 8 * nt + 2 * c4 + (e & 1);
        bool ok = strict ? (tau < t) : (tau <= t);
        ok = ok && ((mask & ((2u << t) - (2u << tau))) == 0u);   // no reset in (tau, t]
        const float v = ok ? gr[nt][e] : 0.f;
        sm.LT[kw][tau][t] = v;
        if (kw == 2) split1(v, sm.Mrbh[t][tau], sm.Mrbl[t][tau]);
      }
  }
  named_bar(1, 128);

  // ---- K3: W = (I - Lab)^-1 diag(m0) At (threads 0..63), X = (I - Lab)^-1 Lak (threads 64..79)
  if (ktid < 80) {
    float u[kChunk];
    const int cc = ktid < 64 ? ktid : ktid - 64;
    if (ktid < 64) {
#pragma unroll
      for (int t = 0; t < kChunk; ++t)
        u[t] = t < fr ? __bfloat162float(sm.GAh[t][cc]) + __bfloat162float(sm.GAl[t][cc]) : 0.f;
    } else {
      const float4* col = reinterpret_cast<const float4*>(&sm.LT[1][cc][0]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 f = col[q];
        u[4 * q] = f.x; u[4 * q + 1] = f.y; u[4 * q + 2] = f.z; u[4 * q + 3] = f.w;
      }
    }
#pragma unroll
    for (int tau = 0; tau < kChunk - 1; ++tau) {
      const float4* lrow = reinterpret_cast<const float4*>(&sm.LT[0][tau][0]);
      float lv[kChunk];
#pragma unroll
      for (int q = (tau + 1) / 4; q < 4; ++q) {
        const float4 f = lrow[q];
        lv[4 * q] = f.x; lv[4 * q + 1] = f.y; lv[4 * q + 2] = f.z; lv[4 * q + 3] = f.w;
      }
#pragma unroll
      for (int t = tau + 1; t < kChunk; ++t) u[t] = fmaf(lv[t], u[tau], u[t]);
    }
    if (ktid < 64) {
#pragma unroll
      for (int t = 0; t < kChunk; ++t) split1(u[t], cx.Wh[t][cc], cx.Wl[t][cc]);
    } else {
#pragma unroll
      for (int t = 0; t < kChunk; ++t) split1(u[t], cx.Xh[t][cc], cx.Xl[t][cc]);
    }
  }
  named_bar(1, 128);

  // ---- K4: Q = m0.Rt + Mrb W (columns 16kw..16kw+15), Z = Mrk + Mrb X (warp kw == 0)
  {
    uint32_t mh[4], ml[4];
    ldsm_x4(mh, a_rowmajor_addr(&sm.Mrbh[0][0], kStrS, 0, 0, lane));
    ldsm_x4(ml, a_rowmajor_addr(&sm.Mrbl[0][0], kStrS, 0, 0, lane));
    const int j0 = 16 * kw;
    float q[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = g + 8 * hh;
        const int j = j0 + 8 * nt + 2 * c4;
        float2 r2 = make_float2(0.f, 0.f);
        if (t < fr) {
          const float2 h2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sm.GAh[16 + t][j]));
          const float2 l2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sm.GAl[16 + t][j]));
          r2 = make_float2(h2.x + l2.x, h2.y + l2.y);
        }
        q[nt][2 * hh] = r2.x;
        q[nt][2 * hh + 1] = r2.y;
      }
    uint32_t wh[4], wl[4];
    ldsm_x4_t(wh, b_kmajor_addr(&cx.Wh[0][0], kStr, 0, j0, lane));
    ldsm_x4_t(wl, b_kmajor_addr(&cx.Wl[0][0], kStr, 0, j0, lane));
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      mma16816(q[nt], ml, wh[2 * nt], wh[2 * nt + 1]);
      mma16816(q[nt], mh, wl[2 * nt], wl[2 * nt + 1]);
      mma16816(q[nt], mh, wh[2 * nt], wh[2 * nt + 1]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        st_split2(&cx.Qh[g + 8 * hh][j0 + 8 * nt + 2 * c4], &cx.Ql[g + 8 * hh][j0 + 8 * nt + 2 * c4],
                  q[nt][2 * hh], q[nt][2 * hh + 1]);
    if (kw == 0) {
      float z[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) z[nt][e] = sm.LT[3][8 * nt + 2 * c4 + (e & 1)][g + 8 * (e >> 1)];
      uint32_t xh[4], xl[4];
      ldsm_x4_t(xh, b_kmajor_addr(&cx.Xh[0][0], kStrS, 0, 0, lane));
      ldsm_x4_t(xl, b_kmajor_addr(&cx.Xl[0][0], kStrS, 0, 0, lane));
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        mma16816(z[nt], ml, xh[2 * nt], xh[2 * nt + 1]);
        mma16816(z[nt], mh, xl[2 * nt], xl[2 * nt + 1]);
        mma16816(z[nt], mh, xh[2 * nt], xh[2 * nt + 1]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          st_split2(&cx.Zh[g + 8 * hh][8 * nt + 2 * c4], &cx.Zl[g + 8 * hh][8 * nt + 2 * c4], z[nt][2 * hh],
                    z[nt][2 * hh + 1]);
    }
  }
}

// ------------------------------------------------------------------ state warps
template <typename T>
__device__ __forceinline__ void state_chunk(FwdSmem2<T>& sm, const Ctx& cx, float (&acc)[8][4], int warp, int lane) {
  constexpr bool kVExact = std::is_same<T, bf16>::value;
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;
  const unsigned mask = unsigned(cx.mask);
  // SA^T, Y^T (rows i, columns t) = S0 [W^T | Q^T] + V^T [X^T | Z^T]
  float sa[2][4] = {}, yy[2][4] = {};
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    uint32_t ah[4], al[4];
    split2(acc[2 * ks][0], acc[2 * ks][1], ah[0], al[0]);
    split2(acc[2 * ks][2], acc[2 * ks][3], ah[1], al[1]);
    split2(acc[2 * ks + 1][0], acc[2 * ks + 1][1], ah[2], al[2]);
    split2(acc[2 * ks + 1][2], acc[2 * ks + 1][3], ah[3], al[3]);
    uint32_t wh[4], wl[4], qh[4], ql[4];
    ldsm_x4(wh, b_nmajor_addr(&cx.Wh[0][0], kStr, 0, 16 * ks, lane));
    ldsm_x4(wl, b_nmajor_addr(&cx.Wl[0][0], kStr, 0, 16 * ks, lane));
    ldsm_x4(qh, b_nmajor_addr(&cx.Qh[0][0], kStr, 0, 16 * ks, lane));
    ldsm_x4(ql, b_nmajor_addr(&cx.Ql[0][0], kStr, 0, 16 * ks, lane));
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      mma16816(sa[nt], al, wh[2 * nt], wh[2 * nt + 1]);
      mma16816(sa[nt], ah, wl[2 * nt], wl[2 * nt + 1]);
      mma16816(sa[nt], ah, wh[2 * nt], wh[2 * nt + 1]);
      mma16816(yy[nt], al, qh[2 * nt], qh[2 * nt + 1]);
      mma16816(yy[nt], ah, ql[2 * nt], ql[2 * nt + 1]);
      mma16816(yy[nt], ah, qh[2 * nt], qh[2 * nt + 1]);
    }
  }
  uint32_t vh[4], vl[4] = {0u, 0u, 0u, 0u};
  ldsm_x4_t(vh, a_kmajor_addr(&cx.Vh[0][0], kStr, 0, row0, lane));
  if constexpr (!kVExact) ldsm_x4_t(vl, a_kmajor_addr(&cx.Vl[0][0], kStr, 0, row0, lane));
  {
    uint32_t xh[4], xl[4], zh[4], zl[4];
    ldsm_x4(xh, b_nmajor_addr(&cx.Xh[0][0], kStrS, 0, 0, lane));
    ldsm_x4(xl, b_nmajor_addr(&cx.Xl[0][0], kStrS, 0, 0, lane));
    ldsm_x4(zh, b_nmajor_addr(&cx.Zh[0][0], kStrS, 0, 0, lane));
    ldsm_x4(zl, b_nmajor_addr(&cx.Zl[0][0], kStrS, 0, 0, lane));
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      mma16816(sa[nt], vh, xl[2 * nt], xl[2 * nt + 1]);
      mma16816(sa[nt], vh, xh[2 * nt], xh[2 * nt + 1]);
      mma16816(yy[nt], vh, zl[2 * nt], zl[2 * nt + 1]);
      mma16816(yy[nt], vh, zh[2 * nt], zh[2 * nt + 1]);
      if constexpr (!kVExact) {
        mma16816(sa[nt], vl, xh[2 * nt], xh[2 * nt + 1]);
        mma16816(yy[nt], vl, zh[2 * nt], zh[2 * nt + 1]);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) sm.ybuf[8 * nt + 2 * c4 + (e & 1)][row0 + g + 8 * (e >> 1)] = yy[nt][e];

  // S_16 = keep.S0 diag(L_15) + (SA^T Bh + V^T Kh) diag(L_15); only the last segment's tokens
  // contribute.  The products go to a separate accumulator so that S0 is scaled exactly and
  // never added to the (1/L-sized) intermediate terms.
  const unsigned seg_last = __popc(mask & 0xfffeu);
  unsigned last_bits = 0u;
#pragma unroll
  for (int t = 0; t < kChunk; ++t) last_bits |= (unsigned(__popc(mask & ((2u << t) - 2u))) == seg_last ? 1u : 0u) << t;
  const float keep = mask == 0u ? 1.f : 0.f;
  uint32_t sh[4], sl[4];
  split2(sa[0][0], sa[0][1], sh[0], sl[0]);
  split2(sa[0][2], sa[0][3], sh[1], sl[1]);
  split2(sa[1][0], sa[1][1], sh[2], sl[2]);
  split2(sa[1][2], sa[1][3], sh[3], sl[3]);
  if (last_bits != 0xffffu) {
    mask_a_k(sh, c4, last_bits);
    mask_a_k(sl, c4, last_bits);
    mask_a_k(vh, c4, last_bits);
    mask_a_k(vl, c4, last_bits);
  }
#pragma unroll
  for (int np = 0; np < 4; ++np) {
    uint32_t bbh[4], bbl[4], kbh[4], kbl[4];
    ldsm_x4_t(bbh, b_kmajor_addr(&cx.Bh[0][0], kStr, 0, 16 * np, lane));
    ldsm_x4_t(bbl, b_kmajor_addr(&cx.Bl[0][0], kStr, 0, 16 * np, lane));
    ldsm_x4_t(kbh, b_kmajor_addr(&cx.Bh[0][0], kStr, 16, 16 * np, lane));
    ldsm_x4_t(kbl, b_kmajor_addr(&cx.Bl[0][0], kStr, 16, 16 * np, lane));
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      mma16816(d, sl, bbh[2 * u], bbh[2 * u + 1]);
      mma16816(d, sh, bbl[2 * u], bbl[2 * u + 1]);
      mma16816(d, sh, bbh[2 * u], bbh[2 * u + 1]);
      mma16816(d, vh, kbl[2 * u], kbl[2 * u + 1]);
      mma16816(d, vh, kbh[2 * u], kbh[2 * u + 1]);
      if constexpr (!kVExact) mma16816(d, vl, kbh[2 * u], kbh[2 * u + 1]);
      const int nt = 2 * np + u;
      const float2 l2 = *reinterpret_cast<const float2*>(&cx.lam15[8 * nt + 2 * c4]);
      acc[nt][0] = fmaf(keep * acc[nt][0], l2.x, d[0] * l2.x);
      acc[nt][1] = fmaf(keep * acc[nt][1], l2.y, d[1] * l2.y);
      acc[nt][2] = fmaf(keep * acc[nt][2], l2.x, d[2] * l2.x);
      acc[nt][3] = fmaf(keep * acc[nt][3], l2.y, d[3] * l2.y);
    }
  }
}

// Token-by-token update of one chunk on the state fragments (decay out of range), inputs read from global.
template <typename T>
__device__ __forceinline__ void state_chunk_tokens(const FwdArgs& p, FwdSmem2<T>& sm, unsigned mask,
                                                   float (&acc)[8][4], int64_t b, int64_t h, int64_t t0, int len,
                                                   int warp, int lane) {
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;
  const T* R = static_cast<const T*>(p.r);
  const T* Wd = static_cast<const T*>(p.w);
  const T* K = static_cast<const T*>(p.k);
  const T* V = static_cast<const T*>(p.v);
  const T* A = static_cast<const T*>(p.a);
  const T* Bb = static_cast<const T*>(p.b);
  for (int tt = 0; tt < len; ++tt) {
    const int64_t o = tok_off(b, t0 + tt, h, p.T, p.H);
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
        const float wv = Elt<T>::to_f32(Wd[o + col]), bv = Elt<T>::to_f32(Bb[o + col]);
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
      sm.ybuf[tt][row0 + g] = y_lo;
      sm.ybuf[tt][row0 + g + 8] = y_hi;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) chunk_fwd_kernel(FwdArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  FwdSmem2<T>& sm = *reinterpret_cast<FwdSmem2<T>*>(smem_raw);

  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_state = warp < 4;
  const int ktid = tid - 128;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;

  // state fragments: acc[nt][e] = S[16*warp + g + 8*(e>>1)][8*nt + 2*c4 + (e&1)]
  float acc[8][4];
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;
  if (is_state) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float2 v2 = make_float2(0.f, 0.f);
        if (p.s0) v2 = *reinterpret_cast<const float2*>(p.s0 + (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4);
        acc[nt][2 * hh] = v2.x;
        acc[nt][2 * hh + 1] = v2.y;
      }
  }

  // prologue: the context warps stage chunk 0 and fetch its reset flags
  unsigned reset_bits_next = 0u;
  if (!is_state) {
    stage_chunk<T>(p, sm.in[0], b, h, 0, int(min64(kChunk, p.T)), ktid);
    if (warp == 4) {
      const int len0 = int(min64(kChunk, p.T));
      const bool f = p.reset && lane < len0 && p.reset[b * p.T + lane] != 0;
      reset_bits_next = __ballot_sync(0xffffffffu, f) & 0xffffu;
    }
    cp_async_wait_all();
  }
  __syncthreads();

  for (int64_t it = 0; it <= nc; ++it) {
    if (!is_state) {
      if (it < nc) {
        const int64_t c = it;
        const int buf = int(c & 1);
        if (warp == 4 && lane == 0) sm.kmask = int(reset_bits_next);
        if (c + 1 < nc) {
          const int64_t t1 = (c + 1) * kChunk;
          const int len1 = int(min64(kChunk, p.T - t1));
          stage_chunk<T>(p, sm.in[buf ^ 1], b, h, t1, len1, ktid);
          if (warp == 4) {
            const bool f = p.reset && lane < len1 && p.reset[b * p.T + t1 + lane] != 0;
            reset_bits_next = __ballot_sync(0xffffffffu, f) & 0xffffu;
          }
        }
        named_bar(1, 128);
        build_context<T>(sm, sm.ctx[buf], sm.in[buf], unsigned(sm.kmask), ktid);
        cp_async_wait_all();
      }
    } else if (it >= 1) {
      const int64_t c = it - 1;
      const Ctx& cx = sm.ctx[c & 1];
      const int64_t t0 = c * kChunk;
      const int len = int(min64(kChunk, p.T - t0));
      if (!cx.unsafe) {
        state_chunk<T>(sm, cx, acc, warp, lane);
      } else {
        state_chunk_tokens<T>(p, sm, unsigned(cx.mask), acc, b, h, t0, len, warp, lane);
      }
      if (p.ckpt) {
        float* base = p.ckpt + (unit * nc + c) * kN * kN;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            *reinterpret_cast<float2*>(base + (row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4) =
                make_float2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
      }
      named_bar(2, 128);   // ybuf complete
      T* y = static_cast<T*>(p.y);
      for (int e = tid; e < len * 8; e += 128) {
        const int tt = e >> 3, part = e & 7;
        alignas(16) T vals[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) vals[u] = Elt<T>::from_f32(sm.ybuf[tt][part * 8 + u]);
        uint4* dst = reinterpret_cast<uint4*>(y + tok_off(b, t0 + tt, h, p.T, p.H) + part * 8);
        const uint4* sv = reinterpret_cast<const uint4*>(vals);
#pragma unroll
        for (int u = 0; u < int(sizeof(vals) / 16); ++u) dst[u] = sv[u];
      }
    }
    __syncthreads();   // context of chunk it handed to the state warps; staged inputs rotate
  }

  if (is_state && p.s_out) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        *reinterpret_cast<float2*>(p.s_out + (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4) =
            make_float2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
  }
}

template <typename T>
cudaError_t launch(const FwdArgs& p, cudaStream_t stream) {
  const size_t smem = sizeof(FwdSmem2<T>);
  cudaError_t e = cudaFuncSetAttribute(chunk_fwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  chunk_fwd_kernel<T><<<dim3(unsigned(p.B * p.H)), dim3(kThreads), smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_fwd(const FwdArgs& p, int dtype, cudaStream_t stream) {
  switch (dtype) {
    case 0: return launch<float>(p, stream);
    case 1: return launch<__nv_bfloat16>(p, stream);
    case 2: return launch<__half>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
