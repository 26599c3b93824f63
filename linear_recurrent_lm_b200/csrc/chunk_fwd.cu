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
// Mrb, Mrk are the same with rt_t (tau <= t).  With T = (I - Lab)^-1 (unit
// lower triangular, solved by substitution -- the triangular inversion the
// rwkv-lab page names for chunked delta rules):
//   SA = W S0^T + X V,   Y = Q S0^T + Z V,
//   W = T At, X = T Lak, Q = Rt + Mrb W, Z = Mrb X + Mrk,
//   S_16 = S0 diag(L_15) + SA^T Bb + V^T Kb,  Bb_t = b_t L_15 / L_t, Kb_t = k_t L_15 / L_t.
// Only the last two lines touch the state: per warp (16 rows of S) they are
// S0 @ [W^T | Q^T] (16x64x32) and [SA^T | V^T] @ [Bb ; Kb] (16x32x64) on
// bf16 mma.sync.  Reset flags inside a chunk become masks: pairs (t, tau)
// separated by a reset are dropped from Lab..Mrk, S0 only reaches tokens
// before the first reset, and only the last segment feeds S_16.
//
// Precision: every product with an fp32 operand uses the 3-term bf16 split
// (hi*hi + hi*lo + lo*hi), about 2^-16 relative per product; bf16 inputs
// (v) enter exactly.  A chunk whose decay product leaves [2^-40, 2^40]
// (e.g. w = 0) cannot use the 1/L scaling and is run token by token instead.
//
// One CTA (4 warps) per (b,h); warp w owns rows 16w..16w+15 of S as mma
// accumulator fragments for the whole sequence.  The next chunk's inputs are
// copied to shared memory with cp.async while the current one is processed.
// The state after every chunk goes to the checkpoint workspace.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace wkv7 {
namespace {

constexpr int kThreads = 128;
constexpr int kStr = 72;    // padded row stride (elements) of 64-wide tiles: conflict-free ldmatrix
constexpr int kStrS = 24;   // padded row stride of 16-wide tiles
constexpr int kIn = 6;      // staged inputs: r, w, k, v, a, b
using bf16 = __nv_bfloat16;

template <typename T>
struct ChunkSmem {
  T in[2][kIn][kChunk][kStr];
  bf16 GAh[32][kStr], GAl[32][kStr];   // rows 0..15 at_t, 16..31 rt_t
  bf16 GBh[32][kStr], GBl[32][kStr];   // rows 0..15 bh_t, 16..31 kh_t
  bf16 BBh[kChunk][kStr], BBl[kChunk][kStr];
  bf16 KBh[kChunk][kStr], KBl[kChunk][kStr];
  bf16 Wh[kChunk][kStr], Wl[kChunk][kStr];
  bf16 Qh[kChunk][kStr], Ql[kChunk][kStr];
  bf16 Vh[kChunk][kStr], Vl[kChunk][kStr];   // split v (16-bit non-bf16 and f32 inputs only)
  bf16 Xh[kChunk][kStrS], Xl[kChunk][kStrS], Zh[kChunk][kStrS], Zl[kChunk][kStrS];
  float A0[kChunk][kN];       // at_t masked to tokens before the first reset
  float R0[kChunk][kN];       // rt_t, same mask
  float LT[4][kChunk][20];    // transposed [tau][t]: Lab, Lak, Mrb, Mrk
  float ybuf[kChunk][kN + 4];
  float lam15[kN];
  int mask;
};

template <typename T>
__device__ __forceinline__ void stage_chunk(const FwdArgs& p, const T* const* src, T (*dst)[kChunk][kStr],
                                            int64_t b, int64_t h, int64_t t0, int len) {
  constexpr int n = Vec16<T>::n;
  constexpr int VPT = kN / n;
  for (int idx = threadIdx.x; idx < kIn * kChunk * VPT; idx += kThreads) {
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

template <typename T>
__global__ void __launch_bounds__(kThreads) chunk_fwd_kernel(FwdArgs p) {
  constexpr bool kVExact = std::is_same<T, bf16>::value;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ChunkSmem<T>& sm = *reinterpret_cast<ChunkSmem<T>*>(smem_raw);

  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;
  const T* src[kIn] = {static_cast<const T*>(p.r), static_cast<const T*>(p.w), static_cast<const T*>(p.k),
                       static_cast<const T*>(p.v), static_cast<const T*>(p.a), static_cast<const T*>(p.b)};

  // state fragments: acc[nt][e] = S[row0 + g + 8*(e>>1)][8*nt + 2*c4 + (e&1)]
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float2 v2 = make_float2(0.f, 0.f);
      if (p.s0) v2 = *reinterpret_cast<const float2*>(p.s0 + (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4);
      acc[nt][2 * hh] = v2.x;
      acc[nt][2 * hh + 1] = v2.y;
    }

  if (nc > 0) {
    stage_chunk<T>(p, src, sm.in[0], b, h, 0, int(min64(kChunk, p.T)));
    cp_async_wait_all();
  }

  for (int64_t c = 0; c < nc; ++c) {
    const int buf = int(c & 1);
    const int64_t t0 = c * kChunk;
    const int len = int(min64(kChunk, p.T - t0));
    if (c + 1 < nc)
      stage_chunk<T>(p, src, sm.in[buf ^ 1], b, h, t0 + kChunk, int(min64(kChunk, p.T - t0 - kChunk)));
    if (warp == 0) {
      const bool f = p.reset && lane < len && p.reset[b * p.T + t0 + lane] != 0;
      const unsigned m = __ballot_sync(0xffffffffu, f) & 0xffffu;
      if (lane == 0) sm.mask = int(m);
    }
    __syncthreads();   // (A) inputs of chunk c visible, mask visible
    const unsigned mask = unsigned(sm.mask);
    const T (*X)[kChunk][kStr] = sm.in[buf];

    // ---- 1) decay products and decay-scaled vectors (elementwise, fp32)
    bool bad = false;
    {
      const int j = tid & 63, hf = tid >> 6;
      const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
      float lam[kChunk];
      float l = 1.f;
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        l *= Elt<T>::to_f32(X[1][t][j]);
        lam[t] = l;
        bad |= !(l >= 0x1p-40f && l <= 0x1p40f);
      }
      if (hf == 0) {
        float prev = 1.f;
#pragma unroll
        for (int t = 0; t < kChunk; ++t) {
          const float at = Elt<T>::to_f32(X[4][t][j]) * prev;
          const float rt = Elt<T>::to_f32(X[0][t][j]) * lam[t];
          prev = lam[t];
          split1(at, sm.GAh[t][j], sm.GAl[t][j]);
          split1(rt, sm.GAh[16 + t][j], sm.GAl[16 + t][j]);
          sm.A0[t][j] = t < fr ? at : 0.f;
          sm.R0[t][j] = t < fr ? rt : 0.f;
        }
        sm.lam15[j] = lam[kChunk - 1];
      } else {
        const int seg_last = __popc(mask & 0xfffeu);
#pragma unroll
        for (int t = 0; t < kChunk; ++t) {
          const float inv = 1.f / lam[t];
          const float bt = Elt<T>::to_f32(X[5][t][j]), kt = Elt<T>::to_f32(X[2][t][j]);
          split1(bt * inv, sm.GBh[t][j], sm.GBl[t][j]);
          split1(kt * inv, sm.GBh[16 + t][j], sm.GBl[16 + t][j]);
          const bool last = __popc(mask & ((2u << t) - 2u)) == seg_last;
          const float ratio = lam[kChunk - 1] * inv;
          split1(last ? bt * ratio : 0.f, sm.BBh[t][j], sm.BBl[t][j]);
          split1(last ? kt * ratio : 0.f, sm.KBh[t][j], sm.KBl[t][j]);
          if constexpr (!kVExact) split1(Elt<T>::to_f32(X[3][t][j]), sm.Vh[t][j], sm.Vl[t][j]);
        }
      }
    }
    const bool unsafe = __syncthreads_or(bad);   // (B)

    if (!unsafe) {
      // ---- 2) 32x32 Gram of [at; rt] and [bh; kh] on tensor cores, masked, stored transposed
      {
        const int m0 = (warp >> 1) * 16, n0 = (warp & 1) * 16;
        float gr[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint32_t ah[4], al[4], bh[4], bl[4];
          ldsm_x4(ah, a_rowmajor_addr(&sm.GAh[0][0], kStr, m0, 16 * ks, lane));
          ldsm_x4(al, a_rowmajor_addr(&sm.GAl[0][0], kStr, m0, 16 * ks, lane));
          ldsm_x4(bh, b_nmajor_addr(&sm.GBh[0][0], kStr, n0, 16 * ks, lane));
          ldsm_x4(bl, b_nmajor_addr(&sm.GBl[0][0], kStr, n0, 16 * ks, lane));
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            mma16816(gr[nt], al, bh[2 * nt], bh[2 * nt + 1]);
            mma16816(gr[nt], ah, bl[2 * nt], bl[2 * nt + 1]);
            mma16816(gr[nt], ah, bh[2 * nt], bh[2 * nt + 1]);
          }
        }
        const bool strict = warp < 2;   // Lab, Lak strictly lower; Mrb, Mrk include the diagonal
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = g + (e >> 1) * 8;
            const int tau = 8 * nt + 2 * c4 + (e & 1);
            bool ok = strict ? (tau < t) : (tau <= t);
            ok = ok && ((mask & ((2u << t) - (2u << tau))) == 0u);   // no reset in (tau, t]
            sm.LT[warp][tau][t] = ok ? gr[nt][e] : 0.f;
          }
      }
      __syncthreads();   // (C)

      // ---- 3) W = T At, Q = Rt + Mrb W (columns 0..63); X = T Lak, Z = Mrb X + Mrk (columns 64..79)
      if (tid < 80) {
        const float (*Lab)[20] = sm.LT[0];
        const float (*Mrb)[20] = sm.LT[2];
        float u[kChunk], o[kChunk];
        const int cc = tid < 64 ? tid : tid - 64;
        if (tid < 64) {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) u[t] = sm.A0[t][cc];
        } else {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) u[t] = sm.LT[1][cc][t];
        }
#pragma unroll
        for (int tau = 0; tau < kChunk; ++tau)
#pragma unroll
          for (int t = tau + 1; t < kChunk; ++t) u[t] = fmaf(Lab[tau][t], u[tau], u[t]);
        if (tid < 64) {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) o[t] = sm.R0[t][cc];
        } else {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) o[t] = sm.LT[3][cc][t];
        }
#pragma unroll
        for (int tau = 0; tau < kChunk; ++tau)
#pragma unroll
          for (int t = tau; t < kChunk; ++t) o[t] = fmaf(Mrb[tau][t], u[tau], o[t]);
        if (tid < 64) {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) {
            split1(u[t], sm.Wh[t][cc], sm.Wl[t][cc]);
            split1(o[t], sm.Qh[t][cc], sm.Ql[t][cc]);
          }
        } else {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) {
            split1(u[t], sm.Xh[t][cc], sm.Xl[t][cc]);
            split1(o[t], sm.Zh[t][cc], sm.Zl[t][cc]);
          }
        }
      }
      __syncthreads();   // (D)

      // ---- 4) state products for this warp's 16 rows
      float sa[2][4] = {}, yy[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t ah[4], al[4];
        split2(acc[2 * ks][0], acc[2 * ks][1], ah[0], al[0]);
        split2(acc[2 * ks][2], acc[2 * ks][3], ah[1], al[1]);
        split2(acc[2 * ks + 1][0], acc[2 * ks + 1][1], ah[2], al[2]);
        split2(acc[2 * ks + 1][2], acc[2 * ks + 1][3], ah[3], al[3]);
        uint32_t wh[4], wl[4], qh[4], ql[4];
        ldsm_x4(wh, b_nmajor_addr(&sm.Wh[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4(wl, b_nmajor_addr(&sm.Wl[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4(qh, b_nmajor_addr(&sm.Qh[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4(ql, b_nmajor_addr(&sm.Ql[0][0], kStr, 0, 16 * ks, lane));
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
      if constexpr (kVExact) {
        ldsm_x4_t(vh, a_kmajor_addr(&X[3][0][0], kStr, 0, row0, lane));
      } else {
        ldsm_x4_t(vh, a_kmajor_addr(&sm.Vh[0][0], kStr, 0, row0, lane));
        ldsm_x4_t(vl, a_kmajor_addr(&sm.Vl[0][0], kStr, 0, row0, lane));
      }
      {
        uint32_t xh[4], xl[4], zh[4], zl[4];
        ldsm_x4(xh, b_nmajor_addr(&sm.Xh[0][0], kStrS, 0, 0, lane));
        ldsm_x4(xl, b_nmajor_addr(&sm.Xl[0][0], kStrS, 0, 0, lane));
        ldsm_x4(zh, b_nmajor_addr(&sm.Zh[0][0], kStrS, 0, 0, lane));
        ldsm_x4(zl, b_nmajor_addr(&sm.Zl[0][0], kStrS, 0, 0, lane));
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

      // S_16 = S0 diag(L_15) + SA^T Bb + V^T Kb
      const bool keep = mask == 0u;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = keep ? acc[nt][e] * sm.lam15[8 * nt + 2 * c4 + (e & 1)] : 0.f;
      uint32_t sh[4], sl[4];
      split2(sa[0][0], sa[0][1], sh[0], sl[0]);
      split2(sa[0][2], sa[0][3], sh[1], sl[1]);
      split2(sa[1][0], sa[1][1], sh[2], sl[2]);
      split2(sa[1][2], sa[1][3], sh[3], sl[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bbh[4], bbl[4], kbh[4], kbl[4];
        ldsm_x4_t(bbh, b_kmajor_addr(&sm.BBh[0][0], kStr, 0, 16 * np, lane));
        ldsm_x4_t(bbl, b_kmajor_addr(&sm.BBl[0][0], kStr, 0, 16 * np, lane));
        ldsm_x4_t(kbh, b_kmajor_addr(&sm.KBh[0][0], kStr, 0, 16 * np, lane));
        ldsm_x4_t(kbl, b_kmajor_addr(&sm.KBl[0][0], kStr, 0, 16 * np, lane));
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          float (&d)[4] = acc[2 * np + u];
          mma16816(d, sl, bbh[2 * u], bbh[2 * u + 1]);
          mma16816(d, sh, bbl[2 * u], bbl[2 * u + 1]);
          mma16816(d, sh, bbh[2 * u], bbh[2 * u + 1]);
          mma16816(d, vh, kbl[2 * u], kbl[2 * u + 1]);
          mma16816(d, vh, kbh[2 * u], kbh[2 * u + 1]);
          if constexpr (!kVExact) mma16816(d, vl, kbh[2 * u], kbh[2 * u + 1]);
        }
      }
    } else {
      // ---- token-by-token fallback on the same fragments (decay product out of range)
      for (int tt = 0; tt < len; ++tt) {
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
            const float av = Elt<T>::to_f32(X[4][tt][8 * nt + 2 * c4 + (e & 1)]);
            if (e < 2) s_lo = fmaf(acc[nt][e], av, s_lo); else s_hi = fmaf(acc[nt][e], av, s_hi);
          }
        s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
        s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
        s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
        s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
        const float v_lo = Elt<T>::to_f32(X[3][tt][row0 + g]);
        const float v_hi = Elt<T>::to_f32(X[3][tt][row0 + g + 8]);
        float y_lo = 0.f, y_hi = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = 8 * nt + 2 * c4 + (e & 1);
            const float wv = Elt<T>::to_f32(X[1][tt][col]), bv = Elt<T>::to_f32(X[5][tt][col]);
            const float kv = Elt<T>::to_f32(X[2][tt][col]), rv = Elt<T>::to_f32(X[0][tt][col]);
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

    if (p.ckpt) {
      float* base = p.ckpt + (unit * nc + c) * kN * kN;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<float2*>(base + (row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4) =
              make_float2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
    }
    cp_async_wait_all();
    __syncthreads();   // (E) ybuf complete; next chunk's inputs landed
    {
      T* y = static_cast<T*>(p.y);
      for (int e = tid; e < len * 8; e += kThreads) {
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
  }

  if (p.s_out) {
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
  const size_t smem = sizeof(ChunkSmem<T>);
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
