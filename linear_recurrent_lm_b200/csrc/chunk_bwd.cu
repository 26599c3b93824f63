// WKV-7 backward in 16-token chunks on tensor cores (algo CHUNKED).
//
// Exact reverse mode of the chunk formulas of the forward (see chunk_fwd.cu):
// inside a chunk with entering state S0, decay products L_t = prod_{s<=t} w_s
// and At = a L_{t-1}, Rt = r L_t, Bh = b / L_t, Kh = k / L_t,
//   SA = m0.At S0^T + Lab SA + Lak V,    Y = m0.Rt S0^T + Mrb SA + Mrk V,
//   S16 = keep.S0 diag(L_15) + SA^T Bb + V^T Kb   (Bb = ls.Bh L_15, Kb = ls.Kh L_15)
// where Lab = At Bh^T, Lak = At Kh^T (strictly lower), Mrb = Rt Bh^T,
// Mrk = Rt Kh^T (lower), all masked to token pairs with no reset between them;
// m0 marks tokens before the chunk's first reset, ls the tokens of its last
// segment, keep = "no reset in the chunk".  Given dY and dS16 (the gradient
// carried from the next chunk):
//   dSA  = Mrb^T dY + Bb dS16^T,   dU = (I - Lab)^-T dSA,
//   dV   = Mrk^T dY + Kb dS16^T + Lak^T dU,
//   dMrb = dY SA^T, dMrk = dY V^T, dLab = dU SA^T, dLak = dU V^T   (masked),
//   dAt  = dLab Bh + dLak Kh + m0.dU S0,   dRt = dMrb Bh + dMrk Kh + m0.dY S0,
//   dBh  = dLab^T At + dMrb^T Rt + ls.L_15.(SA dS16),
//   dKh  = dLak^T At + dMrk^T Rt + ls.L_15.(V dS16),
//   dS0  = keep.dS16 diag(L_15) + (m0.dY)^T Rt + (m0.dU)^T At
// and, through the decay, with d log L_t = dr r + da_{t+1} a_{t+1} - db b - dk k
// (plus, at t = 15, sum_i dS16 o S0 L_15 and sum over the last segment of
// dBb o Bb + dKb o Kb), d log w_s = sum_{t >= s} d log L_t and dw = d log w / w.
// The pages print no backward; this is derived from the chunk forward, which
// itself is the recurrence regrouped (RWKV-MLX page, "Key Design Decisions" 2:
// state checkpoints every 16 tokens; rwkv-metal page: the backward recomputes
// each chunk from its checkpoint).
//
// Gradients need cosine >= 0.999, so every product here is a single bf16
// mma.sync with fp32 accumulation.  A chunk with a decay outside the range
// the 1/L scaling tolerates (some w < 1/16, or L_15 outside [2^-40, 2^40])
// makes the CTA stop and mark its unit in `unit_flags`; the scan backward then
// recomputes exactly those units.
//
// One CTA (4 warps) per (b,h).  Warp w owns rows 16w..16w+15 (value channel i)
// of dS as accumulator fragments, and columns 16w..16w+15 (key channel j) of
// the key-space gradients.  Chunks are visited in reverse; the inputs of the
// next one are staged with cp.async and its checkpoint is prefetched into
// registers while the current one is processed.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace wkv7 {
namespace {

constexpr int kThreads = 128;
constexpr int kStr = 72;
constexpr int kStrS = 24;
constexpr int kStrG = 40;
constexpr int kIn = 7;   // r, w, k, v, a, b, dy
using bf16 = __nv_bfloat16;

template <typename T>
struct CbSmem {
  T in[2][kIn][kChunk][kStr];
  bf16 Vb[std::is_same<T, bf16>::value ? 1 : kChunk][kStr];    // bf16 copies of v, dy (non-bf16 inputs)
  bf16 DYb[std::is_same<T, bf16>::value ? 1 : kChunk][kStr];
  bf16 GA[32][kStr];       // rows 0..15 At, 16..31 Rt
  bf16 GB[32][kStr];       // rows 0..15 Bh, 16..31 Kh
  bf16 BK[32][kStr];       // rows 0..15 Bb, 16..31 Kb
  bf16 S0b[kN][kStr];      // entering state
  bf16 dSb[kN][kStr];      // dS16
  bf16 SAb[kChunk][kStr], DUb[kChunk][kStr], Wb[kChunk][kStr];
  bf16 Tb[kChunk][kStrS], Xb[kChunk][kStrS], Mrbb[kChunk][kStrS], Mrkb[kChunk][kStrS], Lakb[kChunk][kStrS];
  bf16 dG[32][kStrG];      // [dMrb dMrk; dLab dLak]
  __align__(16) float LabT[kChunk][20];
  __align__(16) float LakT[kChunk][20];
  float lam[kChunk][kN];
  float E1[kChunk][kN], E2[kChunk][kN];
  float e3[kN];
  float dlam[4][kN];
  int mask;
};

template <typename T>
__device__ __forceinline__ void stage7(const BwdArgs& p, T (*dst)[kChunk][kStr], int64_t b, int64_t h, int64_t t0,
                                       int len) {
  constexpr int n = Vec16<T>::n;
  constexpr int VPT = kN / n;
  const T* src[kIn] = {static_cast<const T*>(p.r), static_cast<const T*>(p.w), static_cast<const T*>(p.k),
                       static_cast<const T*>(p.v), static_cast<const T*>(p.a), static_cast<const T*>(p.b),
                       static_cast<const T*>(p.dy)};
  for (int idx = threadIdx.x; idx < kIn * kChunk * VPT; idx += kThreads) {
    const int m = idx / (kChunk * VPT);
    const int rem = idx - m * kChunk * VPT;
    const int tt = rem / VPT, vec = rem - (rem / VPT) * VPT;
    T* s = &dst[m][tt][vec * n];
    if (tt < len) {
      cp_async16(s, src[m] + tok_off(b, t0 + tt, h, p.T, p.H) + vec * n);
    } else {   // padding token: w = 1, everything else (dy included) 0
      const T fill = Elt<T>::from_f32(m == 1 ? 1.f : 0.f);
#pragma unroll
      for (int e = 0; e < n; ++e) s[e] = fill;
    }
  }
  cp_async_commit();
}

// State entering chunk c: checkpoint c-1, s0, or zero; as accumulator fragments of rows row0..row0+15.
__device__ __forceinline__ void load_entry_state(const BwdArgs& p, int64_t unit, int64_t nc, int64_t c, int row0,
                                                 int g, int c4, float (&S)[8][4]) {
  const float* src = c > 0 ? p.ckpt + (unit * nc + (c - 1)) * kN * kN : (p.s0 ? p.s0 + unit * kN * kN : nullptr);
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float2 v = make_float2(0.f, 0.f);
      if (src) v = *reinterpret_cast<const float2*>(src + (row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4);
      S[nt][2 * hh] = v.x;
      S[nt][2 * hh + 1] = v.y;
    }
}

__device__ __forceinline__ void frag_to_a(const float (&lo)[4], const float (&hi)[4], uint32_t (&a)[4]) {
  a[0] = pack_bf16(lo[0], lo[1]);
  a[1] = pack_bf16(lo[2], lo[3]);
  a[2] = pack_bf16(hi[0], hi[1]);
  a[3] = pack_bf16(hi[2], hi[3]);
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Zero the bf16 halves of an A fragment whose k index (token) is >= fr.
__device__ __forceinline__ void mask_k(uint32_t (&a)[4], int c4, int fr) {
  const int k0 = 2 * c4, k1 = 8 + 2 * c4;
  const uint32_t m0 = (k0 < fr ? 0x0000ffffu : 0u) | (k0 + 1 < fr ? 0xffff0000u : 0u);
  const uint32_t m1 = (k1 < fr ? 0x0000ffffu : 0u) | (k1 + 1 < fr ? 0xffff0000u : 0u);
  a[0] &= m0;
  a[1] &= m0;
  a[2] &= m1;
  a[3] &= m1;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) chunk_bwd_kernel(BwdArgs p) {
  constexpr bool kBf = std::is_same<T, bf16>::value;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  CbSmem<T>& sm = *reinterpret_cast<CbSmem<T>*>(smem_raw);

  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;    // i-block (rows of dS) and j-block (columns) of this warp
  const int64_t nc = (p.T + kChunk - 1) / kChunk;

  float dS[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float2 v = make_float2(0.f, 0.f);
      if (p.dsT) v = *reinterpret_cast<const float2*>(p.dsT + (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4);
      dS[nt][2 * hh] = v.x;
      dS[nt][2 * hh + 1] = v.y;
    }
  float S0[8][4];
  bool flagged = false;
  if (nc > 0) {
    load_entry_state(p, unit, nc, nc - 1, row0, g, c4, S0);
    const int64_t t0 = (nc - 1) * kChunk;
    stage7<T>(p, sm.in[(nc - 1) & 1], b, h, t0, int(p.T - t0));
    if (warp == 0) {
      const int len = int(p.T - t0);
      const bool f = p.reset && lane < len && p.reset[b * p.T + t0 + lane] != 0;
      const unsigned m = __ballot_sync(0xffffffffu, f) & 0xffffu;
      if (lane == 0) sm.mask = int(m);
    }
  }

  for (int64_t c = nc - 1; c >= 0; --c) {
    const int buf = int(c & 1);
    const int64_t t0 = c * kChunk;
    const int len = int(min64(kChunk, p.T - t0));
    cp_async_wait_all();
    __syncthreads();   // (0) inputs of chunk c landed; previous chunk fully done
    const unsigned mask = unsigned(sm.mask);
    const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
    const bool keep = mask == 0u;
    const int seg_last = __popc(mask & 0xfffeu);
    const T (*X)[kChunk][kStr] = sm.in[buf];
    const bf16 (*Vsrc)[kStr] = kBf ? reinterpret_cast<const bf16(*)[kStr]>(&X[3][0][0]) : sm.Vb;
    const bf16 (*DYsrc)[kStr] = kBf ? reinterpret_cast<const bf16(*)[kStr]>(&X[6][0][0]) : sm.DYb;

    // ---- P1: decay products, decay-scaled vectors (bf16), state copies, sum_i S0 o dS16
    bool bad = false;
    {
      const int jp = tid & 31, grp = tid >> 5;   // columns 2jp, 2jp+1; vector family grp
      const int j = 2 * jp;
      float l0 = 1.f, l1 = 1.f, p0 = 1.f, p1 = 1.f;
      float lam0[kChunk], lam1[kChunk];
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        const float w0 = Elt<T>::to_f32(X[1][t][j]), w1 = Elt<T>::to_f32(X[1][t][j + 1]);
        l0 *= w0;
        l1 *= w1;
        lam0[t] = l0;
        lam1[t] = l1;
        bad |= !(w0 >= 0.0625f && w1 >= 0.0625f && l0 >= 0x1p-40f && l1 >= 0x1p-40f && l0 <= 0x1p40f && l1 <= 0x1p40f);
      }
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        uint32_t* row;
        float x0, x1;
        if (grp == 0) {          // At_t = a_t L_{t-1}
          x0 = Elt<T>::to_f32(X[4][t][j]) * p0;
          x1 = Elt<T>::to_f32(X[4][t][j + 1]) * p1;
          row = reinterpret_cast<uint32_t*>(&sm.GA[t][j]);
          *row = pack_bf16(x0, x1);
        } else if (grp == 1) {   // Rt_t = r_t L_t; L_t itself
          x0 = Elt<T>::to_f32(X[0][t][j]) * lam0[t];
          x1 = Elt<T>::to_f32(X[0][t][j + 1]) * lam1[t];
          *reinterpret_cast<uint32_t*>(&sm.GA[16 + t][j]) = pack_bf16(x0, x1);
          *reinterpret_cast<float2*>(&sm.lam[t][j]) = make_float2(lam0[t], lam1[t]);
        } else {                 // Bh, Bb (grp 2) / Kh, Kb (grp 3)
          const int src = grp == 2 ? 5 : 2;
          const float i0 = rcp_approx(lam0[t]), i1 = rcp_approx(lam1[t]);
          x0 = Elt<T>::to_f32(X[src][t][j]) * i0;
          x1 = Elt<T>::to_f32(X[src][t][j + 1]) * i1;
          const int r = grp == 2 ? t : 16 + t;
          *reinterpret_cast<uint32_t*>(&sm.GB[r][j]) = pack_bf16(x0, x1);
          const bool last = __popc(mask & ((2u << t) - 2u)) == seg_last;
          *reinterpret_cast<uint32_t*>(&sm.BK[r][j]) =
              last ? pack_bf16(x0 * lam0[kChunk - 1], x1 * lam1[kChunk - 1]) : 0u;
        }
        p0 = lam0[t];
        p1 = lam1[t];
      }
      if constexpr (!kBf) {
        for (int e = tid; e < kChunk * kN; e += kThreads) {
          const int t = e >> 6, jj = e & 63;
          sm.Vb[t][jj] = __float2bfloat16_rn(Elt<T>::to_f32(X[3][t][jj]));
          sm.DYb[t][jj] = __float2bfloat16_rn(Elt<T>::to_f32(X[6][t][jj]));
        }
      }
      // this warp's rows of S0 and dS16 in bf16; partial sum_i S0[i][j] dS16[i][j]
      float part[16];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int r = row0 + g + 8 * hh;
          *reinterpret_cast<uint32_t*>(&sm.S0b[r][8 * nt + 2 * c4]) = pack_bf16(S0[nt][2 * hh], S0[nt][2 * hh + 1]);
          *reinterpret_cast<uint32_t*>(&sm.dSb[r][8 * nt + 2 * c4]) = pack_bf16(dS[nt][2 * hh], dS[nt][2 * hh + 1]);
        }
        part[2 * nt] = S0[nt][0] * dS[nt][0] + S0[nt][2] * dS[nt][2];
        part[2 * nt + 1] = S0[nt][1] * dS[nt][1] + S0[nt][3] * dS[nt][3];
      }
      // reduce over the 8 row-lanes (lane bits 2..4); every lane ends with 2 columns
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const bool up = lane & 16;
        const float send = up ? part[k] : part[k + 8];
        const float keepv = up ? part[k + 8] : part[k];
        part[k] = keepv + __shfl_xor_sync(0xffffffffu, send, 16);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const bool up = lane & 8;
        const float send = up ? part[k] : part[k + 4];
        const float keepv = up ? part[k + 4] : part[k];
        part[k] = keepv + __shfl_xor_sync(0xffffffffu, send, 8);
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const bool up = lane & 4;
        const float send = up ? part[k] : part[k + 2];
        const float keepv = up ? part[k + 2] : part[k];
        part[k] = keepv + __shfl_xor_sync(0xffffffffu, send, 4);
      }
      // part[q] (q=0,1) now holds index 8*(lane>>4&1) + 4*(lane>>3&1) + 2*(lane>>2&1) + q = 2*nt + q
      {
        const int idx = 8 * ((lane >> 4) & 1) + 4 * ((lane >> 3) & 1) + 2 * ((lane >> 2) & 1);
        const int nt = idx >> 1;
        sm.dlam[warp][8 * nt + 2 * c4] = part[0];
        sm.dlam[warp][8 * nt + 2 * c4 + 1] = part[1];
      }
    }
    const bool unsafe = __syncthreads_or(bad);   // (1)
    if (unsafe) {
      flagged = true;
      break;
    }

    // prefetch the next (earlier) chunk: inputs, entering state, reset mask
    float S0n[8][4];
    unsigned mask_next = 0u;
    if (c > 0) {
      stage7<T>(p, sm.in[buf ^ 1], b, h, t0 - kChunk, kChunk);
      load_entry_state(p, unit, nc, c - 1, row0, g, c4, S0n);
      if (warp == 0) {
        const bool f = p.reset && lane < kChunk && p.reset[b * p.T + t0 - kChunk + lane] != 0;
        mask_next = __ballot_sync(0xffffffffu, f) & 0xffffu;
      }
    }

    // ---- P2: Gram block of this warp (single bf16), masked
    {
      const int m0 = (warp >> 1) * 16, n0 = (warp & 1) * 16;
      float gr[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a[4], bb[4];
        ldsm_x4(a, a_rowmajor_addr(&sm.GA[0][0], kStr, m0, 16 * ks, lane));
        ldsm_x4(bb, b_nmajor_addr(&sm.GB[0][0], kStr, n0, 16 * ks, lane));
        mma16816(gr[0], a, bb[0], bb[1]);
        mma16816(gr[1], a, bb[2], bb[3]);
      }
      const bool strict = warp < 2;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = g + (e >> 1) * 8;
          const int tau = 8 * nt + 2 * c4 + (e & 1);
          bool ok = strict ? (tau < t) : (tau <= t);
          ok = ok && ((mask & ((2u << t) - (2u << tau))) == 0u);
          const float v = ok ? gr[nt][e] : 0.f;
          if (warp == 0) sm.LabT[tau][t] = v;
          else if (warp == 1) { sm.LakT[tau][t] = v; sm.Lakb[t][tau] = __float2bfloat16_rn(v); }
          else if (warp == 2) sm.Mrbb[t][tau] = __float2bfloat16_rn(v);
          else sm.Mrkb[t][tau] = __float2bfloat16_rn(v);
        }
    }
    __syncthreads();   // (2)

    // ---- P3: T = (I - Lab)^-1, W = T diag(m0) At, X = T Lak by forward substitution (threads 0..95)
    if (tid < 96) {
      float u[kChunk];
      const int cc = tid < 64 ? tid : (tid < 80 ? tid - 64 : tid - 80);
      if (tid < 64) {
#pragma unroll
        for (int t = 0; t < kChunk; ++t) u[t] = t < fr ? __bfloat162float(sm.GA[t][cc]) : 0.f;
      } else if (tid < 80) {
#pragma unroll
        for (int t = 0; t < kChunk; ++t) u[t] = sm.LakT[cc][t];
      } else {
#pragma unroll
        for (int t = 0; t < kChunk; ++t) u[t] = t == cc ? 1.f : 0.f;
      }
#pragma unroll
      for (int tau = 0; tau < kChunk - 1; ++tau) {
        const float4* lrow = reinterpret_cast<const float4*>(&sm.LabT[tau][0]);
        float lv[kChunk];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 f4 = lrow[q];
          lv[4 * q] = f4.x; lv[4 * q + 1] = f4.y; lv[4 * q + 2] = f4.z; lv[4 * q + 3] = f4.w;
        }
#pragma unroll
        for (int t = tau + 1; t < kChunk; ++t) u[t] = fmaf(lv[t], u[tau], u[t]);
      }
      if (tid < 64) {
#pragma unroll
        for (int t = 0; t < kChunk; ++t) sm.Wb[t][cc] = __float2bfloat16_rn(u[t]);
      } else if (tid < 80) {
#pragma unroll
        for (int t = 0; t < kChunk; ++t) sm.Xb[t][cc] = __float2bfloat16_rn(u[t]);
      } else {
#pragma unroll
        for (int t = 0; t < kChunk; ++t) sm.Tb[t][cc] = __float2bfloat16_rn(u[t]);
      }
    }
    __syncthreads();   // (3)

    // ---- P4 (rows i of this warp): SA, dSA, dU, dV
    {
      float sa[2][4] = {}, ds4[4][4] = {};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t as[4], ad[4], bw[4], bb[4], bk[4];
        frag_to_a(S0[2 * ks], S0[2 * ks + 1], as);
        frag_to_a(dS[2 * ks], dS[2 * ks + 1], ad);
        ldsm_x4(bw, b_nmajor_addr(&sm.Wb[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4(bb, b_nmajor_addr(&sm.BK[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4(bk, b_nmajor_addr(&sm.BK[0][0], kStr, 16, 16 * ks, lane));
        mma16816(sa[0], as, bw[0], bw[1]);
        mma16816(sa[1], as, bw[2], bw[3]);
        mma16816(ds4[0], ad, bb[0], bb[1]);
        mma16816(ds4[1], ad, bb[2], bb[3]);
        mma16816(ds4[2], ad, bk[0], bk[1]);
        mma16816(ds4[3], ad, bk[2], bk[3]);
      }
      uint32_t av[4], ay[4], bx[4], bm[4], bk[4];
      ldsm_x4_t(av, a_kmajor_addr(&Vsrc[0][0], kStr, 0, row0, lane));
      ldsm_x4_t(ay, a_kmajor_addr(&DYsrc[0][0], kStr, 0, row0, lane));
      ldsm_x4(bx, b_nmajor_addr(&sm.Xb[0][0], kStrS, 0, 0, lane));
      ldsm_x4_t(bm, b_kmajor_addr(&sm.Mrbb[0][0], kStrS, 0, 0, lane));
      ldsm_x4_t(bk, b_kmajor_addr(&sm.Mrkb[0][0], kStrS, 0, 0, lane));
      mma16816(sa[0], av, bx[0], bx[1]);
      mma16816(sa[1], av, bx[2], bx[3]);
      mma16816(ds4[0], ay, bm[0], bm[1]);
      mma16816(ds4[1], ay, bm[2], bm[3]);
      mma16816(ds4[2], ay, bk[0], bk[1]);
      mma16816(ds4[3], ay, bk[2], bk[3]);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sm.SAb[8 * nt + 2 * c4 + (e & 1)][row0 + g + 8 * (e >> 1)] = __float2bfloat16_rn(sa[nt][e]);
      // dU^T = dSA^T T
      uint32_t adsa[4], bt[4];
      frag_to_a(ds4[0], ds4[1], adsa);
      ldsm_x4_t(bt, b_kmajor_addr(&sm.Tb[0][0], kStrS, 0, 0, lane));
      float du[2][4] = {};
      mma16816(du[0], adsa, bt[0], bt[1]);
      mma16816(du[1], adsa, bt[2], bt[3]);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sm.DUb[8 * nt + 2 * c4 + (e & 1)][row0 + g + 8 * (e >> 1)] = __float2bfloat16_rn(du[nt][e]);
      // dV^T += dU^T Lak
      uint32_t adu[4], bl[4];
      frag_to_a(du[0], du[1], adu);
      ldsm_x4_t(bl, b_kmajor_addr(&sm.Lakb[0][0], kStrS, 0, 0, lane));
      mma16816(ds4[2], adu, bl[0], bl[1]);
      mma16816(ds4[3], adu, bl[2], bl[3]);
      T* dv = static_cast<T*>(p.dv);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tau = 8 * nt + 2 * c4 + (e & 1);
          if (tau < len) dv[tok_off(b, t0 + tau, h, p.T, p.H) + row0 + g + 8 * (e >> 1)] = Elt<T>::from_f32(ds4[2 + nt][e]);
        }
    }
    __syncthreads();   // (4)

    // ---- P5: gradient Gram block; [dRt; dAt] from S0 and [dBb; dKb] from dS16 for this warp's columns
    float xr[2][4] = {}, xa[2][4] = {}, xb[2][4] = {}, xk[2][4] = {};
    {
      const bf16* Asrc = (warp >> 1) ? &sm.DUb[0][0] : &DYsrc[0][0];
      const bf16* Bsrc = (warp & 1) ? &Vsrc[0][0] : &sm.SAb[0][0];
      float gr[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a[4], bb[4];
        ldsm_x4(a, a_rowmajor_addr(Asrc, kStr, 0, 16 * ks, lane));
        ldsm_x4(bb, b_nmajor_addr(Bsrc, kStr, 0, 16 * ks, lane));
        mma16816(gr[0], a, bb[0], bb[1]);
        mma16816(gr[1], a, bb[2], bb[3]);
      }
      const bool strict = (warp >> 1) != 0;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = g + (e >> 1) * 8;
          const int tau = 8 * nt + 2 * c4 + (e & 1);
          bool ok = strict ? (tau < t) : (tau <= t);
          ok = ok && ((mask & ((2u << t) - (2u << tau))) == 0u);
          sm.dG[(warp >> 1) * 16 + t][(warp & 1) * 16 + tau] = __float2bfloat16_rn(ok ? gr[nt][e] : 0.f);
        }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t ay[4], au[4], asa[4], av[4], bs[4], bd[4];
        ldsm_x4(ay, a_rowmajor_addr(&DYsrc[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4(au, a_rowmajor_addr(&sm.DUb[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4(asa, a_rowmajor_addr(&sm.SAb[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4(av, a_rowmajor_addr(&Vsrc[0][0], kStr, 0, 16 * ks, lane));
        ldsm_x4_t(bs, b_kmajor_addr(&sm.S0b[0][0], kStr, 16 * ks, row0, lane));
        ldsm_x4_t(bd, b_kmajor_addr(&sm.dSb[0][0], kStr, 16 * ks, row0, lane));
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          mma16816(xr[nt], ay, bs[2 * nt], bs[2 * nt + 1]);
          mma16816(xa[nt], au, bs[2 * nt], bs[2 * nt + 1]);
          mma16816(xb[nt], asa, bd[2 * nt], bd[2 * nt + 1]);
          mma16816(xk[nt], av, bd[2 * nt], bd[2 * nt + 1]);
        }
      }
    }
    __syncthreads();   // (5)

    // ---- P6 (columns j of this warp): key-space gradients and the per-token outputs
    {
      float dA[2][4] = {}, dR[2][4] = {}, dB[2][4] = {}, dK[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        uint32_t aL[4], aM[4], aLt[4], aLk[4], bg[4], ba[4];
        ldsm_x4(aL, a_rowmajor_addr(&sm.dG[0][0], kStrG, 16, 16 * ks, lane));   // [dLab | dLak]
        ldsm_x4(aM, a_rowmajor_addr(&sm.dG[0][0], kStrG, 0, 16 * ks, lane));    // [dMrb | dMrk]
        ldsm_x4_t(bg, b_kmajor_addr(&sm.GB[0][0], kStr, 16 * ks, row0, lane)); // Bh (ks 0) / Kh (ks 1)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          mma16816(dA[nt], aL, bg[2 * nt], bg[2 * nt + 1]);
          mma16816(dR[nt], aM, bg[2 * nt], bg[2 * nt + 1]);
        }
        // ks 0: dLab^T At / dLak^T At ; ks 1: dMrb^T Rt / dMrk^T Rt
        const int krow = ks == 0 ? 16 : 0;
        ldsm_x4_t(aLt, a_kmajor_addr(&sm.dG[0][0], kStrG, krow, 0, lane));
        ldsm_x4_t(aLk, a_kmajor_addr(&sm.dG[0][0], kStrG, krow, 16, lane));
        ldsm_x4_t(ba, b_kmajor_addr(&sm.GA[0][0], kStr, ks == 0 ? 0 : 16, row0, lane));
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          mma16816(dB[nt], aLt, ba[2 * nt], ba[2 * nt + 1]);
          mma16816(dK[nt], aLk, ba[2 * nt], ba[2 * nt + 1]);
        }
      }
      T* gda = static_cast<T*>(p.da);
      T* gdr = static_cast<T*>(p.dr);
      T* gdb = static_cast<T*>(p.db);
      T* gdk = static_cast<T*>(p.dk);
      float e3p[2][2] = {};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int t = g + 8 * hh;
          const int j = row0 + 8 * nt + 2 * c4;
          const bool m0t = t < fr;
          const bool ls = __popc(mask & ((2u << t) - 2u)) == seg_last;
          float o_da[2], o_dr[2], o_db[2], o_dk[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int e = 2 * hh + q;
            const float Lt = sm.lam[t][j + q];
            const float Lp = t > 0 ? sm.lam[t - 1][j + q] : 1.f;
            const float L15 = sm.lam[kChunk - 1][j + q];
            const float inv = rcp_approx(Lt);
            const float dAt = dA[nt][e] + (m0t ? xa[nt][e] : 0.f);
            const float dRt = dR[nt][e] + (m0t ? xr[nt][e] : 0.f);
            const float dBt = dB[nt][e] + (ls ? L15 * xb[nt][e] : 0.f);
            const float dKt = dK[nt][e] + (ls ? L15 * xk[nt][e] : 0.f);
            o_da[q] = dAt * Lp;
            o_dr[q] = dRt * Lt;
            o_db[q] = dBt * inv;
            o_dk[q] = dKt * inv;
            const float rr = Elt<T>::to_f32(X[0][t][j + q]), aa = Elt<T>::to_f32(X[4][t][j + q]);
            const float bv = Elt<T>::to_f32(X[5][t][j + q]), kv = Elt<T>::to_f32(X[2][t][j + q]);
            sm.E1[t][j + q] = o_dr[q] * rr - o_db[q] * bv - o_dk[q] * kv;
            sm.E2[t][j + q] = o_da[q] * aa;
            if (ls) e3p[nt][q] += (xb[nt][e] * bv + xk[nt][e] * kv) * L15 * inv;
          }
          if (t < len) {
            const int64_t o = tok_off(b, t0 + t, h, p.T, p.H) + j;
            gda[o] = Elt<T>::from_f32(o_da[0]); gda[o + 1] = Elt<T>::from_f32(o_da[1]);
            gdr[o] = Elt<T>::from_f32(o_dr[0]); gdr[o + 1] = Elt<T>::from_f32(o_dr[1]);
            gdb[o] = Elt<T>::from_f32(o_db[0]); gdb[o + 1] = Elt<T>::from_f32(o_db[1]);
            gdk[o] = Elt<T>::from_f32(o_dk[0]); gdk[o + 1] = Elt<T>::from_f32(o_dk[1]);
          }
        }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float v = e3p[nt][q];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          if (g == 0) sm.e3[row0 + 8 * nt + 2 * c4 + q] = v;
        }
    }

    // ---- P7 (rows i of this warp): gradient entering the chunk
    {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dS[nt][e] = keep ? dS[nt][e] * sm.lam[kChunk - 1][8 * nt + 2 * c4 + (e & 1)] : 0.f;
      uint32_t ay[4], au[4];
      ldsm_x4_t(ay, a_kmajor_addr(&DYsrc[0][0], kStr, 0, row0, lane));
      ldsm_x4_t(au, a_kmajor_addr(&sm.DUb[0][0], kStr, 0, row0, lane));
      mask_k(ay, c4, fr);
      mask_k(au, c4, fr);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t br[4], ba[4];
        ldsm_x4_t(br, b_kmajor_addr(&sm.GA[0][0], kStr, 16, 16 * np, lane));
        ldsm_x4_t(ba, b_kmajor_addr(&sm.GA[0][0], kStr, 0, 16 * np, lane));
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          mma16816(dS[2 * np + u], ay, br[2 * u], br[2 * u + 1]);
          mma16816(dS[2 * np + u], au, ba[2 * u], ba[2 * u + 1]);
        }
      }
    }
    __syncthreads();   // (6) E1, E2, e3 complete

    // ---- P8: d log w by a reverse cumulative sum over the chunk, dw = d log w / w
    if (tid < kN) {
      const int j = tid;
      float fin = sm.e3[j];
      if (keep) fin += sm.lam[kChunk - 1][j] * ((sm.dlam[0][j] + sm.dlam[1][j]) + (sm.dlam[2][j] + sm.dlam[3][j]));
      T* gdw = static_cast<T*>(p.dw);
      float cum = 0.f;
#pragma unroll
      for (int t = kChunk - 1; t >= 0; --t) {
        cum += sm.E1[t][j] + (t < kChunk - 1 ? sm.E2[t + 1][j] : fin);
        if (t < len) gdw[tok_off(b, t0 + t, h, p.T, p.H) + j] = Elt<T>::from_f32(cum / Elt<T>::to_f32(X[1][t][j]));
      }
    }
    if (c > 0) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) S0[nt][e] = S0n[nt][e];
      if (tid == 0) sm.mask = int(mask_next);
    }
  }

  cp_async_wait_all();
  if (tid == 0 && p.unit_flags) p.unit_flags[unit] = flagged ? 1 : 0;
  if (!flagged && p.ds0) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        *reinterpret_cast<float2*>(p.ds0 + (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4) =
            make_float2(dS[nt][2 * hh], dS[nt][2 * hh + 1]);
  }
}

template <typename T>
cudaError_t launch(const BwdArgs& p, cudaStream_t stream) {
  const size_t smem = sizeof(CbSmem<T>);
  cudaError_t e = cudaFuncSetAttribute(chunk_bwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  chunk_bwd_kernel<T><<<dim3(unsigned(p.B * p.H)), dim3(kThreads), smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_bwd(const BwdArgs& p, int dtype, cudaStream_t stream) {
  switch (dtype) {
    case 0: return launch<float>(p, stream);
    case 1: return launch<__nv_bfloat16>(p, stream);
    case 2: return launch<__half>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
