// WKV-7 backward in 16-token chunks on tensor cores (algo CHUNKED).
//
// Exact reverse mode of the chunk formulas of the forward (see chunk_fwd.cu):
// inside a chunk with entering state S0, decay products L_t = prod_{s<=t} w_s
// and At = a L_{t-1}, Rt = r L_t, Bh = b / L_t, Kh = k / L_t,
//   SA = m0.At S0^T + Lab SA + Lak V,    Y = m0.Rt S0^T + Mrb SA + Mrk V,
//   S16 = keep.S0 diag(L_15) + (SA^T ls.Bh + V^T ls.Kh) diag(L_15)
// where Lab = At Bh^T, Lak = At Kh^T (strictly lower), Mrb = Rt Bh^T,
// Mrk = Rt Kh^T (lower), all masked to token pairs with no reset between them;
// m0 marks tokens before the chunk's first reset, ls the tokens of its last
// segment, keep = "no reset in the chunk".  Given dY and dS16 (the gradient
// carried from the next chunk), with dSl = dS16 diag(L_15):
//   dSA  = Mrb^T dY + ls.Bh dSl^T,   dU = (I - Lab)^-T dSA,
//   dV   = Mrk^T dY + ls.Kh dSl^T + Lak^T dU,
//   dMrb = dY SA^T, dMrk = dY V^T, dLab = dU SA^T, dLak = dU V^T   (masked),
//   dAt  = dLab Bh + dLak Kh + m0.dU S0,   dRt = dMrb Bh + dMrk Kh + m0.dY S0,
//   dBh  = dLab^T At + dMrb^T Rt + ls.L_15.(SA dS16),
//   dKh  = dLak^T At + dMrk^T Rt + ls.L_15.(V dS16),
//   dS0  = keep.dSl + (m0.dY)^T Rt + (m0.dU)^T At
// and, through the decay, with d log L_t = dr r + da_{t+1} a_{t+1} - db b - dk k
// (plus, at t = 15, keep.L_15 sum_i dS16 o S0 and the last segment's
// dBb o Bb + dKb o Kb), d log w_s = sum_{t >= s} d log L_t and dw = d log w / w.
// The pages print no backward; this is derived from the chunk forward, which
// itself is the recurrence regrouped (RWKV-MLX page, "Key Design Decisions" 2:
// state checkpoints every 16 tokens; rwkv-metal page: the backward recomputes
// each chunk from its checkpoint).
//
// Gradients need cosine >= 0.999, so every product here is a single bf16
// mma.sync (m16n8k16) with fp32 accumulation.  A chunk with a decay outside
// the range the 1/L scaling tolerates (some w < 1/16, or L_15 outside
// [2^-40, 2^40]) makes the CTA stop and mark its unit in `unit_flags`; the
// scan backward then recomputes exactly those units.
//
// Work split (one CTA of 8 warps per (b,h)), chunks in reverse, pipelined:
//   warps 4-7 ("context") for chunk c-1: stage its inputs (one TMA box per
//     input on an mbarrier, bounded waits) and its checkpoint, build the decay-scaled operands, the masked Gram, T,
//     W, X and the recomputed SA = W S0^T + X V into one half of a double
//     buffer;
//   warps 0-3 ("main") for chunk c: warp w owns rows 16w..16w+15 of dS as
//     accumulator fragments (the only quantity carried from chunk to chunk)
//     and columns 16w..16w+15 of the key-space gradients; they run the
//     dS chain, the gradient products and the per-token outputs.
// One CTA barrier per chunk hands the context over.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;
constexpr int kStr = 72;
constexpr int kStrS = 24;
constexpr int kStrG = 40;
constexpr int kIn = 7;   // r, w, k, v, a, b, dy
using bf16 = __nv_bfloat16;

struct __align__(16) BCtx {
  bf16 GA[32][kStr];      // rows 0..15 at, 16..31 rt   [t][j]
  bf16 GB[32][kStr];      // rows 0..15 bh, 16..31 kh   [tau][j]
  bf16 S0b[kN][kStr];     // entering state             [i][j]
  bf16 SAb[kChunk][kStr]; // recomputed SA              [tau][i]
  bf16 Vb[kChunk][kStr];  // v                          [tau][i]
  bf16 DYb[kChunk][kStr]; // dy                         [t][i]
  bf16 Tb[kChunk][kStrS], Mrbb[kChunk][kStrS], Mrkb[kChunk][kStrS], Lakb[kChunk][kStrS];   // [t][tau]
  float lam[kChunk][kN + 4];   // L_t [t][j]
  int mask, unsafe;
  unsigned ls_bits;            // tokens of the chunk's last segment
};

template <typename T>
struct __align__(128) BwdSmem2 {
  BCtx ctx[2];
  __align__(128) T in[kIn][kChunk][kN];   // staged inputs of the chunk being built (TMA boxes)
  __align__(16) float LabT[kChunk][20];
  __align__(16) float LakT[kChunk][20];
  bf16 Wb[kChunk][kStr], Xb[kChunk][kStrS];
  bf16 DUb[kChunk][kStr];     // dU   [tau][i]
  bf16 dSb[kN][kStr];         // dS16 [i][j]
  bf16 dG[32][kStrG];         // [dMrb dMrk; dLab dLak]
  bf16 dVs[kChunk][kStr];     // dv staging [tau][i]
  __align__(16) float DL[kChunk][kN + 4];   // d log L_t without the chunk-end term
  __align__(16) float e3[kN];
  __align__(16) float dlam[4][kN];
  unsigned long long in_bar;   // completion of the bulk copies into `in` (one phase per staged chunk)
  int kbad[4];
  int stop;
};

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void cta_sync() { asm volatile("bar.sync 0;\n" ::: "memory"); }

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void frag_to_a(const float (&lo)[4], const float (&hi)[4], uint32_t (&a)[4]) {
  a[0] = pack_bf16(lo[0], lo[1]);
  a[1] = pack_bf16(lo[2], lo[3]);
  a[2] = pack_bf16(hi[0], hi[1]);
  a[3] = pack_bf16(hi[2], hi[3]);
}

// Keep only the bf16 halves of an m16n8k16 A fragment whose k index is set in `bits`.
__device__ __forceinline__ void mask_k16(uint32_t (&a)[4], int c4, unsigned bits) {
  const int k0 = 2 * c4, k1 = 8 + 2 * c4;
  const uint32_t m0 = ((bits >> k0) & 1u ? 0x0000ffffu : 0u) | ((bits >> (k0 + 1)) & 1u ? 0xffff0000u : 0u);
  const uint32_t m1 = ((bits >> k1) & 1u ? 0x0000ffffu : 0u) | ((bits >> (k1 + 1)) & 1u ? 0xffff0000u : 0u);
  a[0] &= m0;
  a[1] &= m0;
  a[2] &= m1;
  a[3] &= m1;
}

// Stage the seven inputs (r, w, k, v, a, b, dy) of chunk tokens t0..t0+15 into sm.in: one TMA box
// per input, issued by one thread; rows past T arrive as zeros (K1 reads w there as 1).
template <typename T>
__device__ __forceinline__ void stage7(const BwdArgs& p, const InputMaps& tm, BwdSmem2<T>& sm, int64_t b, int64_t h,
                                       int64_t t0, int ktid) {
  if (ktid == 0) {
    mbar_arrive_expect_tx(&sm.in_bar, unsigned(kIn * kChunk * kN * sizeof(T)) + p.extra_tx);
#pragma unroll
    for (int m = 0; m < kIn; ++m) tma_load_4d(&sm.in[m][0][0], &tm.m[m], 0, int(h), int(t0), int(b), &sm.in_bar);
  }
}

// State entering chunk c (checkpoint c-1, s0 or zero) as accumulator fragments: context thread
// (warp kw, lane 4g + c4) holds s[nt] = S[16kw + g][8nt + 2c4 + {0,1}], S[16kw + g + 8][same].
__device__ __forceinline__ void load_entry_rows(const BwdArgs& p, int64_t unit, int64_t nc, int64_t c, int ktid,
                                                float4 (&s)[8]) {
  if (c > 0) {   // tiled checkpoint order: one contiguous 512-byte row of float4 per warp and nt
    const float* src = p.ckpt + (unit * nc + (c - 1)) * kN * kN + (ktid >> 5) * 1024 + (ktid & 31) * 4;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt] = *reinterpret_cast<const float4*>(src + nt * 128);
  } else if (p.s0) {
    const int lane = ktid & 31;
    const float* src = p.s0 + unit * kN * kN + (16 * (ktid >> 5) + (lane >> 2)) * kN + 2 * (lane & 3);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float2 lo = *reinterpret_cast<const float2*>(src + 8 * nt);
      const float2 hi = *reinterpret_cast<const float2*>(src + 8 * kN + 8 * nt);
      s[nt] = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
  } else {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Reset flag of token 16c + lane of batch row b (false past T, for c < 0 or without flags).
__device__ __forceinline__ bool reset_flag(const BwdArgs& p, int64_t b, int64_t c, int lane) {
  const int64_t t = c * kChunk + lane;
  return p.reset && c >= 0 && lane < kChunk && t < p.T && p.reset[b * p.T + t] != 0;
}

// ------------------------------------------------------------------ context warps
// A wait for staged inputs that runs out marks the chunk unsafe (the unit is then recomputed by the
// exact scan, which reads global memory) and sets `timed_out`, after which nothing more is staged.
template <typename T>
__device__ __forceinline__ void build_context(const BwdArgs& p, BwdSmem2<T>& sm, BCtx& cx, unsigned mask,
                                              const float4 (&s0rows)[8], int ktid, int len, unsigned parity,
                                              bool& unsafe, bool& timed_out) {
  const int kw = ktid >> 5, lane = ktid & 31;
  const bool to = !mbar_wait_bounded(&sm.in_bar, parity, kWaitLimitNs);
  const T (*X)[kChunk][kN] = sm.in;

  // ---- K1: decay products, scaled operands, v/dy copies, entering state in bf16.
  // Thread = (column pair 2jp, 2jp+1; token quarter kw), two columns per packed fp32 op.
  bool bad = false;
  {
    const int j = 2 * lane, t0 = 4 * kw;
    // L_{t0-1}: product of the earlier quarters' decays (warp-uniform trip count)
    float2 lam = make_float2(1.f, 1.f);
    auto ldw = [&](int t) { return t < len ? load2(&X[1][t][j]) : make_float2(1.f, 1.f); };   // padding: w = 1
    for (int t = 0; t < t0; ++t) lam = mul2(lam, ldw(t));
    float2 wmin = make_float2(1.f, 1.f), lmin = make_float2(1.f, 1.f), lmax = lmin;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = t0 + u;
      const float2 lp = lam, w2 = ldw(t);
      lam = mul2(lam, w2);
      wmin = make_float2(fminf(wmin.x, w2.x), fminf(wmin.y, w2.y));
      lmin = make_float2(fminf(lmin.x, lam.x), fminf(lmin.y, lam.y));
      lmax = make_float2(fmaxf(lmax.x, lam.x), fmaxf(lmax.y, lam.y));
      const float2 inv = make_float2(rcp_approx(lam.x), rcp_approx(lam.y));
      const float2 at = mul2(load2(&X[4][t][j]), lp), rt = mul2(load2(&X[0][t][j]), lam);
      const float2 bh = mul2(load2(&X[5][t][j]), inv), kh = mul2(load2(&X[2][t][j]), inv);
      *reinterpret_cast<float2*>(&cx.lam[t][j]) = lam;
      *reinterpret_cast<uint32_t*>(&cx.GA[t][j]) = pack_bf16(at.x, at.y);
      *reinterpret_cast<uint32_t*>(&cx.GA[16 + t][j]) = pack_bf16(rt.x, rt.y);
      *reinterpret_cast<uint32_t*>(&cx.GB[t][j]) = pack_bf16(bh.x, bh.y);
      *reinterpret_cast<uint32_t*>(&cx.GB[16 + t][j]) = pack_bf16(kh.x, kh.y);
      if constexpr (std::is_same<T, bf16>::value) {
        *reinterpret_cast<uint32_t*>(&cx.Vb[t][j]) = *reinterpret_cast<const uint32_t*>(&X[3][t][j]);
        *reinterpret_cast<uint32_t*>(&cx.DYb[t][j]) = *reinterpret_cast<const uint32_t*>(&X[6][t][j]);
      } else {
        const float2 v2 = load2(&X[3][t][j]), d2 = load2(&X[6][t][j]);
        *reinterpret_cast<uint32_t*>(&cx.Vb[t][j]) = pack_bf16(v2.x, v2.y);
        *reinterpret_cast<uint32_t*>(&cx.DYb[t][j]) = pack_bf16(d2.x, d2.y);
      }
    }
    // every L_t of the chunk lies in exactly one quarter, so the CTA-wide ballot sees all of them
    bad = !(fminf(wmin.x, wmin.y) >= 0.0625f && fminf(lmin.x, lmin.y) >= 0x1p-40f && fmaxf(lmax.x, lmax.y) <= 0x1p40f);
    const int row = 16 * kw + (lane >> 2), col = 2 * (lane & 3);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      *reinterpret_cast<uint32_t*>(&cx.S0b[row][8 * nt + col]) = pack_bf16(s0rows[nt].x, s0rows[nt].y);
      *reinterpret_cast<uint32_t*>(&cx.S0b[row + 8][8 * nt + col]) = pack_bf16(s0rows[nt].z, s0rows[nt].w);
    }
  }
  const unsigned any_bad = __ballot_sync(0xffffffffu, bad), any_to = __ballot_sync(0xffffffffu, to);
  if (lane == 0) sm.kbad[kw] = (any_bad ? 1 : 0) | (any_to ? 2 : 0);
  named_bar(1, 128);
  const int kb = sm.kbad[0] | sm.kbad[1] | sm.kbad[2] | sm.kbad[3];
  unsafe = kb != 0;
  timed_out = (kb & 2) != 0;
  if (timed_out && ktid == 0 && p.status) atomicOr(p.status, kStatusWaitTimeout);
  if (ktid == 0) {
    cx.mask = int(mask);
    cx.unsafe = unsafe ? 1 : 0;
    cx.ls_bits = last_segment_bits(mask);
  }
}

template <typename T>
__device__ __forceinline__ void finish_context(BwdSmem2<T>& sm, BCtx& cx, unsigned mask, int ktid) {
  const int kw = ktid >> 5, lane = ktid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;

  // ---- K2: Gram block of this warp (single bf16), masked
  {
    const int m0 = (kw >> 1) * 16, n0 = (kw & 1) * 16;
    float gr[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t a[4], bb[4];
      ldsm_x4(a, a_rowmajor_addr(&cx.GA[0][0], kStr, m0, 16 * ks, lane));
      ldsm_x4(bb, b_nmajor_addr(&cx.GB[0][0], kStr, n0, 16 * ks, lane));
      mma16816(gr[0], a, bb[0], bb[1]);
      mma16816(gr[1], a, bb[2], bb[3]);
    }
    const bool strict = kw < 2;
    const int st0 = seg_of(mask, g), st1 = seg_of(mask, g + 8);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = g + (e >> 1) * 8;
        const int tau = 8 * nt + 2 * c4 + (e & 1);
        const bool ok = (strict ? (tau < t) : (tau <= t)) && seg_of(mask, tau) == ((e >> 1) ? st1 : st0);
        const float v = ok ? gr[nt][e] : 0.f;
        if (kw == 0) sm.LabT[tau][t] = v;
        else if (kw == 1) { sm.LakT[tau][t] = v; cx.Lakb[t][tau] = __float2bfloat16_rn(v); }
        else if (kw == 2) cx.Mrbb[t][tau] = __float2bfloat16_rn(v);
        else cx.Mrkb[t][tau] = __float2bfloat16_rn(v);
      }
  }
  named_bar(1, 128);

  // ---- K3: T = (I - Lab)^-1, W = T diag(m0) At, X = T Lak by forward substitution (threads 0..95)
  if (ktid < 96) {
    float u[kChunk];
    const int cc = ktid < 64 ? ktid : (ktid < 80 ? ktid - 64 : ktid - 80);
    if (ktid < 64) {
#pragma unroll
      for (int t = 0; t < kChunk; ++t) u[t] = t < fr ? __bfloat162float(cx.GA[t][cc]) : 0.f;
    } else if (ktid < 80) {
      const float4* col = reinterpret_cast<const float4*>(&sm.LakT[cc][0]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 f = col[q];
        u[4 * q] = f.x; u[4 * q + 1] = f.y; u[4 * q + 2] = f.z; u[4 * q + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int t = 0; t < kChunk; ++t) u[t] = t == cc ? 1.f : 0.f;
    }
    // rows of Lab^T are loaded one step ahead, so each step waits only on its FMAs
    float4 nxt[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) nxt[q] = reinterpret_cast<const float4*>(&sm.LabT[0][0])[q];
#pragma unroll
    for (int tau = 0; tau < kChunk - 1; ++tau) {
      const float4 cur[4] = {nxt[0], nxt[1], nxt[2], nxt[3]};
      if (tau + 1 < kChunk - 1) {
#pragma unroll
        for (int q = (tau + 2) / 4; q < 4; ++q) nxt[q] = reinterpret_cast<const float4*>(&sm.LabT[tau + 1][0])[q];
      }
      const float lv[kChunk] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y, cur[1].z, cur[1].w,
                                cur[2].x, cur[2].y, cur[2].z, cur[2].w, cur[3].x, cur[3].y, cur[3].z, cur[3].w};
#pragma unroll
      for (int t = tau + 1; t < kChunk; ++t) u[t] = fmaf(lv[t], u[tau], u[t]);
    }
    if (ktid < 64) {
#pragma unroll
      for (int t = 0; t < kChunk; ++t) sm.Wb[t][cc] = __float2bfloat16_rn(u[t]);
    } else if (ktid < 80) {
#pragma unroll
      for (int t = 0; t < kChunk; ++t) sm.Xb[t][cc] = __float2bfloat16_rn(u[t]);
    } else {
#pragma unroll
      for (int t = 0; t < kChunk; ++t) cx.Tb[t][cc] = __float2bfloat16_rn(u[t]);
    }
  }
  named_bar(1, 128);

  // ---- K4: SA = W S0^T + X V for rows i = 16kw..16kw+15, stored [tau][i]
  {
    const int i0 = 16 * kw;
    float sa[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t a[4], bs[4];
      ldsm_x4(a, a_rowmajor_addr(&sm.Wb[0][0], kStr, 0, 16 * ks, lane));
      ldsm_x4(bs, b_nmajor_addr(&cx.S0b[0][0], kStr, i0, 16 * ks, lane));
      mma16816(sa[0], a, bs[0], bs[1]);
      mma16816(sa[1], a, bs[2], bs[3]);
    }
    uint32_t ax[4], bv[4];
    ldsm_x4(ax, a_rowmajor_addr(&sm.Xb[0][0], kStrS, 0, 0, lane));
    ldsm_x4_t(bv, b_kmajor_addr(&cx.Vb[0][0], kStr, 0, i0, lane));
    mma16816(sa[0], ax, bv[0], bv[1]);
    mma16816(sa[1], ax, bv[2], bv[3]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        *reinterpret_cast<uint32_t*>(&cx.SAb[g + 8 * hh][i0 + 8 * nt + 2 * c4]) =
            pack_bf16(sa[nt][2 * hh], sa[nt][2 * hh + 1]);
  }
}

// ------------------------------------------------------------------ main warps
template <typename T>
__device__ __forceinline__ void main_chunk(const BwdArgs& p, BwdSmem2<T>& sm, const BCtx& cx, float (&dS)[8][4],
                                           int64_t b, int64_t h, int64_t t0, int len, int warp, int lane) {
  const int tid = threadIdx.x;
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp, j0 = 16 * warp;
  const unsigned mask = unsigned(cx.mask);
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
  const unsigned m0bits = (1u << fr) - 1u;
  const bool keep = mask == 0u;
  const unsigned ls_bits = cx.ls_bits;
  // staging of da, dr, db, dk [q][t][j] in bf16; reuses dSb, which is dead after M8
  bf16 (*gst)[kChunk][kStr] = reinterpret_cast<bf16 (*)[kChunk][kStr]>(&sm.dSb[0][0]);

  // ---- M1: [dSA^T | dV^T] = dSl [ls.Bh | ls.Kh]^T + dY^T [Mrb | Mrk]   (rows i of this warp)
  float acc4[4][4] = {};
  {
    const bool ls_lo = (ls_bits >> g) & 1u, ls_hi = (ls_bits >> (8 + g)) & 1u;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const float2 la = *reinterpret_cast<const float2*>(&cx.lam[kChunk - 1][16 * ks + 2 * c4]);
      const float2 lb = *reinterpret_cast<const float2*>(&cx.lam[kChunk - 1][16 * ks + 8 + 2 * c4]);
      const float2 p0 = mul2(make_float2(dS[2 * ks][0], dS[2 * ks][1]), la);
      const float2 p1 = mul2(make_float2(dS[2 * ks][2], dS[2 * ks][3]), la);
      const float2 p2 = mul2(make_float2(dS[2 * ks + 1][0], dS[2 * ks + 1][1]), lb);
      const float2 p3 = mul2(make_float2(dS[2 * ks + 1][2], dS[2 * ks + 1][3]), lb);
      uint32_t a[4] = {pack_bf16(p0.x, p0.y), pack_bf16(p1.x, p1.y), pack_bf16(p2.x, p2.y), pack_bf16(p3.x, p3.y)};
      uint32_t bb[4], bk[4];
      ldsm_x4(bb, b_nmajor_addr(&cx.GB[0][0], kStr, 0, 16 * ks, lane));
      ldsm_x4(bk, b_nmajor_addr(&cx.GB[0][0], kStr, 16, 16 * ks, lane));
      if (!ls_lo) { bb[0] = 0u; bb[1] = 0u; bk[0] = 0u; bk[1] = 0u; }
      if (!ls_hi) { bb[2] = 0u; bb[3] = 0u; bk[2] = 0u; bk[3] = 0u; }
      mma16816(acc4[0], a, bb[0], bb[1]);
      mma16816(acc4[1], a, bb[2], bb[3]);
      mma16816(acc4[2], a, bk[0], bk[1]);
      mma16816(acc4[3], a, bk[2], bk[3]);
    }
    uint32_t ay[4], bm[4], bk[4];
    ldsm_x4_t(ay, a_kmajor_addr(&cx.DYb[0][0], kStr, 0, row0, lane));
    ldsm_x4_t(bm, b_kmajor_addr(&cx.Mrbb[0][0], kStrS, 0, 0, lane));
    ldsm_x4_t(bk, b_kmajor_addr(&cx.Mrkb[0][0], kStrS, 0, 0, lane));
    mma16816(acc4[0], ay, bm[0], bm[1]);
    mma16816(acc4[1], ay, bm[2], bm[3]);
    mma16816(acc4[2], ay, bk[0], bk[1]);
    mma16816(acc4[3], ay, bk[2], bk[3]);
  }
  // ---- M2: dU^T = dSA^T T ; M3: dV^T += dU^T Lak
  {
    uint32_t adsa[4], bt[4];
    frag_to_a(acc4[0], acc4[1], adsa);
    ldsm_x4_t(bt, b_kmajor_addr(&cx.Tb[0][0], kStrS, 0, 0, lane));
    float du[2][4] = {};
    mma16816(du[0], adsa, bt[0], bt[1]);
    mma16816(du[1], adsa, bt[2], bt[3]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sm.DUb[8 * nt + 2 * c4 + (e & 1)][row0 + g + 8 * (e >> 1)] = __float2bfloat16_rn(du[nt][e]);
    uint32_t adu[4], bl[4];
    frag_to_a(du[0], du[1], adu);
    ldsm_x4_t(bl, b_kmajor_addr(&cx.Lakb[0][0], kStrS, 0, 0, lane));
    mma16816(acc4[2], adu, bl[0], bl[1]);
    mma16816(acc4[3], adu, bl[2], bl[3]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sm.dVs[8 * nt + 2 * c4 + (e & 1)][row0 + g + 8 * (e >> 1)] = __float2bfloat16_rn(acc4[2 + nt][e]);
  }
  // ---- M4: dS16 in bf16 for the column products; partial sum_i S0 o dS16 over this warp's rows
  {
    float part[16];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int col = 8 * nt + 2 * c4;
      float2 s_lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cx.S0b[row0 + g][col]));
      float2 s_hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cx.S0b[row0 + g + 8][col]));
      const float2 pr = fma2(s_lo, make_float2(dS[nt][0], dS[nt][1]), mul2(s_hi, make_float2(dS[nt][2], dS[nt][3])));
      part[2 * nt] = pr.x;
      part[2 * nt + 1] = pr.y;
      *reinterpret_cast<uint32_t*>(&sm.dSb[row0 + g][col]) = pack_bf16(dS[nt][0], dS[nt][1]);
      *reinterpret_cast<uint32_t*>(&sm.dSb[row0 + g + 8][col]) = pack_bf16(dS[nt][2], dS[nt][3]);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool up = lane & 16;
      const float send = up ? part[k] : part[k + 8];
      const float kv = up ? part[k + 8] : part[k];
      part[k] = kv + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool up = lane & 8;
      const float send = up ? part[k] : part[k + 4];
      const float kv = up ? part[k + 4] : part[k];
      part[k] = kv + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const bool up = lane & 4;
      const float send = up ? part[k] : part[k + 2];
      const float kv = up ? part[k + 2] : part[k];
      part[k] = kv + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    const int idx = 8 * ((lane >> 4) & 1) + 4 * ((lane >> 3) & 1) + 2 * ((lane >> 2) & 1);
    sm.dlam[warp][8 * (idx >> 1) + 2 * c4] = part[0];
    sm.dlam[warp][8 * (idx >> 1) + 2 * c4 + 1] = part[1];
  }
  named_bar(2, 128);   // DUb, dVs, dSb, dlam complete

  // ---- M5: gradient entering the chunk: keep.dSl + (m0.dY)^T Rt + (m0.dU)^T At
  {
    if (keep) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float2 l = *reinterpret_cast<const float2*>(&cx.lam[kChunk - 1][8 * nt + 2 * c4]);
        const float2 u0 = mul2(make_float2(dS[nt][0], dS[nt][1]), l);
        const float2 u1 = mul2(make_float2(dS[nt][2], dS[nt][3]), l);
        dS[nt][0] = u0.x; dS[nt][1] = u0.y; dS[nt][2] = u1.x; dS[nt][3] = u1.y;
      }
    } else {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) dS[nt][0] = dS[nt][1] = dS[nt][2] = dS[nt][3] = 0.f;
    }
    uint32_t ay[4], au[4];
    ldsm_x4_t(ay, a_kmajor_addr(&cx.DYb[0][0], kStr, 0, row0, lane));
    ldsm_x4_t(au, a_kmajor_addr(&sm.DUb[0][0], kStr, 0, row0, lane));
    mask_k16(ay, c4, m0bits);
    mask_k16(au, c4, m0bits);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t br[4], ba[4];
      ldsm_x4_t(br, b_kmajor_addr(&cx.GA[0][0], kStr, 16, 16 * np, lane));
      ldsm_x4_t(ba, b_kmajor_addr(&cx.GA[0][0], kStr, 0, 16 * np, lane));
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        mma16816(dS[2 * np + u], ay, br[2 * u], br[2 * u + 1]);
        mma16816(dS[2 * np + u], au, ba[2 * u], ba[2 * u + 1]);
      }
    }
  }
  // ---- dv out (coalesced from the staging tile)
  {
    T* dv = static_cast<T*>(p.dv);
    const int tt = tid >> 3, part = tid & 7;
    if (tt < len) {
      alignas(16) T vals[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) vals[u] = Elt<T>::from_f32(__bfloat162float(sm.dVs[tt][part * 8 + u]));
      uint4* dst = reinterpret_cast<uint4*>(dv + tok_off(b, t0 + tt, h, p.T, p.H) + part * 8);
      const uint4* sv = reinterpret_cast<const uint4*>(vals);
#pragma unroll
      for (int u = 0; u < int(sizeof(vals) / 16); ++u) dst[u] = sv[u];
    }
  }
  // ---- M7: gradient Gram block (warp = block): [dMrb dMrk; dLab dLak], masked
  {
    const bf16* Asrc = (warp >> 1) ? &sm.DUb[0][0] : &cx.DYb[0][0];
    const bf16* Bsrc = (warp & 1) ? &cx.Vb[0][0] : &cx.SAb[0][0];
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
    const int st0 = seg_of(mask, g), st1 = seg_of(mask, g + 8);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = g + (e >> 1) * 8;
        const int tau = 8 * nt + 2 * c4 + (e & 1);
        const bool ok = (strict ? (tau < t) : (tau <= t)) && seg_of(mask, tau) == ((e >> 1) ? st1 : st0);
        sm.dG[(warp >> 1) * 16 + t][(warp & 1) * 16 + tau] = __float2bfloat16_rn(ok ? gr[nt][e] : 0.f);
      }
  }
  // ---- M8: [dRt; dAt] from S0 and [dBb; dKb] from dS16, columns j0..j0+15
  float xr[2][4] = {}, xa[2][4] = {}, xb[2][4] = {}, xk[2][4] = {};
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    uint32_t ay[4], au[4], asa[4], av[4], bs[4], bd[4];
    ldsm_x4(ay, a_rowmajor_addr(&cx.DYb[0][0], kStr, 0, 16 * ks, lane));
    ldsm_x4(au, a_rowmajor_addr(&sm.DUb[0][0], kStr, 0, 16 * ks, lane));
    ldsm_x4(asa, a_rowmajor_addr(&cx.SAb[0][0], kStr, 0, 16 * ks, lane));
    ldsm_x4(av, a_rowmajor_addr(&cx.Vb[0][0], kStr, 0, 16 * ks, lane));
    ldsm_x4_t(bs, b_kmajor_addr(&cx.S0b[0][0], kStr, 16 * ks, j0, lane));
    ldsm_x4_t(bd, b_kmajor_addr(&sm.dSb[0][0], kStr, 16 * ks, j0, lane));
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      mma16816(xr[nt], ay, bs[2 * nt], bs[2 * nt + 1]);
      mma16816(xa[nt], au, bs[2 * nt], bs[2 * nt + 1]);
      mma16816(xb[nt], asa, bd[2 * nt], bd[2 * nt + 1]);
      mma16816(xk[nt], av, bd[2 * nt], bd[2 * nt + 1]);
    }
  }
  named_bar(2, 128);   // dG complete

  // ---- M9/M10: key-space gradients of columns j0..j0+15 and the per-token outputs
  {
    float dA[2][4] = {}, dR[2][4] = {}, dB[2][4] = {}, dK[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t aL[4], aM[4], aLt[4], aLk[4], bg[4], ba[4];
      ldsm_x4(aL, a_rowmajor_addr(&sm.dG[0][0], kStrG, 16, 16 * ks, lane));
      ldsm_x4(aM, a_rowmajor_addr(&sm.dG[0][0], kStrG, 0, 16 * ks, lane));
      ldsm_x4_t(bg, b_kmajor_addr(&cx.GB[0][0], kStr, 16 * ks, j0, lane));
      const int krow = ks == 0 ? 16 : 0;
      ldsm_x4_t(aLt, a_kmajor_addr(&sm.dG[0][0], kStrG, krow, 0, lane));
      ldsm_x4_t(aLk, a_kmajor_addr(&sm.dG[0][0], kStrG, krow, 16, lane));
      ldsm_x4_t(ba, b_kmajor_addr(&cx.GA[0][0], kStr, ks == 0 ? 0 : 16, j0, lane));
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        mma16816(dA[nt], aL, bg[2 * nt], bg[2 * nt + 1]);
        mma16816(dR[nt], aM, bg[2 * nt], bg[2 * nt + 1]);
        mma16816(dB[nt], aLt, ba[2 * nt], ba[2 * nt + 1]);
        mma16816(dK[nt], aLk, ba[2 * nt], ba[2 * nt + 1]);
      }
    }
    T* gda = static_cast<T*>(p.da);
    T* gdr = static_cast<T*>(p.dr);
    T* gdb = static_cast<T*>(p.db);
    T* gdk = static_cast<T*>(p.dk);
    float2 e2v[2][2];   // [nt][hh], columns j, j+1
    float2 e1v[2][2];
    float2 e3p[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    const float2 zero2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int t = g + 8 * hh;
      const bool m0t = t < fr;
      const bool ls = (ls_bits >> t) & 1u;
      const int64_t orow = tok_off(b, t0 + t, h, p.T, p.H);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int j = j0 + 8 * nt + 2 * c4;
        const int e = 2 * hh;
        const float2 Lt = *reinterpret_cast<const float2*>(&cx.lam[t][j]);
        const float2 Lp = t > 0 ? *reinterpret_cast<const float2*>(&cx.lam[t - 1][j]) : make_float2(1.f, 1.f);
        const float2 L15 = *reinterpret_cast<const float2*>(&cx.lam[kChunk - 1][j]);
        const float2 at = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cx.GA[t][j]));
        const float2 rt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cx.GA[16 + t][j]));
        const float2 bh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cx.GB[t][j]));
        const float2 kh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cx.GB[16 + t][j]));
        const float2 xb2 = ls ? make_float2(xb[nt][e], xb[nt][e + 1]) : zero2;
        const float2 xk2 = ls ? make_float2(xk[nt][e], xk[nt][e + 1]) : zero2;
        const float2 dAt = add2(make_float2(dA[nt][e], dA[nt][e + 1]), m0t ? make_float2(xa[nt][e], xa[nt][e + 1]) : zero2);
        const float2 dRt = add2(make_float2(dR[nt][e], dR[nt][e + 1]), m0t ? make_float2(xr[nt][e], xr[nt][e + 1]) : zero2);
        const float2 dBt = fma2(L15, xb2, make_float2(dB[nt][e], dB[nt][e + 1]));
        const float2 dKt = fma2(L15, xk2, make_float2(dK[nt][e], dK[nt][e + 1]));
        const float2 inv = make_float2(rcp_approx(Lt.x), rcp_approx(Lt.y));
        e1v[nt][hh] = sub2(mul2(dRt, rt), fma2(dBt, bh, mul2(dKt, kh)));
        e2v[nt][hh] = mul2(dAt, at);
        e3p[nt] = fma2(fma2(xb2, bh, mul2(xk2, kh)), L15, e3p[nt]);
        if constexpr (std::is_same<T, bf16>::value) {   // staged, written coalesced after the barrier
          store2(&gst[0][t][j], mul2(dAt, Lp));
          store2(&gst[1][t][j], mul2(dRt, Lt));
          store2(&gst[2][t][j], mul2(dBt, inv));
          store2(&gst[3][t][j], mul2(dKt, inv));
        } else if (t < len) {
          store2(gda + orow + j, mul2(dAt, Lp));
          store2(gdr + orow + j, mul2(dRt, Lt));
          store2(gdb + orow + j, mul2(dBt, inv));
          store2(gdk + orow + j, mul2(dKt, inv));
        }
      }
    }
    // d log L_t = E1_t + E2_{t+1}: E2 of row t+1 lives in lane+4 (same half) or, for row 7, in lane c4 (upper half)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float2 dn0, up0, dn1;
      dn0.x = __shfl_down_sync(0xffffffffu, e2v[nt][0].x, 4);
      dn0.y = __shfl_down_sync(0xffffffffu, e2v[nt][0].y, 4);
      up0.x = __shfl_sync(0xffffffffu, e2v[nt][1].x, c4);
      up0.y = __shfl_sync(0xffffffffu, e2v[nt][1].y, c4);
      dn1.x = __shfl_down_sync(0xffffffffu, e2v[nt][1].x, 4);
      dn1.y = __shfl_down_sync(0xffffffffu, e2v[nt][1].y, 4);
      const int j = j0 + 8 * nt + 2 * c4;
      *reinterpret_cast<float2*>(&sm.DL[g][j]) = add2(e1v[nt][0], g < 7 ? dn0 : up0);
      *reinterpret_cast<float2*>(&sm.DL[g + 8][j]) = add2(e1v[nt][1], g < 7 ? dn1 : make_float2(0.f, 0.f));
      float2 v = e3p[nt];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
        v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
      }
      if (g == 0) *reinterpret_cast<float2*>(&sm.e3[j]) = v;
    }
  }
  named_bar(2, 128);   // DL, e3, staged gradients complete

  if constexpr (std::is_same<T, bf16>::value) {
    T* const outs[4] = {static_cast<T*>(p.da), static_cast<T*>(p.dr), static_cast<T*>(p.db), static_cast<T*>(p.dk)};
    const int tt = tid >> 3, part = tid & 7;
    if (tt < len) {
      const int64_t o = tok_off(b, t0 + tt, h, p.T, p.H) + part * 8;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(outs[q] + o) = *reinterpret_cast<const uint4*>(&gst[q][tt][part * 8]);
    }
  }

  // ---- M11: dw = (reverse cumulative sum of d log L) / w.  Thread = (column pair, token quarter
  // q = warp): each thread first adds the rows of the later quarters itself, then walks its four.
  {
    const int j = 2 * lane, q = warp, thi = 4 * q + 3;
    float2 cum = *reinterpret_cast<const float2*>(&sm.e3[j]);
    if (keep) {
      const float2 d01 = add2(*reinterpret_cast<const float2*>(&sm.dlam[0][j]), *reinterpret_cast<const float2*>(&sm.dlam[1][j]));
      const float2 d23 = add2(*reinterpret_cast<const float2*>(&sm.dlam[2][j]), *reinterpret_cast<const float2*>(&sm.dlam[3][j]));
      cum = fma2(*reinterpret_cast<const float2*>(&cx.lam[kChunk - 1][j]), add2(d01, d23), cum);
    }
    for (int t = kChunk - 1; t > thi; --t) cum = add2(cum, *reinterpret_cast<const float2*>(&sm.DL[t][j]));
    T* gdw = static_cast<T*>(p.dw) + tok_off(b, t0, h, p.T, p.H) + j;
    const int64_t rs = p.H * kN;
    float2 Lt = *reinterpret_cast<const float2*>(&cx.lam[thi][j]);
#pragma unroll
    for (int u = 3; u >= 0; --u) {
      const int t = 4 * q + u;
      cum = add2(cum, *reinterpret_cast<const float2*>(&sm.DL[t][j]));
      const float2 Lp = t > 0 ? *reinterpret_cast<const float2*>(&cx.lam[t - 1][j]) : make_float2(1.f, 1.f);
      if (t < len) store2(gdw + t * rs, mul2(cum, mul2(Lp, make_float2(rcp_approx(Lt.x), rcp_approx(Lt.y)))));
      Lt = Lp;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) chunk_bwd_kernel(const BwdArgs p, const __grid_constant__ InputMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  BwdSmem2<T>& sm = *reinterpret_cast<BwdSmem2<T>*>(smem_raw);

  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_main = warp < 4;
  const int ktid = tid - 128;
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;

  if (tid == 0) sm.stop = 0;

  // The two roles run separate loops so that their register sets never overlap; both meet
  // at one CTA barrier per iteration (bar.sync 0, executed by all 256 threads).
  if (is_main) {
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
    cta_sync();   // prologue staged by the context warps
    bool flagged = false;
    for (int64_t it = 0; it <= nc; ++it) {
      if (it >= 1) {
        const int64_t c = nc - it;   // chunk whose gradients are computed now
        const BCtx& cx = sm.ctx[c & 1];
        if (cx.unsafe) {
          if (tid == 0) sm.stop = 1;
        } else {
          const int64_t t0 = c * kChunk;
          main_chunk<T>(p, sm, cx, dS, b, h, t0, int(min64(kChunk, p.T - t0)), warp, lane);
        }
      }
      cta_sync();
      if (sm.stop) {
        flagged = true;
        break;
      }
    }
    if (tid == 0 && p.unit_flags) p.unit_flags[unit] = flagged ? 1 : 0;
    if (!flagged && p.ds0) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<float2*>(p.ds0 + (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4) =
              make_float2(dS[nt][2 * hh], dS[nt][2 * hh + 1]);
    }
  } else {
    // prologue: stage the last chunk, its entering state and reset flags
    float4 s0rows[8];
    unsigned mask_next;
    unsigned phase = 0;        // barrier phase of the next staging to wait for
    bool pending = true;       // a staging was issued and not yet waited for
    bool timed_out = false;
    {
      if (ktid == 0) mbar_init(&sm.in_bar, 1);
      named_bar(1, 128);
      const int64_t c = nc - 1;
      const int64_t t0 = c * kChunk;
      stage7<T>(p, tm, sm, b, h, t0, ktid);
      load_entry_rows(p, unit, nc, c, ktid, s0rows);
      mask_next = __ballot_sync(0xffffffffu, reset_flag(p, b, c, lane)) & 0xffffu;
    }
    // the flag of the chunk staged next is loaded one iteration before its ballot, off the critical path
    bool f_prev = reset_flag(p, b, nc - 2, lane);
    cta_sync();
    for (int64_t it = 0; it <= nc; ++it) {
      const int64_t c = nc - 1 - it;   // chunk whose context is built now
      if (c >= 0 && pending && !timed_out) {   // (an unsafe chunk stages nothing more: the unit stops)
        BCtx& cx = sm.ctx[c & 1];
        const unsigned mask = mask_next;
        bool unsafe = false;
        build_context<T>(p, sm, cx, mask, s0rows, ktid, int(min64(kChunk, p.T - c * kChunk)), phase & 1u, unsafe,
                         timed_out);
        if (!timed_out) {
          pending = false;
          ++phase;
        }
        // the staged inputs and entering state are consumed: prefetch the previous chunk
        if (c > 0 && !unsafe) {
          const int64_t tp = (c - 1) * kChunk;
          stage7<T>(p, tm, sm, b, h, tp, ktid);
          pending = true;
          load_entry_rows(p, unit, nc, c - 1, ktid, s0rows);
          mask_next = __ballot_sync(0xffffffffu, f_prev) & 0xffffu;   // chunk c-1
          f_prev = reset_flag(p, b, c - 2, lane);
        }
        if (!unsafe) finish_context<T>(sm, cx, mask, ktid);
      }
      cta_sync();
      if (sm.stop) break;
    }
    // copies issued but never waited for (the unit stopped early) must land before the CTA exits
    if (pending) mbar_wait_bounded(&sm.in_bar, phase & 1u, timed_out ? kWaitLimitNs / 100 : kWaitLimitNs);
  }
}

template <typename T>
cudaError_t launch(const BwdArgs& p, const InputMaps& tm, cudaStream_t stream) {
  const size_t smem = sizeof(BwdSmem2<T>);
  cudaError_t e = cudaFuncSetAttribute(chunk_bwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  chunk_bwd_kernel<T><<<dim3(unsigned(p.B * p.H)), dim3(kThreads), smem, stream>>>(p, tm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_bwd(const BwdArgs& p, const InputMaps& tm, int dtype, cudaStream_t stream) {
  switch (dtype) {
    case 0: return launch<float>(p, tm, stream);
    case 1: return launch<__nv_bfloat16>(p, tm, stream);
    case 2: return launch<__half>(p, tm, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
