// WKV-7 forward in 16-token chunks with the intra-chunk products on tensor
// cores (algo CHUNKED) -- the chunk-parallel form that the HF model card page
// mentions, derived here from the recurrence.
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
// lower triangular, by substitution -- the triangular solve the rwkv-lab page
// names for chunked delta rules) and M = Mrb T:
//   SA = W S0^T + X V,  Y = Q S0^T + Z V,
//   W = T At,  X = T Lak,  Q = Rt + M At,  Z = Mrk + M Lak,
//   S_16 = S0 diag(L_15) + (SA^T Bh + V^T Kh) diag(L_15).
// Reset flags inside a chunk become masks: pairs (t, tau) separated by a
// reset are dropped from Lab..Mrk, S0 only reaches tokens before the first
// reset (At and Rt rows masked, i.e. columns of T and M), only the last
// segment feeds S_16, and S0 drops out of S_16 if the chunk holds any reset.
//
// Precision: every product is tf32 with fp32 accumulation; operands are
// rounded to tf32 (nearest) except SA^T, which the state product reads back
// from tensor memory as tf32.  An emulation of the rounded operands against
// the fp64 oracle stays ~6x inside the bf16 tolerance.  A chunk whose decay
// product leaves [2^-40, 2^40] (e.g. w = 0) cannot use the 1/L scaling and is
// run token by token instead.
//
// Work split (one CTA of 8 warps per (b,h)), pipelined over chunks:
//   warps 4-7 ("context") for chunk c+1: stage the inputs (one TMA box per
//     input on an mbarrier, bounded waits), build the decay-scaled operands
//     (for the state products in the tcgen05 operand layout, Bh and Kh masked
//     to the last segment) and the masked Gram of [At; Rt] and [Bh; Kh]
//     (mma.sync) into one half of a double-buffered context;
//   warps 0-3 ("state") for chunk c: warp w owns rows 16w..16w+15 of S as
//     fp32 accumulator fragments for the whole sequence; they solve for T,
//     form W, X, M, Q, Z (mma.sync, 16x16 blocks), then one thread issues the
//     two state products as tcgen05 MMAs (M = 64, accumulators in TMEM; see
//     state_chunk), and the warps write y, update S and write the chunk-end
//     checkpoint.
// One CTA barrier per chunk hands the context over.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "epilogue.cuh"
#include "mma.cuh"
#include "tc05.cuh"
#include "token_path.cuh"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;
constexpr int kIn = 6;       // staged inputs: r, w, k, v, a, b
constexpr int kStrY = 72;    // row stride (elements) of the y staging tile
constexpr int S68 = 68, S20 = 20;
using bf16 = __nv_bfloat16;

// Produced by the context warps for one chunk, consumed by the state warps one iteration later.
struct __align__(128) Ctx {
  float Rt[kChunk][S68];    // m0 . rt  [t][j]   (fp32, initial value of Q)
  float AtT[kN][S20];       // at       [j][tau]
  // tcgen05 operands, K-major canonical layout (cidx): rows j (or i), K = tau
  __align__(128) float VTc[kN * kChunk];    // v         (A of both state products)
  __align__(128) float BhTc[kN * kChunk];   // ls . bh   (B of S_16)
  __align__(128) float KhTc[kN * kChunk];   // ls . kh   (B of S_16)
  float LabT[kChunk][S20];  // Lab^T    [tau][t] (fp32, for T)
  float LakT[kChunk][S20];  // Lak^T    [tau][t]
  float Mrb[kChunk][S20];   // Mrb      [t][tau]
  float Mrk[kChunk][S20];   // Mrk      [t][tau] (fp32, initial value of Z)
  float lam15[kN];
  int mask;                 // reset bits of the chunk
  int unsafe;               // decay product out of range: run this chunk token by token
};

template <typename T>
struct __align__(128) FwdSmem3 {
  Ctx ctx[2];
  float GA[32][S68];        // rows 0..15 at_t, 16..31 rt_t   [t][j]
  float GB[32][S68];        // rows 0..15 bh_t, 16..31 kh_t   [tau][j]
  __align__(16) float Tm[kChunk][S20];      // T   [t][tau]  (state warps)
  __align__(16) float TT[kChunk][S20];      // T^T [tau][t]
  __align__(128) float B1[2 * kChunk * kN];      // [W; Q]: rows t (W) and 16 + t (Q), K = j (cidx, K 64)
  __align__(128) float B1v[2 * kChunk * kChunk]; // [X; Z]: rows t and 16 + t, K = tau (cidx, K 16)
  float M[kChunk][S20];
  __align__(128) T in[kIn][kChunk][kN];      // staged inputs of the chunk being built (TMA boxes)
  __align__(16) uint16_t Ys[kChunk][kStrY]; // y of the last chunk [t][i] (16-bit outputs), written next iteration
  __align__(16) float epi_par[3][kN];        // fused epilogue: GroupNorm weight, bias and bonus weights of the head
  unsigned long long in_bar;                 // completion of the bulk copies into `in` (one phase per chunk)
  unsigned long long d1_bar, mma_bar;        // completion of a chunk's D1 MMAs / of all its MMAs (one phase per chunk)
  uint32_t tmem_base;                        // TMEM: S0 (cols 0-63), D1 (64-95), D3 (128-191)
  int kbad[4];
  float qsum[4][kN];                         // log-space decay: sum of -exp(x) over each token quarter
};

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void cta_sync() { asm volatile("bar.sync 0;\n" ::: "memory"); }

// Float index of element (r, k) of a K-major canonical tcgen05 operand with K = kdim (no swizzle:
// 8-row x 16-byte core matrices, K-adjacent ones 128 bytes apart, row groups kdim/4 * 128 apart).
__device__ __forceinline__ int cidx(int r, int k, int kdim) {
  return (r >> 3) * (kdim * 8) + (k >> 2) * 32 + (r & 7) * 4 + (k & 3);
}

constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmS0 = 0, kTmD1 = 64, kTmD3 = 128;   // TMEM column offsets

// Store four 8x8 b16 matrices from accumulator-fragment registers, transposed.
__device__ __forceinline__ void stsm_x4_t(void* row_ptr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};\n"
               ::"r"(smem_u32(row_ptr)), "r"(r0), "r"(r1), "r"(r2), "r"(r3) : "memory");
}

template <typename T>
__device__ __forceinline__ uint32_t pack16(float lo, float hi) {
  if constexpr (std::is_same<T, __half>::value) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    return pack_bf16(lo, hi);
  }
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Keep the A-fragment entries of a natural-k fragment (k = 8s+c and 8s+c+4) whose bit is set.
__device__ __forceinline__ void mask_nat(uint32_t (&a)[4], int s, int c4, unsigned bits) {
  const bool k0 = (bits >> (8 * s + c4)) & 1u, k1 = (bits >> (8 * s + c4 + 4)) & 1u;
  if (!k0) { a[0] = 0u; a[1] = 0u; }
  if (!k1) { a[2] = 0u; a[3] = 0u; }
}

// Stage the six inputs of chunk tokens t0..t0+15 into sm.in: one TMA box per input, issued by one
// thread; rows past T arrive as zeros (K1 reads w there as 1, which leaves the state unchanged).
// The copies complete phase c of sm.in_bar for chunk c.
template <typename T>
__device__ __forceinline__ void stage_chunk(const FwdArgs& p, const InputMaps& tm, FwdSmem3<T>& sm, int64_t b,
                                            int64_t h, int64_t t0, int ktid) {
  if (ktid == 0) {
    if (!in_bounds(h < p.H && b < p.B && t0 >= 0 && t0 < p.T, p.status)) return;   // (debug build)
    mbar_arrive_expect_tx(&sm.in_bar, unsigned(kIn * kChunk * kN * sizeof(T)) + p.extra_tx);
#pragma unroll
    for (int m = 0; m < kIn; ++m) tma_load_4d(&sm.in[m][0][0], &tm.m[m], 0, int(h), int(t0), int(b), &sm.in_bar);
  }
}

// ------------------------------------------------------------------ context warps
// `degraded` (CTA-uniform, sticky): a wait for staged inputs ran out; from then on nothing more is
// staged and every chunk takes the token path, which reads its inputs from global memory.
template <typename T, bool kLog>
__device__ __forceinline__ void build_context(const FwdArgs& p, const InputMaps& tm, FwdSmem3<T>& sm, Ctx& cx,
                                              unsigned mask, int64_t b, int64_t h, int64_t c, int64_t nc, int ktid,
                                              bool& degraded) {
  const int kw = ktid >> 5, lane = ktid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
  const T (*X)[kChunk][kN] = sm.in;
  const int len = int(min64(kChunk, p.T - c * kChunk));

  const bool timed_out = !degraded && !mbar_wait_bounded(&sm.in_bar, unsigned(c & 1), kWaitLimitNs);

  // ---- K1: decay products and decay-scaled operands.  Thread = (token quarter kw; columns lane
  // and lane + 32, as one packed fp32 pair); the transposed copies go out as one float4 per column.
  bool bad = false;
  {
    const int tq = 4 * kw, ja = lane, jb = lane + 32;
    auto ld2 = [&](int m, int t) { return make_float2(Elt<T>::to_f32(X[m][t][ja]), Elt<T>::to_f32(X[m][t][jb])); };
    auto ldw = [&](int t) {   // padding: w = 1
      if (t >= len) return make_float2(1.f, 1.f);
      const float2 x = ld2(1, t);
      return make_float2(decay_of(x.x, kLog), decay_of(x.y, kLog));
    };
    // log-space decay: log L_t = sum_{s<=t} -exp(x_s).  Each warp sums its own quarter's terms and
    // takes the earlier quarters' sums from the other warps (one exponential per input, not a chain
    // of two per token over every earlier token)
    auto ldl = [&](int t) {   // -exp(x_t); padding: 0 (w = 1)
      if (t >= len) return make_float2(0.f, 0.f);
      const float2 x = ld2(1, t);
      return make_float2(-__expf(x.x), -__expf(x.y));
    };
    float2 lam = make_float2(1.f, 1.f);   // L_{tq-1}: product over the earlier quarters (warp-uniform count)
    float2 lsum = make_float2(0.f, 0.f);  // log L_{tq-1} (log-space decay)
    float2 dl[4];
    if (kLog) {
      float2 qs = make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        dl[u] = ldl(tq + u);
        qs = add2(qs, dl[u]);
      }
      sm.qsum[kw][ja] = qs.x;
      sm.qsum[kw][jb] = qs.y;
      named_bar(1, 128);   // (the next writes come after the barrier below, once every warp has read)
      for (int w2 = 0; w2 < kw; ++w2) lsum = add2(lsum, make_float2(sm.qsum[w2][ja], sm.qsum[w2][jb]));
      lam = make_float2(__expf(lsum.x), __expf(lsum.y));
    } else {
      for (int t = 0; t < tq; ++t) lam = mul2(lam, ldw(t));
    }
    float at[2][4], bh[2][4], kh[2][4], vv[2][4];
    const unsigned ls_bits = last_segment_bits(mask);   // S_16 sees only the chunk's last segment
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = tq + u;
      const float2 lp = lam;
      if (kLog) {
        lsum = add2(lsum, dl[u]);
        lam = make_float2(__expf(lsum.x), __expf(lsum.y));
      } else {
        lam = mul2(lam, ldw(t));
      }
      bad |= !(lam.x >= 0x1p-40f && lam.x <= 0x1p40f) || !(lam.y >= 0x1p-40f && lam.y <= 0x1p40f);
      const float2 inv = make_float2(rcp_approx(lam.x), rcp_approx(lam.y));
      const float2 a2 = mul2(ld2(4, t), lp), r2 = mul2(ld2(0, t), lam);
      const float2 b2 = mul2(ld2(5, t), inv), k2 = mul2(ld2(2, t), inv), v2 = ld2(3, t);
      at[0][u] = tf32f(a2.x); at[1][u] = tf32f(a2.y);
      bh[0][u] = tf32f(b2.x); bh[1][u] = tf32f(b2.y);
      kh[0][u] = tf32f(k2.x); kh[1][u] = tf32f(k2.y);
      vv[0][u] = tf32f(v2.x); vv[1][u] = tf32f(v2.y);
      sm.GA[t][ja] = at[0][u];
      sm.GA[t][jb] = at[1][u];
      sm.GA[16 + t][ja] = tf32f(r2.x);
      sm.GA[16 + t][jb] = tf32f(r2.y);
      sm.GB[t][ja] = bh[0][u];
      sm.GB[t][jb] = bh[1][u];
      sm.GB[16 + t][ja] = kh[0][u];
      sm.GB[16 + t][jb] = kh[1][u];
      cx.Rt[t][ja] = t < fr ? r2.x : 0.f;
      cx.Rt[t][jb] = t < fr ? r2.y : 0.f;
    }
    const float l0 = (ls_bits >> tq) & 1u ? 1.f : 0.f, l1 = (ls_bits >> (tq + 1)) & 1u ? 1.f : 0.f;
    const float l2 = (ls_bits >> (tq + 2)) & 1u ? 1.f : 0.f, l3 = (ls_bits >> (tq + 3)) & 1u ? 1.f : 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int j = q ? jb : ja;
      const int ci = cidx(j, tq, kChunk);   // four consecutive tau: one float4
      *reinterpret_cast<float4*>(&cx.AtT[j][tq]) = make_float4(at[q][0], at[q][1], at[q][2], at[q][3]);
      *reinterpret_cast<float4*>(&cx.BhTc[ci]) = make_float4(l0 * bh[q][0], l1 * bh[q][1], l2 * bh[q][2], l3 * bh[q][3]);
      *reinterpret_cast<float4*>(&cx.KhTc[ci]) = make_float4(l0 * kh[q][0], l1 * kh[q][1], l2 * kh[q][2], l3 * kh[q][3]);
      *reinterpret_cast<float4*>(&cx.VTc[ci]) = make_float4(vv[q][0], vv[q][1], vv[q][2], vv[q][3]);
    }
    if (kw == 3) {
      cx.lam15[ja] = lam.x;
      cx.lam15[jb] = lam.y;
    }
  }
  const unsigned any_bad = __ballot_sync(0xffffffffu, bad), any_to = __ballot_sync(0xffffffffu, timed_out);
  if (lane == 0) sm.kbad[kw] = (any_bad ? 1 : 0) | (any_to ? 2 : 0);
  named_bar(1, 128);
  const int kb = sm.kbad[0] | sm.kbad[1] | sm.kbad[2] | sm.kbad[3];
  if ((kb & 2) && !degraded) {
    degraded = true;
    if (ktid == 0 && p.status) atomicOr(p.status, kStatusWaitTimeout);
  }
  const bool unsafe = kb != 0 || degraded;
  if (ktid == 0) {
    cx.mask = int(mask);
    cx.unsafe = unsafe ? 1 : 0;
  }

  // the staged inputs are consumed: fetch the next chunk while the rest is built
  if (c + 1 < nc && !degraded) {
    const int64_t t1 = (c + 1) * kChunk;
    stage_chunk<T>(p, tm, sm, b, h, t1, ktid);
  }
  if (unsafe) return;

  // ---- K2: 32x32 Gram of [at; rt] and [bh; kh] (tf32), masked
  {
    const int m0 = (kw >> 1) * 16, n0 = (kw & 1) * 16;
    float gr[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a[4], bb[4];
      ldsm_x4(a, a32_addr(&sm.GA[0][0], S68, m0, 8 * ks, lane));
      ldsm_x4(bb, b32_2n_addr(&sm.GB[0][0], S68, n0, 8 * ks, lane));
      mma1688(gr[0], a, bb[0], bb[1]);
      mma1688(gr[1], a, bb[2], bb[3]);
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
        if (kw == 0) cx.LabT[tau][t] = v;
        else if (kw == 1) cx.LakT[tau][t] = tf32f(v);
        else if (kw == 2) cx.Mrb[t][tau] = tf32f(v);
        else cx.Mrk[t][tau] = v;
      }
  }
}

// ------------------------------------------------------------------ state warps
// One chunk of the state warps.  Steps a/b (mma.sync, 16x16 blocks) form W, Q, X, Z in the
// tcgen05 operand layout; the state products then run as one batch of tcgen05 MMAs issued by one
// thread (M = 64 rows i, accumulators in TMEM):
//   D1 = S0 [W; Q]^T + V^T [X; Z]^T   (columns 0-15: SA^T, 16-31: Y^T),  S0 from TMEM (tf32)
//   D3 = SA^T ls.Bh + V^T ls.Kh       (SA^T read back from D1 in TMEM as the A operand)
// and S_16 = keep.S0 diag(L_15) + D3 diag(L_15) stays in the fp32 registers.  `mma_phase` counts
// the batches issued so far (the parity of the mbarrier phase to wait for).
template <typename T>
__device__ __forceinline__ void state_chunk(const FwdArgs& p, FwdSmem3<T>& sm, const Ctx& cx, float (&acc)[8][4],
                                            int64_t b, int64_t h, int64_t t0, int len, int warp, int lane,
                                            uint32_t tmem, unsigned& mma_phase, float* ck_prev) {
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;
  const int j0 = 16 * warp;
  const unsigned mask = unsigned(cx.mask);
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
  const unsigned m0bits = (1u << fr) - 1u;   // tokens that S0 reaches
  const uint32_t tlane = uint32_t(32 * warp) << 16;   // this warp's TMEM lanes (rows 16w..16w+15)

  // ---- S0 in tf32 into TMEM (A operand of D1)
  {
    float s0t[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s0t[nt][e] = tf32f(acc[nt][e]);
    tc::st_16x256b_x8(tmem + tlane + kTmS0, s0t);
  }

  // ---- T = (I - Lab)^-1 by forward substitution, one column per lane (warp 0, lanes 0-15)
  if (warp == 0 && lane < kChunk) {
    const int cc = lane;
    float u[kChunk];
#pragma unroll
    for (int t = 0; t < kChunk; ++t) u[t] = t == cc ? 1.f : 0.f;
    // rows of Lab^T are loaded one step ahead, so each step waits only on its FMAs
    float4 nxt[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) nxt[q] = reinterpret_cast<const float4*>(&cx.LabT[0][0])[q];
#pragma unroll
    for (int tau = 0; tau < kChunk - 1; ++tau) {
      const float4 cur[4] = {nxt[0], nxt[1], nxt[2], nxt[3]};
      if (tau + 1 < kChunk - 1) {
#pragma unroll
        for (int q = (tau + 2) / 4; q < 4; ++q) nxt[q] = reinterpret_cast<const float4*>(&cx.LabT[tau + 1][0])[q];
      }
      const float lv[kChunk] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y, cur[1].z, cur[1].w,
                                cur[2].x, cur[2].y, cur[2].z, cur[2].w, cur[3].x, cur[3].y, cur[3].z, cur[3].w};
#pragma unroll
      for (int t = tau + 1; t < kChunk; ++t) u[t] = fmaf(lv[t], u[tau], u[t]);
    }
#pragma unroll
    for (int t = 0; t < kChunk; ++t) {
      const float v = tf32f(u[t]);
      sm.Tm[t][cc] = v;
      sm.TT[cc][t] = v;
    }
  }
  named_bar(2, 128);

  // ---- step a: W = T diag(m0) At (columns j0..j0+15), M = Mrb T (warp 0), X = T Lak (warp 1)
  uint32_t bat[2][4];   // At^T fragments of this warp's columns: [n-tile][k-step pair]
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) ldsm_x4(bat[nt], b32_2k_addr(&cx.AtT[0][0], S20, j0 + 8 * nt, 0, lane));
  {
    uint32_t at[2][4];
#pragma unroll
    for (int s = 0; s < 2; ++s) ldsm_x4(at[s], a32_addr(&sm.Tm[0][0], S20, 0, 8 * s, lane));
    if (warp == 1) {   // X = T Lak (unmasked T)
      float xx[2][4] = {};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t bl[4];
        ldsm_x4(bl, b32_2k_addr(&cx.LakT[0][0], S20, 8 * nt, 0, lane));
        mma1688(xx[nt], at[0], bl[0], bl[1]);
        mma1688(xx[nt], at[1], bl[2], bl[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<float2*>(&sm.B1v[cidx(g + 8 * hh, 8 * nt + 2 * c4, kChunk)]) =
              make_float2(tf32f(xx[nt][2 * hh]), tf32f(xx[nt][2 * hh + 1]));
    }
    mask_nat(at[0], 0, c4, m0bits);
    mask_nat(at[1], 1, c4, m0bits);
    float ww[2][4] = {};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      mma1688(ww[nt], at[0], bat[nt][0], bat[nt][1]);
      mma1688(ww[nt], at[1], bat[nt][2], bat[nt][3]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        *reinterpret_cast<float2*>(&sm.B1[cidx(g + 8 * hh, j0 + 8 * nt + 2 * c4, kN)]) =
            make_float2(tf32f(ww[nt][2 * hh]), tf32f(ww[nt][2 * hh + 1]));
    if (warp == 0) {   // M = Mrb T
      uint32_t am[2][4];
#pragma unroll
      for (int s = 0; s < 2; ++s) ldsm_x4(am[s], a32_addr(&cx.Mrb[0][0], S20, 0, 8 * s, lane));
      float mm[2][4] = {};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t bt[4];
        ldsm_x4(bt, b32_2k_addr(&sm.TT[0][0], S20, 8 * nt, 0, lane));
        mma1688(mm[nt], am[0], bt[0], bt[1]);
        mma1688(mm[nt], am[1], bt[2], bt[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<float2*>(&sm.M[g + 8 * hh][8 * nt + 2 * c4]) =
              make_float2(tf32f(mm[nt][2 * hh]), tf32f(mm[nt][2 * hh + 1]));
    }
  }
  named_bar(2, 128);

  // ---- step b: Q = m0.Rt + M diag(m0) At (columns j0..j0+15), Z = Mrk + M Lak (warp 2)
  {
    uint32_t am[2][4];
#pragma unroll
    for (int s = 0; s < 2; ++s) ldsm_x4(am[s], a32_addr(&sm.M[0][0], S20, 0, 8 * s, lane));
    if (warp == 2) {
      float zz[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float2 m2 = *reinterpret_cast<const float2*>(&cx.Mrk[g + 8 * hh][8 * nt + 2 * c4]);
          zz[nt][2 * hh] = m2.x;
          zz[nt][2 * hh + 1] = m2.y;
        }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t bl[4];
        ldsm_x4(bl, b32_2k_addr(&cx.LakT[0][0], S20, 8 * nt, 0, lane));
        mma1688(zz[nt], am[0], bl[0], bl[1]);
        mma1688(zz[nt], am[1], bl[2], bl[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<float2*>(&sm.B1v[cidx(kChunk + g + 8 * hh, 8 * nt + 2 * c4, kChunk)]) =
              make_float2(tf32f(zz[nt][2 * hh]), tf32f(zz[nt][2 * hh + 1]));
    }
    mask_nat(am[0], 0, c4, m0bits);
    mask_nat(am[1], 1, c4, m0bits);
    float qq[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float2 r2 = *reinterpret_cast<const float2*>(&cx.Rt[g + 8 * hh][j0 + 8 * nt + 2 * c4]);
        qq[nt][2 * hh] = r2.x;
        qq[nt][2 * hh + 1] = r2.y;
      }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      mma1688(qq[nt], am[0], bat[nt][0], bat[nt][1]);
      mma1688(qq[nt], am[1], bat[nt][2], bat[nt][3]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        *reinterpret_cast<float2*>(&sm.B1[cidx(kChunk + g + 8 * hh, j0 + 8 * nt + 2 * c4, kN)]) =
            make_float2(tf32f(qq[nt][2 * hh]), tf32f(qq[nt][2 * hh + 1]));
  }
  // operands visible to the tensor core, S0 in TMEM, then one thread issues the batch
  tc::fence_smem_to_async();
  tc::wait_st();
  tc::fence_before_sync();
  named_bar(2, 128);
  if (warp == 0 && lane == 0) {
    tc::fence_after_sync();
    constexpr uint32_t id32 = tc::idesc_tf32(64, 32), id64 = tc::idesc_tf32(64, 64);
#pragma unroll
    for (int s = 0; s < kN / 8; ++s)   // S0 [W; Q]^T over j, 8 per MMA
      tc::mma_ts(tmem + kTmD1, tmem + kTmS0 + 8 * s, tc::smem_desc(&sm.B1[64 * s], 8 * kN * 4), id32, s > 0);
#pragma unroll
    for (int s = 0; s < 2; ++s)        // + V^T [X; Z]^T over tau
      tc::mma_ss(tmem + kTmD1, tc::smem_desc(&cx.VTc[64 * s], 8 * kChunk * 4),
                 tc::smem_desc(&sm.B1v[64 * s], 8 * kChunk * 4), id32, true);
#pragma unroll
    for (int s = 0; s < 2; ++s)        // D3 = V^T ls.Kh (independent of D1) ...
      tc::mma_ss(tmem + kTmD3, tc::smem_desc(&cx.VTc[64 * s], 8 * kChunk * 4),
                 tc::smem_desc(&cx.KhTc[64 * s], 8 * kChunk * 4), id64, s > 0);
    // D3 reads D1 through the A-operand path: issue it only once D1 is complete
    tc::commit(&sm.d1_bar);
    if (!mbar_wait_bounded(&sm.d1_bar, mma_phase & 1u, kWaitLimitNs) && p.status) atomicOr(p.status, kStatusWaitTimeout);
    tc::fence_after_sync();
#pragma unroll
    for (int s = 0; s < 2; ++s)        // ... + SA^T ls.Bh (SA^T = D1 columns 0-15)
      tc::mma_ts(tmem + kTmD3, tmem + kTmD1 + 8 * s, tc::smem_desc(&cx.BhTc[64 * s], 8 * kChunk * 4), id64, true);
    tc::commit(&sm.mma_bar);
  }
  // while the tensor core works: the checkpoint of the state entering this chunk (the previous
  // chunk's end state, still unchanged in the fragments), 512 contiguous bytes per warp and nt
  if (ck_prev) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<float4*>(ck_prev + nt * 128) = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
  }
  if (!mbar_wait_bounded(&sm.mma_bar, mma_phase & 1u, kWaitLimitNs) && threadIdx.x == 0 && p.status)
    atomicOr(p.status, kStatusWaitTimeout);
  ++mma_phase;
  tc::fence_after_sync();

  float yy[2][4], d[8][4];
  tc::ld_16x256b_x2(tmem + tlane + kTmD1 + kChunk, yy);   // Y^T: D1 columns 16-31
  tc::ld_16x256b_x8(tmem + tlane + kTmD3, d);
  tc::wait_ld();

  if constexpr (sizeof(T) == 2) {   // Y^T fragments -> Ys[t][i]; written out after the next CTA barrier
    const int m = lane >> 3;
    stsm_x4_t(&sm.Ys[8 * (m >> 1) + (lane & 7)][row0 + 8 * (m & 1)], pack16<T>(yy[0][0], yy[0][1]),
              pack16<T>(yy[0][2], yy[0][3]), pack16<T>(yy[1][0], yy[1][1]), pack16<T>(yy[1][2], yy[1][3]));
  } else {
    T* y = static_cast<T*>(p.y);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = 8 * nt + 2 * c4 + (e & 1);
        const int64_t o = tok_off(b, t0 + t, h, p.T, p.H) + row0 + g + 8 * (e >> 1);
        if (t < len && range_ok(o, 1, p.B * p.T * p.H * kN, p.status)) y[o] = Elt<T>::from_f32(yy[nt][e]);
      }
  }

  // ---- S_16 = keep.S0 diag(L_15) + D3 diag(L_15)
  const float keep = mask == 0u ? 1.f : 0.f;
#pragma unroll
  for (int jt = 0; jt < 8; ++jt) {
    const float2 l2 = *reinterpret_cast<const float2*>(&cx.lam15[8 * jt + 2 * c4]);
    acc[jt][0] = fmaf(keep * acc[jt][0], l2.x, d[jt][0] * l2.x);
    acc[jt][1] = fmaf(keep * acc[jt][1], l2.y, d[jt][1] * l2.y);
    acc[jt][2] = fmaf(keep * acc[jt][2], l2.x, d[jt][2] * l2.x);
    acc[jt][3] = fmaf(keep * acc[jt][3], l2.y, d[jt][3] * l2.y);
  }
  // the next batch overwrites D1/D3 and S0: every warp's loads are done before it is issued
  tc::fence_before_sync();
}

// The eight float4 of a checkpoint in the tiled order (ck == nullptr: none due).
__device__ __forceinline__ void store_ck(float* ck, const float (&acc)[8][4]) {
  if (ck) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<float4*>(ck + nt * 128) = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
  }
}

template <typename T, bool kEpi, bool kLog>
__global__ void __launch_bounds__(kThreads, 2) chunk_fwd_kernel(const FwdArgs p, const __grid_constant__ InputMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  FwdSmem3<T>& sm = *reinterpret_cast<FwdSmem3<T>*>(smem_raw);

  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_state = warp < 4;
  const int ktid = tid - 128;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;

  // The two roles run separate loops so that their register sets never overlap; both meet
  // at one CTA barrier per iteration (bar.sync 0, executed by all 256 threads).
  if (is_state) {
    // state fragments: acc[nt][e] = S[16*warp + g + 8*(e>>1)][8*nt + 2*c4 + (e&1)]
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float2 v2 = make_float2(0.f, 0.f);
        const int64_t so = (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4;
        if (p.s0 && range_ok(so, 2, p.B * p.H * kN * kN, p.status)) v2 = *reinterpret_cast<const float2*>(p.s0 + so);
        acc[nt][2 * hh] = v2.x;
        acc[nt][2 * hh + 1] = v2.y;
      }
    if (warp == 0) {   // 256 TMEM columns: two CTAs per SM fill the 512 exactly
      tc::alloc(&sm.tmem_base, kTmemCols);
      tc::relinquish();
    }
    if (tid == 0) {
      mbar_init(&sm.d1_bar, 1);
      mbar_init(&sm.mma_bar, 1);
    }
    if constexpr (kEpi) {   // the head's epilogue parameters
      const float* const par[3] = {p.ln_w, p.ln_b, p.r_k};
      for (int i = tid; i < 3 * kN; i += 128) sm.epi_par[i / kN][i % kN] = par[i / kN][h * kN + i % kN];
    }
    tc::fence_before_sync();
    cta_sync();   // chunk 0 staged; TMEM allocated; the epilogue parameters in place
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    unsigned mma_phase = 0;
    // y of the previous chunk (16-bit outputs): this thread's 16-byte piece of token row tid/8, at
    // element offset yoff; with the fused epilogue also the r, k, v and g of that piece, loaded before
    // the CTA barrier and used after it, and the 8 lanes of the row form one GroupNorm group.
    int64_t yoff = -1;
    const int ytt = tid >> 3, ypart = tid & 7;
    uint4 er = {}, ek = {}, ev = {}, eg = {};
    auto flush_y = [&]() {
      if (yoff < 0) return;
      const uint4 yv = *reinterpret_cast<const uint4*>(&sm.Ys[ytt][ypart * 8]);
      if constexpr (kEpi) {
        float y8[8], r8[8], k8[8], v8[8], g8[8], o8[8];
        unpack16<T>(yv, y8);
        unpack16<T>(er, r8);
        unpack16<T>(ek, k8);
        unpack16<T>(ev, v8);
        unpack16<T>(eg, g8);
        epi_forward<8, 8>(y8, r8, k8, v8, g8, &sm.epi_par[0][ypart * 8], &sm.epi_par[1][ypart * 8],
                          &sm.epi_par[2][ypart * 8], p.eps, 0xffu << (lane & 24), o8);
        uint4 ov;
        T* const oq = reinterpret_cast<T*>(&ov);
#pragma unroll
        for (int e = 0; e < 8; ++e) oq[e] = Elt<T>::from_f32(o8[e]);
        *reinterpret_cast<uint4*>(static_cast<T*>(p.out) + yoff) = ov;
        if (p.y) *reinterpret_cast<uint4*>(static_cast<T*>(p.y) + yoff) = yv;
      } else {
        *reinterpret_cast<uint4*>(static_cast<T*>(p.y) + yoff) = yv;
      }
      yoff = -1;
    };
    float* ck = nullptr;   // checkpoint slot of the state in the fragments (tiled order), if still due
    for (int64_t it = 0; it <= nc; ++it) {
      flush_y();
      if (it >= 1) {
        const int64_t c = it - 1;
        const Ctx& cx = sm.ctx[c & 1];
        const int64_t t0 = c * kChunk;
        const int len = int(min64(kChunk, p.T - t0));
        if (!cx.unsafe) {
          state_chunk<T>(p, sm, cx, acc, b, h, t0, len, warp, lane, tmem, mma_phase, ck);
          if (sizeof(T) == 2 && ytt < len &&
              range_ok(tok_off(b, t0 + ytt, h, p.T, p.H) + ypart * 8, 8, p.B * p.T * p.H * kN, p.status)) {
            yoff = tok_off(b, t0 + ytt, h, p.T, p.H) + ypart * 8;
            if constexpr (kEpi) {
              er = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.r) + yoff);
              ek = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.k) + yoff);
              ev = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.v) + yoff);
              eg = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.g) + yoff);
            }
          }
        } else if constexpr (kEpi) {   // token by token into the y tile, then out like a safe chunk
          store_ck(ck, acc);
          state_chunk_tokens<T>(p, unsigned(cx.mask), acc, b, h, t0, len, warp, lane, &sm.Ys[0][0], kStrY);
          if (ytt < len && range_ok(tok_off(b, t0 + ytt, h, p.T, p.H) + ypart * 8, 8, p.B * p.T * p.H * kN, p.status)) {
            yoff = tok_off(b, t0 + ytt, h, p.T, p.H) + ypart * 8;
            er = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.r) + yoff);
            ek = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.k) + yoff);
            ev = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.v) + yoff);
            eg = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.g) + yoff);
          }
        } else {
          store_ck(ck, acc);
          state_chunk_tokens<T>(p, unsigned(cx.mask), acc, b, h, t0, len, warp, lane);
        }
        // this chunk's end state is checkpointed during the next chunk (or after the loop)
        ck = p.ckpt && range_ok((unit * nc + c) * kN * kN, kN * kN, p.B * p.H * nc * kN * kN, p.status)
                 ? p.ckpt + (unit * nc + c) * kN * kN + warp * 1024 + lane * 4 : nullptr;
      }
      cta_sync();   // context of chunk it handed over; Ys complete
    }
    flush_y();
    store_ck(ck, acc);
    // every batch was waited for and every TMEM load is complete: release TMEM
    named_bar(2, 128);
    tc::fence_after_sync();
    if (warp == 0) tc::dealloc(tmem, kTmemCols);
    if (p.s_out) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int64_t so = (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4;
          if (range_ok(so, 2, p.B * p.H * kN * kN, p.status))
            *reinterpret_cast<float2*>(p.s_out + so) = make_float2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
        }
    }
  } else {
    // prologue: stage chunk 0 and fetch its reset flags
    unsigned reset_bits;
    bool degraded = false;
    unsigned stuck = 0;   // parity of the phase whose wait ran out
    {
      if (ktid == 0) mbar_init(&sm.in_bar, 1);
      named_bar(1, 128);
      const int len0 = int(min64(kChunk, p.T));
      stage_chunk<T>(p, tm, sm, b, h, 0, ktid);
      const bool f = p.reset && lane < len0 && p.reset[b * p.T + lane] != 0;
      reset_bits = __ballot_sync(0xffffffffu, f) & 0xffffu;
    }
    cta_sync();
    for (int64_t it = 0; it <= nc; ++it) {
      if (it < nc) {
        const int64_t c = it;
        const unsigned mask = reset_bits;
        if (c + 1 < nc) {   // reset flags of the next chunk (used next iteration)
          const int64_t t1 = (c + 1) * kChunk;
          const int len1 = int(min64(kChunk, p.T - t1));
          const bool f = p.reset && lane < len1 && p.reset[b * p.T + t1 + lane] != 0;
          reset_bits = __ballot_sync(0xffffffffu, f) & 0xffffu;
        }
        const bool was_degraded = degraded;
        build_context<T, kLog>(p, tm, sm, sm.ctx[c & 1], mask, b, h, c, nc, ktid, degraded);
        if (degraded && !was_degraded) stuck = unsigned(c & 1);
        tc::fence_smem_to_async();   // the tcgen05 operands of the context, for the tensor core
      }
      cta_sync();
    }
    // a wait that ran out may have left copies in flight: give them a bounded chance to land
    if (degraded) mbar_wait_bounded(&sm.in_bar, stuck, kWaitLimitNs / 100);
  }
}

// The log-space decay is a template parameter: the kernel without it has none of its code in K1.
template <typename T, bool kEpi>
cudaError_t launch(const FwdArgs& p, const InputMaps& tm, cudaStream_t stream) {
  const size_t smem = sizeof(FwdSmem3<T>);
  auto kern = p.log_decay ? chunk_fwd_kernel<T, kEpi, true> : chunk_fwd_kernel<T, kEpi, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(unsigned(p.B * p.H)), dim3(kThreads), smem, stream>>>(p, tm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_fwd(const FwdArgs& p, const InputMaps& tm, int dtype, cudaStream_t stream) {
  if (p.out) {   // the fused epilogue: 16-bit types only (their y goes out through the staged tile)
    switch (dtype) {
      case 1: return launch<__nv_bfloat16, true>(p, tm, stream);
      case 2: return launch<__half, true>(p, tm, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (dtype) {
    case 0: return launch<float, false>(p, tm, stream);
    case 1: return launch<__nv_bfloat16, false>(p, tm, stream);
    case 2: return launch<__half, false>(p, tm, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
