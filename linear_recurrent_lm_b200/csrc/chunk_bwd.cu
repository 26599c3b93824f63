// WKV-7 backward in 16-token chunks on the fifth-generation tensor cores (algo CHUNKED).
//
// Exact reverse mode of the chunk formulas of the forward (see chunk_fwd.cu): inside a chunk with
// entering state S0 and decay products L_t = prod_{s<=t} w_s, At = a L_{t-1}, Rt = r L_t,
// Bh = b / L_t, Kh = k / L_t, the masked Gram blocks Lab = At Bh^T, Lak = At Kh^T (strictly lower),
// Mrb = Rt Bh^T, Mrk = Rt Kh^T (lower), T = (I - Lab)^-1, W = T m0.At, X = T Lak and
//   SA = W S0^T + X V,   S16 = keep.S0 diag(L_15) + (SA^T Bl + V^T Kl) diag(L_15)
// (m0: tokens before the chunk's first reset, ls: tokens of its last segment, Bl = ls.Bh,
// Kl = ls.Kh, keep: no reset in the chunk).  Given dY and the gradient dS16 carried from the next
// chunk, with dSl = dS16 diag(L_15):
//   dSA = Mrb^T dY + Bl dSl^T,   dU = T^T dSA,   dV = Mrk^T dY + Kl dSl^T + Lak^T dU,
//   dS0 = keep.dSl + (m0.dY)^T Rt + (m0.dU)^T At,
//   dMrb = dY SA^T, dMrk = dY V^T, dLab = dU SA^T, dLak = dU V^T   (masked like their blocks),
//   dAt = dLab Bh + dLak Kh + m0.dU S0,   dRt = dMrb Bh + dMrk Kh + m0.dY S0,
//   dBh = dLab^T At + dMrb^T Rt + ls.(SA dSl),   dKh = dLak^T At + dMrk^T Rt + ls.(V dSl),
// and through the decays d log L_t = dRt.Rt + dAt_{t+1}.At_{t+1} - dBh.Bh - dKh.Kh, plus at t = 15
// the L_15 terms keep.sum_i dSl o S0 + sum_tau ls.((SA dSl) o Bh + (V dSl) o Kh);
// d log w_s = sum_{t >= s} d log L_t and dw = d log w / w.  The pages print no backward; this is
// derived from the chunk forward, itself the recurrence regrouped (RWKV-MLX page, "Key Design
// Decisions" 2: state checkpoints every 16 tokens; rwkv-metal page: the backward rebuilds each
// chunk from its checkpoint).
//
// Everything runs transposed so that the tensor core's 64-row side is a state dimension: the
// carried gradient is dS^T (TMEM rows = key channel j), G1 = dSl [Bh|Kh]^T and G2 = dY^T [Mrb|Mrk]
// have rows = value channel i (dSA^T = ls o G1b + G2b, dU^T = dSA^T T, dV^T = ls o G1k + G2k +
// dU^T Lak follow on the FP32 cores, one thread per i), and the key-space gradients dAt^T, dRt^T,
// dBh^T, dKh^T have rows = j, so that one thread owns one key channel over all 16 tokens of the
// chunk and keeps the reverse sum for dw in its registers.
//
// Precision: the tensor-core products take bf16 operands split in two, x = hi + lo with
// hi = bf16(x), lo = bf16(x - hi), and accumulate hi.hi + hi.lo + lo.hi in fp32 (lo.lo, about
// 2^-16 of the product, is dropped); the inputs v and dy are exact in bf16 when they arrive in
// bf16 and then skip their lo half.  The carried dS^T, the decay scalings, the small 16x16 solves
// and the per-token outputs are fp32.  A chunk whose decays the 1/L scaling cannot take (some
// w < 1/16, or L_15 outside [2^-40, 2^40]) stops the CTA and marks its unit in `unit_flags`; the
// scan backward then recomputes exactly those units.
//
// Shared-memory operands are "core arrays": a P x Q matrix of bf16 stored as 8-row x 8-column
// (16-byte) core matrices, element (p, q) at (p/8)(8Q) + (q/8)64 + (p%8)8 + q%8.  The tensor core
// reads one either K-major (rows = M or N, columns = K: LBO 128 bytes, SBO 16Q bytes, 256 bytes
// per K step of 16) or MN-major (columns = M or N, rows = K: LBO 16Q bytes, SBO 128 bytes, 32Q
// bytes per K step), so each matrix is stored once whichever way round a product needs it.
// Products with fewer than 64 useful rows read 64 anyway; the extra rows come from the arrays
// that follow (always inside the CTA's shared memory) and their results are never read.
//
// Work split: one CTA of 8 warps per (b,h) (about 200 KB of shared memory and 512 TMEM columns,
// so one CTA per SM), chunks in reverse, pipelined:
//   warps 4-7 ("context") for chunk c-1: stage its inputs (one TMA box per input) and its
//     checkpoint (one bulk copy) on an mbarrier with bounded waits, build the decay-scaled
//     operands, the masked Gram (tcgen05), T by substitution, W, X, and SA^T = S0 W^T + V^T X^T
//     (tcgen05) into one half of a double buffer;
//   warps 0-3 ("main") for chunk c: scale the carried dS^T, then one thread issues the products
//     in three batches (chain: G1, G2, Rt^T m0.dY; then At^T m0.dU, the gradient Gram and the S0
//     and dSl parts of the key-space products; then their Gram parts), while the warps write dv
//     and, per key channel, da, dr, db, dk and dw.
// One CTA barrier per chunk hands the context over.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;
constexpr int kIn = 7;   // r, w, k, v, a, b, dy
constexpr int S20 = 20;
using bf16 = __nv_bfloat16;

// TMEM columns (512 allocated: one CTA per SM).  Every accumulator has M = 64 rows.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDS = 64;     // main: dS^T                     (64; rows j)
constexpr uint32_t kColG1 = 128;    // main: dSl [Bh|Kh]^T            (32; rows i)
constexpr uint32_t kColG2 = 160;    // main: dY^T [Mrb|Mrk]           (32; rows i)
constexpr uint32_t kColGG = 192;    // main: [dY; dU] [SA^T | v^T]     (32; rows t and 16 + t)
constexpr uint32_t kColE = 256;     // main: dAt^T | dRt^T | dBg^T | dKg^T | (SA dSl)^T | (V dSl)^T  (96; rows j)

// bf16 index of element (p, q) of a core array with Q columns.
__device__ __forceinline__ int cb(int p, int q, int Q) { return (p >> 3) * (Q * 8) + (q >> 3) * 64 + (p & 7) * 8 + (q & 7); }

// Device status word of the running launch, for the debug-build bounds checks in helpers that do not
// see the kernel arguments (set by thread 0 before the first CTA barrier).
#ifdef WKV7_DEBUG
__shared__ int* s_dbg_status;
__device__ __forceinline__ int* debug_status() { return s_dbg_status; }
#else
__device__ __forceinline__ int* debug_status() { return nullptr; }
#endif

// A matrix split in two bf16 core arrays (hi, then lo).
template <int P, int Q>
struct Split {
  bf16 hi[P * Q];
  bf16 lo[P * Q];
};

// Split 8 fp32 values into one 16-byte row of hi and one of lo at element index e.
template <int P, int Q>
__device__ __forceinline__ void put8(Split<P, Q>& m, int e, const float (&x)[8]) {
  if (kDebugChecks && !(e >= 0 && e + 8 <= P * Q && (e & 7) == 0)) {   // debug build: one whole 16-byte row
    in_bounds(false, debug_status());
    return;
  }
  uint32_t h[4], l[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * u], x[2 * u + 1]);
    const float2 hf = __bfloat1622float2(hh);
    const __nv_bfloat162 ll = __floats2bfloat162_rn(x[2 * u] - hf.x, x[2 * u + 1] - hf.y);
    h[u] = *reinterpret_cast<const uint32_t*>(&hh);
    l[u] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  *reinterpret_cast<uint4*>(&m.hi[e]) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(&m.lo[e]) = make_uint4(l[0], l[1], l[2], l[3]);
}
// The 8 values (hi + lo) of one 16-byte row at element index e.
template <int P, int Q>
__device__ __forceinline__ void get8(const Split<P, Q>& m, int e, float (&x)[8]) {
  const uint4 h = *reinterpret_cast<const uint4*>(&m.hi[e]), l = *reinterpret_cast<const uint4*>(&m.lo[e]);
  const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[u]));
    const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lw[u]));
    x[2 * u] = a.x + c.x;
    x[2 * u + 1] = a.y + c.y;
  }
}

// ---- warp-level products (mma.sync m16n8k16, bf16 in, fp32 accumulate) on split core arrays.
// ldmatrix reads one 8x8 tile of a core array as 8 rows of 16 bytes; lane l supplies the row address
// of tile l / 8.
// A fragment (16 rows x 16 k) of a K-major core array (rows = M, columns = K) at (m0, k0).
template <int Q>
__device__ __forceinline__ uint32_t afrag_k(const bf16* a, int m0, int k0, int lane) {
  const int mi = lane >> 3, r = lane & 7;
  return smem_u32(a + cb(m0 + (mi & 1) * 8 + r, k0 + (mi >> 1) * 8, Q));
}
// A fragment of a matrix stored transposed (rows = K, columns = M), read with ldmatrix.trans.
template <int Q>
__device__ __forceinline__ uint32_t afrag_mn(const bf16* a, int m0, int k0, int lane) {
  const int mi = lane >> 3, r = lane & 7;
  return smem_u32(a + cb(k0 + (mi >> 1) * 8 + r, m0 + (mi & 1) * 8, Q));
}
// B fragments of two n-tiles (n0..n0+15) x 16 k from a core array with rows = N, columns = K.
template <int Q>
__device__ __forceinline__ uint32_t bfrag_k(const bf16* b, int n0, int k0, int lane) {
  const int mi = lane >> 3, r = lane & 7;
  return smem_u32(b + cb(n0 + (mi >> 1) * 8 + r, k0 + (mi & 1) * 8, Q));
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// acc[nt] (+)= A B over one K step of 16 for two n-tiles, with split operands: hi.hi + hi.lo + lo.hi.
// The lo addresses are the hi ones plus a fixed byte distance; a_exact skips the A lo half.
__device__ __forceinline__ void mma_split2(float (&acc)[2][4], uint32_t a_hi, uint32_t a_lo_off, bool a_mn,
                                           bool a_exact, uint32_t b_hi, uint32_t b_lo_off) {
  uint32_t ah[4], al[4], bh[4], bl[4];
  if (a_mn) ldsm4t(ah, a_hi); else ldsm4(ah, a_hi);
  ldsm4(bh, b_hi);
  ldsm4(bl, b_hi + b_lo_off);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    mma16816(acc[nt], ah, bh[2 * nt], bh[2 * nt + 1]);
    mma16816(acc[nt], ah, bl[2 * nt], bl[2 * nt + 1]);
  }
  if (!a_exact) {
    if (a_mn) ldsm4t(al, a_hi + a_lo_off); else ldsm4(al, a_hi + a_lo_off);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) mma16816(acc[nt], al, bh[2 * nt], bh[2 * nt + 1]);
  }
}

// One operand of a product: a split core array with Q columns, read K-major (rows = M/N, columns
// = K) or MN-major (columns = M/N, rows = K).  The layout is a compile-time constant; only the
// shared-memory addresses of the hi and lo arrays (already offset to the first row used) are not.
template <int Q, bool MN>
struct Op {
  uint32_t hi, lo;   // shared-memory byte addresses; lo == 0: the values are exact in bf16
  // Descriptor of K step ks: the 16-byte start-address field advances by a constant per step.
  __device__ __forceinline__ uint64_t desc(uint32_t base, int ks) const {
    constexpr uint32_t kLbo = MN ? uint32_t(Q) * 16 : 128u, kSbo = MN ? 128u : uint32_t(Q) * 16;
    constexpr uint32_t kStep = MN ? uint32_t(Q) * 32 : 256u;   // bytes per K step of 16
    const uint32_t lo32 = (((base + uint32_t(ks) * kStep) >> 4) & 0x3FFFu) | ((kLbo >> 4) << 16);
    constexpr uint32_t hi32 = (kSbo >> 4) | (1u << 14);          // SBO, descriptor version 1 (bit 46)
    return (uint64_t(hi32) << 32) | lo32;
  }
};
// The operand starting at row row0 and column col0 (both multiples of 8) of a split core array.
template <int Q, bool MN, int P>
__device__ __forceinline__ Op<Q, MN> op(const Split<P, Q>& m, bool exact = false, int row0 = 0, int col0 = 0) {
  const int e = cb(row0, col0, Q);
  return Op<Q, MN>{tc::smem_u32addr(m.hi + e), exact ? 0u : tc::smem_u32addr(m.lo + e)};
}
// Store one value as its hi and lo halves at element index e (a single element of a core row).
template <int P, int Q>
__device__ __forceinline__ void put1(Split<P, Q>& m, int e, float x) {
  if (!in_bounds(e >= 0 && e < P * Q, debug_status())) return;
  const bf16 h = __float2bfloat16_rn(x);
  m.hi[e] = h;
  m.lo[e] = __float2bfloat16_rn(x - __bfloat162float(h));
}
// D (+)= A B over NKS K steps of 16 (M = 64): hi.hi + hi.lo + lo.hi.  Issued by one thread.
template <int N, int NKS, int QA, bool MA, int QB, bool MB>
__device__ __forceinline__ void mma3(uint32_t d, const Op<QA, MA>& a, const Op<QB, MB>& b, bool accumulate) {
  constexpr uint32_t id = tc::idesc_bf16(64, N, MA ? 1 : 0, MB ? 1 : 0);
#pragma unroll
  for (int ks = 0; ks < NKS; ++ks) {
    const uint64_t ah = a.desc(a.hi, ks), bh = b.desc(b.hi, ks);
    tc::mma_bf16(d, ah, bh, id, accumulate || ks > 0);
    if (b.lo) tc::mma_bf16(d, ah, b.desc(b.lo, ks), id, true);
    if (a.lo) tc::mma_bf16(d, a.desc(a.lo, ks), bh, id, true);
  }
}

// Produced by the context warps for one chunk, read by the main warps one iteration later.  The
// order of the arrays matters: 64-row reads of AR and DY run on into the arrays after them.
template <typename T>
struct __align__(128) Ctx {
  Split<32, 64> AR;      // rows 0-15 At [t][j], rows 16-31 Rt [t][j]
  Split<32, 64> BK;      // rows 0-15 Bh [tau][j], rows 16-31 Kh [tau][j]
  Split<32, 64> DYU;     // rows 0-15 dy [t][i]; rows 16-31 dU [t][i], written by the main warps
  Split<64, 32> DUY;     // [i][m0.dU^T (t) | m0.dy^T (t)]: the dU half is written by the main warps
  Split<64, 32> SV;      // [i][SA^T (tau) | v^T (tau)]
  Split<64, 64> S0T;     // S0^T [j][i]
  Split<16, 32> MM;      // [t][Mrb[t][0..15] | Mrk[t][0..15]]
  __align__(16) float Tp[kChunk][kChunk];     // T [t][tau]
  __align__(16) float LakP[kChunk][kChunk];   // Lak [t][tau]
  __align__(16) float lam[kChunk][kN];        // L_t [t][j]
  __align__(16) float lamT[kN][kChunk + 4];   // L_t [j][t] (rows padded against bank conflicts)
  __align__(16) T rabkT[4][kN][kChunk + 8];   // r, a, b, k of the chunk [j][t]
  int mask;                     // reset bits of the chunk
  int unsafe;                   // decay out of range (or staging timed out): the unit is re-run exactly
};

template <typename T>
struct __align__(128) BwdSmem {
  Ctx<T> ctx[2];
  Split<64, 64> dSlT;    // dSl^T [j][i]                                        (main)
  Split<32, 32> G4;      // rows t: [dLab[t] | dLak[t]], rows 16 + t: [dMrb[t] | dMrk[t]]   (main)
  Split<16, 64> WC;      // W [tau][j]                         (context)
  Split<16, 16> XC;      // X [tau][t]                         (context)
  __align__(16) float Atf[kChunk][kN];      // At [t][j] in fp32     (context)
  __align__(16) float LabT[kChunk][S20];    // Lab^T [tau][t]   (context)
  __align__(128) float ck[kN * kN];         // checkpoint entering the chunk being built (tiled order)
  __align__(128) T stg[kIn][kChunk][kN];    // staged inputs of the chunk being built (TMA boxes)
  unsigned long long in_bar;                // staged inputs and checkpoint landed (one phase per staged chunk)
  unsigned long long u_bar, chain_bar, gg_bar, e_bar;   // main MMAs complete (one phase per chunk each)
  uint32_t tmem_base;
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

// Bounded wait on an MMA-completion barrier; a wait that runs out is recorded in the status word.
__device__ __forceinline__ void mma_wait(const BwdArgs& p, unsigned long long* bar, unsigned parity) {
  if (!mbar_wait_bounded(bar, parity, kWaitLimitNs) && p.status) atomicOr(p.status, kStatusWaitTimeout);
  tc::fence_after_sync();
}

// Causal and same-segment mask of one (t, tau) pair of the chunk.
__device__ __forceinline__ bool pair_ok(unsigned mask, int t, int tau, bool strict) {
  return (strict ? tau < t : tau <= t) && (mask & ((2u << t) - (2u << tau))) == 0u;
}

// Reset flag of token 16c + lane of batch row b (false past T, for c < 0 or without flags).
__device__ __forceinline__ bool reset_flag(const BwdArgs& p, int64_t b, int64_t c, int lane) {
  const int64_t t = c * kChunk + lane;
  return p.reset && c >= 0 && lane < kChunk && t < p.T && p.reset[b * p.T + t] != 0;
}

// Stage chunk c: the seven inputs of its tokens (one TMA box each; rows past T arrive as zeros, K1
// reads w there as 1) and, for c > 0, the checkpoint entering it (one bulk copy), issued by one
// thread on in_bar.
template <typename T>
__device__ __forceinline__ void stage(const BwdArgs& p, const InputMaps& tm, BwdSmem<T>& sm, int64_t unit, int64_t b,
                                      int64_t h, int64_t c, int64_t nc, int ktid) {
  if (ktid == 0) {
    if (!in_bounds(h < p.H && b < p.B && c >= 0 && c < nc && c * kChunk < p.T, p.status)) return;
    const unsigned ck_bytes = c > 0 ? unsigned(kN * kN * sizeof(float)) : 0u;
    mbar_arrive_expect_tx(&sm.in_bar, unsigned(kIn * kChunk * kN * sizeof(T)) + ck_bytes + p.extra_tx);
#pragma unroll
    for (int m = 0; m < kIn; ++m)
      tma_load_4d(&sm.stg[m][0][0], &tm.m[m], 0, int(h), int(c * kChunk), int(b), &sm.in_bar);
    if (c > 0 && range_ok((unit * nc + (c - 1)) * kN * kN, kN * kN, p.B * p.H * nc * kN * kN, p.status))
      bulk_g2s(sm.ck, p.ckpt + (unit * nc + (c - 1)) * kN * kN, ck_bytes, &sm.in_bar);
  }
}

// ------------------------------------------------------------------ context warps
// Decay products, decay-scaled operands, v, dy, S0^T, L_t and the raw r, a, b, k for the main
// warps' per-token outputs.  A wait for the staged data that runs out marks the chunk unsafe (the
// unit is then recomputed by the exact scan) and sets `timed_out`, after which nothing more is
// staged.
template <typename T>
__device__ __forceinline__ void context_operands(const BwdArgs& p, BwdSmem<T>& sm, Ctx<T>& cx, unsigned mask,
                                                 int64_t unit, int64_t c, int ktid, int len, unsigned parity,
                                                 bool& unsafe, bool& timed_out) {
  const int kw = ktid >> 5, lane = ktid & 31;
  const bool to = !mbar_wait_bounded(&sm.in_bar, parity, kWaitLimitNs);
  const T (*X)[kChunk][kN] = sm.stg;
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;

  // ---- pass B: thread = (token t, 8 channels from j0); one 16-byte core row per array
  bool bad = false;
  {
    const int t = (lane & 7) + 8 * (kw & 1), j0 = 8 * ((lane >> 3) + 4 * (kw >> 1));
    // L_{t-1} and L_t: products of the staged decays (rows past T count as w = 1)
    float L[8], Lp[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) Lp[u] = 1.f;
    for (int s2 = 0; s2 < t; ++s2) {
      float w[8];
      unpack16<T>(*reinterpret_cast<const uint4*>(&X[1][s2][j0]), w);
#pragma unroll
      for (int u = 0; u < 8; ++u) Lp[u] *= s2 < len ? w[u] : 1.f;
    }
    {
      float w[8];
      unpack16<T>(*reinterpret_cast<const uint4*>(&X[1][t][j0]), w);
      float wmin = 1.f, lmin = 1.f, lmax = 1.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float wu = t < len ? w[u] : 1.f;
        L[u] = Lp[u] * wu;
        wmin = fminf(wmin, wu);
        lmin = fminf(lmin, L[u]);
        lmax = fmaxf(lmax, L[u]);
      }
      bad = !(wmin >= 0.0625f && lmin >= 0x1p-40f && lmax <= 0x1p40f);
    }
    *reinterpret_cast<float4*>(&cx.lam[t][j0]) = make_float4(L[0], L[1], L[2], L[3]);
    *reinterpret_cast<float4*>(&cx.lam[t][j0 + 4]) = make_float4(L[4], L[5], L[6], L[7]);
    float in[kIn][8];
#pragma unroll
    for (int m = 0; m < kIn; ++m) unpack16<T>(*reinterpret_cast<const uint4*>(&X[m][t][j0]), in[m]);
    float at[8], rt[8], bh[8], kh[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float il = rcp_approx(L[u]);
      at[u] = in[4][u] * Lp[u];
      rt[u] = in[0][u] * L[u];
      bh[u] = in[5][u] * il;
      kh[u] = in[2][u] * il;
    }
    *reinterpret_cast<float4*>(&sm.Atf[t][j0]) = make_float4(at[0], at[1], at[2], at[3]);
    *reinterpret_cast<float4*>(&sm.Atf[t][j0 + 4]) = make_float4(at[4], at[5], at[6], at[7]);
#pragma unroll
    for (int u = 0; u < 8; ++u) {   // transposed copies for the per-key-channel outputs (exact)
      cx.lamT[j0 + u][t] = L[u];
      cx.rabkT[0][j0 + u][t] = Elt<T>::from_f32(in[0][u]);
      cx.rabkT[1][j0 + u][t] = Elt<T>::from_f32(in[4][u]);
      cx.rabkT[2][j0 + u][t] = Elt<T>::from_f32(in[5][u]);
      cx.rabkT[3][j0 + u][t] = Elt<T>::from_f32(in[2][u]);
    }
    put8(cx.AR, cb(t, j0, 64), at);
    put8(cx.AR, cb(16 + t, j0, 64), rt);
    put8(cx.BK, cb(t, j0, 64), bh);
    put8(cx.BK, cb(16 + t, j0, 64), kh);
    put8(cx.DYU, cb(t, j0, 64), in[6]);
    const bool m0t = t < fr;
#pragma unroll
    for (int u = 0; u < 8; ++u) {   // v^T and m0.dy^T: column t of rows j0..j0+7
      put1(cx.SV, cb(j0 + u, 16 + t, 32), in[3][u]);
      put1(cx.DUY, cb(j0 + u, 16 + t, 32), m0t ? in[6][u] : 0.f);
    }
  }
  const unsigned any_bad = __ballot_sync(0xffffffffu, bad), any_to = __ballot_sync(0xffffffffu, to);
  if (lane == 0) sm.kbad[kw] = (any_bad ? 1 : 0) | (any_to ? 2 : 0);
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  named_bar(1, 128);
  const int kb = sm.kbad[0] | sm.kbad[1] | sm.kbad[2] | sm.kbad[3];
  unsafe = kb != 0;
  timed_out = (kb & 2) != 0;
  // ---- pass C: S0^T [j][i] from the checkpoint (tiled order), s0 or zero; thread = 4 x (j, 8 i)
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int idx = ktid + 128 * u;
    const int j = (idx & 7) + 8 * (idx >> 6), i0 = 8 * ((idx >> 3) & 7);
    float s[8];
    if (c > 0) {   // rows i0..i0+7 of column j sit 16 floats apart in the tiled order
      const float* src = sm.ck + ckpt_off(i0, j);
#pragma unroll
      for (int e = 0; e < 8; ++e) s[e] = src[16 * e];
    } else if (p.s0 && range_ok((unit * kN + i0) * kN + j, 7 * kN + 1, p.B * p.H * kN * kN, p.status)) {
#pragma unroll
      for (int e = 0; e < 8; ++e) s[e] = p.s0[(unit * kN + i0 + e) * kN + j];
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) s[e] = 0.f;
    }
    put8(cx.S0T, cb(j, i0, 64), s);
  }
  tc::fence_smem_to_async();
  named_bar(1, 128);
  if (timed_out && ktid == 0 && p.status) atomicOr(p.status, kStatusWaitTimeout);
  if (ktid == 0) {
    cx.mask = int(mask);
    cx.unsafe = unsafe ? 1 : 0;
  }
}

// The rest of the context: Gram, T, W, X and SA^T (safe chunks only).
template <typename T>
__device__ __forceinline__ void context_products(BwdSmem<T>& sm, Ctx<T>& cx, unsigned mask, int ktid) {
  constexpr bool kExactIn = std::is_same<T, bf16>::value;   // v and dy have no lo half
  const int kw = ktid >> 5, lane = ktid & 31;
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;

  // ---- the masked Gram [At; Rt] [Bh; Kh]^T: warp kw computes block (kw / 2, kw % 2) of 16 x 16
  // (Lab, Lak, Mrb, Mrk), rows t, columns tau
  {
    const int mb = kw >> 1, nb = kw & 1, g = lane >> 2, c4 = lane & 3;
    float acc[2][4] = {};
    const uint32_t a_lo = uint32_t(sizeof(cx.AR.hi)), b_lo = uint32_t(sizeof(cx.BK.hi));
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      mma_split2(acc, afrag_k<64>(cx.AR.hi, 16 * mb, 16 * ks, lane), a_lo, false, false,
                 bfrag_k<64>(cx.BK.hi, 16 * nb, 16 * ks, lane), b_lo);
    const bool strict = mb == 0;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = g + 8 * hh, tau = 8 * nt + 2 * c4;
        const float v0 = pair_ok(mask, t, tau, strict) ? acc[nt][2 * hh] : 0.f;
        const float v1 = pair_ok(mask, t, tau + 1, strict) ? acc[nt][2 * hh + 1] : 0.f;
        if (kw == 0) {
          sm.LabT[tau][t] = v0;
          sm.LabT[tau + 1][t] = v1;
        } else if (kw == 1) {
          cx.LakP[t][tau] = v0;
          cx.LakP[t][tau + 1] = v1;
        } else {   // [Mrb | Mrk] row t: a split pair
          const int e = cb(t, 16 * nb + tau, 32);
          const __nv_bfloat162 hh2 = __floats2bfloat162_rn(v0, v1);
          const float2 hf = __bfloat1622float2(hh2);
          *reinterpret_cast<__nv_bfloat162*>(&cx.MM.hi[e]) = hh2;
          *reinterpret_cast<__nv_bfloat162*>(&cx.MM.lo[e]) = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
        }
      }
  }
  named_bar(1, 128);

  // ---- T = (I - Lab)^-1 by forward substitution, one column per thread (threads 0-15)
  if (ktid < kChunk) {
    const int cc = ktid;
    float u[kChunk];
#pragma unroll
    for (int t = 0; t < kChunk; ++t) u[t] = t == cc ? 1.f : 0.f;
#pragma unroll
    for (int tau = 0; tau < kChunk - 1; ++tau) {
#pragma unroll
      for (int t = tau + 1; t < kChunk; ++t) u[t] = fmaf(sm.LabT[tau][t], u[tau], u[t]);
    }
#pragma unroll
    for (int t = 0; t < kChunk; ++t) cx.Tp[t][cc] = u[t];
  }
  named_bar(1, 128);

  // ---- X = T Lak: thread -> (tau, two t); W = T m0.At: thread -> (tau, 8 j)
  {
    const int tau = ktid >> 3;
    if ((ktid & 7) < 2) {   // X row tau, columns 8 (ktid & 7) .. +7
      const int t0 = 8 * (ktid & 7);
      float x[8] = {};
#pragma unroll
      for (int s = 0; s < kChunk; ++s) {
        const float tv = cx.Tp[tau][s];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = fmaf(tv, cx.LakP[s][t0 + e], x[e]);
      }
      put8(sm.XC, cb(tau, t0, 16), x);
    }
    const int j0 = 8 * (ktid & 7);
    float w[8] = {};
#pragma unroll
    for (int t = 0; t < kChunk; ++t) {
      const float tv = t < fr ? cx.Tp[tau][t] : 0.f;
      const float4 a0 = *reinterpret_cast<const float4*>(&sm.Atf[t][j0]);
      const float4 a1 = *reinterpret_cast<const float4*>(&sm.Atf[t][j0 + 4]);
      w[0] = fmaf(tv, a0.x, w[0]); w[1] = fmaf(tv, a0.y, w[1]); w[2] = fmaf(tv, a0.z, w[2]); w[3] = fmaf(tv, a0.w, w[3]);
      w[4] = fmaf(tv, a1.x, w[4]); w[5] = fmaf(tv, a1.y, w[5]); w[6] = fmaf(tv, a1.z, w[6]); w[7] = fmaf(tv, a1.w, w[7]);
    }
    put8(sm.WC, cb(tau, j0, 64), w);
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  named_bar(1, 128);

  // ---- SA^T = S0 W^T + V^T X^T: warp kw computes rows i = 16 kw .. 16 kw + 15, columns tau
  {
    const int g = lane >> 2, c4 = lane & 3;
    float acc[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)   // S0 (stored as S0^T) times W^T, K = j
      mma_split2(acc, afrag_mn<64>(cx.S0T.hi, 16 * kw, 16 * ks, lane), uint32_t(sizeof(cx.S0T.hi)), true, false,
                 bfrag_k<64>(sm.WC.hi, 0, 16 * ks, lane), uint32_t(sizeof(sm.WC.hi)));
    mma_split2(acc, afrag_k<32>(cx.SV.hi, 16 * kw, 16, lane), uint32_t(sizeof(cx.SV.hi)), false, kExactIn,   // v^T X^T, K = t
               bfrag_k<16>(sm.XC.hi, 0, 0, lane), uint32_t(sizeof(sm.XC.hi)));
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = 16 * kw + g + 8 * hh, tau = 8 * nt + 2 * c4;
        const int e = cb(i, tau, 32);
        const float v0 = acc[nt][2 * hh], v1 = acc[nt][2 * hh + 1];
        const __nv_bfloat162 hh2 = __floats2bfloat162_rn(v0, v1);
        const float2 hf = __bfloat1622float2(hh2);
        *reinterpret_cast<__nv_bfloat162*>(&cx.SV.hi[e]) = hh2;
        *reinterpret_cast<__nv_bfloat162*>(&cx.SV.lo[e]) = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
      }
  }
  tc::fence_smem_to_async();
}

// ------------------------------------------------------------------ main warps
template <typename T>
__device__ __forceinline__ void main_chunk(const BwdArgs& p, BwdSmem<T>& sm, Ctx<T>& cx, int64_t b, int64_t h,
                                           int64_t t0, int len, int warp, int lane, uint32_t tmem, unsigned phase) {
  constexpr bool kExactIn = std::is_same<T, bf16>::value;   // v and dy have no lo half
  const uint32_t tlane = uint32_t(32 * warp) << 16;
  const unsigned mask = unsigned(cx.mask);
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
  const unsigned ls_bits = last_segment_bits(mask);
  const bool keep = mask == 0u;
  const int row = 16 * warp + (lane & 15);   // TMEM row of this thread (both halves of the warp)
  const int half = lane >> 4;                // which half of a row's columns this thread holds

  // ---- M1: dSl^T = L_15 dS^T (row j = row) into shared memory for the chain products.  This
  // thread holds columns 16 half + (0..15) and 32 + 16 half + (0..15) of its row.
  float d[32];
  {
    float x[16];
    tc::ld_16x32bx2_x16(tmem + tlane + kColDS, x);
#pragma unroll
    for (int e = 0; e < 16; ++e) d[e] = x[e];
    tc::ld_16x32bx2_x16(tmem + tlane + kColDS + 32, x);
#pragma unroll
    for (int e = 0; e < 16; ++e) d[16 + e] = x[e];
  }
  tc::wait_ld();
  {
    const float l15 = cx.lam[kChunk - 1][row];
#pragma unroll
    for (int e = 0; e < 32; ++e) d[e] *= l15;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = d[8 * q + e];
      put8(sm.dSlT, cb(row, 32 * (q >> 1) + 16 * half + 8 * (q & 1), 64), v);
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  named_bar(2, 128);

  // ---- M2: G1 = dSl [Bh|Kh]^T, G2 = dY^T [Mrb|Mrk]
  if (threadIdx.x == 0) {
    tc::fence_after_sync();
    mma3<32, 4>(tmem + kColG1, op<64, true>(sm.dSlT), op<64, false>(cx.BK), false);
    mma3<32, 1>(tmem + kColG2, op<64, true>(cx.DYU, kExactIn), op<32, true>(cx.MM), false);   // dy rows of DYU
    tc::commit(&sm.u_bar);
  }
  // while the tensor core works: keep.dSl^T back into TMEM (the start of dS0^T) and the L_15 term
  // keep.sum_i dSl o S0 of this key channel (each half of the row, then both halves added)
  float dl15 = 0.f;
  {
    if (keep) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float s0[8];
        get8(cx.S0T, cb(row, 32 * (q >> 1) + 16 * half + 8 * (q & 1), 64), s0);
#pragma unroll
        for (int e = 0; e < 8; ++e) dl15 = fmaf(d[8 * q + e], s0[e], dl15);
      }
    }
    dl15 += __shfl_xor_sync(0xffffffffu, dl15, 16);
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      float x[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = keep ? d[16 * h2 + e] : 0.f;
      tc::st_16x32bx2_x16(tmem + tlane + kColDS + 32 * h2, x);
    }
    tc::wait_st();
  }
  mma_wait(p, &sm.u_bar, phase & 1u);

  // ---- M3: dSA^T, dU^T = dSA^T T and dV^T per value channel i = row (FP32 cores); this thread holds
  // tokens 8 half .. 8 half + 7 of its row; dv out, dU into shared memory
  {
    float g1b[8], g1k[8], g2b[8], g2k[8];
    tc::ld_16x32bx2_x8(tmem + tlane + kColG1, g1b);
    tc::ld_16x32bx2_x8(tmem + tlane + kColG1 + 16, g1k);
    tc::ld_16x32bx2_x8(tmem + tlane + kColG2, g2b);
    tc::ld_16x32bx2_x8(tmem + tlane + kColG2 + 16, g2k);
    tc::wait_ld();
    const int i = row, tb = 8 * half;
    float dsa[16], du[8], dv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float mine = ((ls_bits >> (tb + e)) & 1u ? g1b[e] : 0.f) + g2b[e];
      const float other = __shfl_xor_sync(0xffffffffu, mine, 16);
      dsa[e] = half ? other : mine;
      dsa[8 + e] = half ? mine : other;
      du[e] = 0.f;
      dv[e] = ((ls_bits >> (tb + e)) & 1u ? g1k[e] : 0.f) + g2k[e];
    }
    // dU^T[i][tau] = sum_t dSA^T[i][t] T[t][tau] (T is stored with zeros above its diagonal)
#pragma unroll
    for (int t = 0; t < kChunk; ++t) {
      const float4 a = *reinterpret_cast<const float4*>(&cx.Tp[t][tb]);
      const float4 c = *reinterpret_cast<const float4*>(&cx.Tp[t][tb + 4]);
      du[0] = fmaf(dsa[t], a.x, du[0]); du[1] = fmaf(dsa[t], a.y, du[1]);
      du[2] = fmaf(dsa[t], a.z, du[2]); du[3] = fmaf(dsa[t], a.w, du[3]);
      du[4] = fmaf(dsa[t], c.x, du[4]); du[5] = fmaf(dsa[t], c.y, du[5]);
      du[6] = fmaf(dsa[t], c.z, du[6]); du[7] = fmaf(dsa[t], c.w, du[7]);
    }
    // dV^T[i][tau] += sum_t dU^T[i][t] Lak[t][tau] (Lak is zero on and above its diagonal)
#pragma unroll
    for (int t = 0; t < kChunk; ++t) {
      const float mine = du[t & 7], other = __shfl_xor_sync(0xffffffffu, mine, 16);
      const float dut = ((t >> 3) == half) ? mine : other;
      const float4 a = *reinterpret_cast<const float4*>(&cx.LakP[t][tb]);
      const float4 c = *reinterpret_cast<const float4*>(&cx.LakP[t][tb + 4]);
      dv[0] = fmaf(dut, a.x, dv[0]); dv[1] = fmaf(dut, a.y, dv[1]);
      dv[2] = fmaf(dut, a.z, dv[2]); dv[3] = fmaf(dut, a.w, dv[3]);
      dv[4] = fmaf(dut, c.x, dv[4]); dv[5] = fmaf(dut, c.y, dv[5]);
      dv[6] = fmaf(dut, c.z, dv[6]); dv[7] = fmaf(dut, c.w, dv[7]);
    }
    // dU: rows 16 + t of DYU (column i) and, masked to the tokens before the first reset, DUY
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      put1(cx.DYU, cb(16 + tb + e, i, 64), du[e]);
      v[e] = tb + e < fr ? du[e] : 0.f;
    }
    put8(cx.DUY, cb(i, tb, 32), v);
    T* dvp = static_cast<T*>(p.dv) + tok_off(b, t0 + tb, h, p.T, p.H) + i;
    const int64_t rs = p.H * kN, total = p.B * p.T * p.H * kN;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (tb + e < len && range_ok(tok_off(b, t0 + tb + e, h, p.T, p.H) + i, 1, total, p.status))
        *dvp = Elt<T>::from_f32(dv[e]);
      dvp += rs;
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  named_bar(2, 128);

  // ---- M4: rest of dS0^T; gradient Gram; the S0 and dSl parts of the key-space products
  if (threadIdx.x == 0) {
    tc::fence_after_sync();
    mma3<64, 1>(tmem + kColDS, op<64, true>(cx.AR, false, 16), op<32, false>(cx.DUY, kExactIn, 0, 16), true);
    mma3<64, 1>(tmem + kColDS, op<64, true>(cx.AR), op<32, false>(cx.DUY), true);   // dS0^T += Rt^T m0.dy + At^T m0.dU
    tc::commit(&sm.chain_bar);
    const auto SV_M = op<32, true>(cx.SV);
    mma3<32, 4>(tmem + kColGG, op<64, false>(cx.DYU), SV_M, false);   // [dY; dU] [SA^T | v^T]   (rows t, 16 + t)
    mma3<32, 4>(tmem + kColE, op<64, false>(cx.S0T), op<32, true>(cx.DUY), false);   // S0^T [m0.dU^T | m0.dy^T] (rows j)
    mma3<32, 4>(tmem + kColE + 64, op<64, false>(sm.dSlT), SV_M, false);       // dSl^T [SA^T | v^T]
    tc::commit(&sm.gg_bar);
  }
  mma_wait(p, &sm.gg_bar, phase & 1u);

  // ---- M5: masked gradient Gram into the B operand of the key-space products.  Warp 0 holds rows
  // t of [dMrb | dMrk] (causal), warp 1 rows t of [dLab | dLak] (strictly causal).
  if (warp < 2) {   // this thread: row t = lane % 16, columns 16 half .. 16 half + 15 (the b or the k block)
    float g[16];
    tc::ld_16x32bx2_x16(tmem + tlane + kColGG, g);
    tc::wait_ld();
    const int t = lane & 15;
    const bool strict = warp == 1;
#pragma unroll
    for (int tau = 0; tau < kChunk; ++tau) g[tau] = pair_ok(mask, t, tau, strict) ? g[tau] : 0.f;
    const int r = strict ? t : 16 + t;   // G4 rows t: [dLab | dLak]; rows 16 + t: [dMrb | dMrk]
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = g[8 * q + e];
      put8(sm.G4, cb(r, 16 * half + 8 * q, 32), v);
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  named_bar(2, 128);
  if (threadIdx.x == 0) {
    tc::fence_after_sync();
    const auto BK_M = op<64, true>(cx.BK), AR_M = op<64, true>(cx.AR);
    mma3<32, 2>(tmem + kColE, BK_M, op<32, false>(sm.G4), true);        // += [Bh^T|Kh^T] [dLab^T dMrb^T; dLak^T dMrk^T]
    mma3<32, 2>(tmem + kColE + 32, AR_M, op<32, true>(sm.G4), false);   // [At^T|Rt^T] [dLab dLak; dMrb dMrk]
    tc::commit(&sm.e_bar);
  }
  mma_wait(p, &sm.e_bar, phase & 1u);

  // ---- M6: per key channel j = row: da, dr, db, dk and dw over the chunk's tokens; this thread
  // holds tokens tb .. tb + 7 of its channel (tb = 8 half)
  {
    const int j = row, tb = 8 * half;
    float eA[8], eR[8], eB[8], eK[8], xb[8], xk[8];
    tc::ld_16x32bx2_x8(tmem + tlane + kColE, eA);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 16, eR);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 32, eB);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 48, eK);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 64, xb);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 80, xk);
    float Lr[9];   // L_{tb-1} .. L_{tb+7}
    {
      const float4 a = *reinterpret_cast<const float4*>(&cx.lamT[j][tb]);
      const float4 c = *reinterpret_cast<const float4*>(&cx.lamT[j][tb + 4]);
      Lr[1] = a.x; Lr[2] = a.y; Lr[3] = a.z; Lr[4] = a.w; Lr[5] = c.x; Lr[6] = c.y; Lr[7] = c.z; Lr[8] = c.w;
      Lr[0] = half ? cx.lamT[j][tb - 1] : 1.f;
    }
    float rr[8], ar[8], br[8], kr[8];
    unpack16<T>(*reinterpret_cast<const uint4*>(&cx.rabkT[0][j][tb]), rr);
    unpack16<T>(*reinterpret_cast<const uint4*>(&cx.rabkT[1][j][tb]), ar);
    unpack16<T>(*reinterpret_cast<const uint4*>(&cx.rabkT[2][j][tb]), br);
    unpack16<T>(*reinterpret_cast<const uint4*>(&cx.rabkT[3][j][tb]), kr);
    tc::wait_ld();
    float DL[8], il[8], e3 = 0.f, sumDL = 0.f, firstA = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const bool ls = (ls_bits >> (tb + e)) & 1u;
      il[e] = rcp_approx(Lr[e + 1]);
      const float at = ar[e] * Lr[e], rt = rr[e] * Lr[e + 1], bh = br[e] * il[e], kh = kr[e] * il[e];
      const float xbt = ls ? xb[e] : 0.f, xkt = ls ? xk[e] : 0.f;
      eB[e] += xbt;   // dBh
      eK[e] += xkt;   // dKh
      e3 = fmaf(xbt, bh, fmaf(xkt, kh, e3));
      DL[e] = fmaf(eR[e], rt, -fmaf(eB[e], bh, eK[e] * kh));
      const float a_t = eA[e] * at;    // dAt_t At_t, which belongs to d log L_{t-1}
      if (e > 0) DL[e - 1] += a_t; else firstA = a_t;
    }
    // token tb + 7 takes dAt At of token tb + 8 from the other half (none after token 15)
    const float nextA = __shfl_xor_sync(0xffffffffu, firstA, 16);
    if (!half) DL[7] += nextA;
#pragma unroll
    for (int e = 0; e < 8; ++e) sumDL += DL[e];
    e3 += __shfl_xor_sync(0xffffffffu, e3, 16);
    const float upper = __shfl_xor_sync(0xffffffffu, sumDL, 16);   // sum over tokens 8..15, for half 0
    float cum = dl15 + e3 + (half ? 0.f : upper);
    const int64_t rs = p.H * kN, o0 = tok_off(b, t0 + tb, h, p.T, p.H) + j;
    T* const gda = static_cast<T*>(p.da);
    T* const gdr = static_cast<T*>(p.dr);
    T* const gdb = static_cast<T*>(p.db);
    T* const gdk = static_cast<T*>(p.dk);
    T* const gdw = static_cast<T*>(p.dw);
#pragma unroll
    for (int e = 7; e >= 0; --e) {
      cum += DL[e];
      if (tb + e < len && range_ok(o0 + e * rs, 1, p.B * p.T * p.H * kN, p.status)) {
        const int64_t o = o0 + e * rs;
        gda[o] = Elt<T>::from_f32(eA[e] * Lr[e]);
        gdr[o] = Elt<T>::from_f32(eR[e] * Lr[e + 1]);
        gdb[o] = Elt<T>::from_f32(eB[e] * il[e]);
        gdk[o] = Elt<T>::from_f32(eK[e] * il[e]);
        gdw[o] = Elt<T>::from_f32(cum * (Lr[e] * il[e]));
      }
    }
  }
  tc::fence_before_sync();
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) chunk_bwd_kernel(const BwdArgs p, const __grid_constant__ InputMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  BwdSmem<T>& sm = *reinterpret_cast<BwdSmem<T>*>(smem_raw);

  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_main = warp < 4;
  const int ktid = tid - 128;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;

  if (tid == 0) {
#ifdef WKV7_DEBUG
    s_dbg_status = p.status;
#endif
    sm.stop = 0;
    mbar_init(&sm.in_bar, 1);
    mbar_init(&sm.u_bar, 1);
    mbar_init(&sm.chain_bar, 1);
    mbar_init(&sm.gg_bar, 1);
    mbar_init(&sm.e_bar, 1);
  }
  if (warp == 0) {   // 512 TMEM columns: this kernel runs one CTA per SM (its shared memory)
    tc::alloc(&sm.tmem_base, kTmemCols);
    tc::relinquish();
  }
  tc::fence_before_sync();
  cta_sync();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem_base;

  // The two roles run separate loops so that their register sets never overlap; both meet at
  // one CTA barrier per iteration (bar.sync 0, executed by all 256 threads).
  if (is_main) {
    // dS^T entering the last chunk: dsT transposed (row j = TMEM row 16 warp + lane), or zero
    {
      const int j = 16 * warp + lane;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float d[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          d[e] = (p.dsT && lane < 16 && range_ok((unit * kN + 16 * q4 + e) * kN + j, 1, p.B * p.H * kN * kN, p.status))
                     ? p.dsT[(unit * kN + 16 * q4 + e) * kN + j] : 0.f;
        tc::st_32x32b_x16(tmem + (uint32_t(32 * warp) << 16) + kColDS + 16 * q4, d);
      }
      tc::wait_st();
    }
    tc::fence_before_sync();
    cta_sync();   // prologue staged by the context warps
    bool flagged = false;
    unsigned phase = 0;
    for (int64_t it = 0; it <= nc; ++it) {
      if (it >= 1) {
        const int64_t c = nc - it;   // chunk whose gradients are computed now
        Ctx<T>& cx = sm.ctx[c & 1];   // the main warps own this buffer until the next CTA barrier
        if (cx.unsafe) {
          if (tid == 0) sm.stop = 1;
        } else {
          tc::fence_after_sync();
          const int64_t t0 = c * kChunk;
          main_chunk<T>(p, sm, cx, b, h, t0, int(min64(kChunk, p.T - t0)), warp, lane, tmem, phase);
          ++phase;
        }
      }
      cta_sync();
      if (sm.stop) {
        flagged = true;
        break;
      }
    }
    if (tid == 0 && p.unit_flags && range_ok(unit, 1, p.B * p.H, p.status)) p.unit_flags[unit] = flagged ? 1 : 0;
    if (!flagged && p.ds0) {   // every MMA of the last chunk completed before its e_bar phase
      tc::fence_after_sync();
      const int j = 16 * warp + lane;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float d[16];
        tc::ld_32x32b_x16(tmem + (uint32_t(32 * warp) << 16) + kColDS + 16 * q4, d);
        tc::wait_ld();
        if (lane < 16 && range_ok((unit * kN + 16 * q4) * kN + j, 15 * kN + 1, p.B * p.H * kN * kN, p.status)) {
#pragma unroll
          for (int e = 0; e < 16; ++e) p.ds0[(unit * kN + 16 * q4 + e) * kN + j] = d[e];
        }
      }
    }
  } else {
    unsigned mask_next;
    unsigned phase = 0;        // staging phase of the next wait
    bool pending = true;       // a staging was issued and not yet waited for
    bool timed_out = false;
    // prologue: stage the last chunk and fetch its reset flags
    stage<T>(p, tm, sm, unit, b, h, nc - 1, nc, ktid);
    mask_next = __ballot_sync(0xffffffffu, reset_flag(p, b, nc - 1, lane)) & 0xffffu;
    bool f_prev = reset_flag(p, b, nc - 2, lane);
    cta_sync();
    for (int64_t it = 0; it <= nc; ++it) {
      const int64_t c = nc - 1 - it;   // chunk whose context is built now
      if (c >= 0 && pending && !timed_out) {   // (an unsafe chunk stages nothing more: the unit stops)
        Ctx<T>& cx = sm.ctx[c & 1];
        const unsigned mask = mask_next;
        bool unsafe = false;
        context_operands<T>(p, sm, cx, mask, unit, c, ktid, int(min64(kChunk, p.T - c * kChunk)), phase & 1u, unsafe,
                            timed_out);
        if (!timed_out) {
          pending = false;
          ++phase;
        }
        // the staged inputs and checkpoint are consumed: prefetch the previous chunk
        if (c > 0 && !unsafe) {
          stage<T>(p, tm, sm, unit, b, h, c - 1, nc, ktid);
          pending = true;
          mask_next = __ballot_sync(0xffffffffu, f_prev) & 0xffffu;   // chunk c-1
          f_prev = reset_flag(p, b, c - 2, lane);
        }
        if (!unsafe) {
          context_products<T>(sm, cx, mask, ktid);
        }
      }
      cta_sync();
      if (sm.stop) break;
    }
    // copies issued but never waited for (the unit stopped early) must land before the CTA exits
    if (pending) mbar_wait_bounded(&sm.in_bar, phase & 1u, timed_out ? kWaitLimitNs / 100 : kWaitLimitNs);
  }
  // every MMA was waited for and every TMEM load is complete: release TMEM
  tc::fence_before_sync();
  cta_sync();
  tc::fence_after_sync();
  if (warp == 0) tc::dealloc(tmem, kTmemCols);
}

// One CTA per SM: the whole shared memory of an SM (227 KB per CTA at most, static part included).
static_assert(sizeof(BwdSmem<__nv_bfloat16>) + 1024 <= 227 * 1024, "backward shared memory exceeds one SM");

template <typename T>
cudaError_t launch(const BwdArgs& p, const InputMaps& tm, cudaStream_t stream) {
  const size_t smem = sizeof(BwdSmem<T>);
  cudaError_t e = cudaFuncSetAttribute(chunk_bwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  chunk_bwd_kernel<T><<<dim3(unsigned(p.B * p.H)), dim3(kThreads), smem, stream>>>(p, tm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_bwd(const BwdArgs& p, const InputMaps& tm, int dtype, cudaStream_t stream) {
  switch (dtype) {
    case 1: return launch<__nv_bfloat16>(p, tm, stream);
    case 2: return launch<__half>(p, tm, stream);
    default: return cudaErrorInvalidValue;   // f32 inputs run the exact scan backward
  }
}

}  // namespace wkv7
