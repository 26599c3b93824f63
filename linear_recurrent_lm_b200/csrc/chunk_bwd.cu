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
// carried gradient is dS^T (TMEM rows = key channel j), and the key-space gradients dAt^T, dRt^T,
// dBh^T, dKh^T have rows = j, so that one thread owns one key channel over all 16 tokens of the
// chunk and keeps the reverse sum for dw in its registers.  dU and dV come straight out of one
// product, GU = dSl BKx^T + dY^T [Qm | Vq] (rows = value channel i), because the chunk's small
// factors are folded into its operands beforehand: with Tl = ls.T and X = T Lak,
//   BKx = [Tl^T 0; (ls.X)^T diag(ls)] [Bh; Kh],   Qm = Mrb T,   Vq = Mrk + Mrb X,
// so that dU^T = dSA^T T = dSl (Tl^T Bh)^T + dY^T Qm and dV^T = ls.(dSl Kh^T) + dY^T Mrk + dU^T Lak
// = GU's second half.
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
// Work split: one CTA of 9 warps per (b,h) (about 200 KB of shared memory, so one CTA per SM),
// chunks in reverse, pipelined:
//   warps 4-7 ("context") for chunk c-1: stage its inputs (one TMA box per input) and its
//     checkpoint (one bulk copy) on an mbarrier with bounded waits, build the decay-scaled
//     operands, the masked Gram, T by substitution, the folded operands BKx, Qm, Vq, W and X, and
//     SA^T = S0 W^T + V^T X^T (warp-level split products) into one half of a double buffer;
//   warps 0-3 ("main") for chunk c: scale the carried dS^T, then read GU (dU, dV), mask the
//     gradient Gram and, per key channel, write da, dr, db, dk and dw;
//   warp 8 ("issue") for chunk c: one thread issues the tensor-core products as the main warps
//     hand their operands over (named barriers): GU; then the gradient Gram, dSl [SA^T|v^T], the
//     rest of dS0^T and S0^T [m0.dU^T | m0.dy^T]; then the Gram parts of the key-space products,
//     each batch committed to an mbarrier the main warps wait on.
// One CTA barrier per chunk hands the context over.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"

namespace wkv7 {
namespace {

constexpr int kThreads = 288;   // warps 0-3 main, 4-7 context, 8 issue
constexpr int kIssueTid = 256;  // the thread that issues every tensor-core product
constexpr int kIn = 7;   // r, w, k, v, a, b, dy
constexpr int S20 = 20;
using bf16 = __nv_bfloat16;

// TMEM columns (256 allocated; one CTA per SM).  Every accumulator has M = 64 rows.
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColDS = 0;      // dS^T                               (64; rows j)
constexpr uint32_t kColGU = 64;     // [dU^T | dV^T]                       (32; rows i)
constexpr uint32_t kColGG = 96;     // [dU; dY] [SA^T | v^T]               (32; rows t and 16 + t)
constexpr uint32_t kColE = 128;     // dAt^T | dRt^T | dBg^T | dKg^T | (SA dSl)^T | (V dSl)^T  (96; rows j)

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
// The same B fragments from a core array with rows = K, columns = N (read with ldmatrix.trans).
template <int Q>
__device__ __forceinline__ uint32_t bfrag_mn(const bf16* b, int n0, int k0, int lane) {
  const int mi = lane >> 3, r = lane & 7;
  return smem_u32(b + cb(k0 + (mi & 1) * 8 + r, n0 + (mi >> 1) * 8, Q));
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
// The lo addresses are the hi ones plus a fixed byte distance; a_exact skips the A lo half; a_mn and
// b_mn select the transposed (ldmatrix.trans) reads of the fragment helpers above.
__device__ __forceinline__ void mma_split2(float (&acc)[2][4], uint32_t a_hi, uint32_t a_lo_off, bool a_mn,
                                           bool a_exact, uint32_t b_hi, uint32_t b_lo_off, bool b_mn = false) {
  uint32_t ah[4], al[4], bh[4], bl[4];
  if (a_mn) ldsm4t(ah, a_hi); else ldsm4(ah, a_hi);
  if (b_mn) {
    ldsm4t(bh, b_hi);
    ldsm4t(bl, b_hi + b_lo_off);
  } else {
    ldsm4(bh, b_hi);
    ldsm4(bl, b_hi + b_lo_off);
  }
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

// Store two adjacent values (elements e and e + 1 of one core row) as their hi and lo halves.
template <int P, int Q>
__device__ __forceinline__ void put2(Split<P, Q>& m, int e, float v0, float v1) {
  if (!in_bounds(e >= 0 && e + 2 <= P * Q && (e & 1) == 0, debug_status())) return;
  const __nv_bfloat162 hh = __floats2bfloat162_rn(v0, v1);
  const float2 hf = __bfloat1622float2(hh);
  *reinterpret_cast<__nv_bfloat162*>(&m.hi[e]) = hh;
  *reinterpret_cast<__nv_bfloat162*>(&m.lo[e]) = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
}

// Produced by the context warps for one chunk, read by the main and issue warps one iteration
// later.  The order of the arrays matters: the 64-column read of UYT (32 columns) runs on into the
// arrays after it.
template <typename T>
struct __align__(128) Ctx {
  Split<32, 64> AR;      // rows 0-15 At [t][j], rows 16-31 Rt [t][j]
  Split<32, 64> BK;      // rows 0-15 Bh [tau][j], rows 16-31 Kh [tau][j]
  Split<64, 32> UYT;     // [i][dU^T (t) | dy^T (t)]: the dU half is written by the main warps
  Split<64, 32> DUY;     // [i][m0.dU^T (t) | m0.dy^T (t)]: the dU half is written by the main warps
  Split<64, 32> SV;      // [i][SA^T (tau) | v^T (tau)]
  Split<64, 64> S0T;     // S0^T [j][i]
  Split<32, 64> BKx;     // rows 0-15 (Tl^T Bh) [tau][j], rows 16-31 ((ls.X)^T Bh + ls.Kh) [tau][j]
  Split<16, 32> MMx;     // [t][Qm[t][0..15] | Vq[t][0..15]]
  __align__(16) float lam[kChunk][kN + 4];    // L_t [t][j] (rows padded: the float4 stores of 16 tokens
                                              // of one channel group fall in distinct banks)
  int mask;                     // reset bits of the chunk
  int unsafe;                   // decay out of range (or staging timed out): the unit is re-run exactly
};

template <typename T>
struct __align__(128) BwdSmem {
  Ctx<T> ctx[2];
  Split<64, 64> dSlT;    // dSl^T [j][i]                                        (main)
  Split<32, 32> G4;      // rows t: [dLab[t] | dLak[t]], rows 16 + t: [dMrb[t] | dMrk[t]]   (main)
  Split<16, 64> WC;      // W [tau][j]                                (context)
  Split<16, 16> XC;      // X [tau][t]                                (context)
  Split<32, 32> AC;      // [Tl^T 0; (ls.X)^T diag(ls)] [tau'][t']    (context)
  Split<16, 16> TmT;     // (T m0)^T [t][tau]                         (context)
  __align__(16) float LabT[kChunk][S20];     // Lab^T [tau][t]        (context)
  __align__(16) float Tp[kChunk][kChunk];    // T [t][tau]            (context)
  __align__(16) float LakP[kChunk][kChunk];  // Lak [t][tau]          (context)
  __align__(16) float MrbP[kChunk][kChunk];  // Mrb [t][tau]          (context)
  __align__(16) float MrkP[kChunk][kChunk];  // Mrk [t][tau]          (context)
  __align__(16) float Xp[kChunk][kChunk];    // X [t][tau]            (context)
  __align__(128) float ck[kN * kN];         // checkpoint entering the chunk being built (tiled order)
  __align__(128) T stg[kIn][kChunk][kN];    // staged inputs of the chunk being built (TMA boxes)
  __align__(128) float dyf[kChunk][kN];     // dy of that chunk when it comes from the epilogue's fp32 block
  unsigned long long in_bar;                // staged inputs and checkpoint landed (one phase per staged chunk)
  unsigned long long u_bar, gg_bar, e_bar;  // tensor-core batches complete (one phase per chunk each)
  uint32_t tmem_base;
  int kbad[4];
  int stop;
};

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void cta_sync() { asm volatile("bar.sync 0;\n" ::: "memory"); }

// Named barriers: 1 context warps; 3-5 main warps hand operands to the issue warp.
constexpr int kBarCtx = 1, kBarDsl = 3, kBarDu = 4, kBarG4 = 5;
constexpr int kHandOff = 128 + 32;   // main warps arrive, the issue warp waits

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

// Stage chunk c: the seven inputs of its tokens (one TMA box each, dy in fp32 when it comes from the
// epilogue's block; rows past T arrive as zeros, K1 reads w there as 1) and, for c > 0, the
// checkpoint entering it (one bulk copy), issued by one
// thread on in_bar.
template <typename T, bool kLog, bool kEpi>
__device__ __forceinline__ void stage(const BwdArgs& p, const InputMaps& tm, BwdSmem<T>& sm, int64_t unit, int64_t b,
                                      int64_t h, int64_t c, int64_t nc, int ktid) {
  if (ktid == 0) {
    if (!in_bounds(h < p.H && b < p.B && c >= 0 && c < nc && c * kChunk < p.T, p.status)) return;
    const unsigned ck_bytes = c > 0 ? unsigned(kN * kN * sizeof(float)) : 0u;
    const unsigned dy_bytes = unsigned(kChunk * kN * (kEpi ? sizeof(float) : sizeof(T)));
    mbar_arrive_expect_tx(&sm.in_bar, unsigned((kIn - 1) * kChunk * kN * sizeof(T)) + dy_bytes + ck_bytes + p.extra_tx);
#pragma unroll
    for (int m = 0; m < kIn; ++m) {
      void* dst = (m == kIn - 1 && kEpi) ? static_cast<void*>(&sm.dyf[0][0]) : static_cast<void*>(&sm.stg[m][0][0]);
      tma_load_4d(dst, &tm.m[m], 0, int(h), int(c * kChunk), int(b), &sm.in_bar);
    }
    if (c > 0 && range_ok((unit * nc + (c - 1)) * kN * kN, kN * kN, p.B * p.H * nc * kN * kN, p.status))
      bulk_g2s(sm.ck, p.ckpt + (unit * nc + (c - 1)) * kN * kN, ck_bytes, &sm.in_bar);
  }
}

// ------------------------------------------------------------------ context warps
// Decay products, decay-scaled operands, v, dy, S0^T and L_t.  A wait for the staged data that runs
// out marks the chunk unsafe (the unit is then recomputed by the exact scan) and sets `timed_out`,
// after which nothing more is staged.
template <typename T, bool kLog, bool kEpi>
__device__ __forceinline__ void context_operands(const BwdArgs& p, BwdSmem<T>& sm, Ctx<T>& cx, unsigned mask,
                                                 int64_t unit, int64_t c, int ktid, int len, unsigned parity,
                                                 bool& unsafe, bool& timed_out) {
  const int kw = ktid >> 5, lane = ktid & 31;
  const bool to = !mbar_wait_bounded(&sm.in_bar, parity, kWaitLimitNs);
  const T (*X)[kChunk][kN] = sm.stg;
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;

  // ---- pass B: thread = (token t, 8 channels from j0), the 16 tokens of a channel group in one
  // half-warp; one 16-byte core row per array
  bool bad = false;
  {
    const int t = lane & 15, j0 = 8 * ((lane >> 4) + 2 * kw);
    // L_t by a product scan over the half-warp (rows past T count as w = 1); L_{t-1} one lane up
    float L[8], Lp[8];
    {
      float w[8];
      unpack16<T>(*reinterpret_cast<const uint4*>(&X[1][t][j0]), w);
      float wmin = 1.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        L[u] = t < len ? decay_of(w[u], kLog) : 1.f;
        wmin = fminf(wmin, L[u]);
      }
#pragma unroll
      for (int d = 1; d < kChunk; d *= 2)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float o = __shfl_up_sync(0xffffffffu, L[u], d, 16);
          if (t >= d) L[u] *= o;
        }
      float lmin = 1.f, lmax = 1.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float o = __shfl_up_sync(0xffffffffu, L[u], 1, 16);
        Lp[u] = t >= 1 ? o : 1.f;
        lmin = fminf(lmin, L[u]);
        lmax = fmaxf(lmax, L[u]);
      }
      bad = !(wmin >= 0.0625f && lmin >= 0x1p-40f && lmax <= 0x1p40f);
    }
    float r8[8], k8[8], a8[8], b8[8];
    unpack16<T>(*reinterpret_cast<const uint4*>(&X[0][t][j0]), r8);
    unpack16<T>(*reinterpret_cast<const uint4*>(&X[2][t][j0]), k8);
    unpack16<T>(*reinterpret_cast<const uint4*>(&X[4][t][j0]), a8);
    unpack16<T>(*reinterpret_cast<const uint4*>(&X[5][t][j0]), b8);
    float at[8], rt[8], bh[8], kh[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float il = rcp_approx(L[u]);
      at[u] = a8[u] * Lp[u];
      rt[u] = r8[u] * L[u];
      bh[u] = b8[u] * il;
      kh[u] = k8[u] * il;
    }
    *reinterpret_cast<float4*>(&cx.lam[t][j0]) = make_float4(L[0], L[1], L[2], L[3]);
    *reinterpret_cast<float4*>(&cx.lam[t][j0 + 4]) = make_float4(L[4], L[5], L[6], L[7]);
    put8(cx.AR, cb(t, j0, 64), at);
    put8(cx.AR, cb(16 + t, j0, 64), rt);
    put8(cx.BK, cb(t, j0, 64), bh);
    put8(cx.BK, cb(16 + t, j0, 64), kh);
  }
  // ---- v^T, dy^T and m0.dy^T: thread = (channel i, tokens 8 th .. 8 th + 7), one core row each
  {
    const int i = ktid & 63, th = ktid >> 6;
    float v8[8], y8[8], m8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int t = 8 * th + e;
      v8[e] = Elt<T>::to_f32(X[3][t][i]);
      y8[e] = kEpi ? sm.dyf[t][i] : Elt<T>::to_f32(X[6][t][i]);
      m8[e] = t < fr ? y8[e] : 0.f;
    }
    put8(cx.SV, cb(i, 16 + 8 * th, 32), v8);
    put8(cx.UYT, cb(i, 16 + 8 * th, 32), y8);
    put8(cx.DUY, cb(i, 16 + 8 * th, 32), m8);
  }
  const unsigned any_bad = __ballot_sync(0xffffffffu, bad), any_to = __ballot_sync(0xffffffffu, to);
  if (lane == 0) sm.kbad[kw] = (any_bad ? 1 : 0) | (any_to ? 2 : 0);
  tc::fence_smem_to_async();
  named_bar(kBarCtx, 128);
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
  named_bar(kBarCtx, 128);
  if (timed_out && ktid == 0 && p.status) atomicOr(p.status, kStatusWaitTimeout);
  if (ktid == 0) {
    cx.mask = int(mask);
    cx.unsafe = unsafe ? 1 : 0;
  }
}

// The rest of the context (safe chunks only): the masked Gram, T, X, the folded operands BKx, Qm,
// Vq and W, and SA^T.
template <typename T, bool kLog, bool kEpi>
__device__ __forceinline__ void context_products(const BwdArgs& p, const InputMaps& tm, BwdSmem<T>& sm, Ctx<T>& cx,
                                                 unsigned mask, int ktid, int64_t unit, int64_t b, int64_t h,
                                                 int64_t c_stage, int64_t nc) {
  constexpr bool kExactIn = std::is_same<T, bf16>::value;   // v and dy have no lo half
  const int kw = ktid >> 5, lane = ktid & 31;
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
  const unsigned ls_bits = last_segment_bits(mask);

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
    float (*dst)[kChunk] = kw == 1 ? sm.LakP : kw == 2 ? sm.MrbP : sm.MrkP;
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
        } else {
          *reinterpret_cast<float2*>(&dst[t][tau]) = make_float2(v0, v1);
        }
      }
  }
  named_bar(kBarCtx, 128);

  // ---- T = (I - Lab)^-1 by forward substitution, one column cc per thread (threads 0-15), which
  // also writes row cc of Tl^T (the top-left block of AC) and of (T m0)^T; threads 16-31 write the
  // right-hand blocks of AC (zero above, diag(ls) below); thread 32 stages the next chunk (the
  // staged inputs and checkpoint of this one are consumed)
  if (ktid < kChunk) {
    const int cc = ktid;
    float u[kChunk];
#pragma unroll
    for (int t = 0; t < kChunk; ++t) u[t] = t == cc ? 1.f : 0.f;
    // whole rows of Lab^T: its entries on and left of the diagonal are zero, so they add nothing
#pragma unroll
    for (int tau = 0; tau < kChunk - 1; ++tau) {
      float l[kChunk];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(&sm.LabT[tau][4 * q]);
        l[4 * q] = v.x; l[4 * q + 1] = v.y; l[4 * q + 2] = v.z; l[4 * q + 3] = v.w;
      }
#pragma unroll
      for (int t = tau + 1; t < kChunk; ++t) u[t] = fmaf(l[t], u[tau], u[t]);
    }
#pragma unroll
    for (int t = 0; t < kChunk; ++t) sm.Tp[t][cc] = u[t];
    const float m0c = cc < fr ? 1.f : 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float tl[8], tm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int t = 8 * q + e;
        tl[e] = (ls_bits >> t) & 1u ? u[t] : 0.f;   // Tl^T[cc][t] = ls_t T[t][cc]
        tm[e] = m0c * u[t];                         // (T m0)^T[cc][tau] = T[tau][cc] m0_cc
      }
      put8(sm.AC, cb(cc, 8 * q, 32), tl);
      put8(sm.TmT, cb(cc, 8 * q, 16), tm);
    }
  } else if (ktid < 2 * kChunk) {
    const int tau = ktid - kChunk;
    const float lt = (ls_bits >> tau) & 1u ? 1.f : 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float z[8], d[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        z[e] = 0.f;
        d[e] = 8 * q + e == tau ? lt : 0.f;
      }
      put8(sm.AC, cb(tau, 16 + 8 * q, 32), z);
      put8(sm.AC, cb(16 + tau, 16 + 8 * q, 32), d);
    }
  } else if (c_stage >= 0) {
    stage<T, kLog, kEpi>(p, tm, sm, unit, b, h, c_stage, nc, ktid - 2 * kChunk);
  }
  named_bar(kBarCtx, 128);

  // ---- X = T Lak (threads 0-31) and Qm = Mrb T (threads 32-63): thread -> (row r, 8 columns)
  if (ktid < 4 * kChunk) {
    const int r = (ktid >> 1) & 15, c0 = 8 * (ktid & 1);
    const bool isx = ktid < 2 * kChunk;
    const float (*A)[kChunk] = isx ? sm.Tp : sm.MrbP;
    const float (*B)[kChunk] = isx ? sm.LakP : sm.Tp;
    float x[8] = {};
#pragma unroll
    for (int s = 0; s < kChunk; ++s) {
      const float av = A[r][s];
      const float4 b0 = *reinterpret_cast<const float4*>(&B[s][c0]);
      const float4 b1 = *reinterpret_cast<const float4*>(&B[s][c0 + 4]);
      x[0] = fmaf(av, b0.x, x[0]); x[1] = fmaf(av, b0.y, x[1]); x[2] = fmaf(av, b0.z, x[2]); x[3] = fmaf(av, b0.w, x[3]);
      x[4] = fmaf(av, b1.x, x[4]); x[5] = fmaf(av, b1.y, x[5]); x[6] = fmaf(av, b1.z, x[6]); x[7] = fmaf(av, b1.w, x[7]);
    }
    if (isx) {
      put8(sm.XC, cb(r, c0, 16), x);
      *reinterpret_cast<float4*>(&sm.Xp[r][c0]) = make_float4(x[0], x[1], x[2], x[3]);
      *reinterpret_cast<float4*>(&sm.Xp[r][c0 + 4]) = make_float4(x[4], x[5], x[6], x[7]);
    } else {
      put8(cx.MMx, cb(r, c0, 32), x);
    }
  }
  named_bar(kBarCtx, 128);

  // ---- Vq = Mrk + Mrb X (threads 0-31) and the (ls.X)^T block of AC (threads 32-63)
  if (ktid < 2 * kChunk) {
    const int r = ktid >> 1, c0 = 8 * (ktid & 1);
    float x[8];
    {
      const float4 m0v = *reinterpret_cast<const float4*>(&sm.MrkP[r][c0]);
      const float4 m1v = *reinterpret_cast<const float4*>(&sm.MrkP[r][c0 + 4]);
      x[0] = m0v.x; x[1] = m0v.y; x[2] = m0v.z; x[3] = m0v.w; x[4] = m1v.x; x[5] = m1v.y; x[6] = m1v.z; x[7] = m1v.w;
    }
#pragma unroll
    for (int s = 0; s < kChunk; ++s) {
      const float av = sm.MrbP[r][s];
      const float4 b0 = *reinterpret_cast<const float4*>(&sm.Xp[s][c0]);
      const float4 b1 = *reinterpret_cast<const float4*>(&sm.Xp[s][c0 + 4]);
      x[0] = fmaf(av, b0.x, x[0]); x[1] = fmaf(av, b0.y, x[1]); x[2] = fmaf(av, b0.z, x[2]); x[3] = fmaf(av, b0.w, x[3]);
      x[4] = fmaf(av, b1.x, x[4]); x[5] = fmaf(av, b1.y, x[5]); x[6] = fmaf(av, b1.z, x[6]); x[7] = fmaf(av, b1.w, x[7]);
    }
    put8(cx.MMx, cb(r, 16 + c0, 32), x);
  } else if (ktid < 4 * kChunk) {   // AC[16 + tau][t] = ls_t X[t][tau]
    const int tau = (ktid - 2 * kChunk) >> 1, t0 = 8 * (ktid & 1);
    float z[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) z[e] = (ls_bits >> (t0 + e)) & 1u ? sm.Xp[t0 + e][tau] : 0.f;
    put8(sm.AC, cb(16 + tau, t0, 32), z);
  }
  named_bar(kBarCtx, 128);

  // ---- W = (T m0) At (warp kw: columns 16 kw .. 16 kw + 15) and BKx = AC [Bh; Kh] (warp kw: rows
  // 16 (kw % 2) .., columns 32 (kw / 2) ..), warp-level split products
  {
    const int g = lane >> 2, c4 = lane & 3;
    {
      float acc[2][4] = {};
      mma_split2(acc, afrag_mn<16>(sm.TmT.hi, 0, 0, lane), uint32_t(sizeof(sm.TmT.hi)), true, false,
                 bfrag_mn<64>(cx.AR.hi, 16 * kw, 0, lane), uint32_t(sizeof(cx.AR.hi)), true);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          put2(sm.WC, cb(g + 8 * hh, 16 * kw + 8 * nt + 2 * c4, 64), acc[nt][2 * hh], acc[nt][2 * hh + 1]);
    }
    const int mb = kw & 1, n0 = 32 * (kw >> 1);
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      float acc[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        mma_split2(acc, afrag_k<32>(sm.AC.hi, 16 * mb, 16 * ks, lane), uint32_t(sizeof(sm.AC.hi)), false, false,
                   bfrag_mn<64>(cx.BK.hi, n0 + 16 * np, 16 * ks, lane), uint32_t(sizeof(cx.BK.hi)), true);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          put2(cx.BKx, cb(16 * mb + g + 8 * hh, n0 + 16 * np + 8 * nt + 2 * c4, 64), acc[nt][2 * hh],
               acc[nt][2 * hh + 1]);
    }
  }
  named_bar(kBarCtx, 128);

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
      for (int hh = 0; hh < 2; ++hh)
        put2(cx.SV, cb(16 * kw + g + 8 * hh, 8 * nt + 2 * c4, 32), acc[nt][2 * hh], acc[nt][2 * hh + 1]);
  }
  tc::fence_smem_to_async();
}

// ------------------------------------------------------------------ issue warp
// One thread issues every tensor-core product of chunk c, in three batches, each as soon as the
// main warps have handed over its operands (named barriers kBarDsl, kBarDu, kBarG4).
template <typename T>
__device__ __forceinline__ void issue_chunk(BwdSmem<T>& sm, Ctx<T>& cx, uint32_t tmem, bool leader, bool dy_exact) {
  named_bar(kBarDsl, kHandOff);
  if (leader) {
    tc::fence_after_sync();
    // GU = dSl BKx^T + dY^T [Qm | Vq]                          (rows i: dU^T | dV^T)
    mma3<32, 4>(tmem + kColGU, op<64, true>(sm.dSlT), op<64, false>(cx.BKx), false);
    mma3<32, 1>(tmem + kColGU, op<32, false>(cx.UYT, dy_exact, 0, 16), op<32, true>(cx.MMx), true);   // dy^T
    tc::commit(&sm.u_bar);
  }
  named_bar(kBarDu, kHandOff);
  if (leader) {
    tc::fence_after_sync();
    mma3<32, 4>(tmem + kColGG, op<32, true>(cx.UYT), op<32, true>(cx.SV), false);   // [dU; dY] [SA^T | v^T]
    tc::commit(&sm.gg_bar);
    mma3<32, 4>(tmem + kColE + 64, op<64, false>(sm.dSlT), op<32, true>(cx.SV), false);   // dSl^T [SA^T | v^T]
    // dS0^T += Rt^T m0.dy + At^T m0.dU (the carried gradient of the chunk before)
    mma3<64, 1>(tmem + kColDS, op<64, true>(cx.AR, false, 16), op<32, false>(cx.DUY, dy_exact, 0, 16), true);
    mma3<64, 1>(tmem + kColDS, op<64, true>(cx.AR), op<32, false>(cx.DUY), true);
    mma3<32, 4>(tmem + kColE, op<64, false>(cx.S0T), op<32, true>(cx.DUY), false);   // S0^T [m0.dU^T | m0.dy^T]
  }
  named_bar(kBarG4, kHandOff);
  if (leader) {
    tc::fence_after_sync();
    mma3<32, 2>(tmem + kColE, op<64, true>(cx.BK), op<32, false>(sm.G4), true);        // += [Bh^T|Kh^T] [dLab^T dMrb^T; dLak^T dMrk^T]
    mma3<32, 2>(tmem + kColE + 32, op<64, true>(cx.AR), op<32, true>(sm.G4), false);   // [At^T|Rt^T] [dLab dLak; dMrb dMrk]
    tc::commit(&sm.e_bar);
  }
}

// ------------------------------------------------------------------ main warps
template <typename T, bool kLog, bool kEpi>
__device__ __forceinline__ void main_chunk(const BwdArgs& p, BwdSmem<T>& sm, Ctx<T>& cx, int64_t b, int64_t h,
                                           int64_t t0, int len, int warp, int lane, uint32_t tmem, unsigned phase) {
  const uint32_t tlane = uint32_t(32 * warp) << 16;
  const unsigned mask = unsigned(cx.mask);
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
  const unsigned ls_bits = last_segment_bits(mask);
  const bool keep = mask == 0u;
  const int row = 16 * warp + (lane & 15);   // TMEM row of this thread (both halves of the warp)
  const int half = lane >> 4;                // which half of a row's columns this thread holds
  const int tb = 8 * half;                   // first token of this thread in per-token phases
  const int64_t rs = p.H * kN, total = p.B * p.T * p.H * kN;

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
  named_arrive(kBarDsl, kHandOff);

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

  // ---- M3: dU^T and dV^T of value channel i = row for tokens tb .. tb + 7, straight from GU; dU
  // into shared memory (UYT, and DUY masked to the tokens before the first reset), dv out
  {
    float du[8], dv[8];
    tc::ld_16x32bx2_x8(tmem + tlane + kColGU, du);
    tc::ld_16x32bx2_x8(tmem + tlane + kColGU + 16, dv);
    tc::wait_ld();
    const int i = row;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = tb + e < fr ? du[e] : 0.f;
    put8(cx.UYT, cb(i, tb, 32), du);
    put8(cx.DUY, cb(i, tb, 32), v);
    T* dvp = static_cast<T*>(p.dv) + tok_off(b, t0 + tb, h, p.T, p.H) + i;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (tb + e < len && range_ok(tok_off(b, t0 + tb + e, h, p.T, p.H) + i, 1, total, p.status))
        *dvp = Elt<T>::from_f32(kEpi ? dv[e] + static_cast<const float*>(p.dy)[3 * total + tok_off(b, t0 + tb + e, h, p.T, p.H) + i]
                                      : dv[e]);   // + the epilogue's bonus part
      dvp += rs;
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  named_arrive(kBarDu, kHandOff);

  // r, a, b, k of this thread's key channel and tokens for the last phase (cache hits: the context
  // staged the same rows one chunk earlier), loaded while the tensor core works
  const int j = row;
  const int64_t o0 = tok_off(b, t0 + tb, h, p.T, p.H) + j;
  float rr[8], ar[8], br[8], kr[8], xw[8], er[8], ek[8];
  {
    const float* const eg = static_cast<const float*>(p.dy);   // the epilogue's block, under kEpi
    const T* const gw = static_cast<const T*>(p.w);
    const T* const gr = static_cast<const T*>(p.r);
    const T* const ga = static_cast<const T*>(p.a);
    const T* const gb = static_cast<const T*>(p.b);
    const T* const gk = static_cast<const T*>(p.k);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int64_t o = o0 + e * rs;
      const bool ok = tb + e < len && range_ok(o, 1, total, p.status);
      rr[e] = ok ? Elt<T>::to_f32(gr[o]) : 0.f;
      ar[e] = ok ? Elt<T>::to_f32(ga[o]) : 0.f;
      br[e] = ok ? Elt<T>::to_f32(gb[o]) : 0.f;
      kr[e] = ok ? Elt<T>::to_f32(gk[o]) : 0.f;
      xw[e] = ok && kLog ? Elt<T>::to_f32(gw[o]) : 0.f;   // x, for dL/dx
      er[e] = ok && kEpi ? eg[total + o] : 0.f;                 // bonus parts of dr, dk
      ek[e] = ok && kEpi ? eg[2 * total + o] : 0.f;
    }
  }
  mma_wait(p, &sm.gg_bar, phase & 1u);

  // ---- M5: masked gradient Gram into the B operand of the key-space products.  Warp 0 holds rows
  // t of [dLab | dLak] (strictly causal), warp 1 rows t of [dMrb | dMrk] (causal).
  if (warp < 2) {   // this thread: row t = lane % 16, columns 16 half .. 16 half + 15 (the b or the k block)
    float g[16];
    tc::ld_16x32bx2_x16(tmem + tlane + kColGG, g);
    tc::wait_ld();
    const int t = lane & 15;
    const bool strict = warp == 0;
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
  named_arrive(kBarG4, kHandOff);
  mma_wait(p, &sm.e_bar, phase & 1u);

  // ---- M6: per key channel j = row: da, dr, db, dk and dw over the chunk's tokens; this thread
  // holds tokens tb .. tb + 7 of its channel
  {
    float eA[8], eR[8], eB[8], eK[8], xb[8], xk[8];
    tc::ld_16x32bx2_x8(tmem + tlane + kColE, eA);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 16, eR);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 32, eB);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 48, eK);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 64, xb);
    tc::ld_16x32bx2_x8(tmem + tlane + kColE + 80, xk);
    float Lr[9];   // L_{tb-1} .. L_{tb+7}
#pragma unroll
    for (int e = 0; e < 8; ++e) Lr[e + 1] = cx.lam[tb + e][j];
    Lr[0] = half ? cx.lam[tb - 1][j] : 1.f;
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
    T* const gda = static_cast<T*>(p.da);
    T* const gdr = static_cast<T*>(p.dr);
    T* const gdb = static_cast<T*>(p.db);
    T* const gdk = static_cast<T*>(p.dk);
    T* const gdw = static_cast<T*>(p.dw);
#pragma unroll
    for (int e = 7; e >= 0; --e) {
      cum += DL[e];
      if (tb + e < len && range_ok(o0 + e * rs, 1, total, p.status)) {
        const int64_t o = o0 + e * rs;
        gda[o] = Elt<T>::from_f32(eA[e] * Lr[e]);
        gdr[o] = Elt<T>::from_f32(kEpi ? fmaf(eR[e], Lr[e + 1], er[e]) : eR[e] * Lr[e + 1]);
        gdb[o] = Elt<T>::from_f32(eB[e] * il[e]);
        gdk[o] = Elt<T>::from_f32(kEpi ? fmaf(eK[e], il[e], ek[e]) : eK[e] * il[e]);
        // cum = dL/d(log w_t): dw = cum / w_t = cum L_{t-1} / L_t, or dL/dx = -cum exp(x)
        gdw[o] = Elt<T>::from_f32(kLog ? dx_of_dlogw(cum, xw[e]) : cum * (Lr[e] * il[e]));
      }
    }
  }
  tc::fence_before_sync();
}

template <typename T, bool kLog, bool kEpi>
__global__ void __launch_bounds__(kThreads, 1) chunk_bwd_kernel(const BwdArgs p, const __grid_constant__ InputMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  BwdSmem<T>& sm = *reinterpret_cast<BwdSmem<T>*>(smem_raw);

  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ktid = tid - 128;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;

  if (tid == 0) {
#ifdef WKV7_DEBUG
    s_dbg_status = p.status;
#endif
    sm.stop = 0;
    mbar_init(&sm.in_bar, 1);
    mbar_init(&sm.u_bar, 1);
    mbar_init(&sm.gg_bar, 1);
    mbar_init(&sm.e_bar, 1);
  }
  if (warp == 0) {   // this kernel runs one CTA per SM (its shared memory)
    tc::alloc(&sm.tmem_base, kTmemCols);
    tc::relinquish();
  }
  tc::fence_before_sync();
  cta_sync();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem_base;

  // The three roles run separate loops so that their register sets never overlap; all meet at one
  // CTA barrier per iteration (bar.sync 0, executed by all 288 threads).
  if (warp < 4) {
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
    int64_t first_done = nc;   // first chunk whose gradients were written
    for (int64_t it = 0; it <= nc; ++it) {
      if (it >= 1) {
        const int64_t c = nc - it;   // chunk whose gradients are computed now
        Ctx<T>& cx = sm.ctx[c & 1];   // the main and issue warps own this buffer until the next CTA barrier
        if (cx.unsafe) {
          if (tid == 0) sm.stop = 1;
          first_done = c + 1;
        } else {
          tc::fence_after_sync();
          const int64_t t0 = c * kChunk;
          main_chunk<T, kLog, kEpi>(p, sm, cx, b, h, t0, int(min64(kChunk, p.T - t0)), warp, lane, tmem, phase);
          ++phase;
        }
      }
      cta_sync();
      if (sm.stop) {
        flagged = true;
        break;
      }
    }
    if (tid == 0 && p.unit_flags && range_ok(unit, 1, p.B * p.H, p.status))
      p.unit_flags[unit] = flagged ? int(first_done + 1) : 0;
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
  } else if (warp < 8) {
    unsigned mask_next;
    unsigned phase = 0;        // staging phase of the next wait
    bool pending = true;       // a staging was issued and not yet waited for
    bool timed_out = false;
    // prologue: stage the last chunk and fetch its reset flags
    stage<T, kLog, kEpi>(p, tm, sm, unit, b, h, nc - 1, nc, ktid);
    mask_next = __ballot_sync(0xffffffffu, reset_flag(p, b, nc - 1, lane)) & 0xffffu;
    bool f_prev = reset_flag(p, b, nc - 2, lane);
    cta_sync();
    for (int64_t it = 0; it <= nc; ++it) {
      const int64_t c = nc - 1 - it;   // chunk whose context is built now
      if (c >= 0 && pending && !timed_out) {   // (an unsafe chunk stages nothing more: the unit stops)
        Ctx<T>& cx = sm.ctx[c & 1];
        const unsigned mask = mask_next;
        bool unsafe = false;
        context_operands<T, kLog, kEpi>(p, sm, cx, mask, unit, c, ktid, int(min64(kChunk, p.T - c * kChunk)), phase & 1u, unsafe,
                            timed_out);
        if (!timed_out) {
          pending = false;
          ++phase;
        }
        // the staged inputs and checkpoint are consumed: the previous chunk is staged during the
        // products (by a thread idle there)
        if (c > 0 && !unsafe) {
          pending = true;
          mask_next = __ballot_sync(0xffffffffu, f_prev) & 0xffffu;   // chunk c-1
          f_prev = reset_flag(p, b, c - 2, lane);
        }
        if (!unsafe) {
          context_products<T, kLog, kEpi>(p, tm, sm, cx, mask, ktid, unit, b, h, c > 0 ? c - 1 : -1, nc);
        }
      }
      cta_sync();
      if (sm.stop) break;
    }
    // copies issued but never waited for (the unit stopped early) must land before the CTA exits
    if (pending) mbar_wait_bounded(&sm.in_bar, phase & 1u, timed_out ? kWaitLimitNs / 100 : kWaitLimitNs);
  } else {
    cta_sync();   // prologue
    for (int64_t it = 0; it <= nc; ++it) {
      if (it >= 1) {
        const int64_t c = nc - it;
        Ctx<T>& cx = sm.ctx[c & 1];
        // dy has no lo half when it arrives in bf16 (exact); the epilogue's fp32 dy has one
        if (!cx.unsafe) issue_chunk<T>(sm, cx, tmem, tid == kIssueTid, std::is_same<T, bf16>::value && !kEpi);
      }
      cta_sync();
      if (sm.stop) break;
    }
  }
  // every MMA was waited for and every TMEM load is complete: release TMEM
  tc::fence_before_sync();
  cta_sync();
  tc::fence_after_sync();
  if (warp == 0) tc::dealloc(tmem, kTmemCols);
}

// One CTA per SM: the whole shared memory of an SM (227 KB per CTA at most, static part included).
static_assert(sizeof(BwdSmem<__nv_bfloat16>) + 1024 <= 227 * 1024, "backward shared memory exceeds one SM");

// The log-space decay and the epilogue's gradient block are template parameters: the kernel without
// them has none of their code in its hot loops.
template <typename T, bool kLog, bool kEpi>
cudaError_t launch_t(const BwdArgs& p, const InputMaps& tm, cudaStream_t stream) {
  const size_t smem = sizeof(BwdSmem<T>);
  cudaError_t e = cudaFuncSetAttribute(chunk_bwd_kernel<T, kLog, kEpi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  chunk_bwd_kernel<T, kLog, kEpi><<<dim3(unsigned(p.B * p.H)), dim3(kThreads), smem, stream>>>(p, tm);
  return cudaGetLastError();
}
template <typename T>
cudaError_t launch(const BwdArgs& p, const InputMaps& tm, cudaStream_t stream) {
  if (p.log_decay) return p.epi ? launch_t<T, true, true>(p, tm, stream) : launch_t<T, true, false>(p, tm, stream);
  return p.epi ? launch_t<T, false, true>(p, tm, stream) : launch_t<T, false, false>(p, tm, stream);
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
