// WKV-7 forward for few (b,h) units in two phases (algo CHUNKED, split form).
//
// The fused chunked forward (chunk_fwd.cu) runs one CTA per (b,h) unit and is bound by the
// latency of its per-chunk chain; with fewer units than SMs most of the GPU idles.  Everything in
// a chunk that does not depend on the entering state S0 can instead be built for all chunks at
// once -- the chunk-parallel form the HF model card page mentions -- leaving a short sequential
// chain per unit (notation of chunk_fwd.cu: L_t, At, Rt, Bh, Kh, masks m0 and ls, keep):
//
//   phase 1 (chunk_prep_kernel; one CTA per full chunk, every chunk in parallel), from the
//   inputs alone: the decay products, the masked Gram, T = (I - Lab)^-1 and
//       W  = T diag(m0) At,        Q  = m0.Rt + Mrb T diag(m0) At,    Z = Mrk + Mrb T Lak,
//       Bl = ls.Bh,                Kx = (T Lak)^T Bl + ls.Kh,         L_15;
//   phase 2 (chunk_chain_kernel; one CTA per unit, chunks in order), with S0 the state entering
//   the chunk (rows i across four warps as fp32 accumulator fragments):
//       SA0^T = S0 W^T,   Y^T = S0 Q^T + V^T Z^T,
//       S_16  = (keep.S0 + SA0^T Bl + V^T Kx) diag(L_15).
// SA0^T Bl + V^T Kx is the fused form's SA^T Bl + V^T Kl with SA = W S0^T + (T Lak) V split into
// its S0 part and its V part; all products are tf32 mma.sync with fp32 accumulation, operands
// rounded to tf32 (nearest), as in the fused kernel.
//
// Phase 1 hands its results over in memory the call already owns: W, Q, Bl^T and Kx^T fill the
// chunk's 16 KiB checkpoint slot exactly, and Z, L_15 and a completion marker go into the first
// 128 bytes of each of the chunk's 16 rows of y.  Phase 2 reads both (cp.async, two chunks
// ahead) before it writes y and the chunk-end checkpoint over them.  A chunk whose decay product
// leaves [2^-40, 2^40] gets no operands (phase 1 writes marker 0) and, like a ragged last chunk,
// is run token by token in phase 2.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "token_path.cuh"

namespace wkv7 {
namespace {

constexpr int kThreads = 128;
constexpr int kIn = 6;   // r, w, k, v, a, b
constexpr int S68 = 68, S20 = 20, S72 = 72, S24 = 24;
constexpr int kStrY = 72;
constexpr int kRing = 3;   // phase 2 operand buffers (chunks in flight)
constexpr uint32_t kMarker = 0x5A11C0DEu;

// Float offsets inside a checkpoint slot while it carries phase 1's operands.
constexpr int kOffW = 0;       // W    [t][j]   16 x 64
constexpr int kOffQ = 1024;    // Q    [t][j]   16 x 64
constexpr int kOffBl = 2048;   // Bl^T [j][tau] 64 x 16
constexpr int kOffKx = 3072;   // Kx^T [j][tau] 64 x 16
// In row t of the chunk's y (viewed as floats): [0,16) = Z[t][0..15], [16,32) = ext[t][0..15]
// with ext[0][0] = marker, ext[1..4] = L_15[16(t-1) .. 16(t-1)+15].

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
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
__device__ __forceinline__ uint32_t fu(float x) { return __float_as_uint(x); }
// Reset bits of the chunk at t0 (every lane of the calling warp gets them).
__device__ __forceinline__ unsigned chunk_mask(const FwdArgs& p, int64_t b, int64_t t0, int len, int lane) {
  const bool f = p.reset && lane < len && p.reset[b * p.T + t0 + lane] != 0;
  return __ballot_sync(0xffffffffu, f) & 0xffffu;
}

// ------------------------------------------------------------------ phase 1
template <typename T>
struct __align__(16) PrepSmem {
  T in[kIn][kChunk][kN];     // staged inputs [m][t][j]
  float GA[32][S68];         // rows 0..15 at_t, 16..31 rt_t   [t][j]   (tf32)
  float GB[32][S68];         // rows 0..15 bh_t, 16..31 kh_t   [tau][j] (tf32)
  float Rt[kChunk][S68];     // m0 . rt (fp32)
  float AtT[kN][S20];        // at [j][tau]
  float LabT[kChunk][S20], LakT[kChunk][S20], Mrb[kChunk][S20], Mrk[kChunk][S20];
  float Tm[kChunk][S20], TT[kChunk][S20], M[kChunk][S20], X[kChunk][S20];
  float Z[kChunk][kChunk];
  float lam15[kN];
  __align__(16) float out[4096];   // the checkpoint slot image: W | Q | Bl^T | Kx^T
  int kbad[4];
};

template <typename T>
__global__ void __launch_bounds__(kThreads) chunk_prep_kernel(const FwdArgs p, int64_t nfull) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PrepSmem<T>& sm = *reinterpret_cast<PrepSmem<T>*>(smem_raw);
  const int64_t item = blockIdx.x;
  const int64_t unit = item / nfull, c = item - (item / nfull) * nfull;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;
  const int64_t t0 = c * kChunk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  if (!in_bounds(unit < p.B * p.H && c < nfull && t0 + kChunk <= p.T, p.status)) return;   // (debug build)
  const int64_t act_total = p.B * p.T * p.H * kN;

  // ---- stage the six inputs of the chunk (16 rows of 64 elements each)
  {
    constexpr int kPieces = kN * int(sizeof(T)) / 16;   // 16-byte pieces per row
    const void* src[kIn] = {p.r, p.w, p.k, p.v, p.a, p.b};
    for (int idx = tid; idx < kIn * kChunk * kPieces; idx += kThreads) {
      const int m = idx / (kChunk * kPieces), rem = idx - m * (kChunk * kPieces);
      const int t = rem / kPieces, piece = rem - t * kPieces;
      const int64_t o = tok_off(b, t0 + t, h, p.T, p.H) + piece * (16 / int(sizeof(T)));
      if (range_ok(o, 16 / int(sizeof(T)), act_total, p.status))
        cp_async16(&sm.in[m][t][piece * (16 / int(sizeof(T)))], static_cast<const T*>(src[m]) + o);
    }
    cp_async_commit();
  }
  const unsigned mask = chunk_mask(p, b, t0, kChunk, lane);
  const int fr = mask ? __ffs(int(mask)) - 1 : kChunk;
  const unsigned m0bits = (1u << fr) - 1u;
  const unsigned ls_bits = last_segment_bits(mask);
  cp_async_wait_all();
  __syncthreads();

  // ---- K1: decay products and decay-scaled operands.  Thread = (token quarter `warp`; columns
  // lane and lane + 32).
  bool bad = false;
  {
    const int tq = 4 * warp, ja = lane, jb = lane + 32;
    auto ld2 = [&](int m, int t) {
      return make_float2(Elt<T>::to_f32(sm.in[m][t][ja]), Elt<T>::to_f32(sm.in[m][t][jb]));
    };
    auto ldw = [&](int t) {
      const float2 x = ld2(1, t);
      return make_float2(decay_of(x.x, p.log_decay), decay_of(x.y, p.log_decay));
    };
    float2 lam = make_float2(1.f, 1.f);   // L_{tq-1}
    for (int t = 0; t < tq; ++t) lam = mul2(lam, ldw(t));
    float bl[2][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = tq + u;
      const float2 lp = lam;
      lam = mul2(lam, ldw(t));
      bad |= !(lam.x >= 0x1p-40f && lam.x <= 0x1p40f) || !(lam.y >= 0x1p-40f && lam.y <= 0x1p40f);
      const float2 inv = make_float2(rcp_approx(lam.x), rcp_approx(lam.y));
      const float2 a2 = mul2(ld2(4, t), lp), r2 = mul2(ld2(0, t), lam);
      const float2 b2 = mul2(ld2(5, t), inv), k2 = mul2(ld2(2, t), inv);
      const float atx = tf32f(a2.x), aty = tf32f(a2.y);
      const float bhx = tf32f(b2.x), bhy = tf32f(b2.y);
      sm.GA[t][ja] = atx;
      sm.GA[t][jb] = aty;
      sm.GA[16 + t][ja] = tf32f(r2.x);
      sm.GA[16 + t][jb] = tf32f(r2.y);
      sm.GB[t][ja] = bhx;
      sm.GB[t][jb] = bhy;
      sm.GB[16 + t][ja] = tf32f(k2.x);
      sm.GB[16 + t][jb] = tf32f(k2.y);
      sm.Rt[t][ja] = t < fr ? r2.x : 0.f;
      sm.Rt[t][jb] = t < fr ? r2.y : 0.f;
      sm.AtT[ja][t] = atx;
      sm.AtT[jb][t] = aty;
      const float ls = (ls_bits >> t) & 1u ? 1.f : 0.f;
      bl[0][u] = ls * bhx;
      bl[1][u] = ls * bhy;
    }
    // Bl^T rows j, four consecutive tau: one float4 each
    *reinterpret_cast<float4*>(&sm.out[kOffBl + ja * kChunk + tq]) = make_float4(bl[0][0], bl[0][1], bl[0][2], bl[0][3]);
    *reinterpret_cast<float4*>(&sm.out[kOffBl + jb * kChunk + tq]) = make_float4(bl[1][0], bl[1][1], bl[1][2], bl[1][3]);
    if (warp == 3) {
      sm.lam15[ja] = lam.x;
      sm.lam15[jb] = lam.y;
    }
  }
  const unsigned any_bad = __ballot_sync(0xffffffffu, bad);
  if (lane == 0) sm.kbad[warp] = any_bad ? 1 : 0;
  __syncthreads();
  float* yrow0 = reinterpret_cast<float*>(static_cast<T*>(p.y) + tok_off(b, t0, h, p.T, p.H));
  if (sm.kbad[0] | sm.kbad[1] | sm.kbad[2] | sm.kbad[3]) {   // token path in phase 2
    if (tid == 0) reinterpret_cast<uint32_t*>(yrow0)[kChunk] = 0u;
    return;
  }

  // ---- K2: 32x32 Gram of [at; rt] and [bh; kh] (tf32), masked; warp = 16x16 block
  {
    const int m0 = (warp >> 1) * 16, n0 = (warp & 1) * 16;
    float gr[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a[4], bb[4];
      ldsm_x4(a, a32_addr(&sm.GA[0][0], S68, m0, 8 * ks, lane));
      ldsm_x4(bb, b32_2n_addr(&sm.GB[0][0], S68, n0, 8 * ks, lane));
      mma1688(gr[0], a, bb[0], bb[1]);
      mma1688(gr[1], a, bb[2], bb[3]);
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
        const float v = ok ? gr[nt][e] : 0.f;
        if (warp == 0) sm.LabT[tau][t] = v;
        else if (warp == 1) sm.LakT[tau][t] = tf32f(v);
        else if (warp == 2) sm.Mrb[t][tau] = tf32f(v);
        else sm.Mrk[t][tau] = v;
      }
  }
  __syncthreads();

  // ---- K3: T = (I - Lab)^-1 by forward substitution, one column per lane (warp 0, lanes 0-15)
  if (warp == 0 && lane < kChunk) {
    const int cc = lane;
    float u[kChunk];
#pragma unroll
    for (int t = 0; t < kChunk; ++t) u[t] = t == cc ? 1.f : 0.f;
#pragma unroll
    for (int tau = 0; tau < kChunk - 1; ++tau) {
#pragma unroll
      for (int t = tau + 1; t < kChunk; ++t) u[t] = fmaf(sm.LabT[tau][t], u[tau], u[t]);
    }
#pragma unroll
    for (int t = 0; t < kChunk; ++t) {
      const float v = tf32f(u[t]);
      sm.Tm[t][cc] = v;
      sm.TT[cc][t] = v;
    }
  }
  __syncthreads();

  const int j0 = 16 * warp;   // this warp's 16 key columns in the 16 x 64 products
  // ---- step a: W = T diag(m0) At (columns j0..j0+15), M = Mrb T (warp 0), X = T Lak (warp 1)
  uint32_t bat[2][4];   // At^T fragments of this warp's columns: [n-tile][k-step pair]
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) ldsm_x4(bat[nt], b32_2k_addr(&sm.AtT[0][0], S20, j0 + 8 * nt, 0, lane));
  {
    uint32_t at[2][4];
#pragma unroll
    for (int s = 0; s < 2; ++s) ldsm_x4(at[s], a32_addr(&sm.Tm[0][0], S20, 0, 8 * s, lane));
    if (warp == 1) {
      float xx[2][4] = {};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t bl[4];
        ldsm_x4(bl, b32_2k_addr(&sm.LakT[0][0], S20, 8 * nt, 0, lane));
        mma1688(xx[nt], at[0], bl[0], bl[1]);
        mma1688(xx[nt], at[1], bl[2], bl[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<float2*>(&sm.X[g + 8 * hh][8 * nt + 2 * c4]) =
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
        *reinterpret_cast<float2*>(&sm.out[kOffW + (g + 8 * hh) * kN + j0 + 8 * nt + 2 * c4]) =
            make_float2(tf32f(ww[nt][2 * hh]), tf32f(ww[nt][2 * hh + 1]));
    if (warp == 0) {
      uint32_t am[2][4];
#pragma unroll
      for (int s = 0; s < 2; ++s) ldsm_x4(am[s], a32_addr(&sm.Mrb[0][0], S20, 0, 8 * s, lane));
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
  __syncthreads();

  // ---- step b: Q = m0.Rt + M diag(m0) At (columns j0..), Z = Mrk + M Lak (warp 2);
  //      step c: Kx = X^T Bl + ls.Kh (columns j0..)
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
          const float2 m2 = *reinterpret_cast<const float2*>(&sm.Mrk[g + 8 * hh][8 * nt + 2 * c4]);
          zz[nt][2 * hh] = m2.x;
          zz[nt][2 * hh + 1] = m2.y;
        }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t bl[4];
        ldsm_x4(bl, b32_2k_addr(&sm.LakT[0][0], S20, 8 * nt, 0, lane));
        mma1688(zz[nt], am[0], bl[0], bl[1]);
        mma1688(zz[nt], am[1], bl[2], bl[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<float2*>(&sm.Z[g + 8 * hh][8 * nt + 2 * c4]) =
              make_float2(tf32f(zz[nt][2 * hh]), tf32f(zz[nt][2 * hh + 1]));
    }
    mask_nat(am[0], 0, c4, m0bits);
    mask_nat(am[1], 1, c4, m0bits);
    float qq[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float2 r2 = *reinterpret_cast<const float2*>(&sm.Rt[g + 8 * hh][j0 + 8 * nt + 2 * c4]);
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
        *reinterpret_cast<float2*>(&sm.out[kOffQ + (g + 8 * hh) * kN + j0 + 8 * nt + 2 * c4]) =
            make_float2(tf32f(qq[nt][2 * hh]), tf32f(qq[nt][2 * hh + 1]));

    // Kx[tau][j] = sum_t X[t][tau] Bl[t][j] + ls_tau kh[tau][j]: A = X^T (m = tau, k = t), B = Bl (k = t, n = j)
    float kx[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tau = g + 8 * (e >> 1), j = j0 + 8 * nt + 2 * c4 + (e & 1);
        kx[nt][e] = (ls_bits >> tau) & 1u ? sm.GB[16 + tau][j] : 0.f;
      }
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int k0 = 8 * s + c4;   // t of a0/a1; a2/a3 at t + 4
      const uint32_t ax[4] = {fu(sm.X[k0][g]), fu(sm.X[k0][g + 8]), fu(sm.X[k0 + 4][g]), fu(sm.X[k0 + 4][g + 8])};
      const float l0 = (ls_bits >> k0) & 1u ? 1.f : 0.f, l1 = (ls_bits >> (k0 + 4)) & 1u ? 1.f : 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int n = j0 + 8 * nt + g;
        mma1688(kx[nt], ax, fu(l0 * sm.GB[k0][n]), fu(l1 * sm.GB[k0 + 4][n]));
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tau = g + 8 * (e >> 1), j = j0 + 8 * nt + 2 * c4 + (e & 1);
        sm.out[kOffKx + j * kChunk + tau] = tf32f(kx[nt][e]);
      }
  }
  __syncthreads();

  // ---- hand over: the slot image (16 KiB, coalesced), then Z, L_15 and the marker in the y rows
  {
    float4* slot = reinterpret_cast<float4*>(p.ckpt + (unit * nc + c) * (kN * kN));
    const float4* src = reinterpret_cast<const float4*>(sm.out);
    if (range_ok((unit * nc + c) * (kN * kN), kN * kN, p.B * p.H * nc * (kN * kN), p.status))
#pragma unroll
      for (int u = 0; u < 4096 / 4 / kThreads; ++u) slot[tid + u * kThreads] = src[tid + u * kThreads];
    const int t = tid >> 3, part = tid & 7;   // y row t, 16-byte piece `part` of its first 128 bytes
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (part < 4) {
      v = *reinterpret_cast<const float4*>(&sm.Z[t][4 * part]);
    } else if (t >= 1 && t <= 4) {
      v = *reinterpret_cast<const float4*>(&sm.lam15[16 * (t - 1) + 4 * (part - 4)]);
    } else if (t == 0 && part == 4) {
      v.x = __uint_as_float(kMarker);
    }
    float* yrow = reinterpret_cast<float*>(static_cast<T*>(p.y) + tok_off(b, t0 + t, h, p.T, p.H));
    if (range_ok(tok_off(b, t0 + t, h, p.T, p.H) * int64_t(sizeof(T)) + 16 * part, 16, act_total * int64_t(sizeof(T)),
                 p.status))
      *reinterpret_cast<float4*>(yrow + 4 * part) = v;
  }
}

// ------------------------------------------------------------------ phase 2
template <typename T>
struct __align__(16) ChainBuf {
  float W[kChunk][S72];     // [t][j]
  float Q[kChunk][S72];
  float BlT[kN][S24];       // [j][tau]
  float KxT[kN][S24];
  float Z[kChunk][S24];     // [t][tau]
  float ext[kChunk][16];    // marker, L_15
  T v[kChunk][kN];          // v rows of the chunk [tau][i]
};

template <typename T>
struct __align__(16) ChainSmem {
  ChainBuf<T> buf[kRing];
  __align__(16) T Ys[kChunk][kStrY];   // y of the chunk [t][i]
};

// Per-thread sources of phase 2's copies, fixed for the whole sequence: chunk c reads the same rows
// c * 16 tokens further on, and its checkpoint slot c * 4096 floats further on.
template <typename T>
struct StagePlan {
  static constexpr int kPieces = kN * int(sizeof(T)) / 16;   // 16-byte pieces per row of v
  static constexpr int kVPer = kChunk * kPieces / kThreads;   // pieces of v per thread per chunk
  const float* slot0;        // checkpoint slot of chunk 0 of this unit
  const T* yrow0;            // y row (token tid/8) of chunk 0
  const T* vrow0[kVPer];     // v rows of this thread's pieces, chunk 0
  int64_t chunk_elems;       // elements from a row to the same row of the next chunk
  // debug build: the buffers' starts and extents the copies are checked against
  const float* ckpt;
  const T *ybuf, *vbuf;
  int64_t ck_total, act_total;
  int* status;
};

// Issue the copies of chunk c's operands into `bf` (full chunks only; always one commit group).  The
// 16 KiB slot is contiguous: float 4i of it lands in W|Q (rows padded to 72) for i < 512, in
// Bl^T|Kx^T (rows padded to 24) above.
template <typename T>
__device__ __forceinline__ void chain_stage(const StagePlan<T>& sp, ChainBuf<T>& bf, int64_t c, int64_t nfull,
                                            int tid) {
  if (c < nfull) {
    const float* slot = sp.slot0 + c * (kN * kN);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = tid + k * kThreads;
      float* dst;
      if (k < 4) {
        const int q = i >> 8, t = (i >> 4) & 15, piece = i & 15;
        dst = &bf.W[0][0] + q * (kChunk * S72) + t * S72 + 4 * piece;
      } else {
        const int q = (i >> 8) - 2, j = (i >> 2) & 63, piece = i & 3;
        dst = &bf.BlT[0][0] + q * (kN * S24) + j * S24 + 4 * piece;
      }
      if (range_ok(slot + 4 * i - sp.ckpt, 4, sp.ck_total, sp.status)) cp_async16(dst, slot + 4 * i);
    }
    const int64_t off = c * sp.chunk_elems;
    const int part = tid & 7;
    const float* yrow = reinterpret_cast<const float*>(sp.yrow0 + off);
    if (range_ok((sp.yrow0 + off - sp.ybuf) + 16 * part / int(sizeof(T)), 16 / int(sizeof(T)), sp.act_total, sp.status))
      cp_async16(part < 4 ? &bf.Z[tid >> 3][4 * part] : &bf.ext[tid >> 3][4 * (part - 4)], yrow + 4 * part);
#pragma unroll
    for (int k = 0; k < StagePlan<T>::kVPer; ++k) {
      const int idx = tid + k * kThreads;
      const int t = idx / StagePlan<T>::kPieces, piece = idx - t * StagePlan<T>::kPieces;
      const T* src = sp.vrow0[k] + off + piece * (16 / int(sizeof(T)));
      if (range_ok(src - sp.vbuf, 16 / int(sizeof(T)), sp.act_total, sp.status))
        cp_async16(&bf.v[t][piece * (16 / int(sizeof(T)))], src);
    }
  }
  cp_async_commit();
}

// The eight float4 of a checkpoint in the tiled order.
__device__ __forceinline__ void store_ck(float* ck, const float (&acc)[8][4]) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
    *reinterpret_cast<float4*>(ck + nt * 128) = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) chunk_chain_kernel(const FwdArgs p, int64_t nfull) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ChainSmem<T>& sm = *reinterpret_cast<ChainSmem<T>*>(smem_raw);
  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int row0 = 16 * warp;
  if (!in_bounds(unit < p.B * p.H && nfull * kChunk <= p.T, p.status)) return;   // (debug build)
  const int64_t act_total = p.B * p.T * p.H * kN, st_total = p.B * p.H * kN * kN;

  // state fragments: acc[nt][e] = S[16*warp + g + 8*(e>>1)][8*nt + 2*c4 + (e&1)]
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float2 v2 = make_float2(0.f, 0.f);
      const int64_t so = (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4;
      if (p.s0 && range_ok(so, 2, st_total, p.status)) v2 = *reinterpret_cast<const float2*>(p.s0 + so);
      acc[nt][2 * hh] = v2.x;
      acc[nt][2 * hh + 1] = v2.y;
    }

  StagePlan<T> sp;
  sp.slot0 = p.ckpt + unit * nc * (kN * kN);
  sp.chunk_elems = int64_t(kChunk) * p.H * kN;
  sp.ckpt = p.ckpt;
  sp.ybuf = static_cast<const T*>(p.y);
  sp.vbuf = static_cast<const T*>(p.v);
  sp.ck_total = p.B * p.H * nc * (kN * kN);
  sp.act_total = act_total;
  sp.status = p.status;
  sp.yrow0 = static_cast<const T*>(p.y) + tok_off(b, tid >> 3, h, p.T, p.H);
#pragma unroll
  for (int k = 0; k < StagePlan<T>::kVPer; ++k)
    sp.vrow0[k] = static_cast<const T*>(p.v) + tok_off(b, (tid + k * kThreads) / StagePlan<T>::kPieces, h, p.T, p.H);
  T* const ybase = static_cast<T*>(p.y) + tok_off(b, 0, h, p.T, p.H);   // token 0 of this (b,h)
  const int64_t tok_stride = p.H * kN;

#pragma unroll
  for (int k = 0; k < kRing - 1; ++k) chain_stage<T>(sp, sm.buf[k], k, nfull, tid);

  for (int64_t c = 0; c < nc; ++c) {
    // the buffer of chunk c - 1 is free (barrier at the end of the last iteration): refill it
    chain_stage<T>(sp, sm.buf[(c + kRing - 1) % kRing], c + kRing - 1, nfull, tid);
    cp_async_wait_group<kRing - 1>();
    __syncthreads();
    const ChainBuf<T>& bf = sm.buf[c % kRing];
    const int64_t t0 = c * kChunk;
    const int len = int(min64(kChunk, p.T - t0));
    const unsigned mask = chunk_mask(p, b, t0, len, lane);
    const bool ready = c < nfull && __float_as_uint(bf.ext[0][0]) == kMarker;
    float* ck = range_ok((unit * nc + c) * (kN * kN), kN * kN, sp.ck_total, p.status)
                    ? p.ckpt + (unit * nc + c) * (kN * kN) + warp * 1024 + lane * 4 : nullptr;

    if (!ready) {
      state_chunk_tokens<T>(p, mask, acc, b, h, t0, len, warp, lane);
      __syncthreads();   // every thread's reads of this chunk's operand slot (none) and y rows are done
      if (ck) store_ck(ck, acc);
      continue;
    }

    // S0 as tf32 A fragments (accumulator tile read with the permuted k order)
    uint32_t aS[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      aS[ks][0] = to_tf32(acc[ks][0]);
      aS[ks][1] = to_tf32(acc[ks][2]);
      aS[ks][2] = to_tf32(acc[ks][1]);
      aS[ks][3] = to_tf32(acc[ks][3]);
    }
    // V^T as tf32 A fragments (rows i of this warp, k = tau in the permuted order)
    uint32_t aV[2][4];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int tau = 8 * s + 2 * c4;
      aV[s][0] = to_tf32(Elt<T>::to_f32(bf.v[tau][row0 + g]));
      aV[s][1] = to_tf32(Elt<T>::to_f32(bf.v[tau][row0 + g + 8]));
      aV[s][2] = to_tf32(Elt<T>::to_f32(bf.v[tau + 1][row0 + g]));
      aV[s][3] = to_tf32(Elt<T>::to_f32(bf.v[tau + 1][row0 + g + 8]));
    }

    // SA0^T = S0 W^T (the chain) and Y^T = S0 Q^T + V^T Z^T
    float sa[2][4] = {}, yt[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float2 wv = *reinterpret_cast<const float2*>(&bf.W[8 * nt + g][8 * ks + 2 * c4]);
        mma1688(sa[nt], aS[ks], fu(wv.x), fu(wv.y));
      }
    // D = SA0^T Bl + V^T Kx
    float d[8][4] = {};
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float2 kv = *reinterpret_cast<const float2*>(&bf.KxT[8 * nt + g][8 * s + 2 * c4]);
        mma1688(d[nt], aV[s], fu(kv.x), fu(kv.y));
      }
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const uint32_t aA[4] = {to_tf32(sa[s][0]), to_tf32(sa[s][2]), to_tf32(sa[s][1]), to_tf32(sa[s][3])};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float2 bv = *reinterpret_cast<const float2*>(&bf.BlT[8 * nt + g][8 * s + 2 * c4]);
        mma1688(d[nt], aA, fu(bv.x), fu(bv.y));
      }
    }
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float2 qv = *reinterpret_cast<const float2*>(&bf.Q[8 * nt + g][8 * ks + 2 * c4]);
        mma1688(yt[nt], aS[ks], fu(qv.x), fu(qv.y));
      }
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float2 zv = *reinterpret_cast<const float2*>(&bf.Z[8 * nt + g][8 * s + 2 * c4]);
        mma1688(yt[nt], aV[s], fu(zv.x), fu(zv.y));
      }

    // ---- S_16 = (keep.S0 + D) diag(L_15)
    const float keep = mask == 0u ? 1.f : 0.f;
#pragma unroll
    for (int jt = 0; jt < 8; ++jt) {
      const int j = 8 * jt + 2 * c4;
      const float2 l2 = *reinterpret_cast<const float2*>(&bf.ext[1 + (j >> 4)][j & 15]);
      acc[jt][0] = fmaf(keep * acc[jt][0], l2.x, d[jt][0] * l2.x);
      acc[jt][1] = fmaf(keep * acc[jt][1], l2.y, d[jt][1] * l2.y);
      acc[jt][2] = fmaf(keep * acc[jt][2], l2.x, d[jt][2] * l2.x);
      acc[jt][3] = fmaf(keep * acc[jt][3], l2.y, d[jt][3] * l2.y);
    }
    // ---- y: Y^T fragments -> Ys[t][i], then whole rows out (over the consumed scratch)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sm.Ys[8 * nt + 2 * c4 + (e & 1)][row0 + g + 8 * (e >> 1)] = Elt<T>::from_f32(yt[nt][e]);
    __syncthreads();   // Ys complete; every read of this chunk's operand slot is done
    {
      constexpr int kPieces = kN * int(sizeof(T)) / 16;
#pragma unroll
      for (int idx = tid; idx < kChunk * kPieces; idx += kThreads) {
        const int t = idx / kPieces, piece = idx - t * kPieces;
        T* dst = ybase + (t0 + t) * tok_stride + piece * (16 / int(sizeof(T)));
        if (range_ok(dst - static_cast<T*>(p.y), 16 / int(sizeof(T)), act_total, p.status))
          *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(&sm.Ys[t][piece * (16 / int(sizeof(T)))]);
      }
    }
    if (ck) store_ck(ck, acc);
  }
  cp_async_wait_all();   // the empty groups past the last chunk
  if (p.s_out) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int64_t so = (unit * kN + row0 + g + 8 * hh) * kN + 8 * nt + 2 * c4;
        if (range_ok(so, 2, st_total, p.status))
          *reinterpret_cast<float2*>(p.s_out + so) = make_float2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
      }
  }
}

template <typename T>
cudaError_t launch(const FwdArgs& p, cudaStream_t stream) {
  const int64_t units = p.B * p.H;
  const int64_t nfull = p.T / kChunk;
  cudaError_t e;
  if (nfull > 0) {
    const size_t s1 = sizeof(PrepSmem<T>);
    e = cudaFuncSetAttribute(chunk_prep_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(s1));
    if (e != cudaSuccess) return e;
    const int64_t items = units * nfull;
    if (items > 2147483647) return cudaErrorInvalidValue;
    chunk_prep_kernel<T><<<dim3(unsigned(items)), dim3(kThreads), s1, stream>>>(p, nfull);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t s2 = sizeof(ChainSmem<T>);
  e = cudaFuncSetAttribute(chunk_chain_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(s2));
  if (e != cudaSuccess) return e;
  chunk_chain_kernel<T><<<dim3(unsigned(units)), dim3(kThreads), s2, stream>>>(p, nfull);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_split_fwd(const FwdArgs& p, int dtype, cudaStream_t stream) {
  if (!p.ckpt) return cudaErrorInvalidValue;
  switch (dtype) {
    case 0: return launch<float>(p, stream);
    case 1: return launch<__nv_bfloat16>(p, stream);
    case 2: return launch<__half>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
