// WKV-7 backward, token-order scan on the FP32 cores (algo SCAN).
//
// Reverse-mode derivative of S_t = P_t G_t + v_t k_t^T, y_t = S_t r_t with
// G_t = diag(w_t) + a_t b_t^T and P_t the state entering token t (zero after
// a reset).  Carrying D = dL/dS_t backwards, per token:
//   D += dy r^T;  dr = S_t^T dy;  dv = D k;  dk = D^T v;  dsa = D b;
//   db = D^T sa;  dw = diag(D^T P_t);  da = P_t^T dsa;  D = D diag(w) + dsa a^T
// and D = 0 after a token whose reset flag is set.
//
// Checkpointed as on the rwkv-metal page ("The Metal WKV-7 kernel"): the
// backward rebuilds each chunk from the state saved at its start, every 16
// tokens, instead of running the whole sequence backwards through 1/w, which
// would grow like (1/decay)^T:
// chunks are visited in reverse.  Inside a chunk each reset-free segment is
//   A) recomputed forward from its entering state (the previous checkpoint,
//      s0, or zero after a reset), keeping sa_t for every token in shared
//      memory and ending with the segment's last state; then
//   B) walked backwards, rebuilding P_t = (S_t - sa_t b^T - v k^T) diag(1/w)
//      one token at a time.  Step A also keeps the states entering tokens
//      4, 8 and 12 of the segment in shared memory, and the walk restarts from
//      them, so no chain of divisions is longer than three tokens (rounding
//      grows by at most prod(1/w) over three tokens).  When the decay product
//      over the segment is so small that the divisions could amplify rounding
//      by more than 2^16, P_t is instead recomputed forward from the entering
//      state with the stored sa (exact, quadratic in the segment length).
//
// One CTA per (b,h), 256 threads: thread (q, j) holds rows 16q..16q+15 of
// column j of S, P and D, so the five column reductions of the backward
// (dr, dk, db, dw, da) are in-thread sums plus a 4-way combine in shared
// memory, and the row reductions (sa, dv, dsa) are a 16-shuffle
// reduce-scatter across the 32 columns of a warp plus a 2-way combine.
// Every reduction runs in a fixed order (no atomics): results are
// deterministic.
#include "common.cuh"
#include "kernels.h"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;
constexpr int kIn = 7;               // r, w, k, v, a, b, dy
constexpr float kMaxGrowth = 65536.f;  // largest tolerated prod(1/w) over a segment

constexpr int kSub = 4;               // tokens between the states kept by step A

struct BwdSmem {
  float x[kIn][kChunk][kN];
  float sa[kChunk][kN];
  float sub[kChunk / kSub - 1][kN][kN];   // states entering tokens 4, 8, 12 of a segment [row][column]
  float row_red[2][2][kN];     // [column half][quantity][row]
  float col_red[5][4][kN];     // [quantity][row quarter][column]
  int flags[kChunk];
};

// Sum v[0..15] (rows base..base+15 of this thread's column) over the 32
// columns of the warp.  Returns, on every lane, the total of row (lane>>1)&15.
__device__ __forceinline__ float row_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const bool up = lane & 16;
    const float send = up ? v[k] : v[k + 8];
    const float keep = up ? v[k + 8] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const bool up = lane & 8;
    const float send = up ? v[k] : v[k + 4];
    const float keep = up ? v[k + 4] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool up = lane & 4;
    const float send = up ? v[k] : v[k + 2];
    const float keep = up ? v[k + 2] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool up = lane & 2;
    const float send = up ? v[0] : v[1];
    const float keep = up ? v[1] : v[0];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) scan_bwd_kernel(BwdArgs p, bool only_flagged) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem& sm = *reinterpret_cast<BwdSmem*>(smem_raw);

  const int64_t unit = blockIdx.x;
  if (!in_bounds(unit < p.B * p.H, p.status)) return;   // (debug build; block-uniform)
  if (only_flagged && p.unit_flags[unit] == 0) return;
  // the epilogue's block: dy, then the bonus parts of dr, dk, dv (fp32), each B*T*H*64 floats
  const float* const eg = p.epi ? static_cast<const float*>(p.dy) : nullptr;
  const int64_t act_total = p.B * p.T * p.H * kN, st_total = p.B * p.H * kN * kN;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int tid = threadIdx.x, lane = tid & 31;
  const int q = tid >> 6;          // row quarter
  const int j = tid & 63;          // column
  const int half = j >> 5;         // column half = warp within the quarter
  const int myrow = q * 16 + ((lane >> 1) & 15);   // row whose warp-sum this lane ends with
  const int64_t nc = (p.T + kChunk - 1) / kChunk;
  const T* src[kIn] = {static_cast<const T*>(p.r), static_cast<const T*>(p.w), static_cast<const T*>(p.k),
                       static_cast<const T*>(p.v), static_cast<const T*>(p.a), static_cast<const T*>(p.b),
                       static_cast<const T*>(p.dy)};
  T* dst[6] = {static_cast<T*>(p.dr), static_cast<T*>(p.dk), static_cast<T*>(p.db),
               static_cast<T*>(p.dw), static_cast<T*>(p.da), static_cast<T*>(p.dv)};

  float D[16];
#pragma unroll
  for (int ii = 0; ii < 16; ++ii)
    D[ii] = p.dsT && range_ok((unit * kN + q * 16 + ii) * kN + j, 1, st_total, p.status)
                ? p.dsT[(unit * kN + q * 16 + ii) * kN + j] : 0.f;

  for (int64_t c = nc - 1; c >= 0; --c) {
    const int64_t t0 = c * kChunk;
    const int len = int(min64(kChunk, p.T - t0));
    __syncthreads();   // previous chunk is done with sm.x / sm.sa
    for (int e = tid; e < kIn * len * kN; e += kThreads) {
      const int m = e / (len * kN);
      const int rem = e - m * len * kN;
      const int tt = rem / kN, jj = rem - (rem / kN) * kN;
      const int64_t o = tok_off(b, t0 + tt, h, p.T, p.H) + jj;
      if (range_ok(o, 1, act_total, p.status) && in_bounds(tt < kChunk, p.status)) {
        const float x = (m == 6 && eg) ? eg[o] : Elt<T>::to_f32(src[m][o]);
        sm.x[m][tt][jj] = m == 1 ? decay_of(x, p.log_decay) : x;   // input 1 is the decay; 6 is dy
      }
    }
    if (tid < kChunk)
      sm.flags[tid] = (tid < len && p.reset && range_ok(b * p.T + t0 + tid, 1, p.B * p.T, p.status))
                          ? (p.reset[b * p.T + t0 + tid] != 0) : 0;
    __syncthreads();

    // state entering the chunk (before the reset of its first token applies)
    float E[16];
    {
      if (c > 0) {   // checkpoint c-1, in the tiled checkpoint order
        const bool ok = range_ok((unit * nc + (c - 1)) * kN * kN, kN * kN, p.B * p.H * nc * kN * kN, p.status);
        const float* es = p.ckpt + (ok ? (unit * nc + (c - 1)) * kN * kN : 0);
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) E[ii] = es[ckpt_off(q * 16 + ii, j)];
      } else {       // the caller's s0, row-major
        const float* es = p.s0 ? p.s0 + unit * kN * kN : nullptr;
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) E[ii] = es ? es[(q * 16 + ii) * kN + j] : 0.f;
      }
    }

    int seg_end = len;
    while (seg_end > 0) {
      int seg_start = seg_end - 1;
      while (seg_start > 0 && !sm.flags[seg_start]) --seg_start;
      const bool zero_entry = sm.flags[seg_start] != 0;   // segment starts at a reset

      // ---- A) forward recompute of the segment: sa_t to shared memory, S = last state
      float S[16];
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) S[ii] = zero_entry ? 0.f : E[ii];
      float growth = 1.f;
      for (int tt = seg_start; tt < seg_end; ++tt) {
        const float aj = sm.x[4][tt][j];
        float v16[16];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) v16[ii] = S[ii] * aj;
        const float part = row_reduce16(v16, lane);
        if (!(lane & 1)) sm.row_red[half][0][myrow] = part;
        __syncthreads();
        if (tid < kN) sm.sa[tt][tid] = sm.row_red[0][0][tid] + sm.row_red[1][0][tid];
        const float wj = sm.x[1][tt][j], bj = sm.x[5][tt][j], kj = sm.x[2][tt][j];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int row = q * 16 + ii;
          const float sa = sm.row_red[0][0][row] + sm.row_red[1][0][row];
          S[ii] = fmaf(S[ii], wj, fmaf(sa, bj, sm.x[3][tt][row] * kj));
        }
        if (tt > seg_start) growth *= 1.f / wj;
        const int next = tt + 1 - seg_start;   // the state in S enters token tt + 1
        if (next % kSub == 0 && tt + 1 < seg_end) {
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) sm.sub[next / kSub - 1][q * 16 + ii][j] = S[ii];
        }
        __syncthreads();
      }
      // prod(1/w) over the tokens whose entering state is rebuilt by division
      const bool unstable = __syncthreads_or(!(growth <= kMaxGrowth));

      // ---- B) reverse walk
      for (int tt = seg_end - 1; tt >= seg_start; --tt) {
        const int64_t t = t0 + tt;
        const float rj = sm.x[0][tt][j], wj = sm.x[1][tt][j], kj = sm.x[2][tt][j];
        const float aj = sm.x[4][tt][j], bj = sm.x[5][tt][j];
        float P[16];
        if (tt == seg_start) {
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) P[ii] = zero_entry ? 0.f : E[ii];
        } else if (!unstable && (tt - seg_start) % kSub == 0) {   // kept by step A
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) P[ii] = sm.sub[(tt - seg_start) / kSub - 1][q * 16 + ii][j];
        } else if (!unstable) {
          const float iw = 1.f / wj;
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) {
            const int row = q * 16 + ii;
            P[ii] = (S[ii] - sm.sa[tt][row] * bj - sm.x[3][tt][row] * kj) * iw;
          }
        } else {
          // exact: recompute the state entering tt from the segment's entering state
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) P[ii] = zero_entry ? 0.f : E[ii];
          for (int u = seg_start; u < tt; ++u) {
            const float wu = sm.x[1][u][j], bu = sm.x[5][u][j], ku = sm.x[2][u][j];
#pragma unroll
            for (int ii = 0; ii < 16; ++ii) {
              const int row = q * 16 + ii;
              P[ii] = fmaf(P[ii], wu, fmaf(sm.sa[u][row], bu, sm.x[3][u][row] * ku));
            }
          }
        }
        float dr_p = 0.f, dk_p = 0.f, db_p = 0.f, dw_p = 0.f;
        float rv[16], rs[16];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int row = q * 16 + ii;
          const float dyi = sm.x[6][tt][row];
          D[ii] = fmaf(dyi, rj, D[ii]);
          dr_p = fmaf(S[ii], dyi, dr_p);
          dk_p = fmaf(D[ii], sm.x[3][tt][row], dk_p);
          db_p = fmaf(D[ii], sm.sa[tt][row], db_p);
          dw_p = fmaf(D[ii], P[ii], dw_p);
          rv[ii] = D[ii] * kj;
          rs[ii] = D[ii] * bj;
        }
        const float dv_part = row_reduce16(rv, lane);
        const float dsa_part = row_reduce16(rs, lane);
        if (!(lane & 1)) {
          sm.row_red[half][0][myrow] = dv_part;
          sm.row_red[half][1][myrow] = dsa_part;
        }
        __syncthreads();
        if (tid < kN && range_ok(tok_off(b, t, h, p.T, p.H) + tid, 1, act_total, p.status)) {
          const int64_t o = tok_off(b, t, h, p.T, p.H) + tid;
          const float dvv = sm.row_red[0][0][tid] + sm.row_red[1][0][tid];
          dst[5][o] = Elt<T>::from_f32(eg ? dvv + eg[3 * act_total + o] : dvv);
        }
        float da_p = 0.f;
        const bool rst = sm.flags[tt] != 0;
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int row = q * 16 + ii;
          const float dsa = sm.row_red[0][1][row] + sm.row_red[1][1][row];
          da_p = fmaf(P[ii], dsa, da_p);
          D[ii] = rst ? 0.f : fmaf(D[ii], wj, dsa * aj);
          S[ii] = P[ii];
        }
        sm.col_red[0][q][j] = dr_p;
        sm.col_red[1][q][j] = dk_p;
        sm.col_red[2][q][j] = db_p;
        sm.col_red[3][q][j] = dw_p;
        sm.col_red[4][q][j] = da_p;
        __syncthreads();
        for (int o = tid; o < 5 * kN; o += kThreads) {
          const int m = o >> 6, jj = o & 63;
          const float s = (sm.col_red[m][0][jj] + sm.col_red[m][1][jj]) + (sm.col_red[m][2][jj] + sm.col_red[m][3][jj]);
          if (range_ok(tok_off(b, t, h, p.T, p.H) + jj, 1, act_total, p.status)) {
            const int64_t o = tok_off(b, t, h, p.T, p.H) + jj;
            float g = s;
            if (m == 3 && p.log_decay)   // dL/dx = dL/dw . w . (-exp(x)) = dL/d(log w) . (-exp(x))
              g = dx_of_dlogw(s * sm.x[1][t - t0][jj], Elt<T>::to_f32(src[1][o]));
            if (eg && m <= 1) g += eg[(m + 1) * act_total + o];   // dr, dk: the epilogue's bonus parts
            dst[m][o] = Elt<T>::from_f32(g);
          }
        }
      }
      seg_end = seg_start;
    }
  }
  if (p.ds0) {
#pragma unroll
    for (int ii = 0; ii < 16; ++ii)
      if (range_ok((unit * kN + q * 16 + ii) * kN + j, 1, st_total, p.status))
        p.ds0[(unit * kN + q * 16 + ii) * kN + j] = D[ii];
  }
}

template <typename T>
cudaError_t launch(const BwdArgs& p, bool only_flagged, cudaStream_t stream) {
  const size_t smem = sizeof(BwdSmem);
  cudaError_t e = cudaFuncSetAttribute(scan_bwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  scan_bwd_kernel<T><<<dim3(unsigned(p.B * p.H)), dim3(kThreads), smem, stream>>>(p, only_flagged);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_bwd(const BwdArgs& p, int dtype, bool only_flagged, cudaStream_t stream) {
  switch (dtype) {
    case 0: return launch<float>(p, only_flagged, stream);
    case 1: return launch<__nv_bfloat16>(p, only_flagged, stream);
    case 2: return launch<__half>(p, only_flagged, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
