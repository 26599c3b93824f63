// The WKV epilogue: per-head GroupNorm of y, the bonus term and output gating, forward and backward,
// each one streaming kernel (rwkv-metal page, architecture table: ln_x as a per-head GroupNorm;
// rwkv-lab page, "Native RWKV megakernel backend": the state update fused through GroupNorm, the
// RWKV bonus and output gating).  Per (b, t, h), channels i, j:
//   mu, rstd = mean and 1/sqrt(var + eps) of y over the head's channels,  yn = (y - mu) rstd,
//   s = sum_j r_j k_j rk_j,   z = yn gamma + beta + s v,   out = z g;
// and in reverse, from dout:  dg = dout z,  dz = dout g,  dv += s dz,  ds = sum_i dz_i v_i,
//   dr += ds k rk,  dk += ds r rk,  dyn = dz gamma,  dy = rstd (dyn - mean(dyn) - yn mean(dyn yn)),
//   dgamma += dz yn,  dbeta += dz,  drk += ds r k  (the parameter gradients summed over b and t).
// The backward hands dy and the bonus parts of dr, dk, dv to the recurrence's backward in fp32 (one
// block [4][B,T,H,64]): the GroupNorm's gradient can be large where y has a small spread, and the
// bonus parts are added to the recurrence's before the one rounding to the output dtype.
//
// Both kernels are bound by HBM: a token-head is one 16-byte vector per lane over 8 lanes (16-bit
// types) or 16 lanes (fp32), so every load and store is a whole 128- or 256-byte row, and the
// head's reductions are shuffles inside that lane group.  The grid is (slices of the b, t rows) x H:
// a CTA works on one head, so the backward keeps its parameter gradients in registers across its
// rows, reduces them over the CTA in shared memory and adds one partial per CTA with atomics.
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;

template <typename T>
struct Lanes {
  static constexpr int kPer = kN * int(sizeof(T)) / 16;   // lanes per token-head (8 or 16)
  static constexpr int kElts = 16 / int(sizeof(T));       // channels per lane (8 or 4)
  static constexpr int kRows = kThreads / kPer;           // token-heads per CTA pass
};

// Sum over the lane group of one token-head (kPer consecutive lanes).
template <int kPer>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int o = 1; o < kPer; o *= 2) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T>
__device__ __forceinline__ void load_vec(const void* base, int64_t off, float (&x)[Lanes<T>::kElts]) {
  unpack16<T>(*reinterpret_cast<const uint4*>(static_cast<const T*>(base) + off), x);
}
template <typename T>
__device__ __forceinline__ void store_vec(void* base, int64_t off, const float (&x)[Lanes<T>::kElts]) {
  constexpr int E = Lanes<T>::kElts;
  uint4 raw;
  T* q = reinterpret_cast<T*>(&raw);
#pragma unroll
  for (int e = 0; e < E; ++e) q[e] = Elt<T>::from_f32(x[e]);
  *reinterpret_cast<uint4*>(static_cast<T*>(base) + off) = raw;
}
__device__ __forceinline__ void load_param(const float* p, int h, int c0, float* x, int n) {
  for (int e = 0; e < n; ++e) x[e] = __ldg(p + h * kN + c0 + e);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) epilogue_fwd_kernel(const EpiArgs p) {
  constexpr int P = Lanes<T>::kPer, E = Lanes<T>::kElts, RW = Lanes<T>::kRows;
  const int h = blockIdx.y;
  const int q = threadIdx.x % P;            // lane within the token-head's group
  const int c0 = q * E;                     // first channel of this lane
  const int64_t rows = p.B * p.T;
  float gam[E], bet[E], rk[E];
  load_param(p.ln_w, h, c0, gam, E);
  load_param(p.ln_b, h, c0, bet, E);
  load_param(p.r_k, h, c0, rk, E);
  const int64_t total = rows * p.H * kN;
  const int grp = threadIdx.x / P, warp_first = (threadIdx.x / 32) * (32 / P);
  // The loop is warp-uniform (the group shuffles need the whole warp): a group past the last row
  // computes on zeros and stores nothing.
  for (int64_t it0 = int64_t(blockIdx.x) * RW; it0 + warp_first < rows; it0 += int64_t(gridDim.x) * RW) {
    const int64_t row = it0 + grp;
    const int64_t off = (row * p.H + h) * kN + c0;
    const bool act = row < rows && range_ok(off, E, total, p.status);
    float y[E] = {}, r[E] = {}, k[E] = {}, v[E] = {}, g[E] = {};
    if (act) {
      load_vec<T>(p.y, off, y);
      load_vec<T>(p.r, off, r);
      load_vec<T>(p.k, off, k);
      load_vec<T>(p.v, off, v);
      load_vec<T>(p.g, off, g);
    }
    float out[E];
    epi_forward<P, E>(y, r, k, v, g, gam, bet, rk, p.eps, 0xffffffffu, out);
    if (act) store_vec<T>(p.out, off, out);
  }
}

// Two CTAs per SM (128 registers, no spills): at its natural 153 registers one CTA of 8 warps per SM
// could not keep enough loads in flight.
template <typename T>
__global__ void __launch_bounds__(kThreads, 2) epilogue_bwd_kernel(const EpiArgs p) {
  constexpr int P = Lanes<T>::kPer, E = Lanes<T>::kElts, RW = Lanes<T>::kRows;
  __shared__ float red[3][RW][kN];           // per-group partial parameter gradients
  const int h = blockIdx.y;
  const int grp = threadIdx.x / P, q = threadIdx.x % P;
  const int c0 = q * E;
  const int64_t rows = p.B * p.T;
  float gam[E], bet[E], rk[E];
  load_param(p.ln_w, h, c0, gam, E);
  load_param(p.ln_b, h, c0, bet, E);
  load_param(p.r_k, h, c0, rk, E);
  float dgam[E] = {}, dbet[E] = {}, drk[E] = {};
  const int64_t total = rows * p.H * kN;
  const int warp_first = (threadIdx.x / 32) * (32 / P);
  for (int64_t it0 = int64_t(blockIdx.x) * RW; it0 + warp_first < rows; it0 += int64_t(gridDim.x) * RW) {
    const int64_t row = it0 + grp;
    const int64_t off = (row * p.H + h) * kN + c0;
    const bool act = row < rows && range_ok(off, E, total, p.status);
    float y[E] = {}, r[E] = {}, k[E] = {}, v[E] = {}, g[E] = {}, d[E] = {};   // zeros: no gradient
    if (act) {
      load_vec<T>(p.y, off, y);
      load_vec<T>(p.r, off, r);
      load_vec<T>(p.k, off, k);
      load_vec<T>(p.v, off, v);
      load_vec<T>(p.g, off, g);
      load_vec<T>(p.dout, off, d);
    }
    float sy = 0.f, srk = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      sy += y[e];
      srk = fmaf(r[e] * k[e], rk[e], srk);
    }
    const float mu = group_sum<P>(sy) * (1.f / kN);
    float sq = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) sq = fmaf(y[e] - mu, y[e] - mu, sq);
    const float rstd = rsqrtf(group_sum<P>(sq) * (1.f / kN) + p.eps);
    const float s = group_sum<P>(srk);
    float yn[E], dz[E], dg[E], sds = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      yn[e] = (y[e] - mu) * rstd;
      const float z = fmaf(yn[e], gam[e], fmaf(s, v[e], bet[e]));
      dg[e] = d[e] * z;
      dz[e] = d[e] * g[e];
      sds = fmaf(dz[e], v[e], sds);
    }
    const float ds = group_sum<P>(sds);
    float m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float dyn = dz[e] * gam[e];
      m1 += dyn;
      m2 = fmaf(dyn, yn[e], m2);
    }
    m1 = group_sum<P>(m1) * (1.f / kN);
    m2 = group_sum<P>(m2) * (1.f / kN);
    float dy[E], dr[E], dk[E], dv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dy[e] = rstd * (dz[e] * gam[e] - m1 - yn[e] * m2);
      dr[e] = ds * k[e] * rk[e];
      dk[e] = ds * r[e] * rk[e];
      dv[e] = s * dz[e];
      dgam[e] = fmaf(dz[e], yn[e], dgam[e]);
      dbet[e] += dz[e];
      drk[e] = fmaf(ds, r[e] * k[e], drk[e]);
    }
    if (act) {
      store_vec<T>(p.dg, off, dg);
      const float* const parts[4] = {dy, dr, dk, dv};
#pragma unroll
      for (int m = 0; m < 4; ++m) {   // the fp32 block: dy, then the bonus parts of dr, dk, dv
        float4* q4 = reinterpret_cast<float4*>(p.eg + m * total + off);
#pragma unroll
        for (int u = 0; u < E / 4; ++u)
          q4[u] = make_float4(parts[m][4 * u], parts[m][4 * u + 1], parts[m][4 * u + 2], parts[m][4 * u + 3]);
      }
    }
  }
  // the CTA's parameter gradients: groups' partials through shared memory, one atomic per element
#pragma unroll
  for (int e = 0; e < E; ++e) {
    red[0][grp][c0 + e] = dgam[e];
    red[1][grp][c0 + e] = dbet[e];
    red[2][grp][c0 + e] = drk[e];
  }
  __syncthreads();
  float* const dst[3] = {p.dln_w, p.dln_b, p.dr_k};
  for (int idx = threadIdx.x; idx < 3 * kN; idx += kThreads) {
    const int m = idx / kN, c = idx - m * kN;
    float acc = 0.f;
    for (int gi = 0; gi < RW; ++gi) acc += red[m][gi][c];
    if (dst[m] && in_bounds(h < p.H, p.status)) atomicAdd(dst[m] + h * kN + c, acc);
  }
}

template <typename T>
cudaError_t launch(const EpiArgs& p, bool backward, cudaStream_t stream) {
  const int64_t rows = p.B * p.T;
  int sms = 148, dev = 0, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (backward)
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, epilogue_bwd_kernel<T>, kThreads, 0);
  else
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, epilogue_fwd_kernel<T>, kThreads, 0);
  // one wave: the resident CTAs of every SM shared out over the heads (at least one per head), at
  // most one pass of rows per CTA group
  const int64_t slots = int64_t(sms) * (per_sm > 0 ? per_sm : 1);
  const int64_t per_head = slots / p.H > 0 ? slots / p.H : 1;
  const int64_t need = (rows + Lanes<T>::kRows - 1) / Lanes<T>::kRows;
  const unsigned gx = unsigned(need < per_head ? need : per_head);
  if (gx == 0 || p.H > 65535) return p.H > 65535 ? cudaErrorInvalidValue : cudaSuccess;
  const dim3 grid(gx, unsigned(p.H));
  if (backward)
    epilogue_bwd_kernel<T><<<grid, kThreads, 0, stream>>>(p);
  else
    epilogue_fwd_kernel<T><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_epilogue(const EpiArgs& p, int dtype, bool backward, cudaStream_t stream) {
  switch (dtype) {
    case 0: return launch<float>(p, backward, stream);
    case 1: return launch<__nv_bfloat16>(p, backward, stream);
    case 2: return launch<__half>(p, backward, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
