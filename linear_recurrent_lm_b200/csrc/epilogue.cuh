// The WKV epilogue's forward arithmetic for one token-head spread over a group of P lanes (E channels
// each), shared by the standalone epilogue kernel and the chunked forward's fused y write-out so that
// both give the same bits.  Per-head GroupNorm (rwkv-metal page, architecture table), the bonus term
// and output gating (rwkv-lab page, "Native RWKV megakernel backend"):
//   out = ((y - mu) rstd gamma + beta + s v) g,  s = sum_j r_j k_j rk_j.
#pragma once

#include "common.cuh"

namespace wkv7 {

// Sum over the P lanes of a group (xor partners inside the group; `mask` covers the group).
template <int P>
__device__ __forceinline__ float epi_group_sum(float x, unsigned mask) {
#pragma unroll
  for (int o = 1; o < P; o *= 2) x += __shfl_xor_sync(mask, x, o);
  return x;
}

template <int P, int E>
__device__ __forceinline__ void epi_forward(const float (&y)[E], const float (&r)[E], const float (&k)[E],
                                            const float (&v)[E], const float (&g)[E], const float* gam,
                                            const float* bet, const float* rk, float eps, unsigned mask,
                                            float (&out)[E]) {
  float sy = 0.f, srk = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    sy += y[e];
    srk = fmaf(r[e] * k[e], rk[e], srk);
  }
  const float mu = epi_group_sum<P>(sy, mask) * (1.f / kN);
  float sq = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) sq = fmaf(y[e] - mu, y[e] - mu, sq);
  const float rstd = rsqrtf(epi_group_sum<P>(sq, mask) * (1.f / kN) + eps);
  const float s = epi_group_sum<P>(srk, mask);
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] = fmaf((y[e] - mu) * rstd, gam[e], fmaf(s, v[e], bet[e])) * g[e];
}

}  // namespace wkv7
