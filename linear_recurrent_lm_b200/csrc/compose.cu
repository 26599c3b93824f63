// State composition for splitting T across devices: out = S P + U (or S P^T + U) for every (b, h)
// unit's N x N fp32 matrices.  Over a segment of tokens the recurrence is affine in the state that
// enters it, S_end = S_in P + U, with P the product of the segment's transitions diag(w_t) + a_t b_t^T
// (the forward from S_in = I with v = 0) and U the end state from S_in = 0; composing the segments'
// (P, U) in token order gives every segment's entering state, and the same P carries the state
// gradient backwards: dS_in = dS_end P^T + (the segment's own contribution).
//
// One CTA of 256 threads per unit: S and P are staged in shared memory (row-padded), each thread
// accumulates a (N/16) x (N/16) block of out in fp32, in the plain order k = 0..N-1.  The work is
// tiny next to a forward (N^3 FMAs per unit); it is written for exactness, not speed.
#include "common.cuh"
#include "kernels.h"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;

template <int N>
struct ComposeShape {
  static constexpr int kLd = N + 4;            // padded row of the staged matrices
  static constexpr int kBlk = N / 16;          // out block per thread: kBlk x kBlk
  static constexpr size_t kSmem = size_t(2) * N * kLd * sizeof(float);
};

template <int N>
__global__ void __launch_bounds__(kThreads) compose_kernel(const ComposeArgs p) {
  extern __shared__ __align__(16) float csm[];
  constexpr int LD = ComposeShape<N>::kLd, NB = ComposeShape<N>::kBlk;
  float* Ss = csm;              // S [i][k]
  float* Ps = csm + N * LD;     // P [k][j] (P^T staged transposed, so the loop below is the same)
  const int64_t unit = blockIdx.x;
  const int64_t base = unit * N * N;
  const int64_t total = p.units * N * N;
  for (int e = threadIdx.x; e < N * N; e += kThreads) {
    const int r = e / N, c = e - (e / N) * N;
    const bool ok = range_ok(base + e, 1, total, p.status);
    Ss[r * LD + c] = (p.S && ok) ? p.S[base + e] : 0.f;
    const float pv = (p.P && ok) ? p.P[base + e] : 0.f;
    if (p.transpose_p)
      Ps[c * LD + r] = pv;
    else
      Ps[r * LD + c] = pv;
  }
  __syncthreads();
  const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;   // rows ti + 16 m, columns tj + 16 n
  float acc[NB][NB] = {};
  if (p.S) {
    for (int k = 0; k < N; ++k) {
      float sv[NB], pv[NB];
#pragma unroll
      for (int m = 0; m < NB; ++m) sv[m] = Ss[(ti + 16 * m) * LD + k];
#pragma unroll
      for (int n = 0; n < NB; ++n) pv[n] = Ps[k * LD + tj + 16 * n];
#pragma unroll
      for (int m = 0; m < NB; ++m)
#pragma unroll
        for (int n = 0; n < NB; ++n) acc[m][n] = fmaf(sv[m], pv[n], acc[m][n]);
    }
  }
#pragma unroll
  for (int m = 0; m < NB; ++m)
#pragma unroll
    for (int n = 0; n < NB; ++n) {
      const int64_t o = base + int64_t(ti + 16 * m) * N + tj + 16 * n;
      if (!range_ok(o, 1, total, p.status)) continue;
      p.out[o] = acc[m][n] + (p.U ? p.U[o] : 0.f);
    }
}

template <int N>
cudaError_t launch(const ComposeArgs& p, cudaStream_t stream) {
  const size_t smem = ComposeShape<N>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(compose_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  compose_kernel<N><<<dim3(unsigned(p.units)), dim3(kThreads), smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compose(const ComposeArgs& p, int N, cudaStream_t stream) {
  if (p.units == 0) return cudaSuccess;
  if (p.units > int64_t(0x7fffffff)) return cudaErrorInvalidValue;
  switch (N) {
    case 64: return launch<64>(p, stream);
    case 128: return launch<128>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
