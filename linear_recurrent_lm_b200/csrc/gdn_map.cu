// The gated-delta-rule front-end map (rwkv-lab page, "Highlight result -- GDN in RWKV-7"): a gated
// DeltaNet layer's per-token q, k (one per key head), log-decay g and write strength beta (one per
// value head) become the wkv7 recurrence's r, x (log-space decay), k, a, b (one per value head); v
// passes to the recurrence unchanged.  For value head h of key head kh = h / (H / Hk):
//   q^ = q / sqrt(|q|^2 + eps),   k^ = k / sqrt(|k|^2 + eps),
//   r = r_scale q^,   x = log(-g) on every channel (so that exp(-exp(x)) = exp(g)),
//   kw = beta k^,   a = -k^,   b = exp(g) beta k^.
// The page scales the recurrence's output by 1/sqrt(N); y = S r is linear in r, so r_scale carries it.
//
// HBM-bound streaming: one lane group per (b, t, key head) -- 16-byte vectors, N / (16 / sizeof T)
// lanes -- normalises q and k once and writes the G = H / Hk value heads that share them, so every
// input byte is read once and every output byte written once (N = 128 in bf16: 512 B read per key
// token-head; 8 B of g, beta read and 5 x 256 B written per value token-head).
#include "common.cuh"
#include "kernels.h"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;

template <typename T, int N>
struct MapLanes {
  static constexpr int kPer = N * int(sizeof(T)) / 16;   // lanes per token-head: 8, 16 or 32
  static constexpr int kElts = 16 / int(sizeof(T));       // channels per lane
  static constexpr int kRows = kThreads / kPer;           // key token-heads per CTA pass
};

template <int kPer>
__device__ __forceinline__ float lane_group_sum(float x) {
#pragma unroll
  for (int o = 1; o < kPer; o *= 2) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T, int E>
__device__ __forceinline__ void store16(void* base, int64_t off, const float (&x)[E]) {
  uint4 raw;
  T* q = reinterpret_cast<T*>(&raw);
#pragma unroll
  for (int e = 0; e < E; ++e) q[e] = Elt<T>::from_f32(x[e]);
  *reinterpret_cast<uint4*>(static_cast<T*>(base) + off) = raw;
}

template <typename T, int N>
__global__ void __launch_bounds__(kThreads) gdn_map_kernel(const GdnArgs p) {
  constexpr int P = MapLanes<T, N>::kPer, E = MapLanes<T, N>::kElts, RW = MapLanes<T, N>::kRows;
  const int grp = threadIdx.x / P, c0 = (threadIdx.x % P) * E;
  const int64_t rows = p.B * p.T * p.Hk;
  const int64_t G = p.H / p.Hk;
  const int64_t in_total = rows * N, vrows = p.B * p.T * p.H, out_total = vrows * N;
  const int warp_first = (threadIdx.x / 32) * (32 / P);
  // Warp-uniform loop (the lane-group sums need the whole warp): a group past the last row sums
  // zeros and writes nothing.
  for (int64_t it0 = int64_t(blockIdx.x) * RW; it0 + warp_first < rows; it0 += int64_t(gridDim.x) * RW) {
    const int64_t row = it0 + grp;
    const int64_t off = row * N + c0;
    const bool act = row < rows && range_ok(off, E, in_total, p.status);
    float q[E] = {}, k[E] = {};
    if (act) {
      unpack16<T>(*reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) + off), q);
      unpack16<T>(*reinterpret_cast<const uint4*>(static_cast<const T*>(p.k) + off), k);
    }
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      sq = fmaf(q[e], q[e], sq);
      sk = fmaf(k[e], k[e], sk);
    }
    const float rq = rsqrtf(lane_group_sum<P>(sq) + p.eps) * p.r_scale;
    const float rk = rsqrtf(lane_group_sum<P>(sk) + p.eps);
    if (!act) continue;
    float r[E], kn[E], a[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      r[e] = q[e] * rq;
      kn[e] = k[e] * rk;
      a[e] = -kn[e];
    }
    const int64_t bt = row / p.Hk, hk = row - bt * p.Hk;
    for (int64_t j = 0; j < G; ++j) {
      const int64_t vr = bt * p.H + hk * G + j;   // value token-head
      const int64_t o = vr * N + c0;
      if (!range_ok(vr, 1, vrows, p.status) || !range_ok(o, E, out_total, p.status)) continue;
      const float gl = __ldg(p.g + vr), be = __ldg(p.beta + vr);
      const float xl = logf(-gl), eb = expf(gl) * be;
      float x[E], kw[E], b[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        x[e] = xl;
        kw[e] = kn[e] * be;
        b[e] = kn[e] * eb;
      }
      store16<T, E>(p.r, o, r);
      store16<T, E>(p.x, o, x);
      store16<T, E>(p.kw, o, kw);
      store16<T, E>(p.a, o, a);
      store16<T, E>(p.b, o, b);
    }
  }
}

template <typename T, int N>
cudaError_t launch(const GdnArgs& p, cudaStream_t stream) {
  const int64_t rows = p.B * p.T * p.Hk;
  int sms = 148, dev = 0, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gdn_map_kernel<T, N>, kThreads, 0);
  const int64_t need = (rows + MapLanes<T, N>::kRows - 1) / MapLanes<T, N>::kRows;
  const int64_t cap = int64_t(sms) * (per_sm > 0 ? per_sm : 1);   // one wave; a grid-stride loop past that
  const unsigned grid = unsigned(need < cap ? need : cap);
  if (grid == 0) return cudaSuccess;
  gdn_map_kernel<T, N><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_n(const GdnArgs& p, int N, cudaStream_t stream) {
  return N == 128 ? launch<T, 128>(p, stream) : launch<T, 64>(p, stream);
}

}  // namespace

cudaError_t launch_gdn_map(const GdnArgs& p, int dtype, int N, cudaStream_t stream) {
  if (N != 64 && N != 128) return cudaErrorInvalidValue;
  switch (dtype) {
    case 0: return launch_n<float>(p, N, stream);
    case 1: return launch_n<__nv_bfloat16>(p, N, stream);
    case 2: return launch_n<__half>(p, N, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
