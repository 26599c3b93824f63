// WKV-7 single-token decode step on B*H resident fp32 states, in place.
//
// The rwkv-metal page steps one token on a carried state with plain array
// operations and pads ragged batches on the right without changing the
// results of the padded rows.  Here one launch steps every (b,h) state: it is
// a pure stream over the 16 KiB state (read once, written once) and therefore
// HBM-bound.
//
// A persistent grid of (SM count x resident CTAs per SM) CTAs of 512 threads
// walks the B*H units with a grid stride.  Within a unit, thread t owns row
// t/8 and the 8 columns 8*(t%8)..+7, held as two float4 -- each warp reads and
// writes 1 KiB of contiguous state with 16-byte accesses, and few registers per
// thread keep three CTAs (and their loads) in flight per SM.  The two row dot
// products (sa and y) reduce over the 8 lanes of a row with three
// xor-shuffles.  A unit whose batch row has active[b] == 0 is skipped without
// touching its state, which therefore stays bitwise unchanged (and costs no
// bandwidth in a ragged batch), and gets y = 0; skipping costs one loop
// iteration instead of a CTA launch.
//
// Consecutive decode steps are launched with programmatic dependent launch:
// the next step's CTAs take the SM slots of this step's finished CTAs and wait
// (griddepcontrol.wait) until this grid has completed and its writes are
// visible, so the launch latency of step n+1 overlaps the tail of step n.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace wkv7 {
namespace {

// N = 64: 512 threads, three CTAs per SM; N = 128 (the gated-delta-rule heads of the rwkv-lab
// page's GDN map): 1024 threads, 16 columns per thread.
template <int N> struct StepShape {
  static constexpr int kThreads = 8 * N;                 // 8 threads per state row
  static constexpr int kCols = N / 8;                    // columns per thread
  static constexpr int kMinBlocks = N == 64 ? 3 : 1;
};
constexpr int kMaxDevices = 64;

// Eight consecutive elements of T (16-byte aligned) as fp32.
template <typename T>
__device__ __forceinline__ void load8(const T* g, float* out) {
  constexpr int n = Vec16<T>::n;
#pragma unroll
  for (int u = 0; u < 8 / n; ++u) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(g + u * n));
    unpack16<T>(raw, out + u * n);
  }
}

template <typename T, int N>
__global__ void __launch_bounds__(StepShape<N>::kThreads, StepShape<N>::kMinBlocks) step_kernel(StepArgs p) {
  constexpr int C = StepShape<N>::kCols;
  // Everything this grid reads or writes may belong to the grid launched before it.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t = threadIdx.x;
  const int i = t >> 3, q = t & 7;   // row i, columns C q .. C q + C - 1
  const int64_t units = p.B * p.H;
  for (int64_t unit = blockIdx.x; unit < units; unit += gridDim.x) {
    // (debug build: the row of y, the state row and the input rows of this unit)
    if (!range_ok(unit * N, N, units * N, p.status) || !range_ok((unit * N + i) * N + q * C, C, units * N * N, p.status))
      continue;
    T* y = static_cast<T*>(p.y) + unit * N;
    if (p.active && !p.active[unit / p.H]) {   // padded row: its state is not even read
      if (q == 0) y[i] = Elt<T>::from_f32(0.f);
      continue;
    }
    float4* row = reinterpret_cast<float4*>(p.state + (unit * N + i) * N + q * C);
    float S[C];
#pragma unroll
    for (int u = 0; u < C / 4; ++u) {
      const float4 s4 = row[u];
      S[4 * u] = s4.x; S[4 * u + 1] = s4.y; S[4 * u + 2] = s4.z; S[4 * u + 3] = s4.w;
    }
    const int64_t o = unit * N + q * C;
    float wv[C], kv[C], av[C], bv[C], rv[C];
#pragma unroll
    for (int u = 0; u < C / 8; ++u) load8<T>(static_cast<const T*>(p.a) + o + 8 * u, av + 8 * u);
#pragma unroll
    for (int u = 0; u < C / 8; ++u) load8<T>(static_cast<const T*>(p.w) + o + 8 * u, wv + 8 * u);
#pragma unroll
    for (int j = 0; j < C; ++j) wv[j] = decay_of(wv[j], p.log_decay);
#pragma unroll
    for (int u = 0; u < C / 8; ++u) {
      load8<T>(static_cast<const T*>(p.b) + o + 8 * u, bv + 8 * u);
      load8<T>(static_cast<const T*>(p.k) + o + 8 * u, kv + 8 * u);
      load8<T>(static_cast<const T*>(p.r) + o + 8 * u, rv + 8 * u);
    }
    const float vi = Elt<T>::to_f32(static_cast<const T*>(p.v)[unit * N + i]);

    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int j = 0; j < C; j += 2) {
      s0 = fmaf(S[j], av[j], s0);
      s1 = fmaf(S[j + 1], av[j + 1], s1);
    }
    float sa = s0 + s1;
    sa += __shfl_xor_sync(0xffffffffu, sa, 1);
    sa += __shfl_xor_sync(0xffffffffu, sa, 2);
    sa += __shfl_xor_sync(0xffffffffu, sa, 4);

    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int j = 0; j < C; ++j) {
      S[j] = fmaf(S[j], wv[j], fmaf(sa, bv[j], vi * kv[j]));
      if (j & 1) y1 = fmaf(S[j], rv[j], y1); else y0 = fmaf(S[j], rv[j], y0);
    }
#pragma unroll
    for (int u = 0; u < C / 4; ++u) row[u] = make_float4(S[4 * u], S[4 * u + 1], S[4 * u + 2], S[4 * u + 3]);
    float yy = y0 + y1;
    yy += __shfl_xor_sync(0xffffffffu, yy, 1);
    yy += __shfl_xor_sync(0xffffffffu, yy, 2);
    yy += __shfl_xor_sync(0xffffffffu, yy, 4);
    if (q == 0) y[i] = Elt<T>::from_f32(yy);
  }
}

// Resident grid size for this device and element type, looked up once (concurrent first calls
// may both look it up; they store the same value).
template <typename T, int N>
cudaError_t grid_size(int64_t units, unsigned* out) {
  static std::atomic<int> cached[kMaxDevices];   // SMs x resident CTAs per SM; 0 = not looked up yet
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int slots = (dev >= 0 && dev < kMaxDevices) ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (slots == 0) {
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, step_kernel<T, N>, StepShape<N>::kThreads, 0);
    if (e != cudaSuccess) return e;
    slots = sms * (per_sm > 0 ? per_sm : 1);
    if (dev >= 0 && dev < kMaxDevices) cached[dev].store(slots, std::memory_order_relaxed);
  }
  *out = unsigned(units < int64_t(slots) ? units : int64_t(slots));
  return cudaSuccess;
}

template <typename T, int N>
cudaError_t launch(const StepArgs& p, cudaStream_t stream) {
  unsigned grid = 0;
  cudaError_t e = grid_size<T, N>(p.B * p.H, &grid);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(StepShape<N>::kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, step_kernel<T, N>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const StepArgs& p, int dtype, cudaStream_t stream) {
  const bool n128 = p.N == 128;
  switch (dtype) {
    case 0: return n128 ? launch<float, 128>(p, stream) : launch<float, 64>(p, stream);
    case 1: return n128 ? launch<__nv_bfloat16, 128>(p, stream) : launch<__nv_bfloat16, 64>(p, stream);
    case 2: return n128 ? launch<__half, 128>(p, stream) : launch<__half, 64>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
