// WKV-7 forward, token-order scan on the FP32 cores (algo SCAN).
//
// One CTA per (b,h) unit, N threads (head size N = 64, or 128 for the gated-delta-rule heads of the
// rwkv-lab page's GDN map), thread i owns row i of the N x N fp32 state in registers.  Rows of S never interact in the forward (sa[i] and
// y[i] only read row i), so the scan needs no cross-thread reduction.  Each
// 16-token slab of r,w,k,v,a,b is copied to shared memory with cp.async while
// the previous slab is being consumed, widened once to fp32, and then read by
// all threads as broadcasts.  After every 16 tokens (and after the last
// token) the state is written to the checkpoint workspace: the 16-token
// checkpoint interval of the rwkv-metal page ("The Metal WKV-7 kernel") --
// in the chunked kernels' tiled order for N = 64, row-major for N = 128.
#include "common.cuh"
#include "kernels.h"

namespace wkv7 {
namespace {

constexpr int kInputs = 6;   // slab order: r, w, k, v, a, b

template <typename T, int N>
struct FwdSmem {
  static constexpr size_t raw_bytes = size_t(kInputs) * kChunk * N * sizeof(T);
  static constexpr size_t f32_bytes = size_t(kInputs) * kChunk * N * sizeof(float);
  static constexpr size_t total = raw_bytes + f32_bytes;
};

template <typename T, int N>
__device__ __forceinline__ void stage_slab(const FwdArgs& p, const T* const* src, unsigned char* raw,
                                           int64_t b, int64_t h, int64_t t0, int len) {
  constexpr int VPT = N / Vec16<T>::n;  // 16-byte vectors per token vector
  const int total = kInputs * len * VPT;
  for (int idx = threadIdx.x; idx < total; idx += N) {
    const int in = idx / (len * VPT);
    const int rem = idx - in * len * VPT;
    const int tt = rem / VPT;
    const int vec = rem - tt * VPT;
    const int64_t o = tok_offn<N>(b, t0 + tt, h, p.T, p.H) + vec * Vec16<T>::n;
    unsigned char* s = raw + ((size_t(in) * kChunk + tt) * N + vec * Vec16<T>::n) * sizeof(T);
    if (range_ok(o, Vec16<T>::n, p.B * p.T * p.H * N, p.status) && in_bounds(tt < kChunk, p.status))
      cp_async16(s, src[in] + o);
  }
  cp_async_commit();
}

template <typename T, int N>
__device__ __forceinline__ void widen_slab(const unsigned char* raw, float* f32, int len, bool log_decay) {
  const T* src = reinterpret_cast<const T*>(raw);
  for (int in = 0; in < kInputs; ++in)
    for (int e = threadIdx.x; e < len * N; e += N) {
      const float x = Elt<T>::to_f32(src[in * kChunk * N + e]);
      f32[in * kChunk * N + e] = in == 1 ? decay_of(x, log_decay) : x;   // input 1 is the decay
    }
}

template <typename T, int N>
__global__ void __launch_bounds__(N) scan_fwd_kernel(FwdArgs p) {
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char* raw = smem;
  float* f32 = reinterpret_cast<float*>(smem + FwdSmem<T, N>::raw_bytes);

  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H, h = unit - (unit / p.H) * p.H;
  const int i = threadIdx.x;
  const int64_t nc = (p.T + kChunk - 1) / kChunk;
  const T* src[kInputs] = {static_cast<const T*>(p.r), static_cast<const T*>(p.w), static_cast<const T*>(p.k),
                           static_cast<const T*>(p.v), static_cast<const T*>(p.a), static_cast<const T*>(p.b)};

  float S[N];
  const int64_t st_total = p.B * p.H * N * N;
  if (p.s0 && range_ok((unit * N + i) * N, N, st_total, p.status)) {
    const float4* row = reinterpret_cast<const float4*>(p.s0 + (unit * N + i) * N);
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
      float4 v4 = row[q];
      S[4 * q] = v4.x; S[4 * q + 1] = v4.y; S[4 * q + 2] = v4.z; S[4 * q + 3] = v4.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < N; ++j) S[j] = 0.f;
  }

  if (nc > 0) {
    stage_slab<T, N>(p, src, raw, b, h, 0, int(min64(kChunk, p.T)));
    cp_async_wait_all();
    __syncthreads();
    widen_slab<T, N>(raw, f32, int(min64(kChunk, p.T)), p.log_decay);
    __syncthreads();
  }

  T* y = static_cast<T*>(p.y);
  for (int64_t c = 0; c < nc; ++c) {
    const int64_t t0 = c * kChunk;
    const int len = int(min64(kChunk, p.T - t0));
    if (c + 1 < nc) stage_slab<T, N>(p, src, raw, b, h, t0 + kChunk, int(min64(kChunk, p.T - t0 - kChunk)));

    for (int tt = 0; tt < len; ++tt) {
      const int64_t t = t0 + tt;
      if (p.reset && range_ok(b * p.T + t, 1, p.B * p.T, p.status) && p.reset[b * p.T + t]) {
#pragma unroll
        for (int j = 0; j < N; ++j) S[j] = 0.f;
      }
      const float4* r4 = reinterpret_cast<const float4*>(f32 + (0 * kChunk + tt) * N);
      const float4* w4 = reinterpret_cast<const float4*>(f32 + (1 * kChunk + tt) * N);
      const float4* k4 = reinterpret_cast<const float4*>(f32 + (2 * kChunk + tt) * N);
      const float vi = f32[(3 * kChunk + tt) * N + i];
      const float4* a4 = reinterpret_cast<const float4*>(f32 + (4 * kChunk + tt) * N);
      const float4* b4 = reinterpret_cast<const float4*>(f32 + (5 * kChunk + tt) * N);
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int q = 0; q < N / 4; ++q) {
        const float4 av = a4[q];
        s0 = fmaf(S[4 * q], av.x, s0);
        s1 = fmaf(S[4 * q + 1], av.y, s1);
        s2 = fmaf(S[4 * q + 2], av.z, s2);
        s3 = fmaf(S[4 * q + 3], av.w, s3);
      }
      const float sa = (s0 + s1) + (s2 + s3);
      float y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
#pragma unroll
      for (int q = 0; q < N / 4; ++q) {
        const float4 wv = w4[q], bv = b4[q], kv = k4[q], rv = r4[q];
        S[4 * q] = fmaf(S[4 * q], wv.x, fmaf(sa, bv.x, vi * kv.x));
        S[4 * q + 1] = fmaf(S[4 * q + 1], wv.y, fmaf(sa, bv.y, vi * kv.y));
        S[4 * q + 2] = fmaf(S[4 * q + 2], wv.z, fmaf(sa, bv.z, vi * kv.z));
        S[4 * q + 3] = fmaf(S[4 * q + 3], wv.w, fmaf(sa, bv.w, vi * kv.w));
        y0 = fmaf(S[4 * q], rv.x, y0);
        y1 = fmaf(S[4 * q + 1], rv.y, y1);
        y2 = fmaf(S[4 * q + 2], rv.z, y2);
        y3 = fmaf(S[4 * q + 3], rv.w, y3);
      }
      if (range_ok(tok_offn<N>(b, t, h, p.T, p.H) + i, 1, p.B * p.T * p.H * N, p.status))
        y[tok_offn<N>(b, t, h, p.T, p.H) + i] = Elt<T>::from_f32((y0 + y1) + (y2 + y3));
    }

    if (p.ckpt && range_ok((unit * nc + c) * N * N, N * N, p.B * p.H * nc * N * N, p.status)) {
      float* dst = p.ckpt + (unit * nc + c) * N * N;
#pragma unroll
      for (int q = 0; q < N / 2; ++q)
        *reinterpret_cast<float2*>(dst + (N == 64 ? ckpt_off(i, 2 * q) : i * N + 2 * q)) = make_float2(S[2 * q], S[2 * q + 1]);
    }
    cp_async_wait_all();
    __syncthreads();
    if (c + 1 < nc) {
      widen_slab<T, N>(raw, f32, int(min64(kChunk, p.T - t0 - kChunk)), p.log_decay);
      __syncthreads();
    }
  }

  if (p.s_out && range_ok((unit * N + i) * N, N, st_total, p.status)) {
    float4* dst = reinterpret_cast<float4*>(p.s_out + (unit * N + i) * N);
#pragma unroll
    for (int q = 0; q < N / 4; ++q) dst[q] = make_float4(S[4 * q], S[4 * q + 1], S[4 * q + 2], S[4 * q + 3]);
  }
}

template <typename T, int N>
cudaError_t launch(const FwdArgs& p, cudaStream_t stream) {
  const size_t smem = FwdSmem<T, N>::total;
  cudaError_t e = cudaFuncSetAttribute(scan_fwd_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  scan_fwd_kernel<T, N><<<dim3(unsigned(p.B * p.H)), dim3(N), smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_fwd(const FwdArgs& p, int dtype, cudaStream_t stream) {
  const bool n128 = p.N == 128;
  switch (dtype) {
    case 0: return n128 ? launch<float, 128>(p, stream) : launch<float, 64>(p, stream);
    case 1: return n128 ? launch<__nv_bfloat16, 128>(p, stream) : launch<__nv_bfloat16, 64>(p, stream);
    case 2: return n128 ? launch<__half, 128>(p, stream) : launch<__half, 64>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
