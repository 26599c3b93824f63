// Internal launch interface between the C-ABI layer (wkv7_api.cu) and the kernels.
#pragma once

#include <cuda.h>

#include <cuda_runtime.h>
#include <stdint.h>

#include "wkv7.h"

namespace wkv7 {

struct FwdArgs {
  int64_t B, T, H;
  const void *r, *w, *k, *v, *a, *b;
  const float* s0;        // [B,H,64,64] or null
  const uint8_t* reset;   // [B,T] or null
  void* y;                // [B,T,H,64]
  float* s_out;           // [B,H,64,64] or null
  float* ckpt;            // [B,H,ceil(T/16),64,64] or null
  int* status;            // device status word: bits of wkv7 device errors (kStatus* below)
  unsigned extra_tx;      // test hook: bytes a staging expects beyond what it copies (0 in normal use)
  bool log_decay;         // w holds x and the decay is exp(-exp(x)) (WKV7_FLAG_LOG_DECAY)
  // The WKV epilogue fused into the y write-out (chunked fused form, 16-bit types): with `out`
  // non-null the kernel writes out = epilogue(y) (and y only if `y` is non-null).
  const void* g;
  void* out;
  const float *ln_w, *ln_b, *r_k;
  float eps;
  int N;                  // head size: 64, or 128 (token-order scan only)
};

// Bits of the device status word.
constexpr int kStatusWaitTimeout = 1;
constexpr int kStatusNonFinite = 2;
constexpr int kStatusBounds = 4;   // debug build: an index failed its bounds check

// Debug build (compiled with -DWKV7_DEBUG, libwkv7_debug.so): the kernels check the indices they
// compute -- every global-memory access to activations, states, checkpoints and workspace marks,
// every TMA box coordinate and bulk-copy range, every shared-memory operand index -- against the
// extent of the buffer.  A failed check sets kStatusBounds in the device status word and the access
// is skipped; nothing traps.  In the release build the checks compile to nothing.
#ifdef WKV7_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool in_bounds(bool ok, int* status) {
  if (!kDebugChecks) return true;
  if (!ok && status) atomicOr(status, kStatusBounds);
  return ok;
}
// Elements [off, off + n) inside [0, total).
__device__ __forceinline__ bool range_ok(int64_t off, int64_t n, int64_t total, int* status) {
  return in_bounds(off >= 0 && n >= 0 && off + n <= total, status);
}

// Wall-clock limit of one bounded wait on a staging barrier (the copies it waits for take microseconds).
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;

struct BwdArgs {
  int64_t B, T, H;
  const void *r, *w, *k, *v, *a, *b;
  const float* s0;
  const uint8_t* reset;
  const void* dy;
  const float* dsT;
  const float* ckpt;
  void *dr, *dw, *dk, *dv, *da, *db;
  float* ds0;
  int* unit_flags;   // [B*H] in the workspace tail: the chunked backward marks units it could not handle
                     // (0: complete; else 1 + the first chunk whose gradients it did write -- those of
                     // that chunk and every later one are final)
  int* status;       // device status word (see FwdArgs)
  unsigned extra_tx; // test hook (see FwdArgs)
  bool log_decay;    // w holds x (see FwdArgs); dw receives dL/dx
  bool epi;          // WKV7_FLAG_EPILOGUE_GRADS: dy points at the epilogue's fp32 block [4][B,T,H,64]
                     // (dy, then the bonus parts of dr, dk, dv, which are added before rounding)
};

struct StepArgs {
  int64_t B, H;
  const void *r, *w, *k, *v, *a, *b;
  float* state;
  const uint8_t* active;
  void* y;
  int* status;   // device status word (debug-build bounds checks)
  bool log_decay;  // w holds x (see FwdArgs)
  int N;           // head size: 64 or 128
};

// The WKV epilogue (GroupNorm per head, bonus, gating): forward writes `out`; backward writes the
// fp32 block `eg` [4][B,T,H,64] (dy, then the bonus parts of dr, dk, dv) and dg, and adds the
// parameter gradients to dln_w, dln_b, dr_k (each may be null).
struct EpiArgs {
  int64_t B, T, H;
  const void *y, *r, *k, *v, *g, *dout;
  const float *ln_w, *ln_b, *r_k;
  float eps;
  void *out, *dg;
  float* eg;
  float *dln_w, *dln_b, *dr_k;
  int* status;
};

// The gated-delta-rule map: q, k [B,T,Hk,N] -> r, x, kw, a, b [B,T,H,N] (all of dtype T); g, beta
// fp32 [B,T,H].
struct GdnArgs {
  int64_t B, T, H, Hk;
  const void *q, *k;
  const float *g, *beta;
  float eps, r_scale;
  void *r, *x, *kw, *a, *b;
  int* status;
};

// State composition: out = S P + U (P transposed when transpose_p) per unit of N x N fp32; S or U
// null means zero (P may then be null too).
struct ComposeArgs {
  int64_t units;
  const float *S, *P, *U;
  float* out;
  bool transpose_p;
  int* status;
};

// Descriptor checks shared by every entry point (WKV7_OK, or the status the entry points return).
wkv7_status_t validate_desc(const wkv7_desc_t* d);

// dtype: 0 = f32, 1 = bf16, 2 = f16.  Each returns the launch status.
cudaError_t launch_scan_fwd(const FwdArgs& p, int dtype, cudaStream_t stream);
// only_flagged: run only the (b,h) units whose unit_flags entry is non-zero (others exit at once).
cudaError_t launch_scan_bwd(const BwdArgs& p, int dtype, bool only_flagged, cudaStream_t stream);
cudaError_t launch_step(const StepArgs& p, int dtype, cudaStream_t stream);
cudaError_t launch_epilogue(const EpiArgs& p, int dtype, bool backward, cudaStream_t stream);
cudaError_t launch_gdn_map(const GdnArgs& p, int dtype, int N, cudaStream_t stream);
cudaError_t launch_compose(const ComposeArgs& p, int N, cudaStream_t stream);
// Set kStatusNonFinite in *status if any of the n elements at x (dtype as above; 16-byte aligned)
// is NaN or infinite.  x == nullptr or n == 0: nothing is launched.
cudaError_t launch_finite_scan(const void* x, int64_t n, int dtype, int* status, cudaStream_t stream);
// Device address of the current device's status word (looked up on every call).
cudaError_t device_status_ptr(int** out);

// Tensor maps of the token inputs for the chunked kernels' TMA staging.  Each [B,T,H,64] input is
// viewed as the 4-D tensor {64, H, T, B} (innermost first) and one box is {64, 1, 16, 1}: the 16
// tokens of a chunk for one head, rows past T filled with zeros.  Order r, w, k, v, a, b, dy.
struct InputMaps {
  CUtensorMap m[7];
};

cudaError_t launch_chunk_fwd(const FwdArgs& p, const InputMaps& tm, int dtype, cudaStream_t stream);
// Split form of the chunked forward for few (b,h) units: a chunk-parallel pass, then one sequential
// pass per unit.  Needs p.ckpt (the checkpoint slots carry the first pass's results) and uses the
// first 128 bytes of every row of y of each full chunk as scratch before writing y there.
cudaError_t launch_chunk_split_fwd(const FwdArgs& p, int dtype, cudaStream_t stream);
cudaError_t launch_chunk_bwd(const BwdArgs& p, const InputMaps& tm, int dtype, cudaStream_t stream);

}  // namespace wkv7
