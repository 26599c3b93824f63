// C ABI of libwkv7 (declared in include/wkv7.h): argument validation and
// dispatch to the sm_100a kernels.  Nothing here allocates memory or keeps
// state between calls; every kernel runs on the caller's stream.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <initializer_list>
#include <mutex>

#include "kernels.h"
#include "wkv7.h"

namespace {

constexpr int64_t kMaxGrid = 2147483647;   // grid.x limit: one CTA per (b,h)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool mul_ok(int64_t a, int64_t b, int64_t* out) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > INT64_MAX / a) return false;
  *out = a * b;
  return true;
}

// Common descriptor checks.  On success fills the element counts.
wkv7_status_t check_desc(const wkv7_desc_t* d, int64_t* units, int64_t* tok_elems) {
  if (!d) return WKV7_ERR_NULL;
  if ((d->N != 64 && d->N != 128) || (d->flags & ~(WKV7_FLAG_TEST_WAIT_TIMEOUT | WKV7_FLAG_CHECK_FINITE | WKV7_FLAG_LOG_DECAY |
                                  WKV7_FLAG_EPILOGUE_GRADS)) != 0u)
    return WKV7_ERR_UNSUPPORTED;
  if ((d->flags & WKV7_FLAG_TEST_WAIT_TIMEOUT) && (d->T > 16 || d->T < 0)) return WKV7_ERR_UNSUPPORTED;
  if (d->dtype != WKV7_F32 && d->dtype != WKV7_BF16 && d->dtype != WKV7_F16) return WKV7_ERR_DTYPE;
  if (d->algo < WKV7_ALGO_AUTO || d->algo > WKV7_ALGO_CHUNKED_SPLIT) return WKV7_ERR_UNSUPPORTED;
  if (d->B < 0 || d->T < 0 || d->H < 0) return WKV7_ERR_SHAPE;
  int64_t bh, bth, e;
  if (!mul_ok(d->B, d->H, &bh) || bh > kMaxGrid) return WKV7_ERR_SHAPE;
  if (!mul_ok(bh, d->T, &bth) || !mul_ok(bth, d->N * 4, &e)) return WKV7_ERR_SHAPE;   // byte count fits
  int64_t st;
  const int64_t n = d->N;
  if (!mul_ok(bh, n * n * 4, &st)) return WKV7_ERR_SHAPE;
  // the checkpoint workspace (one 16 KiB state per head per 16 tokens, then one int per head) must
  // have a byte count too, so that wkv7_workspace_bytes is non-zero for every accepted T > 0
  int64_t ck;
  if (!mul_ok(bh, (d->T + 15) / 16, &ck) || !mul_ok(ck, n * n * 4, &ck) || ck > INT64_MAX - (bh * 4 + 15))
    return WKV7_ERR_SHAPE;
  *units = bh;
  *tok_elems = bth * d->N;
  return WKV7_OK;
}

// The chunked kernels compute their products in tf32 (11 significant bits): on f32 inputs they
// cannot hold the 1e-4 bound that f32 results must meet, so only the exact scan takes f32.  (A
// decode step has no algorithm choice and is not affected.)
// Heads of 128 (the GDN map's) run the token-order scan only.
wkv7_status_t check_algo_dtype(const wkv7_desc_t* d) {
  if (d->N != 64 && d->algo >= WKV7_ALGO_CHUNKED) return WKV7_ERR_UNSUPPORTED;
  return (d->dtype == WKV7_F32 && d->algo >= WKV7_ALGO_CHUNKED) ? WKV7_ERR_UNSUPPORTED : WKV7_OK;
}

// Every listed pointer must be non-null (when `need`) and 16-byte aligned (when non-null).
wkv7_status_t check_ptrs(bool need, std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs) {
    if (!p) {
      if (need) return WKV7_ERR_NULL;
      continue;
    }
    if (!aligned16(p)) return WKV7_ERR_ALIGN;
  }
  return WKV7_OK;
}

wkv7_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA; }

// Under WKV7_FLAG_CHECK_FINITE: after a call's kernels succeeded, scan its outputs (pointer, element
// count, dtype code) on the same stream.
struct Output {
  const void* ptr;
  int64_t n;
  int dtype;
};
wkv7_status_t check_outputs(const wkv7_desc_t* d, cudaError_t launched, std::initializer_list<Output> outs, int* status,
                            cudaStream_t s) {
  if (launched != cudaSuccess) return WKV7_ERR_CUDA;
  if (!(d->flags & WKV7_FLAG_CHECK_FINITE)) return WKV7_OK;
  for (const Output& o : outs)
    if (wkv7::launch_finite_scan(o.ptr, o.n, o.dtype, status, s) != cudaSuccess) return WKV7_ERR_CUDA;
  return WKV7_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Tensor maps of up to seven [B,T,H,64] inputs as {64, H, T, B} with a {64, 1, 16, 1} box (the
// chunked kernels' staging).  Unused slots stay zero.
// `last_f32`: the last map describes an fp32 tensor whatever desc->dtype (dy under
// WKV7_FLAG_EPILOGUE_GRADS: the first quarter of the epilogue's block).
wkv7_status_t encode_inputs(const wkv7_desc_t* d, std::initializer_list<const void*> ptrs, wkv7::InputMaps* tm,
                            bool last_f32 = false) {
  *tm = wkv7::InputMaps{};
  if (d->T > INT32_MAX || d->H > INT32_MAX || d->B > INT32_MAX) return WKV7_ERR_SHAPE;   // 32-bit box coordinates
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_tiled();
  if (!enc) return WKV7_ERR_CUDA;
  const cuuint64_t es = d->dtype == WKV7_F32 ? 4 : 2;
  const CUtensorMapDataType dt = d->dtype == WKV7_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : d->dtype == WKV7_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dims[4] = {64, cuuint64_t(d->H), cuuint64_t(d->T), cuuint64_t(d->B)};
  const cuuint64_t strides[3] = {64 * es, cuuint64_t(d->H) * 64 * es, cuuint64_t(d->T) * cuuint64_t(d->H) * 64 * es};
  const cuuint32_t box[4] = {64, 1, 16, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const cuuint64_t strides32[3] = {64 * 4, cuuint64_t(d->H) * 64 * 4, cuuint64_t(d->T) * cuuint64_t(d->H) * 64 * 4};
  int i = 0;
  const int n = int(ptrs.size());
  for (const void* ptr : ptrs) {
    const bool f32 = last_f32 && i == n - 1;
    if (enc(&tm->m[i++], f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : dt, 4, const_cast<void*>(ptr), dims,
            f32 ? strides32 : strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return WKV7_ERR_CUDA;
  }
  return WKV7_OK;
}

// Bytes a staging barrier expects beyond its copies: the timeout test hook (see wkv7.h).
unsigned test_extra_tx(const wkv7_desc_t* d) { return (d->flags & WKV7_FLAG_TEST_WAIT_TIMEOUT) ? 16u : 0u; }

bool use_chunked(const wkv7_desc_t* d) {
  if (d->algo == WKV7_ALGO_SCAN || d->N != 64) return false;
  if (d->algo == WKV7_ALGO_AUTO) return d->dtype != WKV7_F32;
  return true;
}

// Split form of the chunked forward: forced, or chosen for few units (at most one per SM) when a
// workspace is there to carry its first pass.  The timeout test hook exercises the fused form only.
wkv7_status_t use_split(const wkv7_desc_t* d, int64_t units, const void* workspace, bool* split) {
  *split = false;
  if (d->algo == WKV7_ALGO_CHUNKED_SPLIT) {
    if (!workspace) return WKV7_ERR_WORKSPACE;
    *split = (d->flags & WKV7_FLAG_TEST_WAIT_TIMEOUT) == 0u;
    return WKV7_OK;
  }
  if (d->algo == WKV7_ALGO_CHUNKED_FUSED || !workspace || (d->flags & WKV7_FLAG_TEST_WAIT_TIMEOUT)) return WKV7_OK;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return WKV7_ERR_CUDA;
  *split = units <= int64_t(sms);
  return WKV7_OK;
}

}  // namespace

namespace wkv7 {
wkv7_status_t validate_desc(const wkv7_desc_t* d) {
  int64_t units = 0, te = 0;
  const wkv7_status_t st = check_desc(d, &units, &te);
  return st != WKV7_OK ? st : check_algo_dtype(d);
}
}  // namespace wkv7

extern "C" {

int wkv7_version(void) { return 100; }

const char* wkv7_status_string(wkv7_status_t s) {
  switch (s) {
    case WKV7_OK: return "ok";
    case WKV7_ERR_NULL: return "a required pointer is NULL";
    case WKV7_ERR_SHAPE: return "invalid or overflowing shape";
    case WKV7_ERR_DTYPE: return "unknown dtype";
    case WKV7_ERR_ALIGN: return "tensor pointer is not 16-byte aligned";
    case WKV7_ERR_WORKSPACE: return "checkpoint workspace is required";
    case WKV7_ERR_UNSUPPORTED: return "unsupported head size, algorithm, flags or step length";
    case WKV7_ERR_CUDA: return "CUDA launch failed";
    case WKV7_ERR_TIMEOUT: return "device-side wait timed out";
    case WKV7_ERR_SCRATCH_LIMIT: return "problem exceeds the fixed scratch of wkv7_train_step_noalloc";
    case WKV7_ERR_NONFINITE: return "an output checked under WKV7_FLAG_CHECK_FINITE holds a NaN or infinity";
    case WKV7_ERR_BOUNDS: return "a kernel index failed its bounds check (debug build)";
  }
  return "unknown status";
}

// Checkpoint bytes (one fp32 64x64 state per head per 16 tokens), or -1 on overflow.
int64_t checkpoint_bytes(const wkv7_desc_t* d, int64_t units) {
  const int64_t nc = (d->T + 15) / 16;
  int64_t n1, n2;
  if (!mul_ok(units, nc, &n1) || !mul_ok(n1, int64_t(d->N) * d->N * 4, &n2)) return -1;
  return n2;
}

// Workspace = checkpoints, then one int per (b,h) for the chunked backward's
// "recompute this unit exactly" marks, rounded up to 16 bytes.
size_t wkv7_workspace_bytes(const wkv7_desc_t* d) {
  int64_t units = 0, te = 0;
  if (check_desc(d, &units, &te) != WKV7_OK) return 0;
  const int64_t ck = checkpoint_bytes(d, units);
  if (ck < 0 || d->T == 0) return 0;
  return static_cast<size_t>(ck + ((units * 4 + 15) / 16) * 16);
}

wkv7_status_t wkv7_forward(const wkv7_desc_t* d, const void* r, const void* w, const void* k, const void* v,
                           const void* a, const void* b, const float* s0, const uint8_t* reset, void* y,
                           float* s_out, void* workspace, void* stream) {
  int64_t units = 0, te = 0;
  wkv7_status_t st = check_desc(d, &units, &te);
  if (st != WKV7_OK) return st;
  st = check_algo_dtype(d);
  if (st != WKV7_OK) return st;
  st = check_ptrs(te > 0, {r, w, k, v, a, b, y});
  if (st != WKV7_OK) return st;
  st = check_ptrs(false, {s0, s_out, workspace});
  if (st != WKV7_OK) return st;
  if (d->algo == WKV7_ALGO_CHUNKED_SPLIT && te > 0 && !workspace) return WKV7_ERR_WORKSPACE;
  if (units == 0) return WKV7_OK;
  int* status = nullptr;
  if (wkv7::device_status_ptr(&status) != cudaSuccess) return WKV7_ERR_CUDA;
  wkv7::FwdArgs p{d->B, d->T, d->H, r, w, k, v, a, b, s0, reset, y, s_out, static_cast<float*>(workspace),
                  status, test_extra_tx(d), (d->flags & WKV7_FLAG_LOG_DECAY) != 0u};
  p.N = int(d->N);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const std::initializer_list<Output> outs = {{y, te, d->dtype}, {s_out, units * d->N * d->N, WKV7_F32}};
  if (d->T == 0 || !use_chunked(d)) return check_outputs(d, wkv7::launch_scan_fwd(p, d->dtype, s), outs, status, s);
  bool split = false;
  st = use_split(d, units, workspace, &split);
  if (st != WKV7_OK) return st;
  if (split) return check_outputs(d, wkv7::launch_chunk_split_fwd(p, d->dtype, s), outs, status, s);
  wkv7::InputMaps tm;
  st = encode_inputs(d, {r, w, k, v, a, b}, &tm);
  if (st != WKV7_OK) return st;
  return check_outputs(d, wkv7::launch_chunk_fwd(p, tm, d->dtype, s), outs, status, s);
}

wkv7_status_t wkv7_backward(const wkv7_desc_t* d, const void* r, const void* w, const void* k, const void* v,
                            const void* a, const void* b, const float* s0, const uint8_t* reset, const void* dy,
                            const float* dsT, const void* workspace, void* dr, void* dw, void* dk, void* dv,
                            void* da, void* db, float* ds0, void* stream) {
  int64_t units = 0, te = 0;
  wkv7_status_t st = check_desc(d, &units, &te);
  if (st != WKV7_OK) return st;
  if (d->N != 64) return WKV7_ERR_UNSUPPORTED;   // the backward kernels are written for heads of 64
  st = check_algo_dtype(d);
  if (st != WKV7_OK) return st;
  st = check_ptrs(te > 0, {r, w, k, v, a, b, dy, dr, dw, dk, dv, da, db});
  if (st != WKV7_OK) return st;
  st = check_ptrs(false, {s0, dsT, ds0, workspace});
  if (st != WKV7_OK) return st;
  if (te > 0 && !workspace) return WKV7_ERR_WORKSPACE;
  if (units == 0) return WKV7_OK;
  int* flags = d->T > 0 ? reinterpret_cast<int*>(static_cast<char*>(const_cast<void*>(workspace)) +
                                                 checkpoint_bytes(d, units))
                        : nullptr;
  int* status = nullptr;
  if (wkv7::device_status_ptr(&status) != cudaSuccess) return WKV7_ERR_CUDA;
  wkv7::BwdArgs p{d->B, d->T, d->H, r, w, k, v, a, b, s0, reset, dy, dsT, static_cast<const float*>(workspace),
                  dr, dw, dk, dv, da, db, ds0, flags, status, test_extra_tx(d),
                  (d->flags & WKV7_FLAG_LOG_DECAY) != 0u, (d->flags & WKV7_FLAG_EPILOGUE_GRADS) != 0u};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const std::initializer_list<Output> outs = {{dr, te, d->dtype}, {dw, te, d->dtype}, {dk, te, d->dtype},
                                              {dv, te, d->dtype}, {da, te, d->dtype}, {db, te, d->dtype},
                                              {ds0, units * 64 * 64, WKV7_F32}};
  if (d->T == 0 || !use_chunked(d))
    return check_outputs(d, wkv7::launch_scan_bwd(p, d->dtype, false, s), outs, status, s);
  // Chunked pass, then the exact scan for the units it marked (decays too small for 1/L scaling).
  wkv7::InputMaps tm;
  st = encode_inputs(d, {r, w, k, v, a, b, dy}, &tm, (d->flags & WKV7_FLAG_EPILOGUE_GRADS) != 0u);
  if (st != WKV7_OK) return st;
  cudaError_t e = wkv7::launch_chunk_bwd(p, tm, d->dtype, s);
  if (e != cudaSuccess) return WKV7_ERR_CUDA;
  return check_outputs(d, wkv7::launch_scan_bwd(p, d->dtype, true, s), outs, status, s);
}

// The epilogue's descriptor: the token tensors as everywhere; flags other than CHECK_FINITE refused.
static wkv7_status_t check_epilogue(const wkv7_desc_t* d, const wkv7_epilogue_t* ep, int64_t* units, int64_t* te) {
  wkv7_status_t st = check_desc(d, units, te);
  if (st != WKV7_OK) return st;
  if ((d->flags & ~WKV7_FLAG_CHECK_FINITE) != 0u || d->N != 64) return WKV7_ERR_UNSUPPORTED;
  if (!ep || !ep->ln_w || !ep->ln_b || !ep->r_k) return WKV7_ERR_NULL;
  if (!(ep->eps > 0.f) || !(ep->eps < 1e30f)) return WKV7_ERR_UNSUPPORTED;   // also refuses NaN
  for (const void* q : {static_cast<const void*>(ep->ln_w), static_cast<const void*>(ep->ln_b),
                        static_cast<const void*>(ep->r_k)})
    if (reinterpret_cast<uintptr_t>(q) % 4u != 0u) return WKV7_ERR_ALIGN;
  return WKV7_OK;
}

wkv7_status_t wkv7_epilogue_forward(const wkv7_desc_t* d, const wkv7_epilogue_t* ep, const void* y, const void* r,
                                    const void* k, const void* v, const void* g, void* out, void* stream) {
  int64_t units = 0, te = 0;
  wkv7_status_t st = check_epilogue(d, ep, &units, &te);
  if (st != WKV7_OK) return st;
  st = check_ptrs(te > 0, {y, r, k, v, g, out});
  if (st != WKV7_OK) return st;
  if (te == 0) return WKV7_OK;
  int* status = nullptr;
  if (wkv7::device_status_ptr(&status) != cudaSuccess) return WKV7_ERR_CUDA;
  wkv7::EpiArgs p{d->B, d->T, d->H, y, r, k, v, g, nullptr, ep->ln_w, ep->ln_b, ep->r_k, ep->eps,
                  out, nullptr, nullptr, nullptr, nullptr, nullptr, status};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return check_outputs(d, wkv7::launch_epilogue(p, d->dtype, false, s), {{out, te, d->dtype}}, status, s);
}

wkv7_status_t wkv7_epilogue_backward(const wkv7_desc_t* d, const wkv7_epilogue_t* ep, const void* y, const void* r,
                                     const void* k, const void* v, const void* g, const void* dout, float* eg,
                                     void* dg, float* dln_w, float* dln_b, float* dr_k, void* stream) {
  int64_t units = 0, te = 0;
  wkv7_status_t st = check_epilogue(d, ep, &units, &te);
  if (st != WKV7_OK) return st;
  st = check_ptrs(te > 0, {y, r, k, v, g, dout, eg, dg});
  if (st != WKV7_OK) return st;
  for (const float* q : {dln_w, dln_b, dr_k})
    if (q && reinterpret_cast<uintptr_t>(q) % 4u != 0u) return WKV7_ERR_ALIGN;
  if (te == 0) return WKV7_OK;
  int* status = nullptr;
  if (wkv7::device_status_ptr(&status) != cudaSuccess) return WKV7_ERR_CUDA;
  wkv7::EpiArgs p{d->B, d->T, d->H, y, r, k, v, g, dout, ep->ln_w, ep->ln_b, ep->r_k, ep->eps,
                  nullptr, dg, eg, dln_w, dln_b, dr_k, status};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return check_outputs(d, wkv7::launch_epilogue(p, d->dtype, true, s),
                       {{eg, 4 * te, WKV7_F32}, {dg, te, d->dtype}, {dln_w, d->H * 64, WKV7_F32}, {dln_b, d->H * 64, WKV7_F32},
                        {dr_k, d->H * 64, WKV7_F32}},
                       status, s);
}

wkv7_status_t wkv7_forward_epilogue(const wkv7_desc_t* d, const wkv7_epilogue_t* ep, const void* r, const void* w,
                                    const void* k, const void* v, const void* a, const void* b, const float* s0,
                                    const uint8_t* reset, const void* g, void* y, void* out, float* s_out,
                                    void* workspace, void* stream) {
  int64_t units = 0, te = 0;
  wkv7_status_t st = check_desc(d, &units, &te);
  if (st != WKV7_OK) return st;
  st = check_algo_dtype(d);
  if (st != WKV7_OK) return st;
  if (d->flags & WKV7_FLAG_EPILOGUE_GRADS) return WKV7_ERR_UNSUPPORTED;
  wkv7_desc_t de = *d;   // the epilogue's own descriptor: only the finite check carries over
  de.flags = d->flags & WKV7_FLAG_CHECK_FINITE;
  st = check_epilogue(&de, ep, &units, &te);
  if (st != WKV7_OK) return st;
  st = check_ptrs(te > 0, {r, w, k, v, a, b, g, out});
  if (st != WKV7_OK) return st;
  st = check_ptrs(false, {s0, s_out, workspace, y});
  if (st != WKV7_OK) return st;
  if (units == 0 || te == 0) return wkv7_forward(d, r, w, k, v, a, b, s0, reset, y ? y : out, s_out, workspace, stream);
  bool split = false;
  const bool fused = d->dtype != WKV7_F32 && use_chunked(d) && use_split(d, units, workspace, &split) == WKV7_OK && !split;
  if (!fused) {   // the recurrence, then the epilogue on its stored y (out holds y in between when y is NULL)
    void* yb = y ? y : out;
    st = wkv7_forward(d, r, w, k, v, a, b, s0, reset, yb, s_out, workspace, stream);
    if (st != WKV7_OK) return st;
    return wkv7_epilogue_forward(&de, ep, yb, r, k, v, g, out, stream);
  }
  int* status = nullptr;
  if (wkv7::device_status_ptr(&status) != cudaSuccess) return WKV7_ERR_CUDA;
  wkv7::FwdArgs p{d->B, d->T, d->H, r, w, k, v, a, b, s0, reset, y, s_out, static_cast<float*>(workspace),
                  status, test_extra_tx(d), (d->flags & WKV7_FLAG_LOG_DECAY) != 0u,
                  g, out, ep->ln_w, ep->ln_b, ep->r_k, ep->eps, int(d->N)};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  wkv7::InputMaps tm;
  st = encode_inputs(d, {r, w, k, v, a, b}, &tm);
  if (st != WKV7_OK) return st;
  return check_outputs(d, wkv7::launch_chunk_fwd(p, tm, d->dtype, s),
                       {{out, te, d->dtype}, {y, te, d->dtype}, {s_out, units * 64 * 64, WKV7_F32}}, status, s);
}

wkv7_status_t wkv7_state_compose(const wkv7_desc_t* d, const float* S, const float* P, const float* U, float* out,
                                 int transpose_p, void* stream) {
  int64_t units = 0, te = 0;
  wkv7_status_t st = check_desc(d, &units, &te);
  if (st != WKV7_OK) return st;
  if ((d->flags & ~WKV7_FLAG_CHECK_FINITE) != 0u) return WKV7_ERR_UNSUPPORTED;
  st = check_ptrs(units > 0, {out});
  if (st != WKV7_OK) return st;
  if (units > 0 && S && !P) return WKV7_ERR_NULL;
  st = check_ptrs(false, {S, P, U});
  if (st != WKV7_OK) return st;
  if (out && (static_cast<const void*>(out) == S || static_cast<const void*>(out) == P)) return WKV7_ERR_UNSUPPORTED;
  if (units == 0) return WKV7_OK;
  int* status = nullptr;
  if (wkv7::device_status_ptr(&status) != cudaSuccess) return WKV7_ERR_CUDA;
  wkv7::ComposeArgs p{units, S, P, U, out, transpose_p != 0, status};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return check_outputs(d, wkv7::launch_compose(p, d->N, s), {{out, units * d->N * d->N, WKV7_F32}}, status, s);
}

wkv7_status_t wkv7_gdn_map(const wkv7_desc_t* d, const wkv7_gdn_t* gd, const void* q, const void* k,
                           const float* g, const float* beta, void* r, void* x, void* kw, void* a, void* b,
                           void* stream) {
  int64_t units = 0, te = 0;
  wkv7_status_t st = check_desc(d, &units, &te);
  if (st != WKV7_OK) return st;
  if ((d->flags & ~WKV7_FLAG_CHECK_FINITE) != 0u) return WKV7_ERR_UNSUPPORTED;
  if (!gd) return WKV7_ERR_NULL;
  if (gd->Hk < 1 || d->H % gd->Hk != 0 || !(gd->eps >= 0.f) || !(gd->eps < 1e30f) ||
      !(gd->r_scale == gd->r_scale) || !(gd->r_scale < 1e30f && gd->r_scale > -1e30f))
    return WKV7_ERR_UNSUPPORTED;
  st = check_ptrs(te > 0, {q, k, r, x, kw, a, b});
  if (st != WKV7_OK) return st;
  if (te > 0 && (!g || !beta)) return WKV7_ERR_NULL;
  for (const float* p : {g, beta})
    if (reinterpret_cast<uintptr_t>(p) % 4u != 0u) return WKV7_ERR_ALIGN;
  if (te == 0) return WKV7_OK;
  int* status = nullptr;
  if (wkv7::device_status_ptr(&status) != cudaSuccess) return WKV7_ERR_CUDA;
  wkv7::GdnArgs p{d->B, d->T, d->H, gd->Hk, q, k, g, beta, gd->eps, gd->r_scale, r, x, kw, a, b, status};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return check_outputs(d, wkv7::launch_gdn_map(p, d->dtype, d->N, s),
                       {{r, te, d->dtype}, {kw, te, d->dtype}, {a, te, d->dtype}, {b, te, d->dtype}}, status, s);
}

wkv7_status_t wkv7_step(const wkv7_desc_t* d, const void* r, const void* w, const void* k, const void* v,
                        const void* a, const void* b, float* state, const uint8_t* active, void* y, void* stream) {
  int64_t units = 0, te = 0;
  wkv7_status_t st = check_desc(d, &units, &te);
  if (st != WKV7_OK) return st;
  if (d->T != 1) return WKV7_ERR_UNSUPPORTED;
  st = check_ptrs(units > 0, {r, w, k, v, a, b, state, y});
  if (st != WKV7_OK) return st;
  if (units == 0) return WKV7_OK;
  int* status = nullptr;
  if (wkv7::device_status_ptr(&status) != cudaSuccess) return WKV7_ERR_CUDA;
  wkv7::StepArgs p{d->B, d->H, r, w, k, v, a, b, state, active, y, status, (d->flags & WKV7_FLAG_LOG_DECAY) != 0u,
                   d->N};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return check_outputs(d, wkv7::launch_step(p, d->dtype, s), {{y, units * d->N, d->dtype}, {state, units * d->N * d->N, WKV7_F32}},
                       status, s);
}

}  // extern "C"
