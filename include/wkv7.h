/*
 * wkv7.h -- C ABI of the B200 (sm_100a) WKV-7 library (libwkv7.so).
 *
 * WKV-7 is the recurrence at the core of RWKV-7 "Goose": the one part of the
 * model that stock array operations cannot express efficiently, which the
 * rwkv-metal page therefore runs as a hand-written kernel with a checkpointed
 * backward (section "The Metal WKV-7 kernel").  Per (batch b, head h) it
 * keeps an fp32 N x N state S (row i = value channel, column j = key channel)
 * and, for each token t,
 *
 *     sa[i]   = sum_j S[i][j] * a_t[j]                 (S before the update)
 *     S[i][j] = S[i][j] * w_t[j] + sa[i] * b_t[j] + v_t[i] * k_t[j]
 *     y_t[i]  = sum_j S[i][j] * r_t[j]                 (S after the update)
 *
 * i.e. S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T, y_t = S_t r_t: a
 * diagonal-plus-rank-one ("generalised delta rule") transition.  The
 * rwkv-lab page ("GDN subset of RWKV-7") shows the gated delta rule as the
 * special case w = exp(g), a = -k, b = k exp(g) beta, k_write = beta k.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Head size N is 64 (the HF model card page limits its kernel to heads
 *   of 64 channels with an fp32 state).  wkv7_forward with the token-order
 *   scan (algo SCAN, or AUTO, which picks it), wkv7_step and wkv7_gdn_map also
 *   take N = 128, the head size of the gated-DeltaNet layers that the rwkv-lab
 *   page maps onto this recurrence; every other entry point and algo returns
 *   WKV7_ERR_UNSUPPORTED for it, as does any other N.  Below, "64" in a shape
 *   stands for N where N = 128 is accepted.
 * - Activations r,w,k,v,a,b,y,dy and the gradients dr..db are [B,T,H,64],
 *   contiguous, row-major, all in the one dtype of the descriptor (f32, bf16
 *   or f16, the three activation types the same page lists).  Outputs in a
 *   16-bit dtype are rounded to nearest even.  w is the multiplicative decay
 *   (normally in (0,1]).
 * - States s0, s_out, dsT, ds0 and the decode state are fp32 [B,H,64,64],
 *   contiguous, S[i][j] at offset i*64+j.
 * - reset is [B,T] bytes: reset[b][t] != 0 zeroes the incoming state before
 *   token t (the HF model card page packs several documents into one row and
 *   zeroes the state where each new one begins).  At t = 0 it overrides s0.  No
 *   gradient crosses a reset.
 * - Every pointer is a DEVICE pointer, 16-byte aligned (reset and active may
 *   have any alignment).  The caller allocates and owns every buffer; the
 *   library allocates nothing, keeps no per-call state and may be called from
 *   several host threads on different streams -- except
 *   wkv7_train_step_noalloc, whose calls share one fixed scratch array of the
 *   library and must not overlap (see there).
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *   asynchronous on it.  The returned status covers argument validation and
 *   the launch itself (cudaGetLastError); on any validation error nothing is
 *   launched and no output is touched.
 * - Any T >= 0 is accepted.  T need not be a multiple of 16 (the checkpoint
 *   interval; the HF model card page pads separate sequences up to a multiple
 *   of it) -- here the padding is internal.
 */
#ifndef WKV7_H
#define WKV7_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WKV7_OK = 0,
  WKV7_ERR_NULL = 1,        /* a required pointer is NULL                                    */
  WKV7_ERR_SHAPE = 2,       /* B, T or H negative, or an element or workspace byte count overflows int64 */
  WKV7_ERR_DTYPE = 3,       /* dtype code is not a wkv7_dtype_t                               */
  WKV7_ERR_ALIGN = 4,       /* a tensor pointer is not 16-byte aligned                        */
  WKV7_ERR_WORKSPACE = 5,   /* backward without a checkpoint workspace                        */
  WKV7_ERR_UNSUPPORTED = 6, /* N != 64, unknown algo or flags, CHUNKED* with f32, T != 1 for a step */
  WKV7_ERR_CUDA = 7,        /* the launch failed; cudaGetLastError() was not cudaSuccess      */
  WKV7_ERR_TIMEOUT = 8,     /* reserved for device-side bounded waits                          */
  WKV7_ERR_SCRATCH_LIMIT = 9, /* the problem needs more than WKV7_NOALLOC_SCRATCH_BYTES of scratch */
  WKV7_ERR_NONFINITE = 10,   /* WKV7_FLAG_CHECK_FINITE found a NaN or infinity in an output       */
  WKV7_ERR_BOUNDS = 11       /* debug build only: a kernel index failed its bounds check          */
} wkv7_status_t;

typedef enum { WKV7_F32 = 0, WKV7_BF16 = 1, WKV7_F16 = 2 } wkv7_dtype_t;

/*
 * Algorithm.  SCAN: token-order scan on FP32 cores, state in registers.
 * CHUNKED: 16-token chunks with the intra-chunk products on tensor cores
 * (the chunk-parallel form that the HF model card page also mentions), in
 * one of two forms for the forward pass:
 *   - fused: one CTA per (b,h) does everything chunk by chunk;
 *   - split: first every chunk's state-independent products in parallel,
 *     then one short sequential pass per (b,h).  It needs the workspace
 *     (its first pass leaves its results in the checkpoint slots and in the
 *     first 128 bytes of each row of y, which the second pass overwrites).
 * CHUNKED picks split when a workspace is passed and B*H is at most the
 * device's SM count, fused otherwise; CHUNKED_FUSED and CHUNKED_SPLIT force
 * one (CHUNKED_SPLIT without a workspace: WKV7_ERR_WORKSPACE).  The
 * backward has one chunked form, which all three select.  AUTO: CHUNKED for
 * 16-bit inputs, SCAN for f32.  The chunked kernels compute their products
 * in tf32 (fp32 accumulation), which cannot hold f32 results to the 1e-4
 * bound that f32 inputs ask for: any CHUNKED* algo with f32 inputs is
 * refused (WKV7_ERR_UNSUPPORTED).  All produce the same result up to
 * floating-point rounding.
 */
typedef enum {
  WKV7_ALGO_AUTO = 0,
  WKV7_ALGO_SCAN = 1,
  WKV7_ALGO_CHUNKED = 2,
  WKV7_ALGO_CHUNKED_FUSED = 3,
  WKV7_ALGO_CHUNKED_SPLIT = 4
} wkv7_algo_t;

typedef struct {
  int64_t B;      /* batch rows                                  */
  int64_t T;      /* tokens per row (for wkv7_step: must be 1)   */
  int64_t H;      /* heads                                       */
  int32_t N;      /* head size: 64 (128 where stated)            */
  int32_t dtype;  /* wkv7_dtype_t of every activation/gradient   */
  int32_t algo;   /* wkv7_algo_t                                 */
  uint32_t flags; /* 0, or the WKV7_FLAG_* bits below            */
} wkv7_desc_t;

/*
 * desc->flags bit (no page counterpart: a test hook for the device status
 * word).  With it, the chunked kernels' staging of input rows expects 16
 * bytes that are never copied, so the bounded wait for them runs out after
 * about one second; the chunk is then computed from global memory instead
 * (forward: token by token; backward: the exact scan), the results stay
 * correct, and wkv7_get_device_status() reports WKV7_ERR_TIMEOUT.  Accepted
 * only with T <= 16; every other flag bit must be 0 (WKV7_ERR_UNSUPPORTED).
 */
#define WKV7_FLAG_TEST_WAIT_TIMEOUT 0x80000000u

/*
 * desc->flags bit: after the call's kernels, scan its floating outputs on the
 * same stream (forward: y and s_out; backward: dr..db and ds0; step: y and
 * the updated state) and record any NaN or infinity in the device status
 * word, which wkv7_get_device_status() then reports as WKV7_ERR_NONFINITE.
 * The scan reads each output once more; the results themselves are
 * unchanged.  It may be combined with WKV7_FLAG_TEST_WAIT_TIMEOUT.
 */
#define WKV7_FLAG_CHECK_FINITE 0x1u

/*
 * Log-space decay input (rwkv-lab page, "Highlight result -- GDN in RWKV-7":
 * the wkv7 kernel there takes its decay in log space).  With this flag the
 * `w` argument of wkv7_forward, wkv7_backward, wkv7_step and
 * wkv7_train_step_noalloc holds x, same dtype and layout, and the kernels use
 * the decay w = exp(-exp(x)) (log w = -exp(x)), computed in fp32 from the
 * stored x -- so a bf16 input no longer rounds w itself, whose spacing near 1
 * is 2^-8.  wkv7_backward then writes dL/dx into its `dw` output.  Every
 * algorithm accepts it; the chunked forms apply their decay-range test
 * (below) to the computed w.
 */
#define WKV7_FLAG_LOG_DECAY 0x2u

/*
 * wkv7_backward (and wkv7_train_step_noalloc) desc->flags bit: `dy` points at
 * the fp32 block that wkv7_epilogue_backward writes, [4][B,T,H,64], 16-byte
 * aligned: dy itself, then the epilogue's (bonus) parts of dr, dk and dv,
 * which the recurrence's backward adds to its own before the one rounding to
 * the output dtype.  Both stay in fp32 on purpose: the GroupNorm's gradient
 * is large on tokens whose y has a small spread (right after a reset, for
 * instance) and, rounded to bf16 first, costs the gradients ~10 % of their
 * RMS there; and rounding the bonus parts before the sum would round dr, dk,
 * dv twice (~2 % of their RMS).
 */
#define WKV7_FLAG_EPILOGUE_GRADS 0x4u

/*
 * Device status word (the device-side error channel of the boundary).
 * Kernels record errors they cannot return from an asynchronous launch --
 * a bounded wait that ran out, a non-finite output found under
 * WKV7_FLAG_CHECK_FINITE, or (debug build) an index that failed its bounds
 * check -- in one word per device.  This call synchronises the current
 * device, reads the word and, if `clear` is non-zero, resets it.  Returns
 * WKV7_OK; else, in this order of precedence, WKV7_ERR_TIMEOUT if a wait ran
 * out since the last clear, WKV7_ERR_BOUNDS if a checked index fell outside
 * its buffer (the access was skipped), WKV7_ERR_NONFINITE if a checked
 * output held a NaN or infinity; or WKV7_ERR_CUDA if synchronising or
 * reading failed (e.g. no device).
 */
wkv7_status_t wkv7_get_device_status(int clear);

/*
 * 1 in the debug build of this library (libwkv7_debug.so, compiled with
 * WKV7_DEBUG), 0 in the release build (libwkv7.so).  The debug build is the
 * same ABI and the same arithmetic; its kernels also check every index they
 * compute -- global offsets of activations, states, checkpoints and
 * workspace marks, TMA box coordinates, bulk-copy ranges and shared-memory
 * operand indices -- against the extent of its buffer, skip an access that
 * fails and set WKV7_ERR_BOUNDS in the device status word instead of
 * faulting.  Results of a run with no failed check are bit-identical to the
 * release build's.
 */
int wkv7_debug_checks(void);

/* Library version, major*10000 + minor*100 + patch. */
int wkv7_version(void);

/* Static string for a status code (never NULL). */
const char* wkv7_status_string(wkv7_status_t status);

/*
 * Bytes of workspace that wkv7_forward writes and wkv7_backward
 * reads: one fp32 64x64 state per (b, h) every 16 tokens, i.e.
 * B*H*ceil(T/16)*64*64*4 bytes (rwkv-metal page: the state is saved once per
 * 16 tokens; RWKV-MLX page, "Key Design Decisions" 2, puts the cost near 12 MB
 * at B=2, T=512, 12 heads -- this formula gives 12.58 MB).
 * Checkpoint c holds the state after token min(16(c+1), T) - 1, its element
 * (i, j) at offset (i/16)*1024 + (j/8)*128 + (4*(i%8) + (j%8)/2)*4
 * + 2*((i/8)%2) + j%2 (the order of the kernels' mma accumulator fragments, so
 * that every warp moves 512 contiguous bytes per store); with N = 128 the
 * checkpoints are 128x128, row-major (no backward reads them).  After the
 * checkpoints come B*H ints (rounded up to 16 bytes) that wkv7_backward uses
 * to mark heads it must recompute with the exact scan.
 * Returns 0 for an invalid descriptor or T == 0.
 */
size_t wkv7_workspace_bytes(const wkv7_desc_t* desc);

/*
 * Forward pass over T tokens (rwkv-metal page, "The Metal WKV-7 kernel": the
 * full sequence is processed by a single forward launch that saves the state
 * once per 16 tokens; entry points wkv7_train / wkv7_train_with_state).
 *
 *   r,w,k,v,a,b  in   [B,T,H,64] desc->dtype
 *   s0           in   [B,H,64,64] fp32 initial state, or NULL for zeros
 *   reset        in   [B,T] u8, or NULL for no resets
 *   y            out  [B,T,H,64] desc->dtype
 *   s_out        out  [B,H,64,64] fp32 final state, or NULL
 *   workspace    out  wkv7_workspace_bytes(desc) bytes of checkpoints for the
 *                     backward, or NULL (inference: no checkpoints written).
 *                     Passing one for inference as well lets a forward with
 *                     B*H at most the SM count run the split chunked form,
 *                     several times faster there.
 * y must not overlap any input.
 */
wkv7_status_t wkv7_forward(const wkv7_desc_t* desc, const void* r, const void* w, const void* k,
                           const void* v, const void* a, const void* b, const float* s0,
                           const uint8_t* reset, void* y, float* s_out, void* workspace, void* stream);

/*
 * Backward pass (rwkv-metal page: a single backward launch that rebuilds each
 * 16-token chunk from its checkpoint, with gradients flowing into the initial
 * state as well).
 * Inputs are those of the forward call that wrote `workspace` (same
 * descriptor, r..b, s0, reset), plus
 *
 *   dy           in   [B,T,H,64] gradient of the loss w.r.t. y
 *   dsT          in   [B,H,64,64] fp32 gradient w.r.t. the final state, or NULL
 *   dr..db       out  [B,T,H,64] desc->dtype gradients w.r.t. r,w,k,v,a,b
 *   ds0          out  [B,H,64,64] fp32 gradient w.r.t. s0, or NULL
 *
 * dw is the derivative with respect to the multiplicative decay w itself.
 * `workspace` must not be NULL when T > 0 (WKV7_ERR_WORKSPACE).
 */
wkv7_status_t wkv7_backward(const wkv7_desc_t* desc, const void* r, const void* w, const void* k,
                            const void* v, const void* a, const void* b, const float* s0,
                            const uint8_t* reset, const void* dy, const float* dsT,
                            const void* workspace, void* dr, void* dw, void* dk, void* dv, void* da,
                            void* db, float* ds0, void* stream);

/*
 * One decode token for B*H resident states, in place (rwkv-metal page: a
 * one-token step on a carried state, with ragged batches padded on the right
 * without changing the padded rows' results).
 *
 *   desc         B, H, N (64 or 128), dtype; T must be 1; algo is ignored
 *   r..b         in      [B,H,64] desc->dtype (one token per row)
 *   state        in/out  [B,H,64,64] fp32
 *   active       in      [B] u8, or NULL for all rows active.  A row with
 *                        active[b] == 0 leaves its state bitwise unchanged
 *                        and gets y = 0.
 *   y            out     [B,H,64] desc->dtype
 */
wkv7_status_t wkv7_step(const wkv7_desc_t* desc, const void* r, const void* w, const void* k,
                        const void* v, const void* a, const void* b, float* state,
                        const uint8_t* active, void* y, void* stream);

/*
 * Forward + backward in one call, allocating nothing -- for callers that
 * cannot call cudaMalloc (device memory owned by another allocator, such as
 * a framework's caching allocator or a serving engine that reserves all free
 * memory up front, or code paths where allocation is not allowed).  The
 * pages have no counterpart to this entry point.
 *
 * Same arguments and results as wkv7_forward followed by wkv7_backward on
 * the same descriptor, except that no workspace is passed: the checkpoints
 * and the backward's per-head marks live in one fixed device array of the
 * library, WKV7_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the
 * library holds until the process exits.  A problem whose
 * wkv7_workspace_bytes() exceeds that size is rejected with
 * WKV7_ERR_SCRATCH_LIMIT before anything is launched (32 MiB holds, e.g.,
 * B=2, T=512, H=12, or B*H*ceil(T/16) <= 2047 checkpoints).
 *
 * Every call looks up the array's device address on the calling device
 * (the runtime's symbol lookup; nothing is cached, so a cudaDeviceReset in
 * between is harmless).  The first call on a device also loads the library's
 * module there; make that first call before any stream capture.  All calls
 * share the array and it keeps the last call's contents (nothing in it needs
 * to start at zero), so calls that overlap on the GPU -- on different streams
 * or different host threads -- race on it and must be serialised by the
 * caller.
 */
#define WKV7_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
wkv7_status_t wkv7_train_step_noalloc(const wkv7_desc_t* desc, const void* r, const void* w, const void* k,
                                      const void* v, const void* a, const void* b, const float* s0,
                                      const uint8_t* reset, void* y, float* s_out, const void* dy,
                                      const float* dsT, void* dr, void* dw, void* dk, void* dv, void* da,
                                      void* db, float* ds0, void* stream);

/*
 * ------------------------------------------------------------------ WKV epilogue
 * The step after the recurrence in an RWKV-7 time-mix block, one streaming
 * kernel each way (rwkv-metal page, architecture table: "ln_x ... GroupNorm
 * (per head)"; rwkv-lab page, "Native RWKV megakernel backend": the state
 * update fused "through GroupNorm, the RWKV bonus, and output gating").  Per
 * (b, t, h), channels i, j = 0..63:
 *   mu, var = mean and variance of y over the head's 64 channels,
 *   yn_i = (y_i - mu) / sqrt(var + eps)                 (GroupNorm, one group per head)
 *   s    = sum_j r_j k_j r_k[h][j]                      (the bonus weight)
 *   out_i = (yn_i ln_w[h][i] + ln_b[h][i] + s v_i) g_i  (bonus, then gating)
 * with r, k, v the recurrence's own inputs and g the gate.  All token
 * tensors [B,T,H,64] in desc->dtype, 16-byte aligned; the parameters
 * ln_w, ln_b, r_k are fp32 [H,64] (4-byte aligned) and eps > 0.  desc->algo
 * is ignored; desc->flags may hold WKV7_FLAG_CHECK_FINITE only (else
 * WKV7_ERR_UNSUPPORTED).  Errors as for wkv7_forward; eps <= 0 or not
 * finite -> WKV7_ERR_UNSUPPORTED.
 */
typedef struct {
  const float* ln_w; /* [H, 64] GroupNorm weight */
  const float* ln_b; /* [H, 64] GroupNorm bias */
  const float* r_k;  /* [H, 64] bonus weights */
  float eps;         /* GroupNorm epsilon, > 0 */
} wkv7_epilogue_t;

/* out = the epilogue of y (formula above).  One launch on `stream`. */
wkv7_status_t wkv7_epilogue_forward(const wkv7_desc_t* desc, const wkv7_epilogue_t* ep, const void* y,
                                    const void* r, const void* k, const void* v, const void* g, void* out,
                                    void* stream);

/*
 * The forward with the epilogue: out = epilogue(y) for the y that
 * wkv7_forward computes from the same arguments (s_out and the checkpoints
 * in `workspace` as there); y itself is written only when `y` is not NULL
 * (the epilogue's backward needs it).  In the fused chunked form (16-bit
 * inputs where wkv7_forward would run that form) the epilogue runs inside
 * the recurrence's kernel as each chunk's y is written out: one launch, y
 * never read back from memory.  The other forms run wkv7_forward and then
 * wkv7_epilogue_forward (with `y` NULL, `out` holds y in between).  Either
 * way out is bit for bit what wkv7_epilogue_forward gives on the stored y.
 * desc->flags as for wkv7_forward (WKV7_FLAG_EPILOGUE_GRADS refused).
 */
wkv7_status_t wkv7_forward_epilogue(const wkv7_desc_t* desc, const wkv7_epilogue_t* ep, const void* r,
                                    const void* w, const void* k, const void* v, const void* a, const void* b,
                                    const float* s0, const uint8_t* reset, const void* g, void* y, void* out,
                                    float* s_out, void* workspace, void* stream);

/*
 * Reverse mode of the epilogue from dout = dL/dout.  Writes `eg`, an fp32
 * block [4][B,T,H,64] (16-byte aligned): dy (the gradient reaching the
 * recurrence), then the bonus parts of dr, dk and dv -- hand it to
 * wkv7_backward as its dy with WKV7_FLAG_EPILOGUE_GRADS, which adds those
 * parts to the recurrence's own; writes dg (desc->dtype); adds the parameter
 * gradients, summed over b and t, to dln_w, dln_b and dr_k (fp32 [H,64];
 * each may be NULL; the caller zeroes them first -- they are summed with
 * float atomics, so their last bits depend on the order of the adds).  One
 * launch on `stream`.
 */
wkv7_status_t wkv7_epilogue_backward(const wkv7_desc_t* desc, const wkv7_epilogue_t* ep, const void* y,
                                     const void* r, const void* k, const void* v, const void* g,
                                     const void* dout, float* eg, void* dg, float* dln_w, float* dln_b,
                                     float* dr_k, void* stream);

/*
 * ------------------------------------------------------------------ GDN map
 * The front end that runs a gated DeltaNet (GDN) layer on this recurrence
 * (rwkv-lab page, "Highlight result -- GDN in RWKV-7": the gated delta rule is
 * the wkv7 recurrence at matched head sizes, fed through a fixed map of GDN's
 * inputs).  Per (b, t) and value head h, reading key head kh = h / (H / Hk):
 *
 *   q^ = q / sqrt(|q|^2 + eps),  k^ = k / sqrt(|k|^2 + eps)   (over N channels)
 *   r  = r_scale q^          (1/sqrt(N) gives GDN's output scale: y is linear in r)
 *   x  = log(-g) on every channel: the log-space decay input, exp(-exp(x)) = exp(g)
 *   kw = beta k^,   a = -k^,   b = exp(g) beta k^
 *
 * after which wkv7_forward / wkv7_step with WKV7_FLAG_LOG_DECAY on (r, x, kw,
 * v, a, b) -- v is GDN's own, unchanged -- compute GDN's output and state:
 * S_t = exp(g_t) S_{t-1} (I - beta_t k^ k^T) + beta_t v_t k^T, o_t = S_t r_t.
 *
 *   desc         B, T, H (value heads), N (64 or 128), dtype; algo is ignored;
 *                flags 0 or WKV7_FLAG_CHECK_FINITE (which scans r, kw, a, b:
 *                x is -inf wherever g = 0, i.e. no decay)
 *   gd           Hk >= 1 key heads with H % Hk == 0; eps >= 0 and r_scale
 *                finite (else WKV7_ERR_UNSUPPORTED)
 *   q, k         in   [B,T,Hk,N] desc->dtype, 16-byte aligned
 *   g, beta      in   [B,T,H] fp32, 4-byte aligned; g <= 0 (GDN's decay is
 *                exp(g) <= 1; g > 0 writes NaN into x)
 *   r, x, kw, a, b  out  [B,T,H,N] desc->dtype, 16-byte aligned, not
 *                overlapping the inputs
 * With eps = 0 a zero q or k row gives non-finite outputs.  Errors as for
 * wkv7_forward.
 */
typedef struct {
  int64_t Hk;    /* key heads: value head h reads key head h / (H / Hk) */
  float eps;     /* L2-normalisation guard, >= 0 */
  float r_scale; /* multiplies q^ into r */
} wkv7_gdn_t;

wkv7_status_t wkv7_gdn_map(const wkv7_desc_t* desc, const wkv7_gdn_t* gd, const void* q, const void* k,
                           const float* g, const float* beta, void* r, void* x, void* kw, void* a, void* b,
                           void* stream);

/*
 * ------------------------------------------------------------------ state composition
 * For splitting a sequence's tokens across devices (context parallelism;
 * the pages have no passage on it).  Over a segment of tokens the
 * recurrence is affine in the state entering it:
 *
 *   S_end = S_in P + U,   P = prod_t (diag(w_t) + a_t b_t^T)   (the forward
 *   from s0 = I with v = 0),   U = the forward's end state from s0 = 0,
 *
 * and the state gradient goes back through the same P:
 * dS_in = dS_end P^T + (the backward's ds0 from dsT = 0).  This call is the
 * composition step: per (b, h) unit,
 *
 *   out = S P + U        (transpose_p == 0)
 *   out = S P^T + U      (transpose_p != 0)
 *
 * in fp32 (plain k order).  desc: B, H, N (64 or 128) give the unit count
 * and size; T, dtype and algo are validated as usual but not used; flags 0
 * or WKV7_FLAG_CHECK_FINITE.  S, P, U, out: fp32 [B,H,N,N], 16-byte
 * aligned; S NULL means zero (then P may be NULL; out = U); U NULL means
 * zero.  out may be U itself but must not overlap S or P (out == S or
 * out == P -> WKV7_ERR_UNSUPPORTED).  Errors as for wkv7_forward.
 */
wkv7_status_t wkv7_state_compose(const wkv7_desc_t* desc, const float* S, const float* P, const float* U,
                                 float* out, int transpose_p, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WKV7_H */
