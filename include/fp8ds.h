/*
 * fp8ds.h -- C ABI of the B200 (sm_100a) FP8 per-tensor delayed-scaling linear.
 *
 * Two operations, both asynchronous on the caller's CUDA stream:
 *
 *   fp8_quantize  cast a bf16/fp16/fp32 tensor to E4M3 or E5M2 with the scale
 *                 held in a delayed-scaling ring, reduce amax over the raw
 *                 values, and fold that amax into the ring in the same kernel.
 *   fp8_mm        Y = bf16(sinv_a * sinv_b * A.B^T + bias), A and B FP8 with K
 *                 contiguous ("NT") or MN-major, fp32 accumulation, optional
 *                 fp32 bias, optional batch with stride-0 broadcast.
 *
 * Around them: fp8_quantize_pair / fp8_mm_pair (two calls in one launch),
 * fp8_quantize_multi (up to eight quantize calls in one launch),
 * fp8_mm_ws (stream-K tail through a caller workspace), fp8_mm_ex (FP8 bias,
 * FP8 output with delayed output scaling), fp8_quantize_current
 * (current scaling), fp8_quantize_local + fp8_ring_fold (data-parallel
 * delayed scaling), fp8_bias_grad and fp8_linear_forward / _backward (the
 * linear composites), fp8_quantize_static_scratch (no caller scratch), and
 * the utilities fp8_status_string, fp8_device_error, fp8_device_info and
 * fp8_launch_count.
 *
 * Sources: the AstrAI commit-log pages "AstrAI commits, branch main,
 * tests/extension" (ring commit, quantize split commit, snapshot commit,
 * bias-fusion commit, 3D batched commit), "AstrAI commit 05463316
 * csrc/kernels/fp8/quantize.cuh" (transposed/dual quantize), and "AstrAI
 * commit 0d0dc648 csrc/kernels/fp8_mm.cu" (amax over raw values, te-style
 * 16-step history ring).
 *
 * Conventions for every entry point:
 *   - Every pointer argument is device memory owned by the caller, unless the
 *     comment says "host".  The library allocates no device memory, never
 *     synchronises the device, and returns as soon as the work is enqueued.
 *   - The return value is FP8_OK (0) or a negative fp8_status.  On an error
 *     nothing was launched unless the status is FP8_ERR_CUDA.
 *   - Kernel-side faults are never raised on purpose: every wait in a kernel
 *     is bounded; a wait that runs out records FP8_ERR_DEVICE_TIMEOUT in a
 *     library-global error word that fp8_device_error() reads.
 */
#ifndef FP8DS_H_
#define FP8DS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* fp8_stream_t;

typedef enum {
  FP8_OK = 0,
  FP8_ERR_INVALID_ARG = -1,    /* bad enum, negative size, missing pointer      */
  FP8_ERR_UNSUPPORTED = -2,    /* valid request outside what the kernels take  */
  FP8_ERR_CUDA = -3,           /* a CUDA runtime/driver call failed             */
  FP8_ERR_DEVICE_TIMEOUT = -4  /* a bounded in-kernel wait ran out              */
} fp8_status;

/* Input element type of fp8_quantize. */
typedef enum { FP8_IN_BF16 = 0, FP8_IN_FP16 = 1, FP8_IN_FP32 = 2 } fp8_in_dtype;

/* FP8 format: E4M3 (largest finite 448) for activations and weights, E5M2
 * (largest finite 57344) for gradients -- the te-style recipe of the
 * "AstrAI commit 5244f1a8" entry on the fp8_mm.cu page. */
typedef enum { FP8_E4M3 = 0, FP8_E5M2 = 1 } fp8_fmt;

/* QuantLayout of the quantize bindings commit ("tests/extension" page):
 * ROW writes out[r*cols + c]; T writes out_t[c*rows + r] (the [cols, rows]
 * transpose); DUAL writes both from a single read of the input. */
typedef enum { FP8_LAYOUT_ROW = 0, FP8_LAYOUT_T = 1, FP8_LAYOUT_DUAL = 2 } fp8_qlayout;

/* History ring of one tensor (x, w or g each own one), the "[hist | scale |
 * counter]" buffer of the ring commit.  All five pointers are device memory,
 * usually slices of one caller-owned buffer.  Before the first call the
 * caller sets history to 0, idx to 0, scale to the initial scale (1.0),
 * scale_inv to 1.0 and scratch to 0; the kernel keeps them consistent after
 * that.  A ring must not be used by two quantize calls that may run at the
 * same time. */
typedef struct {
  float* history;     /* [16] amax of the last 16 calls, float32               */
  int32_t* idx;       /* [1]  slot the next amax is written to, 0..15          */
  float* scale;       /* [1]  scale the NEXT call multiplies by (published     */
                      /*      by the last block of each call)                  */
  float* scale_inv;   /* [1]  1/scale that the MOST RECENT call used: the      */
                      /*      dequantisation factor to hand to fp8_mm          */
  uint32_t* scratch;  /* [4]  amax bits, block ticket, tile counter, spare;    */
                      /*      8-byte aligned; zero between calls (the kernel   */
                      /*      leaves them at zero)                             */
} fp8_ring;

/*
 * fp8_quantize -- delayed-scaling cast to FP8 with in-kernel ring fold.
 *
 * Computes, with s = *ring.scale read at launch:
 *   q[r,c]  = saturate_rne_fp8(fp32(x[r,c]) * s)       (one fp32 multiply)
 *   amax    = max |x[r,c]| over the raw values (NaN ignored), the fix of
 *             "AstrAI commit 69f35c46" (amax of raw, not scaled, values)
 *   then, in the last block to finish (atomic ticket + fences, ring commit):
 *   history[idx] = amax; idx = (idx + 1) % 16; m = max(history);
 *   *scale = FP8_MAX / m (fp32, round-to-nearest) when m > 0 and finite and
 *            the quotient is finite, otherwise unchanged;
 *   *scale_inv = 1 / s  (the inverse of the scale this call used, as the
 *            snapshot commit requires for the GEMM's dequantisation).
 *
 * in      [rows, cols] row-major, contiguous, element type `dtype`; any
 *         address aligned to the element size (e.g. a 2-byte offset for bf16).
 * layout  fp8_qlayout; out is [rows, cols] uint8 (ROW, DUAL), out_t is
 *         [cols, rows] uint8 (T, DUAL); the unused one may be NULL.
 * rows, cols >= 0; rows*cols == 0 still folds amax = 0 into the ring.
 * Errors: FP8_ERR_INVALID_ARG for a bad enum, a negative size, a NULL ring
 *         field, a NULL in with rows*cols > 0, or a NULL out/out_t the
 *         layout needs; FP8_ERR_UNSUPPORTED for an input address not aligned
 *         to its element size or ring.scratch not 8-byte aligned;
 *         FP8_ERR_CUDA if the launch fails.
 */
int fp8_quantize(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt,
                 fp8_ring ring, uint8_t* out, uint8_t* out_t, fp8_stream_t stream);

/*
 * fp8_quantize_static_scratch -- fp8_quantize for callers that cannot allocate.
 *
 * The paper has no counterpart; this entry point exists for callers that
 * cannot allocate device memory at call time, such as operator or plugin
 * interfaces that receive only input and output pointers, or deployments that
 * reserve all device memory at start-up.  It computes exactly what
 * fp8_quantize computes, with the same arguments, except that ring.scratch is
 * ignored (it may be NULL): the four scratch words (amax bits, block ticket,
 * tile counter, spare) live in a 256-byte array owned by the library, which every GPU that
 * loads the library holds until the process exits.  The call itself allocates
 * nothing.
 *
 *   - The array holds 64 words; a call needs 4, whatever rows*cols is, so no
 *     tensor is refused for lack of scratch.  A request needing more than the
 *     array holds would return FP8_ERR_UNSUPPORTED.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is kept for the life of the
 *     process: after a cudaDeviceReset of that device the kept address is
 *     stale, so do not call this entry point again after a reset.
 *   - All calls on a device share the array.  Each call clears the four words
 *     on `stream` before its kernel, and the kernel leaves them at zero, but
 *     two calls that overlap on the GPU (different streams, no ordering
 *     between them) race on the array and give wrong amax and scales.
 *   - Errors are those of fp8_quantize, plus FP8_ERR_CUDA if the array's
 *     address cannot be obtained or the clearing memset fails.  Every
 *     argument check runs before the clearing memset, so a rejected call
 *     enqueues nothing.
 */
int fp8_quantize_static_scratch(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt,
                                fp8_ring ring, uint8_t* out, uint8_t* out_t, fp8_stream_t stream);

/*
 * fp8_quantize_pair -- two fp8_quantize calls (each on its own ring) in one
 * launch, such as a linear's X and W before its forward GEMM.
 *
 * When both resolve to the same kernel (ROW inputs with the same dtype and
 * 16-byte alignment of their data; or T/DUAL inputs with the same dtype and
 * layout, 16-byte aligned bases and rows that are a multiple of 16 bytes;
 * the formats may differ) and neither is empty, one grid is split between
 * them in proportion to their sizes; each set of blocks has its own amax
 * ticket and folds its own ring.  Otherwise the two run one after the other on `stream`.  Each
 * result (codes, ring, scales) is exactly that of the fp8_quantize call with
 * the same arguments.  If both name the same ring the two calls run in order
 * (a ring cannot serve two calls at once).
 *   q0, q1  host structs; each field as the fp8_quantize argument of that name.
 * Errors as fp8_quantize (the first call's checked first).
 * The pages have no counterpart (a B200 scheduling addition).
 */
typedef struct {
  const void* in;
  int dtype;
  int64_t rows, cols;
  int layout, fmt;
  fp8_ring ring;
  uint8_t* out;
  uint8_t* out_t;
} fp8_quantize_args;
int fp8_quantize_pair(const fp8_quantize_args* q0, const fp8_quantize_args* q1, fp8_stream_t stream);

/*
 * fp8_quantize_multi -- n fp8_quantize calls (each on its own ring) in one
 * launch, such as a linear's X, W and G before its GEMMs.
 *
 * When no ring is named twice, every input is non-empty and the calls
 * resolve to one kernel -- all ROW with the same dtype and 16-byte alignment
 * of their data, or all transposed or all dual with the same dtype, 16-byte
 * aligned bases and rows that are a multiple of 16 bytes (in both cases the
 * formats may differ) -- one grid is split between them in proportion to
 * their sizes: each tensor's blocks cast its own elements, reduce its own
 * amax and fold its own ring, so the launch's start-up and end costs are
 * paid once instead of n times.  Otherwise the calls run in order on
 * `stream`.  Each result (codes, ring, scales) is exactly that of
 * the fp8_quantize call with the same arguments.
 *   qs      host array of n structs; each field as the fp8_quantize argument
 *           of that name.
 *   n       1 .. 8.
 * Errors: FP8_ERR_INVALID_ARG for a null qs or n outside 1 .. 8; otherwise as
 * fp8_quantize, every call checked (in order) before anything is launched.
 * FP8_ERR_CUDA from a launch of the in-order fallback leaves the earlier
 * calls enqueued.  The pages have no counterpart (a B200 scheduling
 * addition).
 */
int fp8_quantize_multi(const fp8_quantize_args* qs, int n, fp8_stream_t stream);

/*
 * fp8_quantize_local / fp8_ring_fold -- delayed scaling of a tensor sharded
 * across data-parallel ranks: one scale for all shards.
 *
 * The pages fold each quantize's amax into the ring in the same kernel
 * ("tests/extension" page, ring commit).  With a tensor split across ranks
 * the fold needs the amax of the whole tensor, so the call is split in two
 * around a cross-rank MAX of one float (the reading of the multi-GPU scale
 * consistency item; the pages give no detail):
 *   1. fp8_quantize_local casts with ring.scale exactly as fp8_quantize does
 *      (same codes), writes 1/ring.scale to ring.scale_inv (the GEMM can run
 *      at once) and this rank's amax over the raw values to *amax_out.  It
 *      leaves history, idx and scale untouched (they may be NULL).
 *   2. The caller MAX-reduces *amax_out over the ranks (NCCL or gloo).
 *   3. fp8_ring_fold folds *amax into the ring (history[idx] = amax,
 *      idx = (idx + 1) mod 16, scale = FP8_MAX / max(history) when positive
 *      and finite, else kept; scale_inv = 1 / the scale before the fold).
 * Every rank that starts from the same ring and folds the same global amax
 * keeps an identical ring.  fp8_quantize_local followed by fp8_ring_fold of
 * its own amax equals one fp8_quantize call bit for bit.
 *
 *   amax_out  device float, written by the last block of the call.
 *   amax      device float read by the fold (device memory, never host).
 * Other arguments, layouts and errors as fp8_quantize; ring.scratch follows
 * the same rules.  fp8_ring_fold launches one single-thread kernel and
 * returns FP8_ERR_INVALID_ARG for a NULL ring pointer or amax or a bad fmt.
 */
int fp8_quantize_local(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt, fp8_ring ring,
                       float* amax_out, uint8_t* out, uint8_t* out_t, fp8_stream_t stream);
int fp8_ring_fold(fp8_ring ring, int fmt, const float* amax, fp8_stream_t stream);

/*
 * fp8_quantize_current -- current (dynamic) scaling cast to FP8, no ring.
 *
 * The DynamicScaling path of the FP8Recipe commit ("tests/extension" page:
 * a dynamic flag, zero rings, scales measured inline): the scale comes from
 * this tensor's own amax instead of a history of earlier ones.
 *   amax  = max |x| over the raw values (NaN ignored)
 *   scale = FP8_MAX / amax (fp32, round-to-nearest); 1 when amax is 0 or the
 *           quotient is not finite
 *   q     = saturate_rne_fp8(fp32(x) * scale)
 *   scale_inv = 1 / scale (the GEMM's dequantisation factor)
 * Two kernels on `stream`: an amax pass and the cast (the cast re-reads x,
 * mostly from L2 for tensors that fit there).
 * scale, scale_inv  device float[1] each, written (required).
 * amax              device float[1], written, or NULL.
 * scratch           device uint32[4], 8-byte aligned, zero before the call;
 *                   left at zero.
 * Other arguments and errors as fp8_quantize.
 */
int fp8_quantize_current(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt, float* scale,
                         float* scale_inv, float* amax, uint32_t* scratch, uint8_t* out, uint8_t* out_t,
                         fp8_stream_t stream);

/*
 * fp8_bias_grad -- bias gradient of the linear: db[c] = sum_r g[r, c].
 *
 * The _LinearFp8 backward fix ("tests/extension" page) reduces grad_b over
 * all leading dimensions of the bf16 output gradient; callers pass G
 * flattened to [rows, cols] (row-major, contiguous, element type `dtype`).
 * The float32 sums are deterministic (fixed summation order, no atomics).
 * db      device float[cols], written.
 * Errors: FP8_ERR_INVALID_ARG (bad dtype, negative size, NULL db or g);
 *         FP8_ERR_UNSUPPORTED (g not aligned to its element size);
 *         FP8_ERR_CUDA (launch failed).  cols == 0 is a no-op.
 */
int fp8_bias_grad(const void* g, int dtype, int64_t rows, int64_t cols, float* db, fp8_stream_t stream);

/* fp8_mm layout word: FP8_MM_NT plus optional operand-layout and format bits.
 * NT means A is [M, K] and B is [N, K], both with K contiguous (K-major).
 * The MN-major bits fold a transposed view into the layout tag at zero copy
 * (3D batched commit, "tests/extension" page: inner .t() views fold into the
 * layout tag): with FP8_MM_A_MN_MAJOR, A is stored [K, M] (M contiguous);
 * with FP8_MM_B_MN_MAJOR, B is stored [K, N] (N contiguous).  So dX = G.W
 * takes W as quantized ([N_out, N_in] = [K, N]) and dW = G^T.X takes G and X
 * as quantized, with no transposed copies. */
#define FP8_MM_NT 0
#define FP8_MM_A_MN_MAJOR (1 << 0) /* A stored [K, M]; needs M % 16 == 0 */
#define FP8_MM_B_MN_MAJOR (1 << 1) /* B stored [K, N]; needs N % 16 == 0 */
#define FP8_MM_A_E5M2 (1 << 8)     /* A holds E5M2 codes (default E4M3) */
#define FP8_MM_B_E5M2 (1 << 9)     /* B holds E5M2 codes (default E4M3) */
#define FP8_MM_BIAS_E5M2 (1 << 10) /* fp8_mm_ex: FP8 bias codes are E5M2 (default E4M3) */

/*
 * fp8_mm -- scaled FP8 GEMM with fused scale, bias and bf16 rounding.
 *
 * For b in [0, batch), m in [0, M), n in [0, N):
 *   Y[b,m,n] = bf16_rne( fp32_acc(sum_k A[b,m,k] * B[b,n,k]) * (sinv_a*sinv_b)
 *                        + bias[n] )
 * (bias-fusion commit: the fp32 bias is added before the single bf16
 * rounding; 3D batched commit: size-1 batches broadcast with stride 0).
 *
 * A       uint8 FP8 codes, element (b,m,k) at A[b*strides[0] + m*K + k]
 *         (FP8_MM_A_MN_MAJOR: at A[b*strides[0] + k*M + m]).
 * B       uint8 FP8 codes, element (b,n,k) at B[b*strides[1] + n*K + k]
 *         (FP8_MM_B_MN_MAJOR: at B[b*strides[1] + k*N + n]).
 * out_bf16 bfloat16 (uint16 storage), element (b,m,n) at
 *         out_bf16[b*strides[2] + m*N + n].
 * strides host array of 3 int64 batch strides in elements; may be NULL when
 *         batch == 1.  0 broadcasts that operand over the batch.
 * sinv_a, sinv_b  device pointers to one float each (typically a ring's
 *         scale_inv), read on the device so the scale chain never visits
 *         the host.
 * bias    device pointer to N floats, or NULL for no bias.
 * M, N >= 0, batch >= 1; M*N == 0 is a no-op.  K >= 0 and K % 16 == 0
 *         (the TMA row pitch must be a multiple of 16 bytes); K == 0 gives
 *         Y = bf16(bias) (or 0).
 * Errors: FP8_ERR_INVALID_ARG (negative size, batch < 1, NULL A/B/out/sinv,
 *         unknown layout bits, NULL strides with batch > 1);
 *         FP8_ERR_UNSUPPORTED (K % 16 != 0, an MN-major operand whose M or N
 *         is not a multiple of 16, A/B/stride not 16-byte aligned,
 *         out_bf16 not 2-byte aligned, a dimension beyond 2^31);
 *         FP8_ERR_CUDA (descriptor encoding or launch failed).
 */
int fp8_mm(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
           const int64_t* strides, int layout, const float* sinv_a, const float* sinv_b,
           const float* bias, uint16_t* out_bf16, fp8_stream_t stream);

/*
 * fp8_linear_forward / fp8_linear_backward -- one FP8 delayed-scaling linear.
 *
 * The _LinearFp8 forward/backward pair of the "tests/extension" page (the
 * forward captures its scales for the backward; grad_b is reduced over the
 * leading dims), composed from the calls above on one stream:
 *   forward:  Xq = quantize(X [M,K], E4M3, ring_x); Wq = quantize(W [N,K],
 *             E4M3, ring_w); Y [M,N] = bf16(Xq.Wq^T * sinv_x * sinv_w + bias).
 *   backward: Gq = quantize(G [M,N], E5M2, ring_g);
 *             dX [M,K] = bf16(Gq.Wq * sinv_g * sinv_w)   (Wq read MN-major),
 *             dW [N,K] = bf16(Gq^T.Xq * sinv_g * sinv_x) (Gq, Xq read MN-major),
 *             db [N]   = column sums of G (float32, deterministic).
 * All quantizes use the row layout: the layout tag replaces the transposed
 * copies.  xq [M,K], wq [N,K], gq [M,N] are caller-owned uint8 buffers; the
 * backward reads the forward's xq, wq and their scale_inv (pass ring_x.
 * scale_inv and ring_w.scale_inv; valid while X and W are not quantized
 * again in between).  dx, dw or db may be NULL to skip that output.
 * Sizes: K % 16 == 0 (forward); backward also M % 16 == 0 (dW reduces over
 * tokens) and N % 16 == 0 (MN-major row pitch).
 * Errors: those of the calls it makes.  Every argument check of every call
 * (the quantize, each GEMM, the bias gradient) runs on the host before the
 * first kernel is enqueued, so a call rejected with FP8_ERR_INVALID_ARG or
 * FP8_ERR_UNSUPPORTED launched nothing and left every ring as it was.  Only
 * FP8_ERR_CUDA can come after earlier steps were launched.
 */
int fp8_linear_forward(const void* x, int x_dtype, const void* w, int w_dtype, int64_t M, int64_t N, int64_t K,
                       const float* bias, fp8_ring ring_x, fp8_ring ring_w, uint8_t* xq, uint8_t* wq, uint16_t* y,
                       fp8_stream_t stream);
int fp8_linear_backward(const void* g, int g_dtype, int64_t M, int64_t N, int64_t K, fp8_ring ring_g,
                        const uint8_t* xq, const uint8_t* wq, const float* sinv_x, const float* sinv_w, uint8_t* gq,
                        uint16_t* dx, uint16_t* dw, float* db, fp8_stream_t stream);

/*
 * fp8_mm_ws -- fp8_mm with a caller-owned workspace that lets the library
 * spread the k-blocks of the last waves' output tiles evenly over all CTAs
 * (data-parallel whole tiles, then a stream-K tail), for outputs whose tile
 * count leaves the GPU part-idle in its last wave (for example the dW = G^T.X
 * GEMMs of a linear, whose output is only weight-sized).
 * Same arguments, result and errors as fp8_mm, plus:
 *   workspace       device memory, 256-byte aligned, all zero before its
 *                   first use.  Its first 1024 bytes are per-piece arrival
 *                   flags that every successful call leaves at zero, so the
 *                   same workspace serves later calls on the same stream; the
 *                   rest holds float32 partial tiles.  After a call that
 *                   recorded a device error (fp8_device_error) zero it again.
 *                   NULL (or smaller than fp8_mm_workspace_bytes) means
 *                   whole tiles only, as fp8_mm.
 *   workspace_bytes its size.  Calls that share a workspace must not overlap.
 * A tile cut into pieces is finished by the CTA holding its first k-block,
 * which adds the float32 partials of the later pieces in piece order, so
 * results are deterministic; they may differ from the fp8_mm result in the
 * last bits (both are within the same acceptance bound).
 * The pages have no counterpart: it is a B200 scheduling addition for
 * outputs whose tiles do not fill the last wave of SMs.
 *
 * fp8_mm_workspace_bytes -- the workspace size fp8_mm_ws would use for this
 * problem on the current device (0 when whole tiles are as fast); at most
 * 1024 + 148 x 128 x 256 x 4 bytes (about 19.4 MB) on a 148-SM B200.
 *
 * fp8_mm_launch_shape -- the launch shape fp8_mm (workspace_bytes 0) or
 * fp8_mm_ws (a workspace of workspace_bytes) picks for an M x N x K problem
 * with this layout on the current device, by the library's time model.
 * Writes shape[0] = output tile width BN (256, 128 or 64; tiles are 128
 * rows per CTA), shape[1] = CTAs per cluster (2: a CTA pair runs 256-row
 * tiles, 1: single CTAs), shape[2] = CTAs launched, shape[3] = stream-K
 * pieces (0: whole tiles only).  fp8_mm_pair has its own shared launch and
 * is not described by this.  Host-only: launches nothing.  Errors:
 * FP8_ERR_INVALID_ARG for a null shape or M, N, K < 1 or batch < 1;
 * FP8_ERR_CUDA when no device can be queried.  The pages have no counterpart.
 */
int fp8_mm_ws(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
              const int64_t* strides, int layout, const float* sinv_a, const float* sinv_b, const float* bias,
              uint16_t* out_bf16, void* workspace, size_t workspace_bytes, fp8_stream_t stream);
size_t fp8_mm_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t batch, int layout);
int fp8_mm_launch_shape(int64_t M, int64_t N, int64_t K, int64_t batch, int layout, size_t workspace_bytes,
                        int32_t* shape);

/*
 * fp8_mm_pair -- two independent GEMMs (each exactly an fp8_mm call) in one
 * launch, such as the dX and dW GEMMs of a linear's backward.
 *
 * The persistent grid is split: one set of CTAs works through problem 0's
 * output tiles and the rest through problem 1's, sized so both sets finish
 * together.  A problem whose tiles cannot fill the GPU (the weight-sized dW
 * output) then shares it with the other instead of leaving SMs idle.  When
 * the library's time model says one launch per problem is as fast (or a
 * problem is empty or has K = 0), the two run one after the other on
 * `stream` as fp8_mm_ws calls with `workspace` (which may be NULL; see
 * fp8_mm_ws; a paired launch does not use it).
 *   a0, a1  host structs; each field as the fp8_mm argument of that name.
 * Each output equals the corresponding fp8_mm result within the fp8_mm
 * bound; errors as fp8_mm (the first problem's error is reported first).
 * The pages have no counterpart (a B200 scheduling addition).
 */
typedef struct {
  const uint8_t* A;
  const uint8_t* B;
  int64_t M, N, K, batch;
  const int64_t* strides;
  int layout;
  const float* sinv_a;
  const float* sinv_b;
  const float* bias;
  uint16_t* out_bf16;
} fp8_mm_args;
int fp8_mm_pair(const fp8_mm_args* a0, const fp8_mm_args* a1, void* workspace, size_t workspace_bytes,
                fp8_stream_t stream);

/*
 * fp8_mm_ex -- fp8_mm with the two epilogue variants of the pages' FP8
 * GEMM: FP8 bias storage and FP8 output.
 *
 * Sources: "AstrAI commits, branch main, tests/extension" page, the
 * bias_scale commit (the bias may be FP8 storage with a scale, dequantised
 * in the epilogue after the operand scaling and before any output
 * quantisation) and the FP8-in/FP8-out GEMM commit.  The pages give no
 * formula for either; the reading here keeps every FP8 tensor on per-tensor
 * delayed scaling.  With y the float32 epilogue value
 *   y[b,m,n] = sinv_a * sinv_b * sum_k A[b,m,k] B[b,n,k] + bias[n]
 * (one fused multiply-add on the float32 accumulator, as in fp8_mm):
 *   bias      bias_scale == NULL: float32 [N] (or NULL, no bias), as fp8_mm;
 *             bias_scale != NULL: FP8 codes [N] (E4M3, or E5M2 with
 *             FP8_MM_BIAS_E5M2 in layout), bias[n] = fp32(decode(code) *
 *             *bias_scale).
 *   out       out_kind FP8_MM_OUT_BF16: bf16 [batch, M, N] = bf16_rn(y), as
 *             fp8_mm (out_ring unused).
 *             out_kind FP8_MM_OUT_E4M3 / _E5M2: FP8 codes [batch, M, N] =
 *             saturate_rne_fp8(fp32(y * s)) with s = *out_ring.scale read at
 *             launch -- the output tensor's delayed scale -- and, in the CTA
 *             that finishes last, out_ring folds amax = max |y| over the
 *             output (NaN ignored) exactly as fp8_quantize folds its input's
 *             amax: next scale published, scale_inv = 1/s for the GEMM that
 *             consumes the output.  An empty output folds amax 0; K == 0
 *             gives y = bias.  With out_amax set (one rank's shard of a
 *             data-parallel output) the fold is left to fp8_ring_fold.
 * Arguments, layouts, strides (strides[2] counts output elements), the
 * workspace and the errors are fp8_mm_ws's, plus FP8_ERR_INVALID_ARG for an
 * unknown out_kind, FP8_MM_BIAS_E5M2 without bias_scale, or an FP8 output
 * without out (non-empty output) or without a complete out_ring;
 * FP8_ERR_UNSUPPORTED for an out_ring.scratch that is not 8-byte aligned.
 * Validation happens before any CUDA call.  Codes leave through TMA stores
 * when out is 16-byte aligned and N and the batch stride are multiples of 16,
 * otherwise through guarded stores of staged rows (32 contiguous bytes of
 * one row per warp store).  One ring must not be used by two calls in
 * flight.
 */
typedef enum { FP8_MM_OUT_BF16 = 0, FP8_MM_OUT_E4M3 = 1, FP8_MM_OUT_E5M2 = 2 } fp8_mm_out;
typedef struct {
  const uint8_t* A;
  const uint8_t* B;
  int64_t M, N, K, batch;
  const int64_t* strides;
  int layout;               /* fp8_mm's layout bits, plus FP8_MM_BIAS_E5M2 */
  const float* sinv_a;
  const float* sinv_b;
  const void* bias;         /* NULL, float32 [N], or FP8 codes [N] (bias_scale set) */
  const float* bias_scale;  /* device scalar, or NULL for a float32 bias */
  int out_kind;             /* fp8_mm_out */
  void* out;                /* bf16 or FP8 codes [batch, M, N] */
  fp8_ring out_ring;        /* FP8 output: the output tensor's ring */
  float* out_amax;          /* FP8 output, data-parallel shard: NULL to fold
                               out_ring in the launch; else the launch writes
                               max |y| of this shard here (device float) and
                               1/s to out_ring.scale_inv, and leaves the ring's
                               history, idx and scale to fp8_ring_fold after a
                               cross-rank MAX of the amax (as
                               fp8_quantize_local) */
} fp8_mm_ex_args;
int fp8_mm_ex(const fp8_mm_ex_args* args, void* workspace, size_t workspace_bytes, fp8_stream_t stream);

/* Number of kernels this process has launched through the library so far
 * (every entry point, every device; a host-side counter, safe to call from
 * any thread, never synchronises).  Tracing aid: the difference across a
 * region is the kernel count of that region, e.g. of a captured CUDA graph. */
uint64_t fp8_launch_count(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* fp8_status_string(int status);

/* Reads, and with clear != 0 resets, the library's device error word on the
 * current device.  Synchronises the device.  Returns FP8_OK when no bounded
 * wait has run out since the last clear, FP8_ERR_DEVICE_TIMEOUT when one has
 * (then *where_out, if not NULL, receives a code naming the wait), or
 * FP8_ERR_CUDA. */
int fp8_device_error(int clear, uint32_t* where_out);

/* Number of SMs and the library's build architecture string, for reports. */
int fp8_device_info(int* sm_count, const char** arch);

/*
 * fp8_debug_wait -- testing only: shorten the bounded waits and make one run out.
 *
 * No page counterpart: this exists so tests can exercise the timeout path of
 * the kernels without faulting or hanging a GPU.  It sets, for every launch
 * made afterwards by this process (all threads, all devices):
 *   budget_ns   the budget of each wait on another role's progress (the
 *               producer / consumer / MMA / epilogue handshakes), in
 *               nanoseconds, 1 .. 2e9; 2e9 is the default.  Waits that drain
 *               a kernel's own TMA copies and MMAs before it frees shared
 *               memory or TMEM keep 2 s whatever this says, so a kernel that
 *               gives up never releases memory still being written.
 *   stall_site  0 (default: no stall), or one wait site code at which the
 *               kernels wait on a barrier that nothing completes, so that the
 *               wait runs out after budget_ns:
 *                 4  fp8_mm family: the epilogue's wait for an accumulator;
 *                 6  fp8_quantize family, transposed and dual layouts of
 *                    inputs whose rows are a multiple of 16 bytes (the TMA
 *                    tile kernels, 16-byte aligned or element-aligned base):
 *                    the consumers' wait for a staged input tile.  The row
 *                    layout's kernel and the transposed / dual kernel of
 *                    other row widths (plain loads) have no waits to shorten.
 * A wait that runs out records its site code in the device error word
 * (fp8_device_error), the kernel stops early and returns; its outputs are
 * undefined and the ring of a stalled quantize has folded an amax of 0.
 * Restore the defaults with fp8_debug_wait(2000000000, 0).
 * Errors: FP8_ERR_INVALID_ARG for a budget of 0 or above 2e9, or another site.
 */
int fp8_debug_wait(uint64_t budget_ns, uint32_t stall_site);

#ifdef __cplusplus
}
#endif

#endif /* FP8DS_H_ */
