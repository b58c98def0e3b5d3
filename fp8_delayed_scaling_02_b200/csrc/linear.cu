// fp8_linear_forward / fp8_linear_backward: one FP8 delayed-scaling linear.
//
// The training linear of the AstrAI pages ("tests/extension": _LinearFp8 owns
// the forward/backward pair, the forward captures its scales for the
// backward, grad_b is reduced over leading dims) composed from this
// library's kernels, all launched on one stream with programmatic dependent
// launch between them:
//   forward   Xq = quantize(X, E4M3, ring_x)        (row layout)
//             Wq = quantize(W, E4M3, ring_w)        (row layout; one fp8_quantize_pair launch with X)
//             Y  = bf16(Xq . Wq^T * sinv_x * sinv_w + b)
//   backward  Gq = quantize(G, E5M2, ring_g)        (row layout)
//             dX = bf16(Gq . Wq * sinv_g * sinv_w)  (Wq read MN-major: [K=N, N=K_in])
//             dW = bf16(Gq^T . Xq * sinv_g * sinv_x)  (Gq and Xq read MN-major)
//             (dX and dW in one fp8_mm_pair launch when both are wanted)
//             db = column sums of G (float32, deterministic)
// The backward's sinv_x / sinv_w are the forward's ring_x / ring_w
// scale_inv: valid as long as X and W are not quantized again between the
// two calls (the forward's scales carry to the backward).
#include "common.cuh"

using fp8ds::bias_grad_args_check;
using fp8ds::mm_args_check;

extern "C" int fp8_linear_forward(const void* x, int x_dtype, const void* w, int w_dtype, int64_t M, int64_t N,
                                  int64_t K, const float* bias, fp8_ring ring_x, fp8_ring ring_w, uint8_t* xq,
                                  uint8_t* wq, uint16_t* y, fp8_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return FP8_ERR_INVALID_ARG;
  // The GEMM's checks first: a call it would reject must not advance ring_x
  // or ring_w (the quantize pair checks its own arguments before launching).
  int rc = mm_args_check(xq, wq, M, N, K, 1, nullptr, FP8_MM_NT, ring_x.scale_inv, ring_w.scale_inv, bias, y);
  if (rc != FP8_OK) return rc;
  // X and W in one launch (each with its own ring).
  const fp8_quantize_args qx{x, x_dtype, M, K, FP8_LAYOUT_ROW, FP8_E4M3, ring_x, xq, nullptr};
  const fp8_quantize_args qw{w, w_dtype, N, K, FP8_LAYOUT_ROW, FP8_E4M3, ring_w, wq, nullptr};
  rc = fp8_quantize_pair(&qx, &qw, stream);
  if (rc != FP8_OK) return rc;
  return fp8_mm(xq, wq, M, N, K, 1, nullptr, FP8_MM_NT, ring_x.scale_inv, ring_w.scale_inv, bias, y, stream);
}

extern "C" int fp8_linear_backward(const void* g, int g_dtype, int64_t M, int64_t N, int64_t K, fp8_ring ring_g,
                                   const uint8_t* xq, const uint8_t* wq, const float* sinv_x, const float* sinv_w,
                                   uint8_t* gq, uint16_t* dx, uint16_t* dw, float* db, fp8_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return FP8_ERR_INVALID_ARG;
  if (sinv_x == nullptr || sinv_w == nullptr) return FP8_ERR_INVALID_ARG;
  // dX [M, K] = G [M, N] . W [N, K]: A = Gq K-major (K = N), B = Wq stored [N, K] = MN-major.
  const fp8_mm_args ax{gq, wq, M, K, N, 1, nullptr, FP8_MM_B_MN_MAJOR | FP8_MM_A_E5M2, ring_g.scale_inv, sinv_w,
                       nullptr, dx};
  // dW [N, K] = G^T [N, M] . X [M, K]: A = Gq stored [M, N] = MN-major, B = Xq stored [M, K] = MN-major.
  const fp8_mm_args aw{gq, xq, N, K, M, 1, nullptr, FP8_MM_A_MN_MAJOR | FP8_MM_B_MN_MAJOR | FP8_MM_A_E5M2,
                       ring_g.scale_inv, sinv_x, nullptr, dw};
  // Every later launch's checks run before the quantize of G, so a call that
  // one of them rejects leaves ring_g as it was.
  int rc = FP8_OK;
  if (dx != nullptr) {
    rc = mm_args_check(ax.A, ax.B, ax.M, ax.N, ax.K, 1, nullptr, ax.layout, ax.sinv_a, ax.sinv_b, nullptr, dx);
    if (rc != FP8_OK) return rc;
  }
  if (dw != nullptr) {
    rc = mm_args_check(aw.A, aw.B, aw.M, aw.N, aw.K, 1, nullptr, aw.layout, aw.sinv_a, aw.sinv_b, nullptr, dw);
    if (rc != FP8_OK) return rc;
  }
  if (db != nullptr) {
    rc = bias_grad_args_check(g, g_dtype, M, N, db);
    if (rc != FP8_OK) return rc;
  }
  rc = fp8_quantize(g, g_dtype, M, N, FP8_LAYOUT_ROW, FP8_E5M2, ring_g, gq, nullptr, stream);
  if (rc != FP8_OK) return rc;
  // Both wanted: one launch shares the GPU between them (the weight-sized dW
  // output alone leaves SMs idle).
  if (dx != nullptr && dw != nullptr) {
    rc = fp8_mm_pair(&ax, &aw, nullptr, 0, stream);
  } else if (dx != nullptr) {
    rc = fp8_mm(ax.A, ax.B, ax.M, ax.N, ax.K, 1, nullptr, ax.layout, ax.sinv_a, ax.sinv_b, nullptr, dx, stream);
  } else if (dw != nullptr) {
    rc = fp8_mm(aw.A, aw.B, aw.M, aw.N, aw.K, 1, nullptr, aw.layout, aw.sinv_a, aw.sinv_b, nullptr, dw, stream);
  }
  if (rc != FP8_OK) return rc;
  if (db != nullptr) return fp8_bias_grad(g, g_dtype, M, N, db, stream);
  return FP8_OK;
}
