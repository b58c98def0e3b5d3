// fp8_bias_grad: db[c] = sum_r G[r, c], the bias gradient of the FP8 linear.
//
// The linear's backward reduces the bf16 output gradient over all leading
// (token) dimensions ("AstrAI commits, branch main, tests/extension": the
// _LinearFp8 backward fix flattens [B, L, d] and reduces grad_b over leading
// dims).  B200 design: deterministic float32 sums with no workspace and no
// atomics, in one launch:
//   * a cluster of 8 CTAs owns a strip of 32 columns; CTA k of the cluster
//     sums rows [k*R/8, (k+1)*R/8);
//   * in a CTA, lane l of warp w sums column l over rows w, w+8, w+16, ...
//     (eight rows in flight per warp, 64-byte coalesced row pieces), then the
//     8 warps' sums are added in warp order through shared memory;
//   * after a cluster barrier, CTA 0 reads the 8 CTA sums from the other
//     CTAs' shared memory (distributed shared memory) and adds them in rank
//     order, so every bit of the result is independent of scheduling.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"

namespace fp8ds {
namespace {

constexpr int kBgThreads = 256;
constexpr int kBgCluster = 8;
constexpr int kBgCols = 32;

template <int DT>
__device__ __forceinline__ float load_elem(const uint8_t* base, int64_t idx) {
  if constexpr (DT == FP8_IN_BF16) {
    return __uint_as_float(uint32_t(reinterpret_cast<const uint16_t*>(base)[idx]) << 16);
  } else if constexpr (DT == FP8_IN_FP16) {
    return __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(base)[idx]));
  } else {
    return reinterpret_cast<const float*>(base)[idx];
  }
}

template <int DT>
__global__ void __cluster_dims__(kBgCluster, 1, 1) __launch_bounds__(kBgThreads)
    bias_grad_kernel(const uint8_t* g, int64_t rows, int64_t cols, float* db) {
  __shared__ float warp_sum[kBgThreads / 32][kBgCols];
  __shared__ float cta_sum[kBgCols];
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  uint32_t rank;
  asm volatile("mov.u32 %0, %cluster_ctarank;" : "=r"(rank));
  const int64_t strip = blockIdx.x / kBgCluster;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c = strip * kBgCols + lane;
  const int64_t per = (rows + kBgCluster - 1) / kBgCluster;
  const int64_t r0 = int64_t(rank) * per;
  const int64_t r1 = rows < r0 + per ? rows : r0 + per;
  float acc = 0.0f;
  if (c < cols) {
    const int nw = kBgThreads / 32;
    int64_t r = r0 + warp;
    // Eight rows of this warp per step: loads issued before any add; the adds
    // keep row order.
    for (; r + 7 * nw < r1; r += 8 * nw) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = load_elem<DT>(g, (r + u * nw) * cols + c);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc += v[u];
    }
    for (; r < r1; r += nw) acc += load_elem<DT>(g, r * cols + c);
  }
  warp_sum[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kBgThreads / 32; ++w) s += warp_sum[w][lane];
    cta_sum[lane] = s;
  }
  // Every CTA's sum is in its shared memory before rank 0 reads them.
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (rank == 0 && warp == 0 && c < cols) {
    const uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(&cta_sum[lane]));
    float s = 0.0f;
#pragma unroll
    for (uint32_t k = 0; k < kBgCluster; ++k) {
      uint32_t remote;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(k));
      float v;
      asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
      s += v;
    }
    db[c] = s;
  }
  // No CTA leaves while rank 0 may still read its shared memory.
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace
}  // namespace fp8ds

using namespace fp8ds;

namespace fp8ds {
int bias_grad_args_check(const void* g, int dtype, int64_t rows, int64_t cols, const float* db) {
  if (dtype < FP8_IN_BF16 || dtype > FP8_IN_FP32) return FP8_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0) return FP8_ERR_INVALID_ARG;
  if (cols == 0) return FP8_OK;
  if (db == nullptr || (rows > 0 && g == nullptr)) return FP8_ERR_INVALID_ARG;
  const int eb = dtype == FP8_IN_FP32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(g) % eb != 0) return FP8_ERR_UNSUPPORTED;
  if (cols > (int64_t(1) << 40) / kBgCluster || rows > (int64_t(1) << 40)) return FP8_ERR_UNSUPPORTED;
  const int64_t strips = (cols + kBgCols - 1) / kBgCols;
  if (strips * kBgCluster > INT32_MAX) return FP8_ERR_UNSUPPORTED;
  return FP8_OK;
}
}  // namespace fp8ds

extern "C" int fp8_bias_grad(const void* g, int dtype, int64_t rows, int64_t cols, float* db, fp8_stream_t stream) {
  const int rc = bias_grad_args_check(g, dtype, rows, cols, db);
  if (rc != FP8_OK) return rc;
  if (cols == 0) return FP8_OK;
  const int64_t strips = (cols + kBgCols - 1) / kBgCols;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(unsigned(strips * kBgCluster));
  const uint8_t* gp = static_cast<const uint8_t*>(g);
  cudaError_t e;
  // The cluster shape comes from __cluster_dims__; the launch only adds the
  // programmatic-dependent-launch attribute.
  switch (dtype) {
    case FP8_IN_BF16: e = launch_pdl(bias_grad_kernel<FP8_IN_BF16>, grid, dim3(kBgThreads), 0, st, 1, gp, rows, cols, db); break;
    case FP8_IN_FP16: e = launch_pdl(bias_grad_kernel<FP8_IN_FP16>, grid, dim3(kBgThreads), 0, st, 1, gp, rows, cols, db); break;
    default: e = launch_pdl(bias_grad_kernel<FP8_IN_FP32>, grid, dim3(kBgThreads), 0, st, 1, gp, rows, cols, db); break;
  }
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}
