// Shared device/host helpers of the fp8ds library (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "fp8ds.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "fp8ds is written for sm_100a (B200) only"
#endif

namespace fp8ds {

constexpr int kHistoryLen = 16;
constexpr float kE4M3Max = 448.0f;
constexpr float kE5M2Max = 57344.0f;

// Codes for the device error word: which bounded wait gave up.
enum WaitSite : uint32_t {
  kWaitNone = 0,
  kWaitProducerEmpty = 1,
  kWaitMmaFull = 2,
  kWaitMmaTmemEmpty = 3,
  kWaitEpilogueTmemFull = 4,
  kWaitDrain = 5,
  kWaitQuantizeTma = 6,
  kWaitSplitK = 7,
};

// Library-global device error word (defined in capi.cu, relocatable device code
// is not used, so each translation unit that records errors gets the address
// through error_word_ptr()).
uint32_t* error_word_ptr();

// cuTensorMapEncodeTiled, fetched once through the runtime's driver entry
// point (no link-time dependency on libcuda).  Returns nullptr if unavailable.
void* tensor_map_encoder();

// cuTensorMapEncodeTiled with interleave none and zero OOB fill, memoised in a
// small per-thread cache keyed by every argument, so repeated calls on the
// same buffers (a training loop) skip the encode.  `map` must point to 64-byte
// aligned storage for one CUtensorMap (128 bytes).  Returns false on failure.
bool encode_tiled_cached(void* map, int data_type, int rank, const void* base, const uint64_t* dims,
                         const uint64_t* strides, const uint32_t* box, int swizzle, int l2_promotion);

// Nanosecond budget of every bounded wait in a kernel (the default).
constexpr unsigned long long kWaitBudgetNs = 2000000000ull;  // 2 s

// What launches take for their bounded waits: the budget of every wait on
// another role's or CTA's progress, and the one wait site (0: none) at which
// kernels wait on a barrier that nothing completes, so that the wait runs out
// and the kernel's timeout path runs.  Only fp8_debug_wait changes them (for
// tests of that path); waits that drain a kernel's own copies and MMAs before
// it frees shared memory or TMEM always keep kWaitBudgetNs.
struct WaitCfg {
  unsigned long long budget_ns;
  uint32_t stall_site;
};
WaitCfg wait_cfg();  // defined in capi.cu

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_device_error(uint32_t* word, uint32_t site) {
  if (word != nullptr) atomicCAS(word, 0u, site);
}

// Programmatic dependent launch.  Every kernel of the library lets the next
// kernel in the stream start launching as soon as it begins, and waits for
// the previous kernel to finish (and its memory to be visible) before it
// reads or writes any global memory; only local set-up (barrier init, TMEM
// allocation, descriptor prefetch) runs before the wait.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Host-side argument checks of fp8_mm and fp8_bias_grad: the status the entry
// point would return before launching anything (FP8_OK if it would launch).
// The linear composites run them for every kernel they will launch before
// they enqueue the first one, so a rejected composite changes no ring.
int mm_args_check(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
                  const int64_t* strides, int layout, const float* sinv_a, const float* sinv_b, const float* bias,
                  const uint16_t* out_bf16);
int bias_grad_args_check(const void* g, int dtype, int64_t rows, int64_t cols, const float* db);

// Counts one successful kernel launch (the library-wide launch counter read
// by fp8_launch_count).
void note_launch();

// cudaLaunchKernelEx with programmatic stream serialisation (and a cluster
// shape when cluster_x > 1).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) note_launch();
  return e;
}

}  // namespace fp8ds

#define FP8DS_CUDA_CHECK(expr)                 \
  do {                                         \
    cudaError_t e_ = (expr);                   \
    if (e_ != cudaSuccess) return FP8_ERR_CUDA; \
  } while (0)
