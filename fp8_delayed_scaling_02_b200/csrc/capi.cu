// Status strings, the device error word and device info of the fp8ds C ABI.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"

namespace {
// Written by bounded waits that run out (first site wins); read and cleared
// by fp8_device_error().
__device__ uint32_t g_device_error;

uint32_t* g_error_ptr[64] = {nullptr};
}  // namespace

namespace fp8ds {
uint32_t* error_word_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (g_error_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_error_ptr[dev] = static_cast<uint32_t*>(p);
  }
  return g_error_ptr[dev];
}

void* tensor_map_encoder() {
  static void* fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = p;
  });
  return fn;
}
}  // namespace fp8ds

extern "C" const char* fp8_status_string(int status) {
  switch (status) {
    case FP8_OK: return "FP8_OK";
    case FP8_ERR_INVALID_ARG: return "FP8_ERR_INVALID_ARG: bad enum, negative size or missing pointer";
    case FP8_ERR_UNSUPPORTED: return "FP8_ERR_UNSUPPORTED: alignment or size outside what the kernels take";
    case FP8_ERR_CUDA: return "FP8_ERR_CUDA: a CUDA call or kernel launch failed";
    case FP8_ERR_DEVICE_TIMEOUT: return "FP8_ERR_DEVICE_TIMEOUT: a bounded in-kernel wait ran out";
    default: return "unknown fp8 status";
  }
}

extern "C" int fp8_device_error(int clear, uint32_t* where_out) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FP8_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return FP8_ERR_CUDA;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return FP8_ERR_CUDA;
  }
  if (where_out) *where_out = v;
  return v == 0 ? FP8_OK : FP8_ERR_DEVICE_TIMEOUT;
}

extern "C" int fp8_device_info(int* sm_count, const char** arch) {
  if (arch) *arch = "sm_100a";
  if (sm_count) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP8_ERR_CUDA;
    if (cudaDeviceGetAttribute(sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FP8_ERR_CUDA;
  }
  return FP8_OK;
}
