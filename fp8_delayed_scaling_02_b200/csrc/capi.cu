// Status strings, the device error word and device info of the fp8ds C ABI.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
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

namespace {
using EncodeTiledFnC = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct MapKey {
  const void* base;
  uint64_t dims[3];
  uint64_t strides[2];
  uint32_t box[3];
  int dtype, rank, swizzle, promo;
  bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};

struct MapEntry {
  MapKey key;
  alignas(64) CUtensorMap map;
  bool valid;
};

constexpr int kMapCacheSize = 32;
thread_local MapEntry t_map_cache[kMapCacheSize];
thread_local int t_map_next = 0;
}  // namespace

bool encode_tiled_cached(void* map, int data_type, int rank, const void* base, const uint64_t* dims,
                         const uint64_t* strides, const uint32_t* box, int swizzle, int l2_promotion) {
  if (rank < 1 || rank > 3) return false;
  MapKey k;
  std::memset(&k, 0, sizeof(k));
  k.base = base;
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides[i];
  k.dtype = data_type;
  k.rank = rank;
  k.swizzle = swizzle;
  k.promo = l2_promotion;
  for (int i = 0; i < kMapCacheSize; ++i) {
    if (t_map_cache[i].valid && t_map_cache[i].key == k) {
      std::memcpy(map, &t_map_cache[i].map, sizeof(CUtensorMap));
      return true;
    }
  }
  auto enc = reinterpret_cast<EncodeTiledFnC>(tensor_map_encoder());
  if (!enc) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t bx[3], es[3] = {1u, 1u, 1u};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  MapEntry& e = t_map_cache[t_map_next];
  e.valid = false;
  if (enc(&e.map, CUtensorMapDataType(data_type), cuuint32_t(rank), const_cast<void*>(base), d, st, bx, es,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CUtensorMapSwizzle(swizzle), CUtensorMapL2promotion(l2_promotion),
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  e.key = k;
  e.valid = true;
  t_map_next = (t_map_next + 1) % kMapCacheSize;
  std::memcpy(map, &e.map, sizeof(CUtensorMap));
  return true;
}
}  // namespace fp8ds

namespace fp8ds {
namespace {
std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned long long> g_wait_budget_ns{kWaitBudgetNs};
std::atomic<uint32_t> g_stall_site{0};
}  // namespace
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
WaitCfg wait_cfg() {
  return WaitCfg{g_wait_budget_ns.load(std::memory_order_relaxed), g_stall_site.load(std::memory_order_relaxed)};
}
}  // namespace fp8ds

extern "C" int fp8_debug_wait(uint64_t budget_ns, uint32_t stall_site) {
  if (budget_ns == 0 || budget_ns > fp8ds::kWaitBudgetNs) return FP8_ERR_INVALID_ARG;
  if (stall_site != 0 && stall_site != fp8ds::kWaitEpilogueTmemFull && stall_site != fp8ds::kWaitQuantizeTma)
    return FP8_ERR_INVALID_ARG;
  fp8ds::g_wait_budget_ns.store(budget_ns, std::memory_order_relaxed);
  fp8ds::g_stall_site.store(stall_site, std::memory_order_relaxed);
  return FP8_OK;
}

extern "C" uint64_t fp8_launch_count(void) { return fp8ds::g_launches.load(std::memory_order_relaxed); }

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
