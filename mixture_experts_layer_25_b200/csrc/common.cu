// Host-side helpers: per-thread error message, SM count, version.
#include <stdarg.h>

#include <atomic>
#include <map>
#include <mutex>
#include <stdio.h>
#include <utility>

#include "common.cuh"

namespace moe {

static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

static std::atomic<unsigned long long> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

moe_status_t set_smem_limit(const void* kernel, size_t bytes, const char* what) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;   // (kernel, device) -> bytes set
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_error("%s: no current device", what);
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(kernel, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return MOE_OK;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) {
    set_error("%s: shared-memory limit %zu bytes: %s", what, bytes, cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  done[key] = bytes;
  return MOE_OK;
}

}  // namespace moe

extern "C" const char* moe_last_error(void) { return moe::g_err; }

extern "C" unsigned long long moe_launch_count(void) { return moe::g_launches.load(); }

extern "C" const char* moe_version(void) { return "libmoe 0.1 (sm_100a)"; }
