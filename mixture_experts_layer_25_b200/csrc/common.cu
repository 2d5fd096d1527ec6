// Host-side helpers: per-thread error message, SM count, version.
#include <stdarg.h>

#include <atomic>
#include <stdio.h>

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

}  // namespace moe

extern "C" const char* moe_last_error(void) { return moe::g_err; }

extern "C" unsigned long long moe_launch_count(void) { return moe::g_launches.load(); }

extern "C" const char* moe_version(void) { return "libmoe 0.1 (sm_100a)"; }
