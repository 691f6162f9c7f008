// Error reporting and version of the libqg C ABI.
#include <stdarg.h>

#include <atomic>
#include <mutex>
#include <tuple>
#include <vector>

#include "qg_internal.cuh"

namespace qg {

static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

void clear_error() { g_err[0] = '\0'; }

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// The dynamic shared memory limit is an attribute of a kernel on one device:
// raised once per (kernel, device), to the largest value asked for so far.
void ensure_smem(const void* func, int bytes) {
  static std::mutex mu;
  static std::vector<std::tuple<const void*, int, int>> done;  // kernel, device, bytes
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (auto& d : done) {
    if (std::get<0>(d) == func && std::get<1>(d) == dev) {
      if (std::get<2>(d) >= bytes) return;
      cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      std::get<2>(d) = bytes;
      return;
    }
  }
  cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  done.emplace_back(func, dev, bytes);
}

qg_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("%s: CUDA launch failed: %s", what, cudaGetErrorString(e));
    return QG_ERR_CUDA;
  }
  return QG_OK;
}

}  // namespace qg

extern "C" const char* qg_last_error(void) { return qg::g_err; }

extern "C" int qg_abi_version(void) { return 1; }

extern "C" unsigned long long qg_kernel_launch_count(void) {
  return qg::g_launches.load(std::memory_order_relaxed);
}
