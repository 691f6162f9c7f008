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

// Timeline recording state (qg_timeline_begin / _end), one per process.
static std::mutex g_tl_mu;
static TlRec* g_tl_buf = nullptr;
static int g_tl_cap = 0, g_tl_next = 0;
static std::vector<int> g_tl_kinds;

static thread_local int g_tl_kind = kTlOther;
void tl_set_kind(int kind) { g_tl_kind = kind; }

TlRec* tl_take(int kind) {
  std::lock_guard<std::mutex> lock(g_tl_mu);
  if (!g_tl_buf || g_tl_next >= g_tl_cap) return nullptr;
  g_tl_kinds.push_back(kind ? kind : g_tl_kind);
  return g_tl_buf + g_tl_next++;
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

extern "C" int qg_timeline_available(void) {
#ifdef QG_TIMELINE
  return 1;
#else
  return 0;
#endif
}

extern "C" qg_status qg_timeline_begin(void* records, int cap) {
  qg::clear_error();
#ifndef QG_TIMELINE
  (void)records;
  (void)cap;
  qg::set_error("qg_timeline_begin: this library was built without QG_TIMELINE");
  return QG_ERR_INVALID_ARGUMENT;
#else
  QG_REQUIRE(records && cap > 0, QG_ERR_INVALID_ARGUMENT, "qg_timeline_begin: null records or cap <= 0");
  QG_REQUIRE(qg::aligned(records, 16), QG_ERR_MISALIGNED, "qg_timeline_begin: records misaligned");
  std::lock_guard<std::mutex> lock(qg::g_tl_mu);
  qg::g_tl_buf = reinterpret_cast<qg::TlRec*>(records);
  qg::g_tl_cap = cap;
  qg::g_tl_next = 0;
  qg::g_tl_kinds.clear();
  return QG_OK;
#endif
}

extern "C" int qg_timeline_end(int* kinds, int max_kinds) {
  std::lock_guard<std::mutex> lock(qg::g_tl_mu);
  const int n = qg::g_tl_next;
  for (int i = 0; kinds && i < n && i < max_kinds; ++i) kinds[i] = qg::g_tl_kinds[i];
  qg::g_tl_buf = nullptr;
  qg::g_tl_cap = 0;
  qg::g_tl_next = 0;
  qg::g_tl_kinds.clear();
  return n;
}
