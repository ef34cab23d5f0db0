// Library-wide entry points: version, status names, per-thread error text.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <map>
#include <utility>

#include "host_util.h"

namespace {
thread_local char g_msg[512] = "";
thread_local cudaEvent_t g_prof_start = nullptr;
thread_local cudaEvent_t g_prof_stop = nullptr;
thread_local bool g_prof_started = false;
int g_sms[64] = {0};
}  // namespace

namespace csa {

csa_status fail(csa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

void clear_error() { g_msg[0] = '\0'; }

static std::atomic<uint64_t> g_launches{0};

csa_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return CSA_OK;
}

csa_status check_launch(const char* what, cudaError_t e) {
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  return check_launch(what);
}

uint64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    else
      cudaGetLastError();
  });
  return fn;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (g_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

bool ensure_smem(const void* kernel, int bytes) {
  // The limit is one value per kernel and device: only ever raise it.
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> limit;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  int& cur = limit[std::make_pair(dev, kernel)];
  if (bytes <= cur) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  cur = bytes;
  return true;
}

void prof_begin(cudaStream_t s) {
  if (g_prof_start && g_prof_stop) {
    cudaEventRecord(g_prof_start, s);
    g_prof_started = true;
  }
}

void prof_end(cudaStream_t s) {
  if (g_prof_started) {
    cudaEventRecord(g_prof_stop, s);
    g_prof_start = g_prof_stop = nullptr;
    g_prof_started = false;
  }
}

}  // namespace csa

extern "C" {

uint64_t csa_launch_count(void) { return csa::launch_count(); }

csa_status csa_profile_next_call(void* start_event, void* stop_event) {
  if ((start_event == nullptr) != (stop_event == nullptr))
    return csa::fail(CSA_ERR_INVALID_ARG, "csa_profile_next_call: pass both events or neither");
  g_prof_start = static_cast<cudaEvent_t>(start_event);
  g_prof_stop = static_cast<cudaEvent_t>(stop_event);
  g_prof_started = false;
  return CSA_OK;
}


const char* csa_version(void) { return "csa-b200 0.1.0 sm_100a"; }

const char* csa_status_string(int32_t s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_DEVICE_TIMEOUT: return "CSA_ERR_DEVICE_TIMEOUT";
    default: return "CSA_ERR_UNKNOWN";
  }
}

const char* csa_last_error(void) { return g_msg; }

}  // extern "C"
