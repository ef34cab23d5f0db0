// Host-side helpers shared by the entry points: argument checks, error text.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

// Device error words of the units (attention.cu reads its own): -1 when the
// word cannot be read; `clear` resets a non-zero word.
int indexer_device_error(bool clear);
int compress_device_error(bool clear);
int out_proj_device_error(bool clear);
int cp_merge_device_error(bool clear);

// Records a printf-style message for csa_last_error() and returns `s`.
csa_status fail(csa_status s, const char* fmt, ...);
// Clears the calling thread's message.
void clear_error();
// Maps a pending launch error (cudaGetLastError) to CSA_ERR_CUDA.
// Launches `kernel` with programmatic stream serialization allowed (the kernel
// calls pdl_wait() before touching global memory), plus an optional cluster
// dimension (> 1).
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// The driver's tensor-map encoder, fetched through the runtime so that the
// library carries no link-time dependency on the driver library (null if the
// driver does not provide it).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Checks the launch just enqueued and counts it (csa_launch_count).  Called
// exactly once after every kernel launch of the library.
csa_status check_launch(const char* what);
// The same for a launch whose own return code is `e` (cudaLaunchKernelEx).
csa_status check_launch(const char* what, cudaError_t e);
uint64_t launch_count();
// Streaming multiprocessors of the current device (cached per device).
int num_sms();
// Raises a kernel's dynamic shared memory limit to `bytes` on the current
// device (once per device and kernel).  Returns false if the runtime refuses.
bool ensure_smem(const void* kernel, int bytes);
// Records the pending csa_profile_next_call start/stop event (if any) on `s`.
void prof_begin(cudaStream_t s);
void prof_end(cudaStream_t s);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace csa

#define CSA_REQUIRE(cond, ...)                                   \
  do {                                                           \
    if (!(cond)) return ::csa::fail(CSA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define CSA_REQUIRE_PTR(p)                                                        \
  do {                                                                            \
    if ((p) == nullptr) return ::csa::fail(CSA_ERR_INVALID_ARG, "%s is NULL", #p); \
    if (!::csa::aligned16(p))                                                     \
      return ::csa::fail(CSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p);  \
  } while (0)
