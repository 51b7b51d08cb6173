// launch.h -- host helpers to launch the kernels (internal).
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <set>
#include <utility>

#include "gnorm.h"

namespace gnorm {

struct FwdArgs;
struct BwdArgs;

cudaError_t launch_fwd(const gnorm_plan& p, const FwdArgs& a, cudaStream_t stream, bool pdl);
cudaError_t launch_bwd(const gnorm_plan& p, const BwdArgs& a, cudaStream_t stream, bool pdl);
cudaError_t launch_dw_reduce(const float* partial, int P, int N, void* dw, int dw_fp32,
                             unsigned long long* work_counter, cudaStream_t stream, bool pdl);

// Device address of the current device's error word (the one gnorm_device_error reads);
// every kernel's bounded waits report there.  Returns a gnorm_status.
int device_error_word(unsigned** out);

// Raises a kernel's dynamic shared-memory limit once per (device, kernel).
inline cudaError_t ensure_smem_limit(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({dev, kernel})) return cudaSuccess;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) done.insert({dev, kernel});
  return e;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled while the
// previous kernel on the stream drains; it calls griddepcontrol.wait before touching
// global memory, so the ordering of memory effects is unchanged.
template <typename Kernel, typename... Args>
cudaError_t launch_kernel(Kernel kernel, int grid, int block, int smem, cudaStream_t stream,
                          bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace gnorm
