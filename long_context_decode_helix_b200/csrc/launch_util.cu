// launch_util.cu -- host helpers shared by the kernels' launch functions.
#include <cuda_runtime.h>

#include <mutex>
#include <set>
#include <utility>

#include "internal.h"

namespace helix {

// Raise a kernel's dynamic shared memory limit to the device's opt-in maximum, once per (kernel,
// device): the attribute call costs microseconds, which a short-context step would otherwise pay
// on every launch.
cudaError_t allow_max_dynamic_smem(const void* func) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({func, dev})) return cudaSuccess;
  }
  int max_optin = 0;
  e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, max_optin);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  done.insert({func, dev});
  return cudaSuccess;
}

}  // namespace helix
