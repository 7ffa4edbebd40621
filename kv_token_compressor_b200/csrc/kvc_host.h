// Host-side launch helpers shared by the kernel files (device attributes, occupancy).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

namespace kvc {

struct DeviceInfo {
  int sms = 0;
  size_t smem_optin = 0;
};

// Multiprocessor count and opt-in shared memory of a device, queried once per device.
inline DeviceInfo device_info(int dev) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return DeviceInfo{};
  if (cache[dev].sms == 0) {
    int sms = 0, optin = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return DeviceInfo{};
    cache[dev].sms = sms;
    cache[dev].smem_optin = static_cast<size_t>(optin);
  }
  return cache[dev];
}

// Raises kernel k's dynamic shared-memory limit on the current device to the most the
// device allows beside the kernel's static shared memory.  Every launch path calls this
// and never sets a lower limit, so concurrent host threads that run one kernel with
// different shared-memory needs cannot undercut one another; the limit does not change
// occupancy, which follows the shared memory a launch actually asks for.  The current
// limit is read back each time (a context reset restores the 48 KB default).
inline bool raise_smem_limit(const void* k) {
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const DeviceInfo di = device_info(dev);
  if (di.sms == 0) return false;
  std::lock_guard<std::mutex> lock(mu);
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, k) != cudaSuccess) return false;
  const int want = static_cast<int>(di.smem_optin) - static_cast<int>(fa.sharedSizeBytes);
  if (fa.maxDynamicSharedSizeBytes >= want) return true;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, want) ==
         cudaSuccess;
}

// Name of the kernel that the calling host thread's last successful launch through this
// library ran (a string literal; "" before the first launch).  Read by kvc_last_kernel().
inline const char*& last_kernel() {
  static thread_local const char* name = "";
  return name;
}

// Resident CTAs per SM of kernel k at this block size and dynamic shared memory (0 on
// error); raises the kernel's dynamic shared-memory limit first (raise_smem_limit).
template <typename Kernel>
int resident_blocks(Kernel k, int threads, size_t smem) {
  if (!raise_smem_limit(reinterpret_cast<const void*>(k))) return 0;
  int blocks = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, k, threads, smem) != cudaSuccess)
    return 0;
  return blocks;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// The driver's cuTensorMapEncodeTiled, looked up once through the runtime (no link
// against libcuda); nullptr when the driver does not provide it.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
inline EncodeTiledFn tensor_map_encoder() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace kvc
