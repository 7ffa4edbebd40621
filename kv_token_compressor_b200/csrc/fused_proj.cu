// Fused projection + softmax-pool (tcgen05 / TMEM / TMA) — placeholder until the
// tensor-core kernel lands: the entry points validate and report KVC_ERR_UNSUPPORTED.
#include "kvc_common.cuh"
#include "kvc_launch.h"

namespace kvc {

// Set by kernels whose bounded waits give up; read and cleared by kvc_device_status().
__device__ unsigned int g_device_error = 0;

kvc_status launch_fused(const FusedProblem&, cudaStream_t) { return KVC_ERR_UNSUPPORTED; }

kvc_status read_and_clear_device_error(cudaStream_t st) {
  if (cudaStreamSynchronize(st) != cudaSuccess) return KVC_ERR_CUDA;
  unsigned int v = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return KVC_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return KVC_ERR_CUDA;
  return v ? KVC_ERR_TIMEOUT : KVC_OK;
}

}  // namespace kvc
