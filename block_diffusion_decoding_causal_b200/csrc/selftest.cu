// Failure-detection self-check: the bounded mbarrier wait every kernel uses,
// made to run out on purpose (nothing ever arrives), so that the host can
// see the timeout bit land in the workspace status word and the context
// stay usable.  No fault, trap or unbounded wait is involved.
#include <string>

#include "fdl_common.cuh"
#include "sm100.cuh"

namespace fdl {
namespace {

__global__ void wait_timeout_kernel(unsigned int* status, long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !sm100::mbar_wait_bounded(&bar, 0, limit_cycles))
    atomicOr(status, FDL_DEV_TIMEOUT);
}

}  // namespace

int record_error(int code, const std::string& msg);
int record_ok();

// The self-check kernel against any status word (the workspace's, or the
// allocation-free LM head's static one).
int launch_wait_timeout(unsigned int* status, long long limit_cycles, cudaStream_t stream) {
  if (limit_cycles < 1000 || limit_cycles > 2000000000LL)
    return record_error(FDL_ERR_INVALID_ARG, "limit_cycles must be in [1e3, 2e9]");
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status, limit_cycles);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_error(FDL_ERR_CUDA, cudaGetErrorString(e));
  return record_ok();
}

}  // namespace fdl

extern "C" int fdl_check_wait_timeout(void* ws, size_t ws_bytes, long long limit_cycles,
                                      void* stream) {
  using namespace fdl;
  if (ws == nullptr || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return record_error(FDL_ERR_WORKSPACE, "workspace must be at least 256 aligned bytes");
  return launch_wait_timeout(&static_cast<Control*>(ws)->status, limit_cycles,
                             (cudaStream_t)stream);
}
