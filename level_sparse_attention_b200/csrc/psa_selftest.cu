// Self-test of the failure path: a wait that runs out.
//
// Every mbarrier wait in the tensor-core kernels is bounded; on expiry it
// records a timeout in the workspace error word and the kernel winds down,
// and psa_check_device reports PSA_ERR_DEVICE_TIMEOUT.  This entry point
// exercises exactly that path without any fault: one warp waits, through the
// same bounded-wait helper the kernels use, on an mbarrier that nothing ever
// arrives at, gives up after the caller's limit, and returns.
#include "sm100_ptx.cuh"

namespace psa {
namespace {

using namespace ptx;

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(int* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);       // one arrival expected; none will come
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  if (threadIdx.x == 0) wait_bar_ns(smem_u32(&bar), 0, &abort_flag, err, limit_ns);
  __syncwarp();
}

}  // namespace
}  // namespace psa

extern "C" psa_status_t psa_selftest_wait_timeout(const psa_params_t* params, void* workspace,
                                                   size_t workspace_bytes, uint64_t limit_ns,
                                                   void* stream) {
  using namespace psa;
  if (!params || !workspace) return PSA_ERR_INVALID_ARG;
  if (params->B <= 0 || params->Hq <= 0 || params->Hkv <= 0 || params->N <= 0 || params->d <= 0 ||
      params->q_blk <= 0 || params->kv_blk <= 0)
    return PSA_ERR_INVALID_ARG;
  if (limit_ns == 0 || limit_ns > 1000000000ull) return PSA_ERR_INVALID_ARG;   // at most 1 s
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PSA_ERR_MISALIGNED;
  const Layout L = make_layout(*params);
  if (workspace_bytes < L.total) return PSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  wait_timeout_kernel<<<1, 32, 0, st>>>(reinterpret_cast<int*>(static_cast<char*>(workspace) + L.err),
                                        limit_ns);
  return cudaGetLastError() == cudaSuccess ? PSA_OK : PSA_ERR_CUDA;
}
