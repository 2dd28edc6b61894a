// Failure-detection self-test: one CTA waits, through the bounded mbarrier wait
// that every kernel of the library uses, on a barrier that nothing completes.
// The wait gives up after the given limit, the timeout is recorded in the
// status word like any device-side failure, and the kernel returns: the error
// path is exercised without a trap, a fault or a hang.
#include "common.cuh"
#include "tc.cuh"

namespace sla {

__global__ void selftest_wait_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    tc::mbar_init(smem_u32(&bar), 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  // no thread arrives on `bar`: phase 0 never completes
  if (threadIdx.x == 0 && !tc::mbar_wait_for(smem_u32(&bar), 0, &abort_flag, limit_ns))
    report(status, SLA_ERR_DEVICE_TIMEOUT, kDetailSelftest);
}

}  // namespace sla

using namespace sla;

extern "C" sla_status sla_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t limit_ns, void* stream) {
  if (!ws || ((uintptr_t)ws % 256) != 0 || ws_bytes < 256) return SLA_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 1000000000) return SLA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, 8, s) != cudaSuccess) return SLA_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, s>>>(reinterpret_cast<int*>(ws), (uint64_t)limit_ns);
  return cudaGetLastError() == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}
