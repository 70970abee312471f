// Failure-detection self-test: one bounded in-kernel wait that is made to
// expire, through the same mbarrier wait the forward's kernels use.
//
// Every wait of the attention kernel on an mbarrier gives up after a fixed
// number of SM cycles, records kDevTimeout in the caller's device status word
// and returns, so a lost arrival ends as an error code and never as a hung
// GPU. This entry point runs that code path on purpose and harmlessly: one
// thread initialises an mbarrier in shared memory that nothing ever arrives
// on and waits on it with a short, caller-given limit. No copy, tensor-core
// operation or memory access other than the status word is in flight, so the
// kernel returns normally and the context stays usable.
#include "tc_util.cuh"

namespace {

__global__ void wait_timeout_kernel(int* status, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x != 0) return;
  abort_sh = 0;
  const uint32_t b = sla::smem_u32(&bar);
  sla::tc::mbar_init(b, 1);
  sla::tc::fence_barrier_init();
  // phase 0 never completes: the one expected arrival is never made
  sla::tc::mbar_wait_for(b, 0, reinterpret_cast<volatile int*>(&abort_sh), status, limit);
}

}  // namespace

extern "C" sla_status sla_check_wait_timeout(void* workspace, size_t workspace_bytes, long long limit_cycles,
                                             void* stream) {
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 || workspace_bytes < 256)
    return SLA_ERR_WORKSPACE;
  if (limit_cycles < 1 || limit_cycles > sla::tc::kWaitCycles) return SLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, 256, s);
  if (e == cudaSuccess) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(static_cast<int*>(workspace), limit_cycles);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}
