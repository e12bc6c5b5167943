// Self-test of the bounded-wait machinery used by the tensor-core GEMM: a
// single thread waits on an mbarrier that nothing ever arrives on, with a short
// limit.  The wait must give up, record kErrTimeout with its tag in the
// workspace status word and return, leaving the CUDA context usable.
#include "int8mp.h"
#include "kernels.h"

using namespace i8mp;

namespace {

constexpr uint32_t kSelftestTag = 0x5e1f;

__global__ void wait_timeout_probe_kernel(DevStatus* st, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0;
  fence_barrier_init();
  // parity 0 = the barrier's first phase, which never completes: no arrivals.
  mbar_wait(&bar, 0u, &abort_flag, st, kSelftestTag, limit_ns);
}

}  // namespace

extern "C" i8_status int8_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t limit_us,
                                                cudaStream_t stream) {
  if (workspace == nullptr || reinterpret_cast<uintptr_t>(workspace) % 256 != 0 ||
      workspace_bytes < sizeof(DevStatus))
    return I8_ERR_WORKSPACE;
  if (limit_us == 0 || limit_us > 2000000) return I8_ERR_INVALID_ARG;
  if (note_cuda_error(cudaMemsetAsync(workspace, 0, sizeof(DevStatus), stream)) != cudaSuccess) return I8_ERR_CUDA;
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(static_cast<DevStatus*>(workspace),
                                                  static_cast<uint64_t>(limit_us) * 1000ull);
  return note_cuda_error(cudaGetLastError()) == cudaSuccess ? I8_OK : I8_ERR_CUDA;
}
