// Device-side check of the bounded-wait path that every tcgen05 kernel of this library relies on:
// one thread waits on an mbarrier that nothing arrives on, with a caller-given limit, and must give
// up, record its code in the workspace status word and return (no trap, no fault), so that the host
// sees DMA_ERR_TIMEOUT and the context stays usable.
#include "internal.h"
#include "tc.cuh"

namespace dma {
namespace {

constexpr int kErrSelftestWait = 0x1;   // status bit of this check (no other kernel uses it)

__global__ void selftest_wait_kernel(int32_t* status, long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)tc::mbar_wait(&bar, 0, &abort_flag, status, kErrSelftestWait, limit_cycles);
  __syncthreads();
}

}  // namespace

cudaError_t launch_selftest_wait(const Plan& P, void* ws, long long limit_cycles, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(ws_ptr<int32_t>(ws, P.off_status), limit_cycles);
  return cudaGetLastError();
}

}  // namespace dma
