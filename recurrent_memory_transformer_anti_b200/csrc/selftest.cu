// Check of the failure path every kernel relies on: a bounded mbarrier wait that gives up.
//
// One CTA initialises an mbarrier that nothing ever arrives on and waits on it with the same
// bounded wait the GEMM, attention and memory kernels use (mbar_wait_for), here with a short
// limit. The wait must give up, raise the CTA's abort flag and leave the error word set, so
// that the host sees RMT_ETIMEOUT from rmt_sync; the kernel then returns normally and the
// context stays usable. Nothing faults, traps or spins without a bound.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace rmt {
namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  const uint32_t b = sm100::smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncwarp();
  // phase 0 of a barrier with one expected arrival and no arriving thread never completes
  const bool ok = sm100::mbar_wait_for(b, 0, &abort_flag, limit_ns);
  __syncwarp();
  if (threadIdx.x == 0 && !ok) atomicOr(err, kErrTimeoutSelftest);
}

}  // namespace

cudaError_t launch_wait_selftest(int* err, unsigned long long limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace rmt
