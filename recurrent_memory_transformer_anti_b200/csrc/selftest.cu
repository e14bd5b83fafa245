// Check of the failure path every kernel relies on: bounded waits that give up.
//
// One CTA initialises an mbarrier that nothing ever arrives on and waits on it with the same
// bounded wait the GEMM, attention and memory kernels use (mbar_wait_for), then waits for a
// global counter that nothing increments with the bounded wait of the chained projections
// (counter_wait_for), each with a short limit. Both waits must give up and leave the error
// word set, so that the host sees RMT_ETIMEOUT from rmt_sync; the kernel then returns
// normally and the context stays usable. Nothing faults, traps or spins without a bound.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace rmt {
namespace {

__device__ unsigned g_never_signalled = 0u;  // read by the counter wait below, written by nobody

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
  // a counter that stays 0 never reaches 1
  bool ok2 = true;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    ok2 = sm100::counter_wait_for(&g_never_signalled, 1u, &abort_flag, limit_ns);
  }
  __syncwarp();
  if (threadIdx.x == 0 && !ok && !ok2) atomicOr(err, kErrTimeoutSelftest);
}

#ifdef RMT_DEBUG
// Check of the debug build's bounds checks: one thread hands load_cell a cell whose residual
// slot lies far outside the limits stored with it. load_cell must record kErrBounds and return
// a cell with every index in range (else the kernel also sets kErrBadArgs); nothing is accessed
// through the cell's indices.
__global__ void __launch_bounds__(32) bounds_selftest_kernel(int* err) {
  __shared__ Cell bad[1];
  if (threadIdx.x == 0) {
    Cell c{};
    c.l = 0;
    c.m = 4;
    c.k = 0;
    c.xin = 1 << 20;  // outside lim_slot
    c.xout = 0;
    c.lim_L = 1;
    c.lim_state = 1;
    c.lim_slot = 2;
    c.lim_M = 8;
    c.lim_nmem = 4;
    c.lim_tokens = 0;
    c.lim_err = err;
    bad[0] = c;
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const Cell c = load_cell(bad, 0);
    if (!(c.xin == 0 && c.xout == 0 && c.k == 0 && c.l == 0 && c.m == 4 && c.t0 == 0)) atomicOr(err, kErrBadArgs);
  }
}
#endif

}  // namespace

#ifdef RMT_DEBUG
cudaError_t launch_bounds_selftest(int* err, cudaStream_t st) {
  bounds_selftest_kernel<<<1, 32, 0, st>>>(err);
  return cudaGetLastError();
}
#endif

cudaError_t launch_wait_selftest(int* err, unsigned long long limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace rmt
