// diag.cu -- a check of the bounded on-chip wait, without a GPU fault.
//
// Every pipeline wait of the GEMM kernels is an mbarrier wait bounded in time
// (mbar_wait): when it gives up, the waiting thread sets CHORD_DEV_TIMEOUT in the device
// status word and raises its CTA's abort flag, and the CTA's other waiters see the flag
// and unwind instead of waiting out their own limit. This kernel runs exactly that code
// on an mbarrier that nothing ever arrives at, with a short limit chosen by the caller,
// so a test can make a wait run out and read the result back while the context stays
// usable.
#include "chord_internal.cuh"

namespace chord {
namespace {

// Warp 0 lane 0 waits with the caller's limit and times out; warp 1 lane 0 waits on the
// same phase with the kernels' own limit and must return once the abort flag is up.
// elapsed_ns[0], [1]: how long each waited.
__global__ void __launch_bounds__(64) wait_timeout_kernel(uint32_t* status, uint64_t* elapsed_ns,
                                                          uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_v = &abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0 && warp < 2) {
    const uint64_t t0 = globaltimer_ns();
    const bool done = warp == 0 ? mbar_wait_limit(&bar, 0, abort_v, status, limit_ns)
                                : mbar_wait(&bar, 0, abort_v, status);
    elapsed_ns[warp] = globaltimer_ns() - t0;
    if (done) atomicOr(status, 0x80000000u);  // the phase completed: nothing arrives, so never
  }
}

}  // namespace

cudaError_t launch_wait_timeout(uint32_t* status, uint64_t* elapsed_ns, uint64_t limit_ns, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 64, 0, stream>>>(status, elapsed_ns, limit_ns);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
