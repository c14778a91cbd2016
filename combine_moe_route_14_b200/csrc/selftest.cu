// Diagnostics: exercise the library's bounded device waits on a condition
// that never becomes true, so that tests can check the timeout path end to
// end (the wait gives up after its limit, the kernel records MOE_DEV_TIMEOUT
// in the status word, returns, and the context stays usable).  The waits
// are the same primitives the grouped GEMM uses; nothing here can hang: each
// wait ends after `limit_ns`.
#include "common.cuh"
#include "launch.h"

namespace moe {

// which = 0: global counters that nothing increments (the fused forms'
//            readiness gates, wait_counts_geq);
// which = 1: a shared-memory mbarrier that nothing arrives on (the GEMM's
//            pipeline waits, mbar_wait);
// which = 2: a flag bit in global memory that nothing sets (the combine
//            epilogue's wait for a token's first slot, wait_bits_set);
// which = 3: a shared-memory mbarrier with cluster-scope acquire (the
//            work-item queue's waits, mbar_wait_cluster).
__global__ void selftest_wait_kernel(int which, uint64_t limit_ns, uint32_t* counter,
                                     uint32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  if (which == 0) {
    wait_counts_geq(counter, 1, 1u, status, &abort_flag, limit_ns);
  } else if (which == 2) {
    wait_bits_set(counter, 0x100u, status, &abort_flag, limit_ns);
  } else {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
    if (which == 1) mbar_wait(&bar, 0, status, &abort_flag, limit_ns);
    else mbar_wait_cluster(&bar, 0, status, &abort_flag, limit_ns);
  }
}

cudaError_t launch_selftest_wait(int which, uint64_t limit_ns, uint32_t* counter,
                                 const DeviceInfo& dev, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(which, limit_ns, counter, dev.status);
  return cudaGetLastError();
}

}  // namespace moe
