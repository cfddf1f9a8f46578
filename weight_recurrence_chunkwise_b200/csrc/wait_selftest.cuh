// wait_selftest.cuh -- diagnostic: the bounded waits of the prefill kernels, run out on purpose.
//
// Thread 0 of every CTA initialises an mbarrier that expects one arrival, which nothing ever
// makes, and waits on its first phase through the same helpers the prefill kernels use
// (mbar_wait, or mbar_wait_cluster with cluster-scope acquire, launched as a cluster of two).
// The wait gives up after limit_ns of wall time; the CTA then records STATUS_TIMEOUT in the
// status word and the time it waited, and exits normally, so the context stays usable.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace dr {

__global__ void __launch_bounds__(32) wait_selftest_kernel(int cluster_scope, unsigned long long limit_ns,
                                                           uint32_t *status, unsigned long long *waited_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    const bool ok = cluster_scope ? mbar_wait_cluster(&bar, 0, limit_ns) : mbar_wait(&bar, 0, limit_ns);
    if (!ok) raise_status(status, STATUS_TIMEOUT);
    if (waited_ns) waited_ns[blockIdx.x] = globaltimer_ns() - t0;
  }
}

}  // namespace dr
