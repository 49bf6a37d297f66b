// Self-test of the failure detection used by every pipelined kernel: a bounded mbarrier wait that
// nothing completes gives up after its limit (2 s of %globaltimer), sets the CTA's abort flag and
// the device error word (ERRF_TIMEOUT), and returns, so that the host reads an error status and
// the context stays usable.  One thread of one CTA; the barrier is never arrived on.
#pragma once
#include "tc_common.cuh"

namespace lsa {

__global__ void __launch_bounds__(32) k_selftest_wait(int32_t *__restrict__ status)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    const uint32_t a = tc::smem_u32(&bar);
    tc::mbar_init(a, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const bool completed = tc::mbar_wait(a, 0, (volatile int *)&abort_flag);
    status[0] = completed ? 1 : 0;
    status[1] = abort_flag;
}

}  // namespace lsa
