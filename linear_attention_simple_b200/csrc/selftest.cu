// selftest.cu -- exercises the bounded-wait failure path without a fault.
//
// One thread initialises an mbarrier that expects one arrival and then waits
// on it; nothing ever arrives, so the bounded wait runs out, records
// GLA_ERR_TIMEOUT in the device status word and the kernel returns normally.
// The GPU context stays usable.
#include "gla_device.cuh"

namespace gla {
namespace {

__global__ void wait_selftest_kernel(WaitCtl ctl)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    mbar_init_fence();
    (void)mbar_wait(&bar, 0, ctl);
}

}  // namespace

gla_status launch_wait_selftest(const WaitCtl& ctl, cudaStream_t st)
{
    trace_begin(st);
    wait_selftest_kernel<<<1, 32, 0, st>>>(ctl);
    trace_end(st, "wait_selftest_kernel");
    count_launch();
    return check_launch("wait_selftest_kernel");
}

}  // namespace gla
