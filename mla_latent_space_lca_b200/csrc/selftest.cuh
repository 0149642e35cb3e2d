// selftest.cuh -- exercises the failure path every kernel of this library
// shares: a bounded mbarrier wait that expires records LCA_ERR_DEVICE_TIMEOUT
// (with the kernel id and wait site) in the device status word and returns,
// leaving the context usable.
#pragma once
#include "common.cuh"

namespace lca {

constexpr int K_SELFTEST = 8;

// One warp waits on an mbarrier that nothing ever arrives at.
__global__ void __launch_bounds__(32) selftest_wait_kernel()
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_mbar_init();
    }
    __syncwarp();
    mbar_wait(b, 0, nullptr, K_SELFTEST, 1);   // expires after kWaitLimitNs
}

}  // namespace lca
