// Test tap of the device-side wait discipline (no counterpart on the pages).
#include "internal.h"

namespace schnet {

// The give-up path every mbarrier wait of the fused kernels takes, on its own: one
// CTA holds tensor memory and waits on an mbarrier with a bounded number of polls;
// when nothing completes the barrier (complete = 0) the wait gives up, the CTA
// raises SCHNET_FLAG_TIMEOUT, releases its tensor memory and returns.
__global__ void k_test_timeout(DevMeta* meta, uint32_t max_polls, int complete)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tslot;
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        tmem_alloc(&tslot, 32);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    if (complete && threadIdx.x == 0)
        asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar)) : "memory");
    bool ok = true;
    if (warp == 0) ok = mbar_wait_bounded(&bar, 0u, max_polls);
    if (__syncthreads_or(!ok) && threadIdx.x == 0) set_flag(meta, SCHNET_FLAG_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 32);
    }
}

cudaError_t launch_test_timeout(schnet_ctx* c, uint32_t max_polls, int complete)
{
    k_test_timeout<<<1, 64, 0, c->s>>>(c->ws.meta, max_polls, complete);
    c->launches += 1;
    return cudaGetLastError();
}

}  // namespace schnet
