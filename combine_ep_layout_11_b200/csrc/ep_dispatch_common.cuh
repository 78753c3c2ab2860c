// Device helpers of the dispatch kernels (ep_dispatch.cu: the row copy;
// ep_cast.cu: the FP8 cast): shared-memory zeroing and the work tickets
// they draw from the layout's workspace header.
#pragma once

#include "ep_internal.h"

namespace ep {
namespace dispatch_dev {

constexpr uint32_t kZeroBytes = 2048;   // the zeroed source of padding-row stores

__host__ __device__ __forceinline__ uint32_t round_up_u32(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Zero `bytes` (a multiple of 16) of shared memory starting at p with the threads
// [0, nthreads) of the CTA, then publish the writes to the async proxy.
__device__ __forceinline__ void zero_smem(uint8_t* p, uint32_t bytes, int tid, int nthreads) {
    for (uint32_t o = tid * 16u; o < bytes; o += nthreads * 16u)
        *reinterpret_cast<uint4*>(p + o) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
}

// After all of this CTA's work: count it finished; the last CTA of the grid
// (every ticket drawn) sets the counters back to zero for the next launch.
__device__ __forceinline__ void tickets_done(WsHeader* h) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&h->done, 1u) == gridDim.x - 1) {
            h->tok_ticket = 0;
            h->pad_ticket = 0;
            __threadfence();
            h->done = 0;
        }
    }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

}  // namespace dispatch_dev
}  // namespace ep
