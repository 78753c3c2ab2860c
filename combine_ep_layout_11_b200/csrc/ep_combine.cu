// Combine: ordered weighted reduction of the expert outputs back to token
// order ("DeepEP 测试目标 API 系统性参考" §2.2 combine() weighted reduction,
// §3.2 Buffer.combine() plain sum when no weights are given, §4.1 refs.py
// ordered_accumulate: one fixed accumulation order for bitwise determinism).
//
//   out[t] = bf16_rne( sum_{k ascending, pair_slot[t,k] >= 0} w[t,k] * y[pair_slot[t,k]] )
//
// in fp32 from +0, every step __fmul_rn then __fadd_rn (never contracted into
// an FMA), so the result is the same bits whatever the launch shape.  The
// kernel is bound by HBM reads: K rows of 2H bytes in, one row out per token.
// A work item is (token, 32*V 16-byte columns); a warp issues all K row loads
// of its item before accumulating, so each lane keeps 8*V loads in flight.
// Padding rows are never read.
#include <cuda_bf16.h>

#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kKBatch = 8;

__device__ __forceinline__ void accumulate8(float (&acc)[8], uint4 v, float w) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(w, __uint_as_float(u[i] << 16)));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(w, __uint_as_float(u[i] & 0xffff0000u)));
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}

template <int V>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * kCombineThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kCombineThreads) >> 5;
    const int HV = a.H / 8;              // 16-byte vectors per row
    const int per_item = 32 * V;
    const int nch = (HV + per_item - 1) / per_item;
    const int64_t items = (int64_t)a.T * nch;
    const int K = a.K;
    const uint4* y = reinterpret_cast<const uint4*>(a.y);

    for (int64_t it = gw; it < items; it += nw) {
        const int64_t t = it / nch;
        const int ch = (int)(it % nch);
        int my_slot = -1;
        float my_w = 1.0f;
        if (lane < K) {
            my_slot = a.pair_slot[t * K + lane];
            if (a.w) my_w = a.w[t * K + lane];
            if ((int64_t)my_slot >= a.capacity) my_slot = -1;
        }
        float acc[V][8];
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[v][i] = 0.0f;

        for (int k0 = 0; k0 < K; k0 += kKBatch) {
            uint4 rows[kKBatch][V];
#pragma unroll
            for (int kk = 0; kk < kKBatch; ++kk) {
                const int k = k0 + kk;
                const int slot = __shfl_sync(0xffffffffu, my_slot, k & 31);
                const bool use = (k < K) && slot >= 0;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int col = ch * per_item + v * 32 + lane;
                    rows[kk][v] = (use && col < HV) ? ld_stream_v4(y + (int64_t)slot * HV + col)
                                                    : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int kk = 0; kk < kKBatch; ++kk) {
                const int k = k0 + kk;
                const int slot = __shfl_sync(0xffffffffu, my_slot, k & 31);
                const float w = __shfl_sync(0xffffffffu, my_w, k & 31);
                if (k < K && slot >= 0) {
#pragma unroll
                    for (int v = 0; v < V; ++v) accumulate8(acc[v], rows[kk][v], w);
                }
            }
        }
        uint4* out = reinterpret_cast<uint4*>(a.out) + t * HV;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int col = ch * per_item + v * 32 + lane;
            if (col < HV) {
                uint4 o;
                o.x = pack_bf16x2(acc[v][0], acc[v][1]);
                o.y = pack_bf16x2(acc[v][2], acc[v][3]);
                o.z = pack_bf16x2(acc[v][4], acc[v][5]);
                o.w = pack_bf16x2(acc[v][6], acc[v][7]);
                st_v4(out + col, o);
            }
        }
    }
}

__global__ void selftest_wait_kernel(WsHeader* hdr, uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);   // expects one arrival that never comes
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, timeout_ns)) atomicOr(&hdr->status, kDevTimeout);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
    constexpr int V = 2;
    int blocks_per_sm = 0;
    cudaError_t err =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, combine_kernel<V>, kCombineThreads, 0);
    if (err != cudaSuccess) return err;
    if (blocks_per_sm < 1) blocks_per_sm = 1;
    combine_kernel<V><<<a.sms * blocks_per_sm, kCombineThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(WsHeader* hdr, uint64_t timeout_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(hdr, timeout_ns);
    return cudaGetLastError();
}

}  // namespace ep
