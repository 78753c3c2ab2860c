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

template <int V, int kMinBlocks>
__global__ void __launch_bounds__(kCombineThreads, kMinBlocks) combine_kernel(CombineArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * kCombineThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kCombineThreads) >> 5;
    const int HV = a.H / 8;              // 16-byte vectors per row
    const int per_item = 32 * V;
    const int nch = (HV + per_item - 1) / per_item;
    const int64_t items = (int64_t)a.T * nch;
    const int K = a.K;
    const uint4* y = reinterpret_cast<const uint4*>(a.y);
    pdl_wait();
    pdl_launch_dependents();

    // the (slot, weight) of lane k for the warp's next item is loaded while the
    // current item is processed, so no item starts with a dependent load
    auto fetch = [&](int64_t it, int& slot, float& w) {
        slot = -1;
        w = 1.0f;
        if (it < items && lane < K) {
            const int64_t t = it / nch;
            slot = a.pair_slot[t * K + lane];
            if (a.w) w = a.w[t * K + lane];
        }
    };
    int next_slot;
    float next_w;
    fetch(gw, next_slot, next_w);
    for (int64_t it = gw; it < items; it += nw) {
        const int64_t t = it / nch;
        const int ch = (int)(it % nch);
        int my_slot = next_slot;
        const float my_w = next_w;
        fetch(it + nw, next_slot, next_w);
        if ((int64_t)my_slot >= a.capacity) my_slot = -1;
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

// ---------------------------------------------------------------------------
// TMA-staged variant for K <= 8: the item is (token, 2 KB column segment).  A
// producer warp bulk-loads the K rows' segments into a stage of a ring in
// shared memory (one mbarrier per stage counts the bytes); four consumer warps
// reduce the stage in ascending k, one 16-byte column per thread, and store the
// bf16 result.  The ring keeps many row segments in flight per SM without
// holding them in registers.
// ---------------------------------------------------------------------------
constexpr int kStageK = 8;
constexpr int kSegVec = 128;                 // 16-byte columns per segment (2 KB of bf16)
constexpr int kSegBytes = kSegVec * 16;
constexpr int kConsumerWarps = 4;
constexpr int kTmaThreads = 32 * (1 + kConsumerWarps);

struct StageMeta {
    float w[kStageK];
    int32_t valid;   // bit k: row k was loaded
    int32_t pad[7];
};

__global__ void __launch_bounds__(kTmaThreads) combine_tma_kernel(CombineArgs a, int stages) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem;                                                   // [stages][kStageK][kSegBytes]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * kStageK * kSegBytes);
    uint64_t* empty = full + stages;
    StageMeta* meta = reinterpret_cast<StageMeta*>(empty + stages);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.K, HV = a.H / 8;
    const int nseg = (HV + kSegVec - 1) / kSegVec;
    const int64_t items = (int64_t)a.T * nseg;
    const int64_t G = gridDim.x, first = blockIdx.x;
    const int64_t n = first < items ? (items - first + G - 1) / G : 0;
    const uint32_t row_bytes = (uint32_t)a.H * 2u;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();

    if (warp == 0) {
        // producer; the (slot, weight) of lane k for item j+1 is loaded while
        // item j is issued, so no item waits on a dependent global load
        auto fetch = [&](int64_t j, int32_t& slot, float& w) {
            slot = -1;
            w = 1.0f;
            if (j < n && lane < K) {
                const int64_t t = (first + j * G) / nseg;
                slot = a.pair_slot[t * K + lane];
                if (a.w) w = a.w[t * K + lane];
            }
        };
        int32_t next_slot;
        float next_w;
        fetch(0, next_slot, next_w);
        for (int64_t j = 0; j < n; ++j) {
            const int s = (int)(j % stages);
            int32_t slot = next_slot;
            float w = next_w;
            fetch(j + 1, next_slot, next_w);
            if ((int64_t)slot >= a.capacity) slot = -1;
            if (!mbar_wait(&empty[s], (uint32_t)(((j / stages) & 1) ^ 1))) {
                if (lane == 0) atomicOr(&a.status->status, kDevTimeout);
                break;
            }
            const int64_t item = first + j * G;
            const int g = (int)(item % nseg);
            const uint32_t bytes = (uint32_t)min(kSegVec, HV - g * kSegVec) * 16u;
            const uint32_t valid = __ballot_sync(0xffffffffu, slot >= 0);
            if (lane < kStageK) meta[s].w[lane] = w;
            if (lane == 0) meta[s].valid = (int32_t)valid;
            __syncwarp();   // the metadata writes are ordered before lane 0's release-arrive
            if (lane == 0) mbar_arrive_expect_tx(&full[s], bytes * __popc(valid));
            __syncwarp();
            if (slot >= 0)
                bulk_load(ring + ((size_t)s * kStageK + lane) * kSegBytes,
                          a.y + (int64_t)slot * (row_bytes / 2) + (int64_t)g * kSegVec * 8, bytes, &full[s]);
        }
        return;
    }

    // consumers
    const int ct = tid - 32;   // 0 .. 127: one 16-byte column of the segment
    for (int64_t j = 0; j < n; ++j) {
        const int s = (int)(j % stages);
        const bool ok = mbar_wait(&full[s], (uint32_t)((j / stages) & 1));
        if (!ok) {
            if (ct == 0) atomicOr(&a.status->status, kDevTimeout);
            return;
        }
        const int64_t item = first + j * G;
        const int64_t t = item / nseg;
        const int g = (int)(item % nseg);
        const int col = g * kSegVec + ct;
        const uint32_t valid = (uint32_t)meta[s].valid;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        if (col < HV) {
#pragma unroll
            for (int k = 0; k < kStageK; ++k) {
                if (valid & (1u << k)) {
                    const uint4 v = *reinterpret_cast<const uint4*>(ring + ((size_t)s * kStageK + k) * kSegBytes + ct * 16);
                    accumulate8(acc, v, meta[s].w[k]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&empty[s])) : "memory");
        if (col < HV) {
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            st_v4(reinterpret_cast<uint4*>(a.out) + t * HV + col, o);
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
    if (a.variant == 1 && a.K <= kStageK) {
        const int stages = 6;
        const size_t smem = (size_t)stages * kStageK * kSegBytes + 2 * stages * 8 + stages * sizeof(StageMeta);
        cudaError_t err =
            cudaFuncSetAttribute(combine_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        int per_sm = 0;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_tma_kernel, kTmaThreads, smem);
        if (err != cudaSuccess) return err;
        if (per_sm < 1) per_sm = 1;
        return launch_pdl(combine_tma_kernel, dim3(a.sms * per_sm), dim3(kTmaThreads), smem, s, false, a, stages);
    }
    auto kernel = a.variant == 2 ? combine_kernel<1, 3> : combine_kernel<2, 2>;
    int blocks_per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kernel, kCombineThreads, 0);
    if (err != cudaSuccess) return err;
    if (blocks_per_sm < 1) blocks_per_sm = 1;
    return launch_pdl(kernel, dim3(a.sms * blocks_per_sm), dim3(kCombineThreads), 0, s, false, a);
}

cudaError_t launch_selftest_wait(WsHeader* hdr, uint64_t timeout_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(hdr, timeout_ns);
    return cudaGetLastError();
}

}  // namespace ep
