// Combine: ordered weighted reduction of the expert outputs back to token
// order ("DeepEP 测试目标 API 系统性参考" §2.2 combine() weighted reduction,
// §3.2 Buffer.combine() plain sum when no weights are given, §4.1 refs.py
// ordered_accumulate: one fixed accumulation order for bitwise determinism).
//
//   out[t] = bf16_rne( init[t] + sum_{k ascending, pair_slot[t,k] >= 0} w[t,k] * y[pair_slot[t,k]] )
//
// in fp32, every step __fmul_rn then __fadd_rn (never contracted into an FMA),
// so the result is the same bits whatever the launch shape.  init[t] is +0, or
// the output bias of §2.2 combine() (bias0, or bias0 + bias1 rounded once),
// the initial value of the reference accumulation in §4.1.  The
// kernel is bound by HBM reads: K rows of 2H bytes in, one row out per token.
// A work item is (token, 32*V 16-byte columns); a warp issues the loads of KB
// rows of its item together before summing them, so each lane keeps KB*V
// loads in flight, and every row is read in contiguous 32*V*16-byte pieces.
// The item's selected entries are first packed to the front of the warp (in
// ascending k), so -1 entries take no place in a batch.  Padding rows are
// never read.
#include <cuda_bf16.h>

#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kCombineThreads = 256;

__device__ __forceinline__ void accumulate8(float (&acc)[8], uint4 v, float w) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(w, __uint_as_float(u[i] << 16)));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(w, __uint_as_float(u[i] & 0xffff0000u)));
    }
}

// acc := float(b0), then acc := acc + float(b1) (one rounded sum) when two biases
__device__ __forceinline__ void init_bias8(float (&acc)[8], uint4 b0, uint4 b1, bool two) {
    const uint32_t u[4] = {b0.x, b0.y, b0.z, b0.w};
    const uint32_t p[4] = {b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __uint_as_float(u[i] << 16);
        acc[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
        if (two) {
            acc[2 * i] = __fadd_rn(acc[2 * i], __uint_as_float(p[i] << 16));
            acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __uint_as_float(p[i] & 0xffff0000u));
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}

// V: 16-byte columns per lane per row (a row segment of V * 512 bytes per
// item); KB: rows whose loads are issued together before they are summed;
// kBias: the sum starts from the output bias (a.bias0 is set).
// kRegions: the rows come from the regions of CombineArgs (ep_combine_regions),
// each selected entry carrying its row's address instead of a receive row.
template <int V, int kMinBlocks, int KB, bool kBias, bool kRegions = false>
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
    // the next grid in the stream is not let in early (no launch_dependents):
    // its CTAs would sit resident beside this bandwidth-bound kernel, which
    // measured slower (dispatch -> combine: 765 against 733 us per
    // large-prefill step); it starts when this grid ends
    pdl_wait();

    // the (slot, weight) of lane k for the warp's next item is loaded while the
    // current item is processed, so no item starts with a dependent load; with
    // regions, also the address of the entry's row (slot then only marks it used)
    auto fetch = [&](int64_t it, int& slot, float& w, const uint4*& rp) {
        slot = -1;
        w = 1.0f;
        rp = nullptr;
        if (it < items && lane < K) {
            const int64_t t = it / nch;
            slot = a.pair_slot[t * K + lane];
            if (a.w) w = a.w[t * K + lane];
            if (kRegions && slot >= 0) {
                const int64_t e = a.topk_idx[t * K + lane];
                const int64_t row = (e >= 0 && e < (int64_t)a.El * a.R) ? (int64_t)slot + a.row_delta[e] : -1;
                if (row >= 0 && row < a.region_capacity)
                    rp = reinterpret_cast<const uint4*>(a.regions[e / a.El]) + row * (a.H / 8);
                slot = rp ? 0 : -1;
            }
        }
    };
    int next_slot;
    float next_w;
    const uint4* next_rp;
    fetch(gw, next_slot, next_w, next_rp);
    // per warp: the item's selected entries moved to the front, in ascending k
    __shared__ int2 packed[kCombineThreads / 32][32];
    __shared__ const uint4* packed_rp[kRegions ? kCombineThreads / 32 : 1][32];
    int2* my_packed = packed[threadIdx.x >> 5];
    const uint4** my_packed_rp = packed_rp[kRegions ? threadIdx.x >> 5 : 0];
    for (int64_t it = gw; it < items; it += nw) {
        const int64_t t = it / nch;
        const int ch = (int)(it % nch);
        int my_slot = next_slot;
        float my_w = next_w;
        const uint4* my_rp = next_rp;
        fetch(it + nw, next_slot, next_w, next_rp);
        if (!kRegions && (int64_t)my_slot >= a.capacity) my_slot = -1;
        // compaction: lane k with a selected entry writes it to position
        // popc(selected below k); the loop below then runs over nsel entries
        // with no holes, in the same ascending-k order
        const uint32_t sel = __ballot_sync(0xffffffffu, lane < K && my_slot >= 0);
        const int nsel = __popc(sel);
        if ((sel >> lane) & 1u) {
            const int pos = __popc(sel & lanemask_lt());
            my_packed[pos] = make_int2(my_slot, __float_as_int(my_w));
            if (kRegions) my_packed_rp[pos] = my_rp;
        }
        __syncwarp();
        if (lane < nsel) {
            const int2 p = my_packed[lane];
            my_slot = p.x;
            my_w = __int_as_float(p.y);
            if (kRegions) my_rp = my_packed_rp[lane];
        }
        __syncwarp();
        float acc[V][8];
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[v][i] = 0.0f;

        // the biases of this item, loaded before the first batch of rows and
        // folded in after that batch is in flight
        uint4 b0[V], b1[V];
        if (kBias) {
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int col = ch * per_item + v * 32 + lane;
                const bool in = col < HV;
                b0[v] = in ? ld_stream_v4(reinterpret_cast<const uint4*>(a.bias0) + t * HV + col)
                           : make_uint4(0, 0, 0, 0);
                b1[v] = (in && a.bias1) ? ld_stream_v4(reinterpret_cast<const uint4*>(a.bias1) + t * HV + col)
                                        : make_uint4(0, 0, 0, 0);
            }
        }

        for (int k0 = 0; k0 < max(nsel, 1); k0 += KB) {
            uint4 rows[KB][V];
#pragma unroll
            for (int kk = 0; kk < KB; ++kk) {
                const int k = k0 + kk;
                const bool use = k < nsel;
                const uint4* row;
                if (kRegions) {
                    const uint64_t p = __shfl_sync(0xffffffffu, reinterpret_cast<uint64_t>(my_rp), k & 31);
                    row = reinterpret_cast<const uint4*>(p);
                } else {
                    row = y + (int64_t)__shfl_sync(0xffffffffu, my_slot, k & 31) * HV;
                }
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int col = ch * per_item + v * 32 + lane;
                    rows[kk][v] = (use && col < HV) ? ld_stream_v4(row + col) : make_uint4(0, 0, 0, 0);
                }
            }
            if (kBias && k0 == 0) {
#pragma unroll
                for (int v = 0; v < V; ++v) init_bias8(acc[v], b0[v], b1[v], a.bias1 != nullptr);
            }
#pragma unroll
            for (int kk = 0; kk < KB; ++kk) {
                const int k = k0 + kk;
                const float w = __shfl_sync(0xffffffffu, my_w, k & 31);
                if (k < nsel) {
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
    // 1 KB of each row per item, two rows in flight per lane without a bias,
    // eight with one: the fastest of the (columns per lane, rows per batch)
    // pairs measured on the prefill and decode workloads, expand and per-rank
    // handles, once the selected entries are packed (2-8 rows per batch,
    // 512 B - 4 KB per row and item).  Without a bias the kernel is held to
    // 64 registers so four CTAs (32 warps) share an SM instead of three:
    // more loads in flight per SM, 328 against 337 us at large prefill
    // (five or six CTAs spill; with a bias the 8-row batches need the
    // registers).
    auto kernel = a.regions ? (a.bias0 ? combine_kernel<2, 2, 8, true, true> : combine_kernel<2, 4, 2, false, true>)
                            : (a.bias0 ? combine_kernel<2, 2, 8, true> : combine_kernel<2, 4, 2, false>);
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
