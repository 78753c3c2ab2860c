// Dispatch: scatter token rows into the expert-contiguous receive buffer
// ("DeepEP 测试目标 API 系统性参考" §2.1 dispatch(): x or (fp8, scales) in, rows
// of the same type out, do_zero_padding; §4.2 math.py for the fused cast).
//
// The work is pure data movement, bound by HBM bandwidth: each token row is
// read once and written K times, padding rows are written once.  Rows travel
// through shared memory on the TMA engine: one bulk load per row segment into
// a multi-stage ring guarded by mbarriers, then one bulk store per destination
// row, issued by K different lanes so the K stores of a row go out together.
// Threads never touch the payload in the copy kernel; in the cast kernel they
// read the staged bf16 row from shared memory, write the e4m3 row and its
// scales to shared memory, and TMA stores those.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ep_internal.h"

namespace ep {

namespace {

constexpr uint32_t kMaxSegBytes = 16384;   // one bulk copy per row segment
constexpr int kCastThreads = 256;

__host__ __device__ __forceinline__ uint32_t round_up_u32(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Zero `bytes` (a multiple of 16) of shared memory starting at p with the threads
// [0, nthreads) of the CTA, then publish the writes to the async proxy.
__device__ __forceinline__ void zero_smem(uint8_t* p, uint32_t bytes, int tid, int nthreads) {
    for (uint32_t o = tid * 16u; o < bytes; o += nthreads * 16u)
        *reinterpret_cast<uint4*>(p + o) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
}

// ---------------------------------------------------------------------------
// Copy kernel: one warp per CTA, several CTAs per SM.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) dispatch_copy_kernel(DispatchArgs a, uint32_t row_bytes, uint32_t seg_bytes,
                                                           int nseg, int stages) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t stride = round_up_u32(seg_bytes, 128);
    uint8_t* stage = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * stride);
    int32_t* slots = reinterpret_cast<int32_t*>(full + stages);
    const int lane = threadIdx.x;
    const int K = a.K;

    if (lane == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
    pdl_wait();
    pdl_launch_dependents();

    const int64_t G = gridDim.x;
    const int64_t items = (int64_t)a.T * nseg;
    const int64_t first = blockIdx.x;
    const int64_t n = first < items ? (items - first + G - 1) / G : 0;

    auto issue = [&](int64_t j) {
        const int64_t item = first + j * G;
        const int64_t t = item / nseg;
        const uint32_t off = (uint32_t)(item % nseg) * seg_bytes;
        const uint32_t bytes = min(seg_bytes, row_bytes - off);
        const int s = (int)(j % stages);
        if (lane < K) slots[s * 32 + lane] = a.pair_slot[t * K + lane];
        if (lane == 0) {
            mbar_arrive_expect_tx(&full[s], bytes);
            bulk_load(stage + (size_t)s * stride, a.x + t * row_bytes + off, bytes, &full[s]);
        }
    };

    int64_t issued = 0;
    for (; issued < n && issued < stages; ++issued) issue(issued);

    for (int64_t j = 0; j < n; ++j) {
        const int s = (int)(j % stages);
        if (!mbar_wait(&full[s], (uint32_t)((j / stages) & 1))) {
            // A load never landed: report, wait a bounded time for the loads
            // still in flight so no copy outlives the CTA, and stop.
            if (lane == 0) atomicOr(&a.status_hdr->status, kDevTimeout);
            for (int64_t jj = j + 1; jj < issued; ++jj)
                mbar_wait(&full[jj % stages], (uint32_t)((jj / stages) & 1), 100000000ull);
            bulk_wait_all<0>();
            return;
        }
        __syncwarp();
        const int64_t item = first + j * G;
        const int64_t t = item / nseg;
        const int sg = (int)(item % nseg);
        const uint32_t off = (uint32_t)sg * seg_bytes;
        const uint32_t bytes = min(seg_bytes, row_bytes - off);
        if (lane < K) {
            const int32_t slot = slots[s * 32 + lane];
            if (slot >= 0 && (int64_t)slot < a.capacity)
                bulk_store(a.recv + (int64_t)slot * row_bytes + off, stage + (size_t)s * stride, bytes);
        }
        if (a.x_scales != nullptr && sg == 0) {
            // e4m3 input: carry the token's scale row to every destination
            for (int k = 0; k < K; ++k) {
                const int32_t slot = slots[s * 32 + k];
                if (slot < 0 || (int64_t)slot >= a.capacity) continue;
                for (int b = lane; b < a.nb; b += 32)
                    a.recv_scales[(int64_t)slot * a.nb + b] = a.x_scales[t * a.nb + b];
            }
        }
        bulk_commit();
        // refill the stage of item j-1 (its stores have finished reading it)
        if (j >= 1 && issued < n) {
            bulk_wait_read<1>();
            __syncwarp();
            issue(issued);
            ++issued;
        }
    }
    bulk_wait_all<0>();

    if (!a.zero_pad) return;
    // padding rows: bulk stores from a zeroed stage
    __syncwarp();
    zero_smem(stage, stride, lane, 32);
    __syncwarp();
    const int64_t pitems = (int64_t)a.hdr->num_pad * nseg;
    for (int64_t q = first * 32 + lane; q < pitems; q += G * 32) {
        const int32_t row = a.pad_rows[q / nseg];
        const uint32_t off = (uint32_t)(q % nseg) * seg_bytes;
        if (row < 0 || (int64_t)row >= a.capacity) continue;
        bulk_store(a.recv + (int64_t)row * row_bytes + off, stage, min(seg_bytes, row_bytes - off));
        if (a.recv_scales != nullptr && off == 0)
            for (int b = 0; b < a.nb; ++b) a.recv_scales[(int64_t)row * a.nb + b] = 0.0f;
    }
    bulk_commit();
    bulk_wait_all<0>();
}

// ---------------------------------------------------------------------------
// Cast kernel: bf16 rows in, e4m3 rows + fp32 per-128-column scales out.
// ---------------------------------------------------------------------------

// Quantise 4 consecutive values of one 128-column block held by this lane;
// the warp holds the whole block (32 lanes x 4 values).
__device__ __forceinline__ uint32_t cast_block4(uint2 raw, float* scale_out) {
    const float f0 = __uint_as_float(raw.x << 16), f1 = __uint_as_float(raw.x & 0xffff0000u);
    const float f2 = __uint_as_float(raw.y << 16), f3 = __uint_as_float(raw.y & 0xffff0000u);
    float m = fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3)));
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
    const float s = __fdiv_rn(fmaxf(m, 1e-4f), 448.0f);
    *scale_out = s;
    const __nv_fp8x2_storage_t lo =
        __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(f0, s), __fdiv_rn(f1, s)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi =
        __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(f2, s), __fdiv_rn(f3, s)), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

__global__ void __launch_bounds__(kCastThreads) dispatch_cast_kernel(DispatchArgs a, int stages) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int H = a.H, nb = a.nb, K = a.K;
    const uint32_t in_stride = round_up_u32(2u * H, 128);
    const uint32_t out_bytes = (uint32_t)H + 4u * nb;       // e4m3 row, then its scales
    const uint32_t out_stride = round_up_u32(out_bytes, 128);
    uint8_t* in = smem;
    uint8_t* out = smem + (size_t)stages * in_stride;
    uint64_t* full = reinterpret_cast<uint64_t*>(out + 2 * (size_t)out_stride);
    int32_t* slots = reinterpret_cast<int32_t*>(full + stages);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool bulk_scales = ((4u * nb) % 16u) == 0;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();

    const int64_t G = gridDim.x;
    const int64_t first = blockIdx.x;
    const int64_t n = first < a.T ? (a.T - first + G - 1) / G : 0;

    // warp 0 only
    auto issue = [&](int64_t j) {
        const int64_t t = first + j * G;
        const int s = (int)(j % stages);
        if (lane < K) slots[s * 32 + lane] = a.pair_slot ? a.pair_slot[t * K + lane] : (int32_t)t;
        if (lane == 0) {
            mbar_arrive_expect_tx(&full[s], 2u * H);
            bulk_load(in + (size_t)s * in_stride, a.x + t * 2 * H, 2u * H, &full[s]);
        }
    };

    int64_t issued = 0;
    if (warp == 0)
        for (; issued < n && issued < stages; ++issued) issue(issued);

    for (int64_t j = 0; j < n; ++j) {
        const int s = (int)(j % stages);
        const int o = (int)(j & 1);
        if (warp == 0) bulk_wait_read<1>();   // output stage o: stores of item j-2 done reading
        const bool landed = mbar_wait(&full[s], (uint32_t)((j / stages) & 1));
        if (__syncthreads_or(!landed)) {
            if (tid == 0 && a.status_hdr != nullptr) atomicOr(&a.status_hdr->status, kDevTimeout);
            if (warp == 0) {
                for (int64_t jj = j; jj < issued; ++jj)
                    mbar_wait(&full[jj % stages], (uint32_t)((jj / stages) & 1), 100000000ull);
                bulk_wait_all<0>();
            }
            return;
        }
        const uint8_t* src = in + (size_t)s * in_stride;
        uint8_t* dst = out + (size_t)o * out_stride;
        float* dst_scales = reinterpret_cast<float*>(dst + H);
        for (int b = warp; b < nb; b += kCastThreads / 32) {
            const uint2 raw = *reinterpret_cast<const uint2*>(src + (size_t)b * 256 + lane * 8);
            float sc;
            const uint32_t q = cast_block4(raw, &sc);
            *reinterpret_cast<uint32_t*>(dst + (size_t)b * 128 + lane * 4) = q;
            if (lane == 0) dst_scales[b] = sc;
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (warp == 0) {
            if (lane < K) {
                const int32_t slot = slots[s * 32 + lane];
                if (slot >= 0 && (int64_t)slot < a.capacity) {
                    bulk_store(a.recv + (int64_t)slot * H, dst, (uint32_t)H);
                    if (bulk_scales) bulk_store(a.recv_scales + (int64_t)slot * nb, dst_scales, 4u * nb);
                }
            }
            if (!bulk_scales) {
                for (int k = 0; k < K; ++k) {
                    const int32_t slot = slots[s * 32 + k];
                    if (slot < 0 || (int64_t)slot >= a.capacity) continue;
                    for (int b = lane; b < nb; b += 32) a.recv_scales[(int64_t)slot * nb + b] = dst_scales[b];
                }
            }
            bulk_commit();
            if (issued < n) {
                __syncwarp();
                issue(issued);   // into stage s: every thread finished reading it before the barrier
                ++issued;
            }
        }
    }
    if (warp == 0) bulk_wait_all<0>();

    if (!a.zero_pad) return;
    __syncthreads();
    uint8_t* zero = out;   // output stage 0, zeroed: an e4m3 row of zeros followed by zero scales
    zero_smem(zero, out_stride, tid, kCastThreads);
    __syncthreads();
    if (warp == 0) {
        const int64_t npad = a.hdr->num_pad;
        for (int64_t q = first * 32 + lane; q < npad; q += G * 32) {
            const int32_t row = a.pad_rows[q];
            if (row < 0 || (int64_t)row >= a.capacity) continue;
            bulk_store(a.recv + (int64_t)row * H, zero, (uint32_t)H);
            if (bulk_scales)
                bulk_store(a.recv_scales + (int64_t)row * nb, zero + H, 4u * nb);
            else
                for (int b = 0; b < nb; ++b) a.recv_scales[(int64_t)row * nb + b] = 0.0f;
        }
        bulk_commit();
        bulk_wait_all<0>();
    }
}

}  // namespace

cudaError_t launch_dispatch_copy(const DispatchArgs& a, int elem_bytes, cudaStream_t s) {
    const uint32_t row_bytes = (uint32_t)a.H * (uint32_t)elem_bytes;
    const int nseg = (int)((row_bytes + kMaxSegBytes - 1) / kMaxSegBytes);
    const uint32_t seg_bytes = round_up_u32((row_bytes + nseg - 1) / nseg, 16);
    const uint32_t stride = round_up_u32(seg_bytes, 128);
    // about 56 KB of stages per CTA, 2..8 stages, 4 CTAs (warps) per SM
    int stages = (int)((57344u + stride - 1) / stride);
    stages = stages < 2 ? 2 : (stages > 8 ? 8 : stages);
    const size_t smem = (size_t)stages * stride + (size_t)stages * 8 + (size_t)stages * 32 * 4;
    cudaError_t err =
        cudaFuncSetAttribute(dispatch_copy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int ctas_per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, dispatch_copy_kernel, 32, smem);
    if (err != cudaSuccess) return err;
    if (ctas_per_sm > 4) ctas_per_sm = 4;
    if (ctas_per_sm < 1) ctas_per_sm = 1;
    const int grid = a.sms * ctas_per_sm;
    return launch_pdl(dispatch_copy_kernel, dim3(grid), dim3(32), smem, s, false, a, row_bytes, seg_bytes, nseg, stages);
}

cudaError_t launch_dispatch_cast(const DispatchArgs& a, cudaStream_t s) {
    const uint32_t in_stride = round_up_u32(2u * a.H, 128);
    const uint32_t out_stride = round_up_u32((uint32_t)a.H + 4u * a.nb, 128);
    const int stages = 3;   // H <= 16384: at most 130 KB of stages
    const size_t smem = (size_t)stages * in_stride + 2 * (size_t)out_stride + (size_t)stages * 8 +
                        (size_t)stages * 32 * 4;
    cudaError_t err =
        cudaFuncSetAttribute(dispatch_cast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int ctas_per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, dispatch_cast_kernel, kCastThreads, smem);
    if (err != cudaSuccess) return err;
    if (ctas_per_sm > 4) ctas_per_sm = 4;
    if (ctas_per_sm < 1) ctas_per_sm = 1;
    return launch_pdl(dispatch_cast_kernel, dim3(a.sms * ctas_per_sm), dim3(kCastThreads), smem, s, false, a, stages);
}

}  // namespace ep
