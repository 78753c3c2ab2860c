// Layout and dispatch in one kernel, the way DeepEP V2's dispatch() derives
// its routing layout from topk_idx inside the call ("DeepEP 测试目标 API 系统性参考"
// §2.1 and the V1/V2 comparison table in §3.1).
//
// One cooperative CTA per SM, and CTA c owns layout chunk c (a run of whole
// tokens).  Before any layout work, up to four copy warps each start TMA bulk
// loads of their first rows of the chunk into their own shared-memory ring, so
// the row reads overlap the layout's latency chain (count, grid barrier, scan,
// slot assignment).  Then each copy warp walks its rows: when a row has
// landed, lanes k < K each issue one bulk store to receive row pair_slot[t, k]
// (written moments before by this CTA), and the freed stage is refilled.  Four
// more warps meanwhile zero-fill a contiguous 1/C share of all padding rows
// with bulk stores from a zeroed segment.  The bytes moved are exactly those
// of ep_layout + ep_dispatch.
#include "ep_layout_body.cuh"

namespace ep {

namespace {

constexpr uint32_t kMaxSegBytes = 16384;

__host__ __device__ __forceinline__ uint32_t rup(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// A fused-kernel plan: `copy_warps` warps each drive a ring of `stages` row
// stages (warp w copies rows w, w + copy_warps, ... of the chunk); the next
// kPadWarps warps zero-fill this CTA's share of the padding rows.
struct FusedPlan {
    uint32_t row_bytes, seg_bytes, layout_bytes;
    int nseg, copy_warps, stages;
};
constexpr int kPadWarps = 4;

template <int NT>
__global__ void __launch_bounds__(NT, 1) layout_dispatch_kernel(LayoutArgs la, DispatchArgs da, FusedPlan fp) {
    extern __shared__ __align__(128) uint8_t smem[];
    int32_t* lsm = reinterpret_cast<int32_t*>(smem);
    const uint32_t row_bytes = fp.row_bytes, seg_bytes = fp.seg_bytes;
    const int nseg = fp.nseg, W = fp.copy_warps, S = fp.stages;
    const uint32_t stride = rup(seg_bytes, 128);
    uint8_t* stage = smem + fp.layout_bytes;                 // [W][S] row stages
    uint8_t* zero = stage + (size_t)W * S * stride;          // one zeroed segment
    uint64_t* full = reinterpret_cast<uint64_t*>(zero + stride);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = la.K;
    const int c = blockIdx.x;

    if (tid == 0) {
        for (int i = 0; i < W * S; ++i) mbar_init(&full[i], 1);
        fence_barrier_init();
    }
    for (uint32_t o = tid * 16u; o < stride; o += NT * 16u)
        *reinterpret_cast<uint4*>(zero + o) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();

    // this CTA's rows: the tokens of its layout chunk, all segments of a token
    // in a row; copy warp w owns rows w, w + W, ...
    const int64_t t0 = (int64_t)c * la.CT;
    const int64_t t1 = min(t0 + la.CT, (int64_t)la.T);
    const int64_t n = (t1 > t0 ? t1 - t0 : 0) * nseg;
    const bool copier = warp < W;
    const int64_t mine = (copier && n > warp) ? (n - warp + W - 1) / W : 0;
    uint8_t* my_stage = stage + (size_t)(copier ? warp : 0) * S * stride;
    uint64_t* my_full = full + (copier ? warp : 0) * S;
    auto row_of = [&](int64_t u) { return warp + u * W; };
    auto issue = [&](int64_t u) {   // lane 0 of a copy warp
        const int64_t j = row_of(u);
        const int64_t t = t0 + j / nseg;
        const uint32_t off = (uint32_t)(j % nseg) * seg_bytes;
        const uint32_t bytes = min(seg_bytes, row_bytes - off);
        const int s = (int)(u % S);
        mbar_arrive_expect_tx(&my_full[s], bytes);
        bulk_load(my_stage + (size_t)s * stride, da.x + t * row_bytes + off, bytes, &my_full[s]);
    };
    int64_t issued = mine < S ? mine : S;
    if (copier && lane == 0)
        for (int64_t u = 0; u < issued; ++u) issue(u);

    if (!layout_dev::layout_body<NT>(la, lsm)) {
        // grid barrier timed out (reported): let the row loads in flight land, then stop
        if (copier && lane == 0)
            for (int64_t u = 0; u < issued; ++u) mbar_wait(&my_full[u % S], (uint32_t)((u / S) & 1), 100000000ull);
        return;
    }

    if (copier) {
        for (int64_t u = 0; u < mine; ++u) {
            const int s = (int)(u % S);
            if (!mbar_wait(&my_full[s], (uint32_t)((u / S) & 1))) {
                if (lane == 0) {
                    atomicOr(&la.hdr->status, kDevTimeout);
                    for (int64_t uu = u + 1; uu < issued; ++uu)
                        mbar_wait(&my_full[uu % S], (uint32_t)((uu / S) & 1), 100000000ull);
                }
                bulk_wait_all<0>();
                return;
            }
            __syncwarp();
            const int64_t j = row_of(u);
            const int64_t t = t0 + j / nseg;
            const int sg = (int)(j % nseg);
            const uint32_t off = (uint32_t)sg * seg_bytes;
            const uint32_t bytes = min(seg_bytes, row_bytes - off);
            int32_t slot = -1;
            if (lane < K) {
                slot = la.pair_slot[t * K + lane];
                if (slot >= 0 && (int64_t)slot < la.capacity)
                    bulk_store(da.recv + (int64_t)slot * row_bytes + off, my_stage + (size_t)s * stride, bytes);
            }
            if (da.x_scales != nullptr && sg == 0) {
                // e4m3 input: carry the token's scale row to every destination
                for (int k = 0; k < K; ++k) {
                    const int32_t sk = __shfl_sync(0xffffffffu, slot, k);
                    if (sk < 0 || (int64_t)sk >= la.capacity) continue;
                    for (int b = lane; b < da.nb; b += 32)
                        da.recv_scales[(int64_t)sk * da.nb + b] = da.x_scales[t * da.nb + b];
                }
            }
            bulk_commit();
            if (u >= 1 && issued < mine) {       // refill the stage of row u-1
                bulk_wait_read<1>();
                __syncwarp();
                if (lane == 0) issue(issued);
                ++issued;
            }
        }
        bulk_wait_all<0>();
    } else if (warp < W + kPadWarps && da.zero_pad) {
        layout_dev::LayoutSmem L(lsm, la.E);
        const int E = la.E;
        const int64_t P = L.padpre[E];
        const int64_t j0 = P * c / gridDim.x, j1 = P * (c + 1) / gridDim.x;
        for (int64_t j = j0 + (int64_t)(warp - W) * 32 + lane; j < j1; j += kPadWarps * 32) {
            int lo = 0, hi = E + 1;              // last e with padpre[e] <= j
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (L.padpre[mid] <= j) lo = mid + 1;
                else hi = mid;
            }
            const int e = lo - 1;
            const int64_t row = (int64_t)L.off[e] + L.cnt[e] + (j - L.padpre[e]);
            if (row >= la.capacity) continue;
            for (int sg = 0; sg < nseg; ++sg) {
                const uint32_t off = (uint32_t)sg * seg_bytes;
                bulk_store(da.recv + row * row_bytes + off, zero, min(seg_bytes, row_bytes - off));
            }
            if (da.recv_scales != nullptr)
                for (int b = 0; b < da.nb; ++b) da.recv_scales[row * da.nb + b] = 0.0f;
        }
        bulk_commit();
        bulk_wait_all<0>();
    }
}

template <int NT>
cudaError_t launch_fused_nt(LayoutArgs la, DispatchArgs da, int elem_bytes, cudaStream_t s) {
    FusedPlan fp;
    fp.row_bytes = (uint32_t)da.H * (uint32_t)elem_bytes;
    fp.nseg = (int)((fp.row_bytes + kMaxSegBytes - 1) / kMaxSegBytes);
    fp.seg_bytes = rup((fp.row_bytes + fp.nseg - 1) / fp.nseg, 16);
    const uint32_t stride = rup(fp.seg_bytes, 128);
    fp.layout_bytes = rup((uint32_t)(layout_dev::layout_smem_ints(la.E) * sizeof(int32_t)), 128);
    int max_smem = 0, dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err != cudaSuccess) return err;
    const size_t fixed = (size_t)fp.layout_bytes + stride + 2048;
    int total = (int)(((size_t)max_smem > fixed ? (size_t)max_smem - fixed : 0) / (stride + 8));
    if (total > 12) total = 12;
    if (total < 2) {   // rows too large to stage beside the layout scratch: two kernels
        cudaError_t e2 = launch_layout(la, da.sms, s);
        return e2 == cudaSuccess ? launch_dispatch_copy(da, elem_bytes, s) : e2;
    }
    // up to four copy warps with at least three stages each
    fp.copy_warps = total >= 12 ? 4 : total >= 9 ? 3 : total >= 6 ? 2 : 1;
    fp.stages = total / fp.copy_warps;
    const size_t smem = (size_t)fp.layout_bytes + ((size_t)fp.copy_warps * fp.stages + 1) * stride +
                        (size_t)fp.copy_warps * fp.stages * 8;
    err = cudaFuncSetAttribute(layout_dispatch_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    // one chunk (CTA) per SM, whole tokens per chunk
    const int64_t ct = ((int64_t)la.T + da.sms - 1) / da.sms;
    la.CT = (int)ct;
    la.C = (int)(((int64_t)la.T + ct - 1) / ct);
    return launch_pdl(layout_dispatch_kernel<NT>, dim3(la.C), dim3(NT), smem, s, true, la, da, fp);
}

}  // namespace

cudaError_t launch_layout_dispatch(LayoutArgs la, DispatchArgs da, int elem_bytes, cudaStream_t s) {
    return layout_dev::layout_threads(la.E) == layout_dev::kWideThreads
               ? launch_fused_nt<layout_dev::kWideThreads>(la, da, elem_bytes, s)
               : launch_fused_nt<layout_dev::kNarrowThreads>(la, da, elem_bytes, s);
}

}  // namespace ep
