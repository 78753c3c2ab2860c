// Dispatch: scatter token rows into the expert-contiguous receive buffer
// ("DeepEP 测试目标 API 系统性参考" §2.1 dispatch(): x or (fp8, scales) in, rows
// of the same type out, do_zero_padding).  The FP8 cast on the way is in
// ep_cast.cu.
//
// The work is pure data movement, bound by HBM bandwidth: each token row is
// read once and written K times, padding rows are written once.  Rows travel
// through shared memory on the TMA engine: one bulk load per row segment into
// a multi-stage ring guarded by mbarriers, then one bulk store per destination
// row, issued by K different lanes so the K stores of a row go out together.
// The copy kernel takes its rows by ticket from counters in the workspace, so
// no SM idles while others finish a larger share.
// Threads never touch the payload.
#include "ep_dispatch_common.cuh"

namespace ep {

namespace {

using namespace dispatch_dev;

constexpr uint32_t kMaxSegBytes = 16384;   // one bulk copy per row segment
constexpr uint32_t kTailSegBytes = 4096;   // segments of the last tokens

// ---------------------------------------------------------------------------
// Copy kernel.  Work is handed out by tickets (atomic counters in the layout's
// workspace header), not by a fixed stride: an ncu capture of a fixed split
// showed the SMs active only 84 % of the kernel on average (some finished at
// 67 %) while the rest worked through their share, so DRAM idled in the tail.
// Two warps per CTA, several CTAs per SM:
//   warp 0  token rows: a ring of `stages` row segments; it takes tickets
//           (one row segment each) from tok_ticket, bulk-loads the segment
//           and, once it lands, lanes k < K bulk-store it to receive rows
//           pair_slot[t, k]; a stage is refilled once its stores have read it;
//   warp 1  padding rows (do_zero_padding): bulk stores of a zeroed buffer of
//           zero_bytes, 32 pieces per ticket from pad_ticket, concurrently
//           with the token rows, so the zero writes fill the gaps of the copy
//           stream instead of forming a tail of their own.
// The CTA that finishes last resets the tickets for the next launch.
// ---------------------------------------------------------------------------
constexpr int kCopyThreads = 64;

// kRegions: the destinations are rows of the regions in DispatchArgs (bf16
// rows; ep_dispatch_regions) instead of the one receive buffer.
template <bool kRegions>
__device__ __forceinline__ uint8_t* region_row(const DispatchArgs& a, int64_t e, int32_t slot, uint32_t row_bytes) {
    if (slot < 0 || e < 0 || e >= (int64_t)a.El * a.R) return nullptr;
    const int64_t row = (int64_t)slot + a.row_delta[e];
    if (row < 0 || row >= a.region_capacity) return nullptr;
    return a.regions[e / a.El] + row * row_bytes;
}

// Items: tokens [0, t_full) in nseg segments of seg_bytes, then the last
// tokens [t_full, T) in nseg2 smaller segments of seg2_bytes, so the work
// drawn last is small and the SMs finish together.
struct CopyItems {
    uint32_t row_bytes, seg_bytes, seg2_bytes;
    int nseg, nseg2;
    uint32_t t_full;
    __device__ __forceinline__ uint32_t count(uint32_t T) const {
        return t_full * (uint32_t)nseg + (T - t_full) * (uint32_t)nseg2;
    }
    // token, byte offset and length of item i
    __device__ __forceinline__ void locate(uint32_t i, int64_t& t, uint32_t& off, uint32_t& bytes) const {
        const uint32_t nf = t_full * (uint32_t)nseg;
        uint32_t seg;
        if (i < nf) {
            t = i / nseg;
            off = (i % nseg) * seg_bytes;
            seg = seg_bytes;
        } else {
            t = t_full + (i - nf) / nseg2;
            off = ((i - nf) % nseg2) * seg2_bytes;
            seg = seg2_bytes;
        }
        bytes = min(seg, row_bytes - off);
    }
};

template <bool kRegions>
__global__ void __launch_bounds__(kCopyThreads) dispatch_copy_kernel(DispatchArgs a, CopyItems it, int stages) {
    const uint32_t row_bytes = it.row_bytes, seg_bytes = it.seg_bytes;
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t stride = round_up_u32(seg_bytes, 128);
    uint8_t* ring = smem;
    uint8_t* zero = ring + (size_t)stages * stride;
    uint64_t* full = reinterpret_cast<uint64_t*>(zero + kZeroBytes);
    uint8_t** dsts = reinterpret_cast<uint8_t**>(full + stages);     // [stages][32] (regions only)
    int32_t* slots = reinterpret_cast<int32_t*>(dsts + (kRegions ? stages * 32 : 0));   // [stages][32]
    uint32_t* stage_item = reinterpret_cast<uint32_t*>(slots + stages * 32);   // [stages]: item held
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.K;
    WsHeader* h = a.status_hdr;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    zero_smem(zero, kZeroBytes, tid, kCopyThreads);
    __syncthreads();

    // token rows: one ticket per (token, segment) item; the row of a stage is
    // loaded by load_row, its destinations by load_slots
    const uint32_t items = it.count((uint32_t)a.T);
    auto load_row = [&](int s, uint32_t item) {
        int64_t t;
        uint32_t off, bytes;
        it.locate(item, t, off, bytes);
        if (lane == 0) {
            stage_item[s] = item;
            mbar_arrive_expect_tx(&full[s], bytes);
            bulk_load(ring + (size_t)s * stride, a.x + t * row_bytes + off, bytes, &full[s]);
        }
    };
    auto load_slots = [&](int s, uint32_t item) {
        int64_t t;
        uint32_t off, bytes;
        it.locate(item, t, off, bytes);
        if (lane < K) {
            const int32_t slot = a.pair_slot[t * K + lane];
            if (kRegions) dsts[s * 32 + lane] = region_row<kRegions>(a, a.topk_idx[t * K + lane], slot, row_bytes);
            else slots[s * 32 + lane] = slot;
        }
    };
    // the first `stages` tickets in one draw (the counters are not written by
    // the preceding grid, and x is complete when a.early is set)
    uint32_t first = 0;
    int64_t issued = 0;
    if (warp == 0) {
        if (lane == 0) first = atomicAdd(&h->tok_ticket, (uint32_t)stages);
        first = __shfl_sync(0xffffffffu, first, 0);
        if (a.early)
            for (; issued < stages && first + issued < items; ++issued) load_row((int)issued, first + (uint32_t)issued);
    }
    // no launch_dependents: a successor's CTAs resident beside this kernel
    // slowed the step (765 against 733 us at large prefill); it starts when
    // this grid ends
    pdl_wait();

    if (warp == 1) {
        // ---- padding rows: pieces of kZeroBytes, 32 per ticket ----
        if (a.zero_pad) {
            const uint32_t npiece = (row_bytes + kZeroBytes - 1) / kZeroBytes;
            const int64_t pieces = (kRegions ? a.num_pad_list : (int64_t)a.hdr->num_pad) * npiece;
            const int64_t tickets = (pieces + 31) / 32;
            const uint32_t sf_bytes = (uint32_t)a.nb * 4u;   // e4m3 rows: their fp32 scale row
            for (;;) {
                uint32_t tk = 0;
                if (lane == 0) tk = atomicAdd(&h->pad_ticket, 1u);
                tk = __shfl_sync(0xffffffffu, tk, 0);
                if ((int64_t)tk >= tickets) break;
                const int64_t q = (int64_t)tk * 32 + lane;
                if (q < pieces && kRegions) {
                    const int64_t pr = q / npiece;
                    const uint32_t off = (uint32_t)(q - pr * npiece) * kZeroBytes;
                    const int64_t entry = a.pad_list[pr];
                    const int64_t r = entry >> 32, row = entry & 0xffffffffll;
                    if (r >= 0 && r < a.R && row < a.region_capacity)
                        bulk_store(a.regions[r] + row * row_bytes + off, zero, min(kZeroBytes, row_bytes - off));
                } else if (q < pieces) {
                    const int64_t pr = q / npiece;
                    const uint32_t off = (uint32_t)(q - pr * npiece) * kZeroBytes;
                    const int32_t row = a.pad_rows[pr];
                    if (row >= 0 && (int64_t)row < a.capacity) {
                        bulk_store(a.recv + (int64_t)row * row_bytes + off, zero, min(kZeroBytes, row_bytes - off));
                        if (a.recv_scales != nullptr && off == 0) {
                            if (sf_bytes % 16u == 0 && sf_bytes <= kZeroBytes)
                                bulk_store(a.recv_scales + (int64_t)row * a.nb, zero, sf_bytes);
                            else
                                for (int b = 0; b < a.nb; ++b) a.recv_scales[(int64_t)row * a.nb + b] = 0.0f;
                        }
                    }
                }
                bulk_commit();
            }
            bulk_wait_all<0>();
        }
        tickets_done(h);
        return;
    }

    // ---- token rows (warp 0) ----
    // the row's bulk load goes out first: it does not need the slots, which
    // are read only when the row has landed
    auto issue = [&](int s, uint32_t item) {
        load_row(s, item);
        load_slots(s, item);
    };
    if (a.early) {
        for (int64_t j = 0; j < issued; ++j) load_slots((int)j, first + (uint32_t)j);
    } else {
        for (; issued < stages && first + issued < items; ++issued) issue((int)issued, first + (uint32_t)issued);
    }
    // then one ticket drawn ahead of its use
    bool more = first + (uint32_t)stages < items;
    uint32_t next = 0;
    if (lane == 0 && more) next = atomicAdd(&h->tok_ticket, 1u);

    for (int64_t j = 0; j < issued; ++j) {
        const int s = (int)(j % stages);
        if (!mbar_wait(&full[s], (uint32_t)((j / stages) & 1))) {
            // A load never landed: report, wait a bounded time for the loads
            // still in flight so no copy outlives the CTA, and stop.
            if (lane == 0) atomicOr(&h->status, kDevTimeout);
            for (int64_t jj = j + 1; jj < issued; ++jj)
                mbar_wait(&full[jj % stages], (uint32_t)((jj / stages) & 1), 100000000ull);
            break;
        }
        __syncwarp();
        const uint32_t item = stage_item[s];
        int64_t t;
        uint32_t off, bytes;
        it.locate(item, t, off, bytes);
        if (lane < K && kRegions) {
            uint8_t* dst = dsts[s * 32 + lane];
            if (dst != nullptr) bulk_store(dst + off, ring + (size_t)s * stride, bytes);
        } else if (lane < K) {
            const int32_t slot = slots[s * 32 + lane];
            if (slot >= 0 && (int64_t)slot < a.capacity)
                bulk_store(a.recv + (int64_t)slot * row_bytes + off, ring + (size_t)s * stride, bytes);
        }
        if (!kRegions && a.x_scales != nullptr && off == 0) {
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
        if (j >= 1 && more) {
            bulk_wait_read<1>();
            __syncwarp();
            const uint32_t tk = __shfl_sync(0xffffffffu, next, 0);
            if (tk < items) {
                issue((int)((j - 1) % stages), tk);
                ++issued;
                if (lane == 0) next = atomicAdd(&h->tok_ticket, 1u);
            } else {
                more = false;
            }
        }
    }
    bulk_wait_all<0>();
    tickets_done(h);
}

}  // namespace

cudaError_t launch_dispatch_copy(const DispatchArgs& a, int elem_bytes, cudaStream_t s, bool regions) {
    CopyItems it{};
    it.row_bytes = (uint32_t)a.H * (uint32_t)elem_bytes;
    it.nseg = (int)((it.row_bytes + kMaxSegBytes - 1) / kMaxSegBytes);
    it.seg_bytes = round_up_u32((it.row_bytes + it.nseg - 1) / it.nseg, 16);
    it.nseg2 = (int)((it.row_bytes + kTailSegBytes - 1) / kTailSegBytes);
    if (it.nseg2 < it.nseg) it.nseg2 = it.nseg;
    it.seg2_bytes = round_up_u32((it.row_bytes + it.nseg2 - 1) / it.nseg2, 16);
    const uint32_t stride = round_up_u32(it.seg_bytes, 128);
    // three row stages of at most 16 KB, up to four CTAs per SM: a sweep of
    // 2-4 stages, 3-4 CTAs per SM and 2-4 KB zero buffers on the prefill,
    // large-prefill and decode workloads put every setting within 2 %
    const int stages = 3;
    const size_t smem = (size_t)stages * stride + kZeroBytes + (size_t)stages * 8 + (size_t)stages * 33 * 4 +
                        (regions ? (size_t)stages * 32 * 8 : 0);
    auto kernel = regions ? dispatch_copy_kernel<true> : dispatch_copy_kernel<false>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int ctas_per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, kernel, kCopyThreads, smem);
    if (err != cudaSuccess) return err;
    if (ctas_per_sm > 4) ctas_per_sm = 4;
    if (ctas_per_sm < 1) ctas_per_sm = 1;
    const int grid = a.sms * ctas_per_sm;
    // The last 2 * grid tokens go in segments of at most 4 KB, so the SMs run
    // out of work together (decode: 82-83 against 86 us; large prefill: 381
    // against 386-389 us; 3 or 4 * grid measured the same, 2 KB segments and
    // a tail of grid / 2 or grid tokens less well).  Not where padding may
    // exceed a fifth of the rows: its 2 KB pieces already keep the SMs busy
    // to the end, and the small segments cost more than they save (prefill:
    // 137.7 against 134.6 us).
    const int64_t pads = a.zero_pad ? (regions ? a.num_pad_list : a.max_pad_rows) : 0;
    const bool split = pads * 4 <= (int64_t)a.T * a.K;
    const int64_t tail = 2 * (int64_t)grid;
    it.t_full = !split ? (uint32_t)a.T : a.T > tail ? (uint32_t)(a.T - tail) : 0u;
    return launch_pdl(kernel, dim3(grid), dim3(kCopyThreads), smem, s, false, a, it, stages);
}

}  // namespace ep
