// Routing layout of the expand dispatch ("DeepEP 测试目标 API 系统性参考" §2.1:
// the layout V2 derives from topk_idx, expert_alignment, do_expand; the
// count -> prefix-sum placement -> reorder stages of the Ascend dispatch on the
// "URMA" tag page).
//
// One cooperative kernel, one CTA per chunk of whole tokens (at most 128, all
// resident at once):
//   1. count: the chunk's per-expert histogram with warp-aggregated shared
//      atomics (__match_any_sync groups lanes holding the same expert; one
//      leader adds the group size), published as row c of table[C][E] and
//      added into the sum of its super-chunk (16 consecutive chunks);
//   2. one grid barrier (bounded wait);
//   3. scan, redundantly in every CTA: for each expert the total over all
//      chunks (the super-chunk sums) and the sum over chunks before c (the
//      super-chunk sums before c's, then the rows of c's own super-chunk
//      before c): at most 8 + 15 rows of 16-byte loads at 128 chunks, over
//      eight thread groups; off[e] = sum_{e'<e} align(cnt, A) and the padding
//      prefix by block scans;
//   4. assign: each warp owns a contiguous run of the chunk's pairs; a first
//      pass counts per (warp, expert), a scan across warps gives each warp its
//      starting row, a second pass ranks lanes of the same expert with
//      __match_any_sync + popc(lanemask_lt).  With the chunk base this is the
//      stable (token-major, k-minor) order, equal to the sequential definition
//      bit for bit;
//   5. padding rows of the experts e = c, c + C, ...
// The kernel waits for its predecessor in the stream before touching global
// memory and lets its successor launch early (programmatic dependent launch).
#include "ep_layout_body.cuh"

namespace ep {

namespace {

// The layout alone uses at most this many chunks (of about 512 pairs each).
// Measured: 64 and 128 give the same 14.4 us at 32 k pairs, and 128 gives
// 16.5 us against 18.4 at 131 k pairs; 32 or fewer are slower everywhere
// but on a single-chunk batch (the scan's table reads are cheap next to the
// per-chunk count and assign work).
constexpr int kLayoutChunks = 128;

template <int NT, bool kRankKeys>
__global__ void __launch_bounds__(NT, 1) layout_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int32_t sm[];
    pdl_wait();
    pdl_launch_dependents();
    layout_dev::layout_body<NT, kRankKeys>(a, sm);
}

template <int NT, bool kRankKeys>
cudaError_t launch_layout_nt(LayoutArgs a, int sms, cudaStream_t s) {
    auto kernel = layout_kernel<NT, kRankKeys>;
    const size_t smem = layout_dev::layout_smem_ints(a.E, kRankKeys ? a.src_E : 0) * sizeof(int32_t);
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, NT, smem);
    if (err != cudaSuccess) return err;
    int max_chunks = sms * (per_sm > 0 ? per_sm : 1);
    if (max_chunks > kLayoutChunks) max_chunks = kLayoutChunks;
    // the fixed-slab form lists up to E * slab padding rows, far more than its
    // pairs: as many chunks as the tokens allow, so every SM shares that work
    Chunking ch = chunking(a.T, a.K, max_chunks, a.slab > 0 ? 1 : NT);
    if (ch.num_chunks == 0) {   // no tokens (the fixed-slab form still has its padding rows to list)
        ch.num_chunks = 1;
        ch.chunk_tokens = 0;
    }
    a.C = ch.num_chunks;
    a.CT = ch.chunk_tokens;
    return launch_pdl(kernel, dim3(a.C), dim3(NT), smem, s, true, a);
}

}  // namespace

cudaError_t launch_layout(LayoutArgs a, int sms, cudaStream_t s) {
    const bool wide = layout_dev::layout_threads(a.E) == layout_dev::kWideThreads;
    if (a.src_idx != nullptr)   // per-rank keys: E = R <= 32, always the wide CTA
        return launch_layout_nt<layout_dev::kWideThreads, true>(a, sms, s);
    return wide ? launch_layout_nt<layout_dev::kWideThreads, false>(a, sms, s)
                : launch_layout_nt<layout_dev::kNarrowThreads, false>(a, sms, s);
}

}  // namespace ep
