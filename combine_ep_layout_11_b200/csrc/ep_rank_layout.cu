// Per-token-per-rank layout: the default receive form of dispatch when the
// expand layout is off ("DeepEP 测试目标 API 系统性参考" §2.1 dispatch(),
// do_expand), with the V1 layout quantities of §3.1 Buffer.dispatch()
// (num_tokens_per_rank, is_token_in_rank, num_tokens_per_expert) and its
// receive outputs (recv_topk_idx, recv_topk_weights,
// num_recv_tokens_per_expert_list).
//
// A token reaches rank r when one of its experts lives there (e / (E/R) == r).
// The receive rows are the (rank, token) pairs in rank-major, token-ascending
// order.  That is exactly the expand layout of a derived routing table with
// one "expert" per rank - entry (t, r) = r if the token reaches r, else -1 -
// with E' = K' = R and alignment 1, so the rows come from the same layout
// kernel (per-chunk counts, one grid barrier, scan, stable slots):
//   1. rank_prep_kernel reads topk_idx once and writes the derived table
//      [T, R] to the workspace, is_token_in_rank [T, R], and the per-expert
//      pair counts (a shared-memory histogram per CTA, then one global add
//      per expert and CTA; integer sums, so the result does not depend on
//      the order of the adds);
//   2. layout_kernel on the derived table gives num_tokens_per_rank, the rank
//      offsets, token_slot [T, R] and recv_src_token;
//   3. rank_post_kernel writes recv_topk_idx / recv_topk_weights row by row
//      and the expert counts, plain and aligned.
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kRankThreads = 256;

__global__ void __launch_bounds__(kRankThreads) rank_prep_kernel(const int64_t* topk_idx, int T, int K, int E,
                                                                 int R, int64_t* rank_idx, uint8_t* in_rank,
                                                                 int32_t* counts, WsHeader* hdr) {
    extern __shared__ int32_t hist[];   // [E]
    for (int e = threadIdx.x; e < E; e += kRankThreads) hist[e] = 0;
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    const int El = E / R;
    const int64_t stride = (int64_t)gridDim.x * kRankThreads;
    bool bad = false;
    for (int64_t t = (int64_t)blockIdx.x * kRankThreads + threadIdx.x; t < T; t += stride) {
        uint32_t mask = 0;
        for (int k = 0; k < K; ++k) {
            const int64_t e = topk_idx[t * K + k];
            if (e >= 0 && e < E) {
                mask |= 1u << (int)(e / El);
                atomicAdd(&hist[e], 1);
            } else if (e != -1) {
                bad = true;   // outside [-1, E): reported, treated as -1
            }
        }
        for (int r = 0; r < R; ++r) {
            const bool in = (mask >> r) & 1u;
            rank_idx[t * R + r] = in ? r : -1;
            if (in_rank) in_rank[t * R + r] = in ? 1 : 0;
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(&hdr->pending, kDevBadExpert);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kRankThreads)
        if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

// Rank of receive row `row`: the r with rank_off[r] <= row < rank_off[r + 1].
__device__ __forceinline__ int row_rank(const int32_t* rank_off, int R, int row) {
    int lo = 0, hi = R - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rank_off[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kRankThreads) rank_post_kernel(RankPostArgs a) {
    pdl_wait();
    pdl_launch_dependents();
    const int El = a.E / a.R, K = a.K;
    const int64_t stride = (int64_t)gridDim.x * kRankThreads;
    const int64_t gid = (int64_t)blockIdx.x * kRankThreads + threadIdx.x;
    int64_t rows = a.rank_off[a.R];
    if (rows > a.capacity) rows = a.capacity;
    if (a.recv_topk_idx || a.recv_topk_w) {
        for (int64_t row = gid; row < rows; row += stride) {
            const int r = row_rank(a.rank_off, a.R, (int)row);
            const int64_t t = a.recv_src[row];
            for (int k = 0; k < K; ++k) {
                const int64_t e = a.topk_idx[t * K + k];
                const bool local = e >= 0 && e < a.E && e / El == r;
                if (a.recv_topk_idx) a.recv_topk_idx[row * K + k] = local ? e - (int64_t)r * El : -1;
                if (a.recv_topk_w)
                    a.recv_topk_w[row * K + k] = local ? (a.topk_weights ? a.topk_weights[t * K + k] : 1.0f) : 0.0f;
            }
        }
    }
    for (int64_t e = gid; e < a.E; e += stride) {
        const int32_t c = a.counts[e];
        if (a.num_tokens_per_expert) a.num_tokens_per_expert[e] = c;
        if (a.num_recv_per_expert) a.num_recv_per_expert[e] = (c + a.A - 1) / a.A * a.A;
    }
}

}  // namespace

RankWsLayout rank_ws_layout(int T, int R, int E) {
    RankWsLayout w;
    w.expand = ws_layout(T, R, R, 1);
    const size_t n = (size_t)(T > 0 ? T : 0) * (size_t)R;
    w.rank_idx_off = w.expand.total;
    w.scratch_w_off = round_up(w.rank_idx_off + n * 8, 256);
    w.scratch_lexp_off = round_up(w.scratch_w_off + n * 4, 256);
    w.counts_off = round_up(w.scratch_lexp_off + n * 4, 256);
    w.total = round_up(w.counts_off + (size_t)E * 4, 256);
    return w;
}

cudaError_t launch_rank_layout(const RankPrepArgs& p, LayoutArgs la, const RankPostArgs& post, int sms,
                               cudaStream_t s) {
    cudaError_t err = cudaMemsetAsync(p.counts, 0, (size_t)p.E * 4, s);
    if (err != cudaSuccess) return err;
    const size_t smem = (size_t)p.E * 4;
    int grid = (p.T + kRankThreads - 1) / kRankThreads;
    if (grid > 2 * sms) grid = 2 * sms;
    if (grid < 1) grid = 1;
    err = launch_pdl(rank_prep_kernel, dim3(grid), dim3(kRankThreads), smem, s, false, p.topk_idx, p.T, p.K, p.E,
                     p.R, p.rank_idx, p.in_rank, p.counts, p.hdr);
    if (err != cudaSuccess) return err;
    err = launch_layout(la, sms, s);
    if (err != cudaSuccess) return err;
    const int64_t rows = (int64_t)p.T * p.R;
    int64_t pg = (rows + kRankThreads - 1) / kRankThreads;
    if (pg > 2 * sms) pg = 2 * sms;
    if (pg < 1) pg = 1;
    return launch_pdl(rank_post_kernel, dim3((unsigned)pg), dim3(kRankThreads), 0, s, false, post);
}

}  // namespace ep
