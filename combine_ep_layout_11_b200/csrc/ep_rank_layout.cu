// Per-token-per-rank layout: the default receive form of dispatch when the
// expand layout is off ("DeepEP 测试目标 API 系统性参考" §2.1 dispatch(),
// do_expand), with the V1 layout quantities of §3.1 Buffer.dispatch()
// (num_tokens_per_rank, is_token_in_rank, num_tokens_per_expert) and its
// receive outputs (recv_topk_idx, recv_topk_weights,
// num_recv_tokens_per_expert_list).
//
// A token reaches rank r when one of its experts lives there (e / (E/R) == r).
// The receive rows are the (rank, token) pairs in rank-major, token-ascending
// order.  That is exactly the expand layout of a (token, rank) table with one
// "expert" per rank - entry (t, r) = r if the token reaches r, else -1 - with
// E' = K' = R and alignment 1, so the rows come from the same layout kernel
// (per-chunk counts, one grid barrier, scan, stable slots), whose keys are
// computed from topk_idx on the fly (LayoutArgs::src_idx):
//   1. layout_kernel with per-rank keys: num_tokens_per_rank, the rank
//      offsets, token_slot [T, R], recv_src_token and is_token_in_rank;
//   2. rank_post_kernel, over the (token, rank) pairs: recv_topk_idx /
//      recv_topk_weights of every row, and the per-expert pair counts - each
//      selected (t, k) is local to exactly one reached rank, so counting the
//      local entries of every row counts every pair once.  A shared-memory
//      histogram per CTA goes to a zeroed workspace array with one atomic add
//      per expert; the last CTA to finish (a counter, after a fence) writes
//      the plain and aligned counts and zeroes the array and the counter for
//      the next call.  Integer sums, so the result does not depend on the
//      order of the adds.
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kRankThreads = 256;

__global__ void __launch_bounds__(kRankThreads) rank_post_kernel(RankPostArgs a) {
    extern __shared__ int32_t hist[];   // [E]
    __shared__ int s_last;
    for (int e = threadIdx.x; e < a.E; e += kRankThreads) hist[e] = 0;
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    const int El = a.E / a.R, K = a.K;
    const int64_t stride = (int64_t)gridDim.x * kRankThreads;
    const int64_t n = (int64_t)a.T * a.R;
    for (int64_t i = (int64_t)blockIdx.x * kRankThreads + threadIdx.x; i < n; i += stride) {
        const int32_t slot = a.token_slot[i];
        if (slot < 0) continue;
        const int64_t t = i / a.R;
        const int r = (int)(i - t * a.R);
        const bool write = (int64_t)slot < a.capacity;
        // the token's ids and weights eight at a time, all loads before any use
        for (int k0 = 0; k0 < K; k0 += 8) {
            int64_t ev[8];
            float wv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const bool in = k0 + j < K;
                ev[j] = in ? a.topk_idx[t * K + k0 + j] : -1;
                wv[j] = (in && a.topk_weights) ? a.topk_weights[t * K + k0 + j] : 1.0f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int k = k0 + j;
                if (k >= K) break;
                const int64_t e = ev[j];
                const bool local = e >= 0 && e < a.E && e / El == r;
                if (local) atomicAdd(&hist[e], 1);
                if (write && a.recv_topk_idx) a.recv_topk_idx[(int64_t)slot * K + k] = local ? e - (int64_t)r * El : -1;
                if (write && a.recv_topk_w) a.recv_topk_w[(int64_t)slot * K + k] = local ? wv[j] : 0.0f;
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += kRankThreads)
        if (hist[e]) atomicAdd(&a.counts[e], hist[e]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(a.done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();   // every other CTA's adds are visible before the counter said so
    for (int e = threadIdx.x; e < a.E; e += kRankThreads) {
        const int32_t c = __ldcg(&a.counts[e]);
        if (a.num_tokens_per_expert) a.num_tokens_per_expert[e] = c;
        if (a.num_recv_per_expert) a.num_recv_per_expert[e] = (c + a.A - 1) / a.A * a.A;
        a.counts[e] = 0;
    }
    if (threadIdx.x == 0) *a.done = 0;
}

}  // namespace

RankWsLayout rank_ws_layout(int T, int R, int E) {
    RankWsLayout w;
    w.expand = ws_layout(T, R, R, 1);
    const size_t n = (size_t)(T > 0 ? T : 0) * (size_t)R;
    w.scratch_w_off = w.expand.total;
    w.scratch_lexp_off = round_up(w.scratch_w_off + n * 4, 256);
    w.counts_off = round_up(w.scratch_lexp_off + n * 4, 256);
    w.done_off = round_up(w.counts_off + (size_t)E * 4, 256);
    w.total = round_up(w.done_off + 4, 256);
    return w;
}

cudaError_t launch_rank_layout(LayoutArgs la, const RankPostArgs& post, int sms, cudaStream_t s) {
    cudaError_t err = launch_layout(la, sms, s);
    if (err != cudaSuccess) return err;
    const int64_t n = (int64_t)post.T * post.R;
    int64_t grid = (n + kRankThreads - 1) / kRankThreads;
    if (grid > 2 * sms) grid = 2 * sms;
    if (grid < 1) grid = 1;
    return launch_pdl(rank_post_kernel, dim3((unsigned)grid), dim3(kRankThreads), (size_t)post.E * 4, s, false,
                      post);
}

}  // namespace ep
