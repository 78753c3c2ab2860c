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
// E' = K' = R and alignment 1, so the rows come from the layout kernel
// (per-chunk counts, one grid barrier, scan, stable slots) in its per-rank
// mode (LayoutArgs::src_idx), one kernel in all:
//   - a pair's key is computed on the fly from the token's K expert ids, and
//     the same pass counts the ids that are local to the pair's rank in a
//     shared-memory histogram of the E experts - each selected (t, k) is
//     local to exactly one reached rank, so every pair is counted once;
//   - each chunk adds its histogram to a workspace array before the grid
//     barrier; after it CTA 0 writes the plain and aligned per-expert counts
//     and zeroes the array for the next call (integer sums: the result does
//     not depend on the order of the adds);
//   - the assign phase writes token_slot [T, R], recv_src_token,
//     is_token_in_rank and each reached row's recv_topk_idx /
//     recv_topk_weights.
// This file holds the workspace layout; the kernel is layout_kernel<.., true>.
#include "ep_internal.h"

namespace ep {

RankWsLayout rank_ws_layout(int T, int R, int E) {
    RankWsLayout w;
    w.expand = ws_layout(T, R, R, 1);
    const size_t n = (size_t)(T > 0 ? T : 0) * (size_t)R;
    w.scratch_w_off = w.expand.base_total;
    w.scratch_lexp_off = round_up(w.scratch_w_off + n * 4, 256);
    w.counts_off = round_up(w.scratch_lexp_off + n * 4, 256);
    w.total = round_up(w.counts_off + (size_t)E * 4, 256);
    return w;
}

}  // namespace ep
