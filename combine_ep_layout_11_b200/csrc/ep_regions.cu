// Expert parallelism over several source groups (GPUs): the receive regions of
// the R destination ranks as separate buffers, filled by several source groups
// ("DeepEP 测试目标 API 系统性参考" §2.1 dispatch(): every rank sends its tokens'
// rows to the ranks owning their experts, over NVLink inside a node; §2.2
// combine(): the rows come back and are reduced at the source).
//
// The receive order is that of one layout over the concatenated batch (the
// tokens of group 0, then group 1, ...): expert e's rows are its pairs in
// (source group, token, k) order, then its alignment padding, and region r
// holds experts [r*E/R, (r+1)*E/R).  So group g's pair (t, k) with expert e
// lands at region row
//     off[e] - off[r*El] + sum_{g' < g} cnt[g'][e] + (pair_slot[t, k] - off1_g[e])
// where off is the aligned prefix of the summed counts, cnt[g'][e] the pairs of
// group g' (what an all-gather of every group's ep_layout counts delivers) and
// pair_slot / off1_g come from group g's own ep_layout with alignment 1.  Every
// term but pair_slot depends on e alone: row_delta[e].
#include <limits.h>

#include <vector>

#include "ep_internal.h"

extern "C" {

int ep_source_offsets(const int32_t* counts, int num_groups, int num_experts, int num_ranks, int expert_alignment,
                      int group, int32_t* row_delta, int64_t* region_rows, int64_t* pad_list,
                      int64_t pad_list_capacity, int64_t* num_pad) {
    const int G = num_groups, E = num_experts, R = num_ranks, A = expert_alignment;
    if (!counts || !row_delta || G < 1 || E < 1 || R < 1 || A < 1 || E % R != 0 || group < 0 || group >= G)
        return EP_ERR_INVALID_ARG;
    if (E > EP_MAX_EXPERTS) return EP_ERR_UNSUPPORTED;
    if (pad_list_capacity < 0 || (pad_list && !num_pad)) return EP_ERR_INVALID_ARG;
    const int El = E / R;
    std::vector<int64_t> tot(E, 0), before(E, 0), off(E + 1, 0);
    for (int g = 0; g < G; ++g) {
        for (int e = 0; e < E; ++e) {
            const int32_t c = counts[(size_t)g * E + e];
            if (c < 0) return EP_ERR_INVALID_ARG;
            tot[e] += c;
            if (g < group) before[e] += c;
        }
    }
    for (int e = 0; e < E; ++e) off[e + 1] = off[e] + (tot[e] + A - 1) / A * A;
    if (off[E] > INT_MAX) return EP_ERR_UNSUPPORTED;
    // group `group`'s own alignment-1 layout: its pairs of expert e start at off1
    int64_t off1 = 0;
    for (int e = 0; e < E; ++e) {
        const int64_t base = off[(e / El) * El];
        row_delta[e] = (int32_t)(off[e] - base + before[e] - off1);
        off1 += counts[(size_t)group * E + e];
    }
    if (region_rows)
        for (int r = 0; r < R; ++r) region_rows[r] = off[(r + 1) * El] - off[r * El];
    int64_t n = 0;
    for (int e = 0; e < E; ++e) {
        const int r = e / El;
        const int64_t base = off[r * El];
        for (int64_t row = off[e] + tot[e]; row < off[e + 1]; ++row, ++n)
            if (pad_list && n < pad_list_capacity) pad_list[n] = ((int64_t)r << 32) | (row - base);
    }
    if (num_pad) *num_pad = n;
    if (pad_list && n > pad_list_capacity) return EP_ERR_CAPACITY;
    return EP_OK;
}

}  // extern "C"
