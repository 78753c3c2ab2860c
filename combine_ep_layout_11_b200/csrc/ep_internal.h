// Internal launch interface between the C ABI (ep_abi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep_common.cuh"

namespace ep {

struct LayoutArgs {
    const int64_t* topk_idx;
    const float* topk_weights;  // nullable
    int T, K, E, R, A;
    int C, CT;                  // chunking, chosen by launch_layout
    int64_t capacity;
    int32_t* cnt;
    int32_t* off;
    int32_t* pair_slot;
    int32_t* recv_src;
    float* recv_w;
    int32_t* recv_lexp;
    WsHeader* hdr;
    int32_t* table;
    int32_t* sup;               // [2][kSupRows][round4(E)], zero before the first call
    int32_t* padpre;
    int32_t* pad_rows;
    int32_t* stats;             // [E] running receive counts, nullable
    // Low-latency form: > 0 gives every expert a fixed slab of `slab` rows
    // (off[e] = e * slab, the rest of the slab is padding); 0: aligned counts.
    int slab;
    // Per-rank keys (ep_rank_layout): nullptr for the expand layout.  Otherwise
    // pair i = (t, r) of a [T, R] table (K = E = R here), whose key is r when
    // token t has an expert on rank r, read from src_idx [T, src_K] with src_E
    // experts; in_rank [T*R] (nullable) gets 1 / 0 per pair.
    const int64_t* src_idx;
    int src_K, src_E;
    uint8_t* in_rank;
    // Per-rank keys only, all nullable: the per-expert pair counts (plain and
    // aligned to src_A), counted through src_counts ([src_E] workspace, zero
    // between calls), and each reached row's rank-local expert ids and weights.
    const float* src_w;
    int src_A;
    int32_t* src_counts;
    int32_t* n_exp_out;
    int32_t* n_recv_out;
    int64_t* rank_topk_idx;
    float* rank_topk_w;
};

// One cooperative kernel: per-chunk counts, a grid barrier, the scans and the
// slot assignment (see ep_layout.cu).
cudaError_t launch_layout(LayoutArgs a, int sms, cudaStream_t s);

struct DispatchArgs {
    const uint8_t* x;          // token rows, row_bytes each (bf16 or e4m3)
    const float* x_scales;     // [T][nb] for e4m3 input
    uint8_t* recv;             // receive rows of the output type
    float* recv_scales;        // e4m3 output: [capacity][nb] fp32 (copy); cast: see sf_* below
    const int32_t* pair_slot;  // [T*K]; nullptr: row t goes to row t (plain cast)
    const WsHeader* hdr;       // num_pad
    const int32_t* pad_rows;
    WsHeader* status_hdr;      // status word
    int T, K, H;
    int64_t capacity;
    int nb;                    // 128-column blocks per row (H/128) when FP8 is involved
    int zero_pad;
    int64_t max_pad_rows;      // a bound on the padding rows, known on the host
    int sms;
    // scale output of the cast (EP_SF_* bits): ng scales per row (nb, or 1 per
    // row), sf_elem bytes each (4: fp32, 1: UE8M0); scale (row, g) at byte
    // (row * ng + g) * sf_elem, or (g * sf_ld + row) * sf_elem column-major
    int sf_format;
    int ng;
    int sf_elem;
    int sf_col_major;
    int64_t sf_ld;
    // Column-major scales through the staging area of an expand handle's
    // workspace (when it holds one): the cast kernel bulk-stores each token's
    // scale row to sf_stage + t * sf_stage_ld, then a second kernel writes the
    // column-major array receive row by receive row, scale (row, g) =
    // staged[recv_src[row]][g] (zero for padding rows), so that a warp's
    // stores cover consecutive rows.  nullptr: one store per scale from the
    // cast kernel.
    uint8_t* sf_stage;
    int64_t sf_stage_ld;
    const int32_t* recv_src;
    const int32_t* num_rows;   // device word: receive rows in use (expert_offset[E])
    // Regions (ep_dispatch_regions; bf16 rows): pair (t, k) with expert
    // e = topk_idx[t, k] goes to regions[e / El], row pair_slot[t, k] +
    // row_delta[e]; padding rows come from pad_list ((r << 32) | row).
    const int64_t* topk_idx;
    const int32_t* row_delta;
    uint8_t* const* regions;
    int64_t region_capacity;
    int El, R;
    const int64_t* pad_list;
    int64_t num_pad_list;
    // Copy kernel: 1 when x is known to be complete before the grid that
    // precedes the kernel has finished (ep_layout_dispatch: x is an input of
    // the same call, so the layout kernel waited for its producer); the first
    // row loads are then issued before waiting for that grid.
    int early;
};

// Fill the sf_* fields for `rows` output rows; returns false for an invalid
// format (unknown bits, UE8M0 without power-of-two rounding).
bool set_scale_format(DispatchArgs* a, int scale_format, int64_t rows);

// bf16 -> bf16 or e4m3 -> e4m3 row scatter through TMA bulk copies; with
// `regions`, bf16 rows into the regions of DispatchArgs.
cudaError_t launch_dispatch_copy(const DispatchArgs& a, int elem_bytes, cudaStream_t s, bool regions = false);
// bf16 -> e4m3 scatter with the per-128-column cast fused in.
cudaError_t launch_dispatch_cast(const DispatchArgs& a, cudaStream_t s);


struct CombineArgs {
    const uint16_t* y;         // bf16 [capacity][H]
    const int32_t* pair_slot;  // [T*K]
    const float* w;            // [T*K] or nullptr
    const uint16_t* bias0;     // bf16 [T][H] or nullptr
    const uint16_t* bias1;     // bf16 [T][H] or nullptr (only with bias0)
    uint16_t* out;             // bf16 [T][H]
    WsHeader* status;          // status word (timeouts)
    int T, K, H;
    int64_t capacity;
    int sms;
    // Regions (ep_combine_regions): the row of pair (t, k) with expert
    // e = topk_idx[t, k] is regions[e / El] row pair_slot[t, k] + row_delta[e]
    // (rows below region_capacity); y and capacity are then unused.
    const int64_t* topk_idx;
    const int32_t* row_delta;
    const uint16_t* const* regions;
    int64_t region_capacity;
    int El, R;
};

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);


cudaError_t launch_selftest_wait(WsHeader* hdr, uint64_t timeout_ns, cudaStream_t s);

// ep_layout's argument checks, then its launch on `s`.  With clear_header the
// workspace header words are zeroed on the stream first, but only once every
// check has passed: a rejected call enqueues nothing (ep_abi.cu).
int layout_call(const int64_t* topk_idx, const float* topk_weights, int T, int K, int E, int R, int A,
                int num_max_tokens_per_rank, ep_layout_t* layout, cudaStream_t s, bool clear_header);

// Per-token-per-rank layout (ep_rank_layout.cu).  Workspace: the expand-layout
// workspace of the [T, R] (token, rank) table (E' = K' = R, A = 1), scratch
// targets for the layout kernel's per-row weight and local-expert writes
// (meaningless here) and the per-expert pair counts (int32 [E], zero between
// calls).
struct RankWsLayout {
    WsLayout expand;
    size_t scratch_w_off;
    size_t scratch_lexp_off;
    size_t counts_off;
    size_t total;
};
RankWsLayout rank_ws_layout(int T, int R, int E);

}  // namespace ep
