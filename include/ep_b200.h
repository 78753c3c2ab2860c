/*
 * ep_b200.h - C ABI of the B200 (sm_100a) MoE expert-parallel dispatch /
 * combine library, DeepEP style, with R virtual ranks held in one GPU's HBM.
 *
 * The operations follow "DeepEP 测试目标 API 系统性参考" (the DeepEP test-target
 * API reference):
 *   ep_layout    §2.1 dispatch(): the routing layout V2 derives from topk_idx
 *                (-1 = unselected), expert_alignment, the expand layout
 *                (do_expand: one receive row per (token, expert) pair), the
 *                handle; §3.1: the per-expert receive counts V1 returns.
 *   ep_dispatch  §2.1 dispatch(): rows to the owning ranks' receive regions,
 *                same type as the input ((fp8, scales) stays (fp8, scales)),
 *                do_zero_padding; §4.2 math.py for the fused FP8 cast.
 *   ep_combine   §2.2 combine(): weighted reduction back to [T, hidden] bf16 in
 *                the order the handle records; §3.2: no weights = plain sum;
 *                §4.1 refs.py ordered_accumulate: one fixed order, so results
 *                are bitwise reproducible.
 *   ep_cast_fp8  §4.2 math.py per_token_cast_to_fp8, with one fp32 scale per
 *                128-column block of a token row (or the §3.3 / §2.1 scale
 *                variants: per row, power of two, UE8M0, column-major).
 *   ep_rank_layout  §2.1 dispatch() without do_expand (one receive row per
 *                token and destination rank) with §3.1's V1 layout quantities;
 *                its handle serves ep_dispatch and §3.2's unweighted combine.
 *   ep_ll_layout §3.3 low_latency_dispatch: a fixed slab of R * max_tokens
 *                receive rows per expert.
 *   ep_layout_dispatch  ep_layout and ep_dispatch in one call (§2.1: V2's
 *                dispatch() derives its layout from topk_idx).
 *   ep_source_offsets, ep_dispatch_regions, ep_combine_regions  several source
 *                groups (the NVLink intranode path of §2.1 dispatch() seen
 *                from one GPU): each group's write offsets in the layout of
 *                the whole batch, and dispatch / combine over R receive
 *                regions given as separate buffers.
 * The placement also matches the last stages of the Ascend full-mesh dispatch
 * on the "URMA" tag page (count reconciliation, prefix-sum placement, reorder).
 *
 * Conventions for every entry point
 *   - Memory: every array is allocated by the caller; the library never
 *     allocates or frees memory and keeps no state between calls outside the
 *     caller's workspace (the one exception, ep_layout_no_alloc, uses a fixed
 *     array of the library's own).  "device" means a pointer to memory of the
 *     current CUDA device.
 *   - Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 *     Every call only enqueues work on that stream and returns; results are
 *     ready when the stream reaches them.  Nothing synchronises the host except
 *     ep_get_status.
 *   - Errors: host-side argument checks return a status before anything is
 *     enqueued (EP_ERR_INVALID_ARG, EP_ERR_CAPACITY, EP_ERR_UNSUPPORTED); a
 *     failed launch returns EP_ERR_CUDA.  Problems only the device can see
 *     (a bad expert id, too many receive rows, a bounded wait that ran out) set
 *     bits in the layout's device status word, read by ep_get_status; the
 *     kernels then skip the affected writes, never write out of bounds, never
 *     trap and never spin without limit.
 *   - Precision: integer and byte work is exact; combine accumulates in fp32 in
 *     ascending k with separately rounded multiply and add, then rounds to bf16
 *     to nearest even, so results are bitwise reproducible run to run and
 *     independent of how many tokens share a call.
 *
 * Layout of the receive buffers (expand layout): expert e's rows are
 * [off[e], off[e] + cnt[e]) holding its (token, k) pairs in token-major,
 * k-minor order, followed by align(cnt[e], A) - cnt[e] padding rows;
 * off[e] = sum over e' < e of align(cnt[e'], A).  Virtual rank r owns experts
 * [r*E/R, (r+1)*E/R), so its region is [off[r*E/R], off[(r+1)*E/R]) and rows
 * are ordered by (destination rank, local expert, source token).  Token t
 * belongs to source rank t / (T/R).
 */
#ifndef EP_B200_H
#define EP_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EP_B200_VERSION 5

/* Host return codes. */
#define EP_OK 0
#define EP_ERR_INVALID_ARG 1   /* null / misaligned pointer, bad size or shape   */
#define EP_ERR_CAPACITY 2      /* receive rows or tokens per rank above a limit  */
#define EP_ERR_BAD_EXPERT 3    /* (device) an expert id outside [-1, E)          */
#define EP_ERR_TIMEOUT 4       /* (device) a bounded wait ran out                */
#define EP_ERR_CUDA 5          /* a CUDA call failed                             */
#define EP_ERR_UNSUPPORTED 6   /* valid arguments outside the supported range    */

/* Bits of the device status word (see ep_get_status). */
#define EP_DEV_BAD_EXPERT 0x1u
#define EP_DEV_CAPACITY 0x2u
#define EP_DEV_TIMEOUT 0x4u

/* Element types of token rows. */
#define EP_DTYPE_BF16 0
#define EP_DTYPE_FP8_E4M3 1

/*
 * Scale formats of the FP8 cast (bits of `scale_format`; 0 = one fp32 scale
 * per 128-column block, row-major [rows, H/128], the default).
 *   EP_SF_PER_ROW    one scale per row, [rows] (§4.2 per_token_cast_to_fp8:
 *                    amax over the whole row)
 *   EP_SF_POW2       each scale rounded up to the smallest power of two not
 *                    below amax / 448 (§3.3 round_scale), so no value saturates
 *   EP_SF_UE8M0      scales stored as one UE8M0 byte each, value 2^(b - 127)
 *                    (§3.3 use_ue8m0); needs EP_SF_POW2
 *   EP_SF_COL_MAJOR  TMA-aligned column-major scales (§2.1
 *                    use_tma_aligned_col_major_sf): scale (row, g) at element
 *                    g * ld + row, ld = rows rounded up to a multiple of 16
 *                    bytes of elements (4 fp32 or 16 UE8M0 entries); entries
 *                    [rows, ld) of each column are not written
 * ep_scale_bytes gives the size of the scale array for a row count.
 */
#define EP_SF_PER_ROW 0x1
#define EP_SF_POW2 0x2
#define EP_SF_UE8M0 0x4
#define EP_SF_COL_MAJOR 0x8

/* Supported ranges (EP_ERR_UNSUPPORTED beyond them). */
#define EP_MAX_TOPK 32
#define EP_MAX_EXPERTS 4096

/*
 * The handle ("handle" / EPHandle in §2.1 and §2.2): the routing layout of one
 * batch, reused as is by ep_dispatch and ep_combine (a cached layout).
 *
 * The caller fills the pointer fields and `capacity` and `workspace_bytes`
 * before ep_layout; ep_layout fills the shape fields.  All arrays are device
 * memory owned by the caller and must stay alive while work that uses the
 * handle is pending.
 *   num_recv_tokens_per_expert [E]     int32  cnt[e]: pairs that chose expert e
 *   expert_offset              [E+1]   int32  aligned exclusive prefix of cnt;
 *                                             expert_offset[E] = rows used (Np)
 *   pair_slot                  [T*K]   int32  receive row of pair (t, k), -1 if
 *                                             topk_idx[t, k] == -1
 *   recv_src_token             [capacity] int32  source token of each row, -1 on
 *                                             padding rows
 *   recv_weight                [capacity] fp32   topk weight of each row (1 when
 *                                             ep_layout got no weights), 0 on padding
 *   recv_local_expert          [capacity] int32  expert id local to the
 *                                             destination rank (e mod E/R), -1 on padding
 *   workspace                  ep_workspace_bytes() bytes, 256-byte aligned,
 *                              zero-filled by the caller before its first use
 *                              (every later ep_layout leaves it ready again;
 *                              after a call reported EP_ERR_TIMEOUT, zero it
 *                              again before the next one);
 *                              holds the device status word and scan scratch,
 *                              and last a staging area of 512 bytes per token
 *                              for ep_dispatch's column-major FP8 scales.  A
 *                              workspace of ep_workspace_bytes() - 512 * T
 *                              bytes (the layout's own part) is accepted too:
 *                              ep_dispatch then stores column-major scales one
 *                              by one, which is slower (see ep_dispatch).
 *                              One workspace serves one call at a time.
 *   cumulative_local_expert_recv_stats [E] int32 or NULL (§2.1 dispatch() and
 *                              §3.3 low_latency_dispatch() argument of that
 *                              name): a running per-expert receive count owned
 *                              by the caller; when set, every ep_layout adds
 *                              cnt[e] to entry e (virtual rank r's local
 *                              experts are entries [r*E/R, (r+1)*E/R)).  Not
 *                              cleared by the library.
 * Rows at and beyond expert_offset[E] are not written by ep_layout.
 */
typedef struct ep_layout_t {
    int32_t* num_recv_tokens_per_expert;
    int32_t* expert_offset;
    int32_t* pair_slot;
    int32_t* recv_src_token;
    float* recv_weight;
    int32_t* recv_local_expert;
    void* workspace;
    uint64_t workspace_bytes;
    int64_t capacity;
    /* filled by ep_layout */
    int32_t num_tokens;
    int32_t num_topk;
    int32_t num_experts;
    int32_t num_ranks;
    int32_t expert_alignment;
    int32_t num_max_tokens_per_rank;
    uint32_t magic;
    uint32_t kind;                                 /* EP_LAYOUT_*, set by the layout call */
    int32_t* cumulative_local_expert_recv_stats;   /* optional, see above */
} ep_layout_t;

/* Receive forms of a handle (its `kind` field). */
#define EP_LAYOUT_EXPAND 0     /* ep_layout: one row per selected (token, k) pair */
#define EP_LAYOUT_PER_RANK 1   /* ep_rank_layout: one row per (token, rank) reached */
#define EP_LAYOUT_LL_SLAB 2    /* ep_ll_layout: a fixed slab of rows per expert */

/* Bytes of workspace for these sizes: the layout's own part plus the
 * 512-byte-per-token scale staging area (a pure host function). */
size_t ep_workspace_bytes(int num_tokens, int num_topk, int num_experts, int expert_alignment);

/* Worst-case receive rows: T*K + E*(A-1); a capacity of this many rows can
 * never overflow (a pure host function). */
int64_t ep_capacity_rows(int num_tokens, int num_topk, int num_experts, int expert_alignment);

/* Bytes of the scale array of `rows` FP8 rows of `hidden` columns in
 * `scale_format` (EP_SF_* bits); -1 if the arguments are invalid (rows < 0,
 * hidden not a positive multiple of 128, unknown bits, UE8M0 without
 * EP_SF_POW2).  A pure host function.  For ep_dispatch, rows = the handle's
 * capacity; for ep_cast_fp8, rows = num_tokens. */
int64_t ep_scale_bytes(int64_t rows, int hidden, int scale_format);

/*
 * Routing layout (§2.1: V2 derives the layout from topk_idx; §3.1: the
 * per-expert receive counts).
 *   topk_idx      device int64 [T, K] row-major; -1 = unselected; NULL only if T == 0
 *   topk_weights  device fp32 [T, K] or NULL (then recv_weight = 1 on real rows)
 *   num_tokens T >= 0 with T % R == 0; num_topk 1 <= K <= EP_MAX_TOPK;
 *   num_experts 1 <= E <= EP_MAX_EXPERTS with E % R == 0; num_ranks R >= 1;
 *   expert_alignment A >= 1;
 *   num_max_tokens_per_rank  0 = no limit; else T/R must not exceed it
 *                             (EP_ERR_CAPACITY), as §3.3 requires of the
 *                             per-rank dispatch budget;
 *   layout        in: pointers, capacity, workspace; out: shape fields.
 * Device-side: an id outside [-1, E) sets EP_DEV_BAD_EXPERT and is treated as
 * -1; more than `capacity` rows sets EP_DEV_CAPACITY and rows past capacity are
 * not written.  Replaces the device status word with the flags of this call.
 * Deterministic: the same input gives the same bytes on every call.
 */
int ep_layout(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
              int num_experts, int num_ranks, int expert_alignment, int num_max_tokens_per_rank,
              ep_layout_t* layout, void* stream);

/*
 * Per-token-per-rank layout: the receive form of §2.1 dispatch() without
 * do_expand, with the V1 layout quantities of §3.1 (num_tokens_per_rank,
 * is_token_in_rank, num_tokens_per_expert) and V1's receive outputs
 * (recv_topk_idx, recv_topk_weights, num_recv_tokens_per_expert_list).
 * Token t reaches rank r when some topk_idx[t, k] is one of r's experts
 * [r*E/R, (r+1)*E/R); it then gets one receive row in r's region.  Rows of
 * rank r are [off[r], off[r+1]) in ascending token order (source rank, then
 * token).  No padding rows.
 *   topk_idx, topk_weights, T, K, E, R as for ep_layout; 1 <= R <= 32
 *   expert_alignment A >= 1: only for num_recv_tokens_per_expert
 *   is_token_in_rank            device uint8 [T, R] or NULL: 1 / 0
 *   num_tokens_per_expert       device int32 [E] or NULL: pairs per expert
 *   num_recv_tokens_per_expert  device int32 [E] or NULL: align(that, A)
 *   recv_topk_idx               device int64 [capacity, K] or NULL: for row
 *                               (t, r), topk_idx[t, k] - r*E/R where that
 *                               expert is on r, else -1
 *   recv_topk_weights           device fp32 [capacity, K] or NULL: the topk
 *                               weight (1 without weights) on those entries, else 0
 *   layout  in: the handle's pointers, capacity (T*R rows never overflow),
 *           workspace of ep_rank_workspace_bytes(T, R, E) bytes (zero-filled
 *           before first use, like ep_layout's);
 *           the fields then mean: num_recv_tokens_per_expert = num_tokens_per_rank
 *           [R], expert_offset = rank offsets [R+1] (off[R] = rows used),
 *           pair_slot = token_slot [T, R] (row of (t, r) or -1),
 *           recv_src_token [capacity]; recv_weight and recv_local_expert are
 *           not used and may be NULL.
 *           out: kind = EP_LAYOUT_PER_RANK, num_tokens = T, and num_topk =
 *           num_experts = num_ranks = R (each token has R possible
 *           destinations), expert_alignment = 1.
 * The handle works with ep_dispatch (rows per (token, rank)) and ep_combine
 * (§3.2 V1: topk_weights must be NULL; out[t] = the plain sum over the ranks
 * the token reached, in ascending rank order, plus the biases).  Device-side
 * errors as for ep_layout.  One kernel; its workspace holds per-expert
 * counters that the call leaves at zero (zero the workspace again after an
 * EP_ERR_TIMEOUT, and before reusing a workspace that served another layout
 * call).
 */
size_t ep_rank_workspace_bytes(int num_tokens, int num_ranks, int num_experts);
int ep_rank_layout(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
                   int num_experts, int num_ranks, int expert_alignment, uint8_t* is_token_in_rank,
                   int32_t* num_tokens_per_expert, int32_t* num_recv_tokens_per_expert, int64_t* recv_topk_idx,
                   float* recv_topk_weights, ep_layout_t* layout, void* stream);

/*
 * Low-latency fixed-slab layout (§3.3 low_latency_dispatch: every rank has
 * the same num_max_dispatch_tokens_per_rank M; a rank receives
 * [E/R, R*M, H]).  With S = R*M, expert e owns receive rows [e*S, (e+1)*S):
 * its pairs first, in token-major, k-minor order (as ep_layout), then padding
 * rows up to the end of the slab.  Arguments and results as for ep_layout with
 * expert_alignment 1 and num_max_tokens_per_rank M (T/R > M is
 * EP_ERR_CAPACITY), except that expert_offset[e] = e*S, the receive buffers
 * need capacity >= E*S rows, and the workspace is
 * ep_ll_workspace_bytes(T, K, E, R, M) bytes.  An expert with more than S
 * pairs (only possible when a token repeats an expert) sets EP_DEV_CAPACITY;
 * its pairs past the slab get pair_slot -1 and are not written.  Sets kind =
 * EP_LAYOUT_LL_SLAB; the handle serves ep_dispatch (do_zero_padding zeroes
 * the unused slab rows) and ep_combine (weighted, as §3.4's low-latency
 * combine).  T = 0 is allowed: every slab row is then padding.
 */
size_t ep_ll_workspace_bytes(int num_tokens, int num_topk, int num_experts, int num_ranks,
                             int num_max_dispatch_tokens_per_rank);
int ep_ll_layout(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
                 int num_experts, int num_ranks, int num_max_dispatch_tokens_per_rank, ep_layout_t* layout,
                 void* stream);

/*
 * Dispatch (§2.1): for every selected pair (t, k), receive row
 * pair_slot[t, k] := token row t.
 *   x            device, 16-byte aligned: bf16 [T, H] if x_dtype == EP_DTYPE_BF16,
 *                e4m3 bytes [T, H] if x_dtype == EP_DTYPE_FP8_E4M3
 *   x_scales     device fp32 [T, H/128] for FP8 input, else ignored
 *   hidden H     > 0; H % 8 == 0 for bf16, H % 128 == 0 whenever FP8 is involved
 *   cast_to_fp8  1: bf16 input is cast on the way (§4.2, the same bytes
 *                ep_cast_fp8 writes for that scale_format) and the receive rows
 *                are FP8
 *   scale_format EP_SF_* bits of the cast's scales (0: fp32 per 128-column
 *                block, row-major); must be 0 unless cast_to_fp8
 *   do_zero_padding  1: the alignment padding rows (and their scales) are zeroed;
 *                0: they are left untouched
 *   recv_x       device, 16-byte aligned: [capacity, H] of the output type
 *   recv_scales  device, 16-byte aligned, when the output is FP8: fp32
 *                [capacity, H/128] for FP8 input, else ep_scale_bytes(capacity,
 *                H, scale_format) bytes in that format; ignored for bf16 output
 * Rows that no pair selects and that are not padding are left untouched.
 * One kernel, except for column-major per-block scales (EP_SF_COL_MAJOR
 * without EP_SF_PER_ROW) on an ep_layout / ep_layout_no_alloc handle whose
 * workspace holds the staging area: the cast kernel then stages each token's
 * scale row once, and a second kernel writes the column-major array receive
 * row by receive row, so that neighbouring threads store neighbouring rows.
 * Otherwise each of the K * H/128 scales of a token is one store.  Both write
 * the same bytes.
 */
int ep_dispatch(const ep_layout_t* layout, const void* x, int x_dtype, const float* x_scales,
                int hidden, int cast_to_fp8, int scale_format, int do_zero_padding, void* recv_x,
                void* recv_scales, void* stream);

/*
 * Layout and dispatch in one call, as V2's dispatch() derives its layout from
 * topk_idx itself (§2.1; §3.1's V1/V2 comparison).  Arguments and results are
 * exactly those of ep_layout followed by ep_dispatch on the same handle; the
 * handle is then reusable by ep_combine and by further ep_dispatch calls.  Two
 * kernels: the layout, then the dispatch, launched behind it with programmatic
 * dependent launch.  x is an input of this call, so x must be complete when
 * the call is made (as for every input).  For bf16 or e4m3 rows, the dispatch
 * kernel may then load its first rows of x while the layout kernel still
 * runs.
 */
int ep_layout_dispatch(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
                       int num_experts, int num_ranks, int expert_alignment, int num_max_tokens_per_rank,
                       ep_layout_t* layout, const void* x, int x_dtype, const float* x_scales, int hidden,
                       int cast_to_fp8, int scale_format, int do_zero_padding, void* recv_x,
                       void* recv_scales, void* stream);

/*
 * Combine (§2.2 weighted, with 0, 1 or 2 output biases; §3.2 unweighted when
 * topk_weights is NULL; §4.1 ordered accumulation and its initial value):
 *   out[t] = bf16_rne( init[t] + sum over k = 0..K-1 with pair_slot[t, k] >= 0
 *                      of w[t, k] * float(y[pair_slot[t, k]]) )
 * accumulated in fp32 in ascending k, each step one rounded product and one
 * rounded sum.  init[t] is +0 without bias, float(bias0[t]) with one bias, and
 * the rounded sum float(bias0[t]) + float(bias1[t]) with two.  A token with no
 * selected entry gives bf16(init[t]).
 *   y            device bf16 [capacity, H], 16-byte aligned: expert outputs in
 *                receive order; padding rows are never read
 *   hidden H     > 0, H % 8 == 0
 *   topk_weights device fp32 [T, K] or NULL (unit weights); must be NULL for
 *                a per-rank handle (EP_LAYOUT_PER_RANK: K = R, a plain sum)
 *   bias0, bias1 device bf16 [T, H], 16-byte aligned, or NULL; bias1 without
 *                bias0 is EP_ERR_INVALID_ARG
 *   out          device bf16 [T, H], 16-byte aligned; may not alias y, and may
 *                alias a bias only if it is that very array
 */
int ep_combine(const ep_layout_t* layout, const void* y, int hidden, const float* topk_weights,
               const void* bias0, const void* bias1, void* out, void* stream);

/*
 * FP8 cast (§4.2 per_token_cast_to_fp8; by default with 128-column blocks):
 * for token t and group g (a 128-column block, or the whole row with
 * EP_SF_PER_ROW), amax = max |x| over the group (clamped below at 1e-4),
 * s = amax / 448 (fp32 division), with EP_SF_POW2 rounded up to a power of two,
 * q = e4m3(x / s) with an fp32 division, round-to-nearest-even and saturation
 * to +-448; scale (t, g) = s, stored as fp32 or as a UE8M0 byte, row-major or
 * column-major as scale_format says.  Dequantisation is float(q) * s.
 *   x             device bf16 [T, H], 16-byte aligned, H % 128 == 0, H <= 16384
 *   scale_format  EP_SF_* bits
 *   x_fp8         device e4m3 [T, H], 16-byte aligned
 *   scales        device, 16-byte aligned, ep_scale_bytes(T, H, scale_format) bytes
 */
int ep_cast_fp8(const void* x, int num_tokens, int hidden, int scale_format, void* x_fp8, void* scales,
                void* stream);

/*
 * Expert parallelism over G source groups (one per GPU in a multi-GPU run),
 * §2.1 dispatch() / §2.2 combine() across ranks: each group g runs ep_layout
 * on its own tokens with expert_alignment 1; the groups exchange their
 * per-expert counts (an all-gather of num_recv_tokens_per_expert); then every
 * group writes its rows straight into the destination ranks' receive regions
 * (separate buffers, one per rank: on several GPUs, peer pointers).  The
 * regions then hold exactly the rows one ep_layout over the concatenated batch
 * (group 0's tokens, then group 1's, ...) with alignment A would give, region r
 * being that layout's rows [off[r*E/R], off[(r+1)*E/R]).
 *
 * ep_source_offsets (a pure host function): from counts, host int32 [G][E]
 * (row g = group g's num_recv_tokens_per_expert), for group `group`:
 *   row_delta    host int32 [E] out: group `group`'s pair (t, k) with expert e
 *                goes to region e / (E/R), row pair_slot[t, k] + row_delta[e]
 *                (pair_slot of its own alignment-1 ep_layout)
 *   region_rows  host int64 [R] out or NULL: rows region r holds, padding included
 *   pad_list     host int64 [pad_list_capacity] out or NULL: every padding row
 *                of every region, (r << 32) | row, in ascending order
 *   num_pad      out (required with pad_list): the number of padding rows
 * Returns EP_ERR_CAPACITY (after filling what fits) when pad_list is too short,
 * EP_ERR_UNSUPPORTED when the rows exceed 2^31 - 1.
 */
int ep_source_offsets(const int32_t* counts, int num_groups, int num_experts, int num_ranks, int expert_alignment,
                      int group, int32_t* row_delta, int64_t* region_rows, int64_t* pad_list,
                      int64_t pad_list_capacity, int64_t* num_pad);

/*
 * Dispatch of one source group's bf16 rows into the regions (§2.1).
 *   layout         the group's handle from ep_layout with expert_alignment 1
 *                  (EP_ERR_INVALID_ARG otherwise); its num_ranks R and
 *                  num_experts E give the regions' experts (E/R each)
 *   topk_idx       device int64 [T, K]: the routing that layout was made from
 *   row_delta      device int32 [E]: ep_source_offsets' row_delta for this group
 *   regions        device array of R device pointers, 16-byte aligned: region r's
 *                  bf16 rows [region_capacity, H] (on several GPUs, peer memory
 *                  mapped into this process)
 *   region_capacity rows each region holds (at least ep_source_offsets'
 *                  region_rows); a row at or past it is not written
 *   x              device bf16 [T, H], 16-byte aligned; H % 8 == 0
 *   pad_list, num_pad  device int64 [num_pad] ((r << 32) | row) or NULL / 0:
 *                  the padding rows this call zero-fills (give them to one call,
 *                  e.g. the last group's)
 * Rows go out as TMA bulk stores from shared memory: plain stores, no
 * multicast.  No kernel reads a region.  The handle's workspace serves the
 * work tickets, so one call per handle at a time.
 */
int ep_dispatch_regions(const ep_layout_t* layout, const int64_t* topk_idx, const int32_t* row_delta,
                        void* const* regions, int64_t region_capacity, const void* x, int hidden,
                        const int64_t* pad_list, int64_t num_pad, void* stream);

/*
 * Combine of one source group's tokens from the regions (§2.2): as ep_combine,
 * with the row of pair (t, k) read from region topk_idx[t, k] / (E/R), row
 * pair_slot[t, k] + row_delta[topk_idx[t, k]] (rows at or past
 * region_capacity are skipped).  Arguments as for ep_dispatch_regions and
 * ep_combine (no biases); regions hold the expert outputs, bf16.
 */
int ep_combine_regions(const ep_layout_t* layout, const int64_t* topk_idx, const int32_t* row_delta,
                       const void* const* regions, int64_t region_capacity, int hidden, const float* topk_weights,
                       void* out, void* stream);

/* Size of the library-owned workspace behind ep_layout_no_alloc. */
#define EP_NO_ALLOC_SCRATCH_BYTES ((size_t)4 << 20)

/*
 * ep_layout for callers that cannot allocate device memory themselves: a plain
 * C host program that links this library but owns no device allocator, or a
 * process whose device memory is entirely reserved by another framework's pool
 * that it cannot extend, so it has no buffer to offer as the workspace.  (The
 * pages have no counterpart; this is an addition of this library.)
 *
 * Same arguments, checks and results as ep_layout, except that layout->workspace
 * and layout->workspace_bytes are ignored on entry: the call uses a fixed 4 MiB
 * array in the library's own device memory (EP_NO_ALLOC_SCRATCH_BYTES), and on
 * success stores that array's device address in the handle, so ep_dispatch,
 * ep_combine and ep_get_status work on the handle as usual.  The caller still
 * provides every input and output array.  It calls no cudaMalloc or cudaFree.
 *
 *   - Sizes whose layout part (ep_workspace_bytes - 512 * T) exceeds 4 MiB
 *     are rejected with EP_ERR_UNSUPPORTED, and every other argument error is
 *     returned as ep_layout returns it; a rejected call enqueues nothing and
 *     leaves the array as it was.  The scale staging area is used only when
 *     the whole of ep_workspace_bytes fits in the array.
 *   - Every GPU that loads the library holds the 4 MiB until the process exits.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (each accepted call clears the words that must start at zero).
 *     Calls whose work overlaps on the GPU - from other streams or threads, or
 *     a dispatch or combine of an older handle still pending - race on it.
 *   - Each accepted call also replaces what every earlier no-alloc handle on
 *     that device reads from the array: the list of padding rows, their
 *     number and the device status word.  After a later ep_layout_no_alloc,
 *     an older no-alloc handle is still valid for ep_dispatch with
 *     do_zero_padding = 0 and for ep_combine (their arrays are the caller's),
 *     but ep_dispatch with do_zero_padding = 1 would zero the later call's
 *     padding rows and ep_get_status would report the later call's flags.
 *     Use only the most recent no-alloc handle for those two.
 *   - The first call on a device looks up the array's device address with that
 *     device current (cudaGetSymbolAddress) and caches it; make that first call
 *     before any stream capture.
 */
int ep_layout_no_alloc(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
                       int num_experts, int num_ranks, int expert_alignment, int num_max_tokens_per_rank,
                       ep_layout_t* layout, void* stream);

/*
 * Synchronises `stream`, then reads the layout's device status word into
 * *device_flags (EP_DEV_* bits, 0 = no device-side error since the last
 * ep_layout on this handle).  Returns EP_OK when the word is 0, else
 * EP_ERR_TIMEOUT, EP_ERR_BAD_EXPERT or EP_ERR_CAPACITY (in that priority), or
 * EP_ERR_CUDA if the synchronisation or the read failed.
 */
int ep_get_status(const ep_layout_t* layout, void* stream, uint32_t* device_flags);

/*
 * Self-test of the bounded wait every kernel uses: launches one CTA that waits
 * on a shared-memory barrier nothing will complete, with a limit of
 * `timeout_ns` (at most 10^9), sets EP_DEV_TIMEOUT in the layout's status word
 * and returns.  Lets a test check on a GPU that a wait which runs out reports an
 * error instead of hanging.
 */
int ep_selftest_bounded_wait(const ep_layout_t* layout, uint64_t timeout_ns, void* stream);

/* Static description of a status code. */
const char* ep_status_string(int status);

/* EP_B200_VERSION of the built library. */
int ep_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_H */
