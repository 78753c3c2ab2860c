// extern "C" entry points declared in include/ep_b200.h: host-side argument
// checks, then kernel launches on the caller's stream.  No allocation, no
// state kept between calls, no host synchronisation except ep_get_status.
#include <limits.h>

#include "ep_internal.h"

namespace {

constexpr uint32_t kLayoutMagic = 0x45504c31u;   // set by ep_layout on a filled handle

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int device_sms(int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return EP_ERR_CUDA;
    return EP_OK;
}

int check_handle(const ep_layout_t* L) {
    if (!L || L->magic != kLayoutMagic || !L->workspace || !L->pair_slot) return EP_ERR_INVALID_ARG;
    return EP_OK;
}

ep::WsHeader* header(const ep_layout_t* L) { return reinterpret_cast<ep::WsHeader*>(L->workspace); }

// Argument checks of ep_layout; on success fills the handle's shape fields and
// the kernel arguments (chunking is chosen at launch).
int prepare_layout(const int64_t* topk_idx, const float* topk_weights, int T, int K, int E, int R, int A,
                   int num_max_tokens_per_rank, ep_layout_t* layout, ep::LayoutArgs* a) {
    if (!layout) return EP_ERR_INVALID_ARG;
    if (T < 0 || K < 1 || E < 1 || R < 1 || A < 1 || num_max_tokens_per_rank < 0) return EP_ERR_INVALID_ARG;
    if (K > EP_MAX_TOPK || E > EP_MAX_EXPERTS) return EP_ERR_UNSUPPORTED;
    if (E % R != 0 || T % R != 0) return EP_ERR_INVALID_ARG;
    if ((int64_t)T * K + (int64_t)E * (A - 1) > INT_MAX) return EP_ERR_UNSUPPORTED;
    if (layout->capacity < 0) return EP_ERR_INVALID_ARG;
    if (layout->capacity > INT_MAX) return EP_ERR_UNSUPPORTED;
    if (num_max_tokens_per_rank > 0 && T / R > num_max_tokens_per_rank) return EP_ERR_CAPACITY;
    if ((T > 0 && !topk_idx) || !layout->num_recv_tokens_per_expert || !layout->expert_offset ||
        !layout->pair_slot || !layout->recv_src_token || !layout->recv_weight || !layout->recv_local_expert ||
        !layout->workspace)
        return EP_ERR_INVALID_ARG;
    if (!aligned(topk_idx, 8) || !aligned(topk_weights, 4) || !aligned(layout->num_recv_tokens_per_expert, 4) ||
        !aligned(layout->expert_offset, 4) || !aligned(layout->pair_slot, 4) ||
        !aligned(layout->recv_src_token, 4) || !aligned(layout->recv_weight, 4) ||
        !aligned(layout->recv_local_expert, 4) || !aligned(layout->workspace, 256) ||
        !aligned(layout->cumulative_local_expert_recv_stats, 4))
        return EP_ERR_INVALID_ARG;
    // the layout's own part is the minimum; the scale staging area behind it
    // is optional (see prepare_dispatch)
    const ep::WsLayout ws = ep::ws_layout(T, K, E, A);
    if (layout->workspace_bytes < ws.base_total) return EP_ERR_INVALID_ARG;

    layout->num_tokens = T;
    layout->num_topk = K;
    layout->num_experts = E;
    layout->num_ranks = R;
    layout->expert_alignment = A;
    layout->num_max_tokens_per_rank = num_max_tokens_per_rank;
    layout->magic = kLayoutMagic;
    layout->kind = EP_LAYOUT_EXPAND;

    uint8_t* wsb = reinterpret_cast<uint8_t*>(layout->workspace);
    a->topk_idx = topk_idx;
    a->topk_weights = topk_weights;
    a->T = T; a->K = K; a->E = E; a->R = R; a->A = A;
    a->C = 0;
    a->CT = 0;
    a->capacity = layout->capacity;
    a->cnt = layout->num_recv_tokens_per_expert;
    a->off = layout->expert_offset;
    a->pair_slot = layout->pair_slot;
    a->recv_src = layout->recv_src_token;
    a->recv_w = layout->recv_weight;
    a->recv_lexp = layout->recv_local_expert;
    a->hdr = reinterpret_cast<ep::WsHeader*>(wsb);
    a->table = reinterpret_cast<int32_t*>(wsb + ws.table_off);
    a->sup = reinterpret_cast<int32_t*>(wsb + ws.sup_off);
    a->padpre = reinterpret_cast<int32_t*>(wsb + ws.padpre_off);
    a->pad_rows = reinterpret_cast<int32_t*>(wsb + ws.padrows_off);
    a->stats = layout->cumulative_local_expert_recv_stats;
    a->slab = 0;
    a->src_idx = nullptr;
    a->src_K = 0;
    a->src_E = 0;
    a->in_rank = nullptr;
    a->src_w = nullptr;
    a->src_A = 1;
    a->src_counts = nullptr;
    a->n_exp_out = nullptr;
    a->n_recv_out = nullptr;
    a->rank_topk_idx = nullptr;
    a->rank_topk_w = nullptr;
    return EP_OK;
}

// A layout of zero tokens: no kernels, just zero counts and offsets.
int empty_layout(ep_layout_t* layout, cudaStream_t s) {
    if (cudaMemsetAsync(layout->workspace, 0, ep::kHeaderClearBytes, s) != cudaSuccess ||
        cudaMemsetAsync(layout->num_recv_tokens_per_expert, 0, (size_t)layout->num_experts * 4, s) != cudaSuccess ||
        cudaMemsetAsync(layout->expert_offset, 0, (size_t)(layout->num_experts + 1) * 4, s) != cudaSuccess)
        return EP_ERR_CUDA;
    return EP_OK;
}

// Argument checks of ep_dispatch against a filled handle; fills the kernel arguments.
int prepare_dispatch(const ep_layout_t* layout, const void* x, int x_dtype, const float* x_scales, int H,
                     int cast_to_fp8, int scale_format, int do_zero_padding, void* recv_x, void* recv_scales,
                     ep::DispatchArgs* a, int* elem_bytes) {
    int rc = check_handle(layout);
    if (rc != EP_OK) return rc;
    const int T = layout->num_tokens;
    if (H <= 0 || (x_dtype != EP_DTYPE_BF16 && x_dtype != EP_DTYPE_FP8_E4M3)) return EP_ERR_INVALID_ARG;
    if (cast_to_fp8 && x_dtype != EP_DTYPE_BF16) return EP_ERR_INVALID_ARG;
    if (scale_format != 0 && !cast_to_fp8) return EP_ERR_INVALID_ARG;
    const bool fp8_in = x_dtype == EP_DTYPE_FP8_E4M3;
    const bool fp8_out = fp8_in || cast_to_fp8;
    if (H % 8 != 0 || (fp8_out && H % 128 != 0)) return EP_ERR_INVALID_ARG;
    if ((T > 0 && !x) || !recv_x || (fp8_out && !recv_scales) || (fp8_in && T > 0 && !x_scales))
        return EP_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(recv_x, 16) || !aligned(x_scales, 4) || !aligned(recv_scales, 16))
        return EP_ERR_INVALID_ARG;
    if (cast_to_fp8 && H > 16384) return EP_ERR_UNSUPPORTED;

    const uint8_t* wsb = reinterpret_cast<const uint8_t*>(layout->workspace);
    const ep::WsLayout ws = ep::ws_layout(T, layout->num_topk, layout->num_experts, layout->expert_alignment);
    a->x = reinterpret_cast<const uint8_t*>(x);
    a->x_scales = fp8_in ? x_scales : nullptr;
    a->recv = reinterpret_cast<uint8_t*>(recv_x);
    a->recv_scales = fp8_out ? reinterpret_cast<float*>(recv_scales) : nullptr;
    a->pair_slot = layout->pair_slot;
    a->hdr = reinterpret_cast<const ep::WsHeader*>(wsb);
    a->pad_rows = reinterpret_cast<const int32_t*>(wsb + ws.padrows_off);
    a->status_hdr = header(layout);
    a->T = T;
    a->K = layout->num_topk;
    a->H = H;
    a->capacity = layout->capacity;
    a->nb = fp8_out ? H / 128 : 0;
    a->zero_pad = do_zero_padding ? 1 : 0;
    // padding rows: E*(A-1) at most for the expand form, the whole slab of an
    // expert for the fixed-slab form, none for the per-rank form
    if (layout->kind == EP_LAYOUT_LL_SLAB)
        a->max_pad_rows = (int64_t)layout->num_experts * layout->num_ranks * layout->num_max_tokens_per_rank;
    else if (layout->kind == EP_LAYOUT_EXPAND)
        a->max_pad_rows = (int64_t)layout->num_experts * (layout->expert_alignment - 1);
    if (!ep::set_scale_format(a, scale_format, layout->capacity)) return EP_ERR_INVALID_ARG;
    // column-major per-block scales go through the staging area when the
    // handle's workspace holds it (per-row scales are K words per token: one
    // store each is cheaper than a second kernel)
    if (cast_to_fp8 && a->sf_col_major && a->ng > 1 && layout->kind == EP_LAYOUT_EXPAND &&
        layout->workspace_bytes >= ws.total) {
        a->sf_stage = reinterpret_cast<uint8_t*>(layout->workspace) + ws.stage_off;
        a->sf_stage_ld = (int64_t)ep::round_up((size_t)a->ng * a->sf_elem, 16);
        a->recv_src = layout->recv_src_token;
        a->num_rows = layout->expert_offset + layout->num_experts;
    }
    *elem_bytes = fp8_in ? 1 : 2;
    return device_sms(&a->sms);
}

}  // namespace

namespace ep {

int layout_call(const int64_t* topk_idx, const float* topk_weights, int T, int K, int E, int R, int A,
                int num_max_tokens_per_rank, ep_layout_t* layout, cudaStream_t s, bool clear_header) {
    LayoutArgs a{};
    int rc = prepare_layout(topk_idx, topk_weights, T, K, E, R, A, num_max_tokens_per_rank, layout, &a);
    if (rc != EP_OK) return rc;
    if (T == 0) return empty_layout(layout, s);   // clears the header itself
    int sms = 0;
    if ((rc = device_sms(&sms)) != EP_OK) return rc;
    // only now, with every check passed, may the call touch the workspace
    if (clear_header && cudaMemsetAsync(layout->workspace, 0, kHeaderClearBytes, s) != cudaSuccess)
        return EP_ERR_CUDA;
    return launch_layout(a, sms, s) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace ep

extern "C" {

int ep_version(void) { return EP_B200_VERSION; }

const char* ep_status_string(int status) {
    switch (status) {
        case EP_OK: return "ok";
        case EP_ERR_INVALID_ARG: return "invalid argument";
        case EP_ERR_CAPACITY: return "capacity exceeded";
        case EP_ERR_BAD_EXPERT: return "expert id outside [-1, num_experts)";
        case EP_ERR_TIMEOUT: return "bounded wait ran out";
        case EP_ERR_CUDA: return "CUDA error";
        case EP_ERR_UNSUPPORTED: return "unsupported size";
        default: return "unknown status";
    }
}

size_t ep_workspace_bytes(int num_tokens, int num_topk, int num_experts, int expert_alignment) {
    if (num_tokens < 0 || num_topk < 1 || num_experts < 1 || expert_alignment < 1) return 0;
    return ep::ws_layout(num_tokens, num_topk, num_experts, expert_alignment).total;
}

int64_t ep_capacity_rows(int num_tokens, int num_topk, int num_experts, int expert_alignment) {
    if (num_tokens < 0 || num_topk < 1 || num_experts < 1 || expert_alignment < 1) return 0;
    return (int64_t)num_tokens * num_topk + (int64_t)num_experts * (expert_alignment - 1);
}

int ep_layout(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
              int num_experts, int num_ranks, int expert_alignment, int num_max_tokens_per_rank,
              ep_layout_t* layout, void* stream) {
    return ep::layout_call(topk_idx, topk_weights, num_tokens, num_topk, num_experts, num_ranks, expert_alignment,
                           num_max_tokens_per_rank, layout, (cudaStream_t)stream, false);
}

size_t ep_rank_workspace_bytes(int num_tokens, int num_ranks, int num_experts) {
    if (num_tokens < 0 || num_ranks < 1 || num_experts < 1) return 0;
    return ep::rank_ws_layout(num_tokens, num_ranks, num_experts).total;
}

int ep_rank_layout(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
                   int num_experts, int num_ranks, int expert_alignment, uint8_t* is_token_in_rank,
                   int32_t* num_tokens_per_expert, int32_t* num_recv_tokens_per_expert, int64_t* recv_topk_idx,
                   float* recv_topk_weights, ep_layout_t* layout, void* stream) {
    const int T = num_tokens, K = num_topk, E = num_experts, R = num_ranks, A = expert_alignment;
    if (!layout) return EP_ERR_INVALID_ARG;
    if (T < 0 || K < 1 || E < 1 || R < 1 || A < 1) return EP_ERR_INVALID_ARG;
    if (K > EP_MAX_TOPK || E > EP_MAX_EXPERTS || R > EP_MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if (E % R != 0 || T % R != 0) return EP_ERR_INVALID_ARG;
    if ((int64_t)T * R > INT_MAX) return EP_ERR_UNSUPPORTED;
    if (layout->capacity < 0) return EP_ERR_INVALID_ARG;
    if (layout->capacity > INT_MAX) return EP_ERR_UNSUPPORTED;
    if ((T > 0 && !topk_idx) || !layout->num_recv_tokens_per_expert || !layout->expert_offset ||
        !layout->pair_slot || !layout->recv_src_token || !layout->workspace)
        return EP_ERR_INVALID_ARG;
    if (!aligned(topk_idx, 8) || !aligned(topk_weights, 4) || !aligned(num_tokens_per_expert, 4) ||
        !aligned(num_recv_tokens_per_expert, 4) || !aligned(recv_topk_idx, 8) || !aligned(recv_topk_weights, 4) ||
        !aligned(layout->num_recv_tokens_per_expert, 4) || !aligned(layout->expert_offset, 4) ||
        !aligned(layout->pair_slot, 4) || !aligned(layout->recv_src_token, 4) || !aligned(layout->workspace, 256))
        return EP_ERR_INVALID_ARG;
    const ep::RankWsLayout ws = ep::rank_ws_layout(T, R, E);
    if (layout->workspace_bytes < ws.total) return EP_ERR_INVALID_ARG;

    layout->num_tokens = T;
    layout->num_topk = R;
    layout->num_experts = R;
    layout->num_ranks = R;
    layout->expert_alignment = 1;
    layout->num_max_tokens_per_rank = 0;
    layout->magic = kLayoutMagic;
    layout->kind = EP_LAYOUT_PER_RANK;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* wsb = reinterpret_cast<uint8_t*>(layout->workspace);
    if (T == 0) {
        if (cudaMemsetAsync(layout->workspace, 0, ep::kHeaderClearBytes, s) != cudaSuccess ||
            cudaMemsetAsync(layout->num_recv_tokens_per_expert, 0, (size_t)R * 4, s) != cudaSuccess ||
            cudaMemsetAsync(layout->expert_offset, 0, (size_t)(R + 1) * 4, s) != cudaSuccess ||
            (num_tokens_per_expert && cudaMemsetAsync(num_tokens_per_expert, 0, (size_t)E * 4, s) != cudaSuccess) ||
            (num_recv_tokens_per_expert &&
             cudaMemsetAsync(num_recv_tokens_per_expert, 0, (size_t)E * 4, s) != cudaSuccess))
            return EP_ERR_CUDA;
        return EP_OK;
    }
    ep::LayoutArgs la{};
    la.topk_idx = nullptr;   // keys come from src_idx
    la.topk_weights = nullptr;
    la.T = T; la.K = R; la.E = R; la.R = R; la.A = 1;
    la.C = 0;
    la.CT = 0;
    la.capacity = layout->capacity;
    la.cnt = layout->num_recv_tokens_per_expert;
    la.off = layout->expert_offset;
    la.pair_slot = layout->pair_slot;
    la.recv_src = layout->recv_src_token;
    la.recv_w = reinterpret_cast<float*>(wsb + ws.scratch_w_off);
    la.recv_lexp = reinterpret_cast<int32_t*>(wsb + ws.scratch_lexp_off);
    la.hdr = header(layout);
    la.table = reinterpret_cast<int32_t*>(wsb + ws.expand.table_off);
    la.sup = reinterpret_cast<int32_t*>(wsb + ws.expand.sup_off);
    la.padpre = reinterpret_cast<int32_t*>(wsb + ws.expand.padpre_off);
    la.pad_rows = reinterpret_cast<int32_t*>(wsb + ws.expand.padrows_off);
    la.stats = nullptr;
    la.slab = 0;
    la.src_idx = topk_idx;
    la.src_K = K;
    la.src_E = E;
    la.in_rank = is_token_in_rank;
    la.src_w = topk_weights;
    la.src_A = A;
    la.src_counts = reinterpret_cast<int32_t*>(wsb + ws.counts_off);
    la.n_exp_out = num_tokens_per_expert;
    la.n_recv_out = num_recv_tokens_per_expert;
    la.rank_topk_idx = recv_topk_idx;
    la.rank_topk_w = recv_topk_weights;

    int sms = 0;
    int rc = device_sms(&sms);
    if (rc != EP_OK) return rc;
    return ep::launch_layout(la, sms, s) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

size_t ep_ll_workspace_bytes(int num_tokens, int num_topk, int num_experts, int num_ranks,
                             int num_max_dispatch_tokens_per_rank) {
    if (num_tokens < 0 || num_topk < 1 || num_experts < 1 || num_ranks < 1 || num_max_dispatch_tokens_per_rank < 1)
        return 0;
    const int64_t slab = (int64_t)num_ranks * num_max_dispatch_tokens_per_rank;
    if (slab > INT_MAX - 1) return 0;
    // the padding-row list holds up to E * slab rows: the expand sizing with A = slab + 1
    return ep::ws_layout(num_tokens, num_topk, num_experts, (int)(slab + 1)).base_total;
}

int ep_ll_layout(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
                 int num_experts, int num_ranks, int num_max_dispatch_tokens_per_rank, ep_layout_t* layout,
                 void* stream) {
    const int M = num_max_dispatch_tokens_per_rank;
    if (!layout || M < 1 || num_ranks < 1 || num_experts < 1) return EP_ERR_INVALID_ARG;
    const int64_t slab = (int64_t)num_ranks * M;
    if (slab * num_experts > INT_MAX) return EP_ERR_UNSUPPORTED;
    if (layout->workspace_bytes <
        ep_ll_workspace_bytes(num_tokens, num_topk, num_experts, num_ranks, M))
        return EP_ERR_INVALID_ARG;
    ep_layout_t tmp = *layout;   // the handle changes only once every check has passed
    ep::LayoutArgs a{};
    int rc = prepare_layout(topk_idx, topk_weights, num_tokens, num_topk, num_experts, num_ranks, 1, M, &tmp, &a);
    if (rc != EP_OK) return rc;
    a.slab = (int)slab;
    tmp.kind = EP_LAYOUT_LL_SLAB;
    *layout = tmp;
    cudaStream_t s = (cudaStream_t)stream;
    // with no tokens the kernel still runs (one CTA): every slab row is padding
    int sms = 0;
    if ((rc = device_sms(&sms)) != EP_OK) return rc;
    return ep::launch_layout(a, sms, s) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int64_t ep_scale_bytes(int64_t rows, int hidden, int scale_format) {
    if (rows < 0 || hidden <= 0 || hidden % 128 != 0) return -1;
    ep::DispatchArgs a{};
    a.nb = hidden / 128;
    if (!ep::set_scale_format(&a, scale_format, rows)) return -1;
    return (a.sf_col_major ? a.sf_ld : rows) * a.ng * a.sf_elem;
}

int ep_dispatch(const ep_layout_t* layout, const void* x, int x_dtype, const float* x_scales, int hidden,
                int cast_to_fp8, int scale_format, int do_zero_padding, void* recv_x, void* recv_scales,
                void* stream) {
    ep::DispatchArgs a{};
    int elem_bytes = 0;
    int rc = prepare_dispatch(layout, x, x_dtype, x_scales, hidden, cast_to_fp8, scale_format, do_zero_padding,
                              recv_x, recv_scales, &a, &elem_bytes);
    if (rc != EP_OK) return rc;
    // no tokens: no pairs, and no padding rows except in the fixed-slab form
    if (layout->num_tokens == 0 && layout->kind != EP_LAYOUT_LL_SLAB) return EP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t err = cast_to_fp8 ? ep::launch_dispatch_cast(a, s) : ep::launch_dispatch_copy(a, elem_bytes, s);
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int ep_layout_dispatch(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
                       int num_experts, int num_ranks, int expert_alignment, int num_max_tokens_per_rank,
                       ep_layout_t* layout, const void* x, int x_dtype, const float* x_scales, int hidden,
                       int cast_to_fp8, int scale_format, int do_zero_padding, void* recv_x, void* recv_scales,
                       void* stream) {
    if (!layout) return EP_ERR_INVALID_ARG;
    ep_layout_t tmp = *layout;   // the handle changes only once every check has passed
    ep::LayoutArgs la{};
    ep::DispatchArgs da{};
    int elem_bytes = 0;
    int rc = prepare_layout(topk_idx, topk_weights, num_tokens, num_topk, num_experts, num_ranks,
                            expert_alignment, num_max_tokens_per_rank, &tmp, &la);
    if (rc != EP_OK) return rc;
    rc = prepare_dispatch(&tmp, x, x_dtype, x_scales, hidden, cast_to_fp8, scale_format, do_zero_padding, recv_x,
                          recv_scales, &da, &elem_bytes);
    if (rc != EP_OK) return rc;
    *layout = tmp;
    cudaStream_t s = (cudaStream_t)stream;
    if (num_tokens == 0) return empty_layout(layout, s);
    // the layout kernel, then the dispatch kernel launched behind it; x is an
    // input of this call, so the layout kernel has waited for its producer and
    // the copy kernel may load its first rows while the layout runs
    cudaError_t err = ep::launch_layout(la, da.sms, s);
    if (err == cudaSuccess) {
        if (cast_to_fp8) {
            err = ep::launch_dispatch_cast(da, s);
        } else {
            da.early = 1;
            err = ep::launch_dispatch_copy(da, elem_bytes, s);
        }
    }
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int ep_combine(const ep_layout_t* layout, const void* y, int hidden, const float* topk_weights, const void* bias0,
               const void* bias1, void* out, void* stream) {
    int rc = check_handle(layout);
    if (rc != EP_OK) return rc;
    const int H = hidden, T = layout->num_tokens;
    if (H <= 0 || H % 8 != 0) return EP_ERR_INVALID_ARG;
    if (T > 0 && (!y || !out)) return EP_ERR_INVALID_ARG;
    if (bias1 && !bias0) return EP_ERR_INVALID_ARG;
    if (layout->kind == EP_LAYOUT_PER_RANK && topk_weights) return EP_ERR_INVALID_ARG;
    if (!aligned(y, 16) || !aligned(out, 16) || !aligned(topk_weights, 4) || !aligned(bias0, 16) ||
        !aligned(bias1, 16))
        return EP_ERR_INVALID_ARG;
    if (T == 0) return EP_OK;
    ep::CombineArgs a{};
    a.y = reinterpret_cast<const uint16_t*>(y);
    a.pair_slot = layout->pair_slot;
    a.w = topk_weights;
    a.bias0 = reinterpret_cast<const uint16_t*>(bias0);
    a.bias1 = reinterpret_cast<const uint16_t*>(bias1);
    a.out = reinterpret_cast<uint16_t*>(out);
    a.T = T;
    a.K = layout->num_topk;
    a.H = H;
    a.capacity = layout->capacity;
    a.status = header(layout);
    if ((rc = device_sms(&a.sms)) != EP_OK) return rc;
    return ep::launch_combine(a, (cudaStream_t)stream) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

// Checks shared by the two region calls: an expand handle of alignment 1 and
// the routing it was made from.
static int check_region_handle(const ep_layout_t* layout, const int64_t* topk_idx, const int32_t* row_delta,
                               const void* regions, int64_t region_capacity) {
    int rc = check_handle(layout);
    if (rc != EP_OK) return rc;
    if (layout->kind != EP_LAYOUT_EXPAND || layout->expert_alignment != 1) return EP_ERR_INVALID_ARG;
    if (region_capacity < 0) return EP_ERR_INVALID_ARG;
    if (layout->num_tokens > 0 && (!topk_idx || !row_delta || !regions)) return EP_ERR_INVALID_ARG;
    if (!aligned(topk_idx, 8) || !aligned(row_delta, 4) || !aligned(regions, 8)) return EP_ERR_INVALID_ARG;
    return EP_OK;
}

int ep_dispatch_regions(const ep_layout_t* layout, const int64_t* topk_idx, const int32_t* row_delta,
                        void* const* regions, int64_t region_capacity, const void* x, int hidden,
                        const int64_t* pad_list, int64_t num_pad, void* stream) {
    int rc = check_region_handle(layout, topk_idx, row_delta, regions, region_capacity);
    if (rc != EP_OK) return rc;
    if (num_pad < 0 || (num_pad > 0 && (!pad_list || !regions)) || !aligned(pad_list, 8)) return EP_ERR_INVALID_ARG;
    const int T = layout->num_tokens, H = hidden;
    if (H <= 0 || H % 8 != 0 || (T > 0 && !x) || !aligned(x, 16)) return EP_ERR_INVALID_ARG;
    ep::DispatchArgs a{};
    a.x = reinterpret_cast<const uint8_t*>(x);
    a.pair_slot = layout->pair_slot;
    a.hdr = header(layout);
    a.status_hdr = header(layout);
    a.T = T;
    a.K = layout->num_topk;
    a.H = H;
    a.capacity = 0;            // no single receive buffer
    a.zero_pad = num_pad > 0 ? 1 : 0;
    if ((rc = device_sms(&a.sms)) != EP_OK) return rc;
    a.topk_idx = topk_idx;
    a.row_delta = row_delta;
    a.regions = reinterpret_cast<uint8_t* const*>(regions);
    a.region_capacity = region_capacity;
    a.R = layout->num_ranks;
    a.El = layout->num_experts / layout->num_ranks;
    a.pad_list = pad_list;
    a.num_pad_list = num_pad;
    if (layout->num_tokens == 0 && num_pad == 0) return EP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    return ep::launch_dispatch_copy(a, 2, s, true) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int ep_combine_regions(const ep_layout_t* layout, const int64_t* topk_idx, const int32_t* row_delta,
                       const void* const* regions, int64_t region_capacity, int hidden, const float* topk_weights,
                       void* out, void* stream) {
    int rc = check_region_handle(layout, topk_idx, row_delta, regions, region_capacity);
    if (rc != EP_OK) return rc;
    const int H = hidden, T = layout->num_tokens;
    if (H <= 0 || H % 8 != 0) return EP_ERR_INVALID_ARG;
    if (T > 0 && !out) return EP_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(topk_weights, 4)) return EP_ERR_INVALID_ARG;
    if (T == 0) return EP_OK;
    ep::CombineArgs a{};
    a.pair_slot = layout->pair_slot;
    a.w = topk_weights;
    a.out = reinterpret_cast<uint16_t*>(out);
    a.T = T;
    a.K = layout->num_topk;
    a.H = H;
    a.status = header(layout);
    a.topk_idx = topk_idx;
    a.row_delta = row_delta;
    a.regions = reinterpret_cast<const uint16_t* const*>(regions);
    a.region_capacity = region_capacity;
    a.R = layout->num_ranks;
    a.El = layout->num_experts / layout->num_ranks;
    if ((rc = device_sms(&a.sms)) != EP_OK) return rc;
    return ep::launch_combine(a, (cudaStream_t)stream) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int ep_cast_fp8(const void* x, int num_tokens, int hidden, int scale_format, void* x_fp8, void* scales,
                void* stream) {
    const int T = num_tokens, H = hidden;
    if (T < 0 || H <= 0 || H % 128 != 0) return EP_ERR_INVALID_ARG;
    if (H > 16384) return EP_ERR_UNSUPPORTED;
    if (T > 0 && (!x || !x_fp8 || !scales)) return EP_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(x_fp8, 16) || !aligned(scales, 16)) return EP_ERR_INVALID_ARG;
    if (ep_scale_bytes(T, H, scale_format) < 0) return EP_ERR_INVALID_ARG;
    if (T == 0) return EP_OK;
    ep::DispatchArgs a{};
    a.x = reinterpret_cast<const uint8_t*>(x);
    a.x_scales = nullptr;
    a.recv = reinterpret_cast<uint8_t*>(x_fp8);
    a.recv_scales = reinterpret_cast<float*>(scales);
    a.pair_slot = nullptr;   // row t -> row t
    a.hdr = nullptr;
    a.pad_rows = nullptr;
    a.status_hdr = nullptr;
    a.T = T;
    a.K = 1;
    a.H = H;
    a.capacity = T;
    a.nb = H / 128;
    a.zero_pad = 0;
    if (!ep::set_scale_format(&a, scale_format, T)) return EP_ERR_INVALID_ARG;
    int rc = device_sms(&a.sms);
    if (rc != EP_OK) return rc;
    return ep::launch_dispatch_cast(a, (cudaStream_t)stream) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int ep_get_status(const ep_layout_t* layout, void* stream, uint32_t* device_flags) {
    int rc = check_handle(layout);
    if (rc != EP_OK) return rc;
    if (!device_flags) return EP_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t flags = 0;
    if (cudaMemcpyAsync(&flags, &header(layout)->status, sizeof(flags), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return EP_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return EP_ERR_CUDA;
    *device_flags = flags;
    if (flags & EP_DEV_TIMEOUT) return EP_ERR_TIMEOUT;
    if (flags & EP_DEV_BAD_EXPERT) return EP_ERR_BAD_EXPERT;
    if (flags & EP_DEV_CAPACITY) return EP_ERR_CAPACITY;
    return EP_OK;
}

int ep_selftest_bounded_wait(const ep_layout_t* layout, uint64_t timeout_ns, void* stream) {
    int rc = check_handle(layout);
    if (rc != EP_OK) return rc;
    if (timeout_ns > 1000000000ull) return EP_ERR_INVALID_ARG;
    return ep::launch_selftest_wait(header(layout), timeout_ns, (cudaStream_t)stream) == cudaSuccess
               ? EP_OK
               : EP_ERR_CUDA;
}

}  // extern "C"
