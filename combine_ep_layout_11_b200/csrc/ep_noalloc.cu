// ep_layout_no_alloc: ep_layout for callers that cannot allocate device memory
// themselves.  The layout's workspace (status word, grid-barrier words, count
// table, padding list) lives in a fixed-size array in this library's own
// device memory instead of a caller-provided buffer.
//
// Every GPU that loads the library holds the array (kStaticScratchBytes) until
// the process exits.  All calls share it and it keeps the last call's contents,
// so calls whose work overlaps on the GPU (other streams, other threads) race on
// it; the header words that must start at zero are cleared on every call.
#include <mutex>

#include "ep_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = EP_NO_ALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_layout_scratch[kStaticScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device, with that device current, and cached.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return EP_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return EP_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || !p) return EP_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return EP_OK;
}

}  // namespace

extern "C" {

int ep_layout_no_alloc(const int64_t* topk_idx, const float* topk_weights, int num_tokens, int num_topk,
                       int num_experts, int num_ranks, int expert_alignment, int num_max_tokens_per_rank,
                       ep_layout_t* layout, void* stream) {
    if (!layout) return EP_ERR_INVALID_ARG;
    if (ep_workspace_bytes(num_tokens, num_topk, num_experts, expert_alignment) == 0) return EP_ERR_INVALID_ARG;
    // the layout's own part; the dispatch uses the scale staging area behind
    // it only where the array has room for it
    const size_t need = ep::ws_layout(num_tokens, num_topk, num_experts, expert_alignment).base_total;
    if (need > kStaticScratchBytes) return EP_ERR_UNSUPPORTED;
    void* ws = nullptr;
    int rc = scratch_address(&ws);
    if (rc != EP_OK) return rc;
    ep_layout_t tmp = *layout;
    tmp.workspace = ws;
    tmp.workspace_bytes = kStaticScratchBytes;
    // ep_layout's checks first; only a call that passes them clears the
    // header words that must start at zero (the barrier counter, the pending
    // flags) and launches, so a rejected call leaves the shared array as it was
    rc = ep::layout_call(topk_idx, topk_weights, num_tokens, num_topk, num_experts, num_ranks, expert_alignment,
                         num_max_tokens_per_rank, &tmp, (cudaStream_t)stream, true);
    if (rc == EP_OK) *layout = tmp;
    return rc;
}

}  // extern "C"
