// Device helpers shared by the dispatch / combine kernels (sm_100a only):
// inline-PTX wrappers for shared-memory barriers and TMA bulk copies, the
// bounded wait every kernel uses, and the workspace layout that ep_layout
// writes and ep_dispatch reads.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cstddef>

#include "ep_b200.h"

namespace ep {

// ---------------------------------------------------------------------------
// Device status word bits (mirrors EP_DEV_* in the public header)
// ---------------------------------------------------------------------------
constexpr uint32_t kDevBadExpert = EP_DEV_BAD_EXPERT;
constexpr uint32_t kDevCapacity = EP_DEV_CAPACITY;
constexpr uint32_t kDevTimeout = EP_DEV_TIMEOUT;

// A wait on a barrier that hardware completes (a TMA load landing in shared
// memory) gives up after this long and reports EP_DEV_TIMEOUT instead of
// spinning forever.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---------------------------------------------------------------------------
// Workspace: [0, 256) header words, then the (chunk x expert) count table, the
// padding prefix and the list of padding rows.
// ---------------------------------------------------------------------------
// Every word before `bar_gen` must be zero before the first ep_layout on a
// workspace; the layout and dispatch kernels leave them at zero again (apart
// from the status word and num_pad, which the next layout rewrites), and the
// host clears them (kHeaderClearBytes) where a call skips the layout kernel.
struct WsHeader {
    uint32_t status;      // EP_DEV_* bits of the last ep_layout and what followed it
    int32_t num_pad;      // padding rows (expert_offset[E] - pairs)
    uint32_t pending;     // flags raised by layout CTAs before the grid barrier
    uint32_t tok_ticket;  // dispatch: next token-row ticket
    uint32_t pad_ticket;  // dispatch: next padding ticket
    uint32_t done;        // dispatch: CTAs finished (the last one resets the tickets)
    uint32_t bar_count;       // layout grid barrier: CTAs arrived, even generations
    uint32_t bar_count_odd;   // the same for odd generations
    uint32_t bar_gen;         // layout grid barrier generation (any value will do)
};
constexpr size_t kHeaderClearBytes = offsetof(WsHeader, bar_gen);
static_assert(sizeof(WsHeader) <= 256, "the header fits its 256 bytes");

// Most chunks (CTAs of the layout kernel) a layout uses.
constexpr int kMaxChunks = 256;
// Chunks per super-chunk: the layout also sums the chunk counts of every run
// of kSupChunks chunks, so that a chunk's scan reads at most
// kMaxChunks / kSupChunks super-chunk rows and kSupChunks - 1 chunk rows.
constexpr int kSupChunks = 16;
constexpr int kSupRows = kMaxChunks / kSupChunks;

struct Chunking {
    int num_chunks;       // C: CTAs of the counting / slot kernels
    int chunk_tokens;     // CT: tokens per chunk
};

// Chunks of whole tokens, about `target_pairs` pairs each, at most `max_chunks`.
inline Chunking chunking(int T, int K, int max_chunks, int target_pairs) {
    Chunking c{0, 0};
    if (T <= 0) return c;
    int64_t pairs = (int64_t)T * K;
    int64_t n = (pairs + target_pairs - 1) / target_pairs;
    if (n > max_chunks) n = max_chunks;
    if (n < 1) n = 1;
    int64_t ct = ((int64_t)T + n - 1) / n;
    c.chunk_tokens = (int)ct;
    c.num_chunks = (int)(((int64_t)T + ct - 1) / ct);
    return c;
}

__host__ __device__ inline int round4(int x) { return (x + 3) / 4 * 4; }

// Bytes per token of the scale staging area: one row of up to 128 fp32
// scales (H <= 16384 for the cast).
constexpr size_t kStageRowBytes = 512;

struct WsLayout {
    size_t table_off;    // int32 [kMaxChunks][round4(E)]: per-chunk expert counts
    size_t sup_off;      // int32 [2][kSupRows][round4(E)]: per-super-chunk sums, two
                         // buffers used by alternate calls (grid-barrier generation parity)
    size_t padpre_off;   // int32 [E+1]: exclusive prefix of padding rows per expert
    size_t padrows_off;  // int32 [E*(A-1)]: receive row of every padding row
    size_t base_total;   // what the layout itself needs
    size_t stage_off;    // [T][kStageRowBytes]: the FP8 dispatch's per-token scale rows
    size_t total;        // with the staging area
};

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WsLayout ws_layout(int T, int K, int E, int A) {
    (void)K;
    WsLayout w;
    w.table_off = 256;
    w.sup_off = round_up(w.table_off + (size_t)kMaxChunks * round4(E) * 4, 256);
    w.padpre_off = round_up(w.sup_off + 2 * (size_t)kSupRows * round4(E) * 4, 256);
    w.padrows_off = round_up(w.padpre_off + ((size_t)E + 1) * 4, 256);
    w.base_total = round_up(w.padrows_off + (size_t)E * (size_t)(A > 1 ? A - 1 : 0) * 4 + 4, 256);
    w.stage_off = w.base_total;
    w.total = w.stage_off + (size_t)(T > 0 ? T : 0) * kStageRowBytes;
    return w;
}

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation and generic-proxy shared-memory writes visible
// to the async proxy (the TMA engine).
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the barrier phase with the given parity to complete; false if it
// has not completed within limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// TMA bulk copy global -> shared, completion counted in bytes on `bar`.
// (No multicast: a plain CTA-local copy.)
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// TMA bulk copy shared -> global, tracked in this thread's bulk async-group.
__device__ __forceinline__ void bulk_store(void* gdst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N of this thread's committed bulk groups are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch: wait until the preceding grid in the stream
// has completed and its writes are visible (a no-op when launched without the
// attribute), and allow the next grid to be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// 16-byte streaming load that does not allocate in L1 (each row is read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while its predecessor in the stream finishes; it must call pdl_wait() before
// touching global memory.
// With `cooperative`, all CTAs of the grid are guaranteed to be resident at
// once (needed by a grid barrier).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              bool cooperative, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cooperative ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace ep
