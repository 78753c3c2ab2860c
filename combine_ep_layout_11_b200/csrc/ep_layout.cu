// Routing layout of the expand dispatch ("DeepEP 测试目标 API 系统性参考" §2.1:
// the layout V2 derives from topk_idx, expert_alignment, do_expand; the
// count -> prefix-sum placement -> reorder stages of the Ascend dispatch on the
// "URMA" tag page).
//
// Kernel 1, count: one CTA per chunk of whole tokens builds its per-expert
// histogram with warp-aggregated shared-memory atomics (__match_any_sync groups
// the lanes that hold the same expert; one leader adds the group size).  The
// last CTA to finish (arrival ticket) loads the whole (chunk x expert) table
// into shared memory and turns it into
//   cnt[e], off[e] = sum_{e'<e} align(cnt[e'], A), the per-chunk row bases
//   base[c][e] = off[e] + sum_{c'<c} hist[c'][e], and the padding prefix.
// No CTA ever waits for another, so there is no spin at all.
//
// Kernel 2, assign: one CTA per chunk; each warp owns a contiguous run of the
// chunk's pairs.  A first pass counts per (warp, expert), a scan across warps
// gives each warp its starting row per expert, and a second pass ranks lanes
// of the same expert with __match_any_sync + popc(lanemask_lt).  Together with
// the chunk base this is exactly the stable (token-major, k-minor) order, so
// the result is deterministic and equal to the sequential definition.
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kCountThreads = 512;
constexpr int kAssignThreads = 256;
constexpr int kAssignWarps = kAssignThreads / 32;

__device__ __forceinline__ int align_up_i(int x, int a) { return (x + a - 1) / a * a; }

// Exclusive scan of one int per thread across the block; *total gets the sum.
// `scratch` needs 32 ints of shared memory.
template <int NT>
__device__ int block_exclusive_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
    }
    if (lane == 31) scratch[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int t = lane < NT / 32 ? scratch[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, t, d);
            if (lane >= d) t += y;
        }
        if (lane < NT / 32) scratch[lane] = t;
    }
    __syncthreads();
    int prefix = (wid > 0 ? scratch[wid - 1] : 0) + x - v;
    *total = scratch[NT / 32 - 1];
    __syncthreads();
    return prefix;
}

__device__ __forceinline__ int valid_expert(int64_t e, int E) { return (e >= 0 && e < E) ? (int)e : -1; }

__global__ void __launch_bounds__(kCountThreads) layout_count_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int32_t sm[];
    __shared__ int s_last;
    __shared__ int s_scratch[32];
    const int tid = threadIdx.x, lane = tid & 31;
    const int c = blockIdx.x, E = a.E;

    // ---- per-chunk histogram ----
    int32_t* h = sm;
    for (int e = tid; e < E; e += kCountThreads) h[e] = 0;
    __syncthreads();
    const int64_t p0 = (int64_t)c * a.CT * a.K;
    const int64_t p1 = min((int64_t)(c + 1) * a.CT, (int64_t)a.T) * a.K;
    bool bad = false;
    for (int64_t base = p0; base < p1; base += kCountThreads) {
        const int64_t i = base + tid;
        int key = -1;
        if (i < p1) {
            const int64_t e = a.topk_idx[i];
            key = valid_expert(e, E);
            bad |= (key < 0 && e != -1);
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) atomicAdd(&h[key], __popc(peers));
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&a.hdr->status, kDevBadExpert);
    __syncthreads();
    for (int e = tid; e < E; e += kCountThreads) a.table[(size_t)c * E + e] = h[e];

    // ---- the last CTA to arrive scans the whole table ----
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&a.hdr->ticket, 1u) == (uint32_t)(a.C - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int C = a.C;
    int32_t* tab = sm;                    // [C][E]
    int32_t* cnt_s = sm + (size_t)C * E;  // [E]
    int32_t* off_s = cnt_s + E;           // [E+1]
    for (int i = tid; i < C * E; i += kCountThreads) tab[i] = __ldcg(a.table + i);
    __syncthreads();

    // column scan: exclusive prefix over chunks, per expert
    for (int e = tid; e < E; e += kCountThreads) {
        int run = 0;
        for (int cc = 0; cc < C; ++cc) {
            const int v = tab[cc * E + e];
            tab[cc * E + e] = run;
            run += v;
        }
        cnt_s[e] = run;
    }
    __syncthreads();

    // aligned offsets and padding prefix: scans over experts, each thread owns
    // a consecutive run of experts
    const int ipt = (E + kCountThreads - 1) / kCountThreads;
    const int e0 = min(tid * ipt, E), e1 = min(e0 + ipt, E);
    int loc_rows = 0, loc_pad = 0;
    for (int e = e0; e < e1; ++e) {
        const int al = align_up_i(cnt_s[e], a.A);
        loc_rows += al;
        loc_pad += al - cnt_s[e];
    }
    int total_rows = 0, total_pad = 0;
    int row_prefix = block_exclusive_scan<kCountThreads>(loc_rows, s_scratch, &total_rows);
    int pad_prefix = block_exclusive_scan<kCountThreads>(loc_pad, s_scratch, &total_pad);
    for (int e = e0; e < e1; ++e) {
        const int al = align_up_i(cnt_s[e], a.A);
        off_s[e] = row_prefix;
        a.off[e] = row_prefix;
        a.padpre[e] = pad_prefix;
        a.cnt[e] = cnt_s[e];
        row_prefix += al;
        pad_prefix += al - cnt_s[e];
    }
    if (tid == 0) {
        a.off[E] = total_rows;
        a.padpre[E] = total_pad;
        a.hdr->num_pad = total_pad;
        if ((int64_t)total_rows > a.capacity) atomicOr(&a.hdr->status, kDevCapacity);
        a.hdr->ticket = 0;
    }
    __syncthreads();
    for (int i = tid; i < C * E; i += kCountThreads) {
        const int e = i % E;
        a.table[i] = off_s[e] + tab[i];
    }
}

__global__ void __launch_bounds__(kAssignThreads) layout_assign_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int32_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int c = blockIdx.x, E = a.E, K = a.K;
    int32_t* base_s = sm;     // [E] first row of each expert for this chunk
    int32_t* wh = sm + E;     // [warps][E] per-warp counts, then per-warp starts
    for (int e = tid; e < E; e += kAssignThreads) {
        base_s[e] = a.table[(size_t)c * E + e];
#pragma unroll
        for (int j = 0; j < kAssignWarps; ++j) wh[j * E + e] = 0;
    }
    __syncthreads();

    const int64_t p0 = (int64_t)c * a.CT * K;
    const int64_t p1 = min((int64_t)(c + 1) * a.CT, (int64_t)a.T) * K;
    const int64_t n = p1 - p0;
    const int64_t per = ((n + kAssignWarps - 1) / kAssignWarps + 31) / 32 * 32;
    const int64_t q0 = min(p0 + w * per, p1), q1 = min(q0 + per, p1);
    int32_t* my = wh + w * E;

    // pass 1: per-warp counts
    for (int64_t qb = q0; qb < q1; qb += 32) {
        const int64_t i = qb + lane;
        const int key = (i < q1) ? valid_expert(a.topk_idx[i], E) : -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) my[key] += __popc(peers);
    }
    __syncthreads();
    // exclusive scan across warps, per expert
    for (int e = tid; e < E; e += kAssignThreads) {
        int run = 0;
#pragma unroll
        for (int j = 0; j < kAssignWarps; ++j) {
            const int v = wh[j * E + e];
            wh[j * E + e] = run;
            run += v;
        }
    }
    __syncthreads();

    // pass 2: ranks within the warp, rows, inverse maps
    const int El = E / a.R;
    const uint32_t lt = lanemask_lt();
    for (int64_t qb = q0; qb < q1; qb += 32) {
        const int64_t i = qb + lane;
        const int key = (i < q1) ? valid_expert(a.topk_idx[i], E) : -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        int slot = -1;
        if (key >= 0) slot = base_s[key] + my[key] + __popc(peers & lt);
        __syncwarp();
        if (key >= 0 && lane == __ffs(peers) - 1) my[key] += __popc(peers);
        __syncwarp();
        if (i < q1) {
            a.pair_slot[i] = slot;
            if (slot >= 0 && (int64_t)slot < a.capacity) {
                a.recv_src[slot] = (int32_t)(i / K);
                a.recv_w[slot] = a.topk_weights ? a.topk_weights[i] : 1.0f;
                a.recv_lexp[slot] = key % El;
            }
        }
    }

    // padding rows of the experts e = c, c + C, ...
    for (int e = c; e < E; e += gridDim.x) {
        const int r0 = a.off[e] + a.cnt[e], r1 = a.off[e + 1];
        const int pp = a.padpre[e];
        for (int r = r0 + tid; r < r1; r += kAssignThreads) {
            a.pad_rows[pp + (r - r0)] = r;
            if ((int64_t)r < a.capacity) {
                a.recv_src[r] = -1;
                a.recv_w[r] = 0.0f;
                a.recv_lexp[r] = -1;
            }
        }
    }
}

}  // namespace

cudaError_t launch_layout(const LayoutArgs& a, cudaStream_t s) {
    const size_t count_smem =
        (size_t)max((size_t)a.E, (size_t)a.C * a.E + 2 * (size_t)a.E + 1) * sizeof(int32_t);
    const size_t assign_smem = (size_t)(1 + kAssignWarps) * a.E * sizeof(int32_t);
    cudaError_t err = cudaFuncSetAttribute(layout_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)count_smem);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(layout_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)assign_smem);
    if (err != cudaSuccess) return err;
    layout_count_kernel<<<a.C, kCountThreads, count_smem, s>>>(a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    layout_assign_kernel<<<a.C, kAssignThreads, assign_smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ep
