// Device side of the routing layout, shared by the layout kernel and the fused
// layout + dispatch kernel.  See ep_layout.cu for the algorithm.
#pragma once

#include "ep_internal.h"

namespace ep {
namespace layout_dev {



constexpr int kLayoutThreads = 256;
constexpr int kThreads = kLayoutThreads;
constexpr int kWarps = kThreads / 32;
constexpr int kGroups = 4;                 // thread groups over the chunk range in the scan
constexpr int kGroupThreads = kThreads / kGroups;

__device__ __forceinline__ int align_up_i(int x, int a) { return (x + a - 1) / a * a; }

// Exclusive scan of one int per thread across the block; *total gets the sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
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
        int t = lane < kWarps ? scratch[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, t, d);
            if (lane >= d) t += y;
        }
        if (lane < kWarps) scratch[lane] = t;
    }
    __syncthreads();
    int prefix = (wid > 0 ? scratch[wid - 1] : 0) + x - v;
    *total = scratch[kWarps - 1];
    __syncthreads();
    return prefix;
}

__device__ __forceinline__ int valid_expert(int64_t e, int E) { return (e >= 0 && e < E) ? (int)e : -1; }

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier over `n` co-resident CTAs (generation counting, so it
// needs no reset between calls).  Bounded: false if the other CTAs have not
// all arrived within kWaitLimitNs.
__device__ __forceinline__ bool grid_barrier(WsHeader* hdr, uint32_t n) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t gen0 = ld_acquire_u32(&hdr->bar_gen);
        __threadfence();
        const uint32_t arrived = atomicAdd(&hdr->bar_count, 1u);
        int ok = 1;
        if (arrived == n - 1) {
            hdr->bar_count = 0;
            __threadfence();
            st_release_u32(&hdr->bar_gen, gen0 + 1);
        } else {
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_u32(&hdr->bar_gen) == gen0) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    ok = 0;
                    break;
                }
            }
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// The layout work of one CTA (chunk c = blockIdx.x of a.C co-resident CTAs of
// kLayoutThreads threads).  `sm` holds layout_smem_ints(E) ints; on return
// (true) it keeps LayoutSmem's arrays for this chunk.  False: the grid barrier
// timed out (reported in the status word) and nothing past the count was written.
__device__ __forceinline__ bool layout_body(const LayoutArgs& a, int32_t* sm) {
    __shared__ int s_scratch[32];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int c = blockIdx.x, C = a.C, E = a.E, Ep = round4(E), K = a.K;
    int32_t* cnt_s = sm;                 // [Ep] histogram of this chunk, then totals
    int32_t* base_s = cnt_s + Ep;        // [Ep] first row of each expert for this chunk
    int32_t* off_s = base_s + Ep;        // [Ep + 4] aligned offsets
    int32_t* padpre_s = off_s + Ep + 4;  // [Ep + 4] padding prefix
    int32_t* wh = padpre_s + Ep + 4;     // [kWarps][Ep]: scan partials, then per-warp counts

    for (int e = tid; e < Ep; e += kThreads) cnt_s[e] = 0;
    if (c == 0 && tid == 0) a.hdr->status = 0;
    __syncthreads();

    // ---- 1. count ----
    const int64_t p0 = (int64_t)c * a.CT * K;
    const int64_t p1 = min((int64_t)(c + 1) * a.CT, (int64_t)a.T) * K;
    bool bad = false;
    for (int64_t base = p0; base < p1; base += kThreads) {
        const int64_t i = base + tid;
        int key = -1;
        if (i < p1) {
            const int64_t e = a.topk_idx[i];
            key = valid_expert(e, E);
            bad |= (key < 0 && e != -1);
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) atomicAdd(&cnt_s[key], __popc(peers));
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&a.hdr->pending, kDevBadExpert);
    __syncthreads();
    for (int e4 = tid; e4 < Ep / 4; e4 += kThreads)
        reinterpret_cast<int4*>(a.table + (size_t)c * Ep)[e4] = reinterpret_cast<const int4*>(cnt_s)[e4];

    // ---- 2. grid barrier ----
    if (!grid_barrier(a.hdr, (uint32_t)C)) {
        if (tid == 0) atomicOr(&a.hdr->status, kDevTimeout);
        return false;
    }

    // ---- 3. scan ----
    {
        const int g = tid / kGroupThreads, q = tid % kGroupThreads;
        const int c_lo = (int)((int64_t)C * g / kGroups), c_hi = (int)((int64_t)C * (g + 1) / kGroups);
        int32_t* part_tot = wh;                 // [kGroups][Ep]
        int32_t* part_pre = wh + kGroups * Ep;  // [kGroups][Ep]
        for (int e4 = q; e4 < Ep / 4; e4 += kGroupThreads) {
            int4 tot = make_int4(0, 0, 0, 0), pre = make_int4(0, 0, 0, 0);
            const int4* col = reinterpret_cast<const int4*>(a.table) + e4;
#pragma unroll 8
            for (int cc = c_lo; cc < c_hi; ++cc) {
                const int4 v = __ldcg(col + (size_t)cc * (Ep / 4));
                tot.x += v.x; tot.y += v.y; tot.z += v.z; tot.w += v.w;
                if (cc < c) { pre.x += v.x; pre.y += v.y; pre.z += v.z; pre.w += v.w; }
            }
            reinterpret_cast<int4*>(part_tot + g * Ep)[e4] = tot;
            reinterpret_cast<int4*>(part_pre + g * Ep)[e4] = pre;
        }
        __syncthreads();
        for (int e = tid; e < E; e += kThreads) {
            int tot = 0, pre = 0;
#pragma unroll
            for (int j = 0; j < kGroups; ++j) {
                tot += part_tot[j * Ep + e];
                pre += part_pre[j * Ep + e];
            }
            cnt_s[e] = tot;
            base_s[e] = pre;
        }
        __syncthreads();
    }
    // aligned offsets and padding prefix: each thread owns a run of experts
    const int ipt = (E + kThreads - 1) / kThreads;
    const int e0 = min(tid * ipt, E), e1 = min(e0 + ipt, E);
    int loc_rows = 0, loc_pad = 0;
    for (int e = e0; e < e1; ++e) {
        const int al = align_up_i(cnt_s[e], a.A);
        loc_rows += al;
        loc_pad += al - cnt_s[e];
    }
    int total_rows = 0, total_pad = 0;
    int row_prefix = block_exclusive_scan(loc_rows, s_scratch, &total_rows);
    int pad_prefix = block_exclusive_scan(loc_pad, s_scratch, &total_pad);
    for (int e = e0; e < e1; ++e) {
        const int al = align_up_i(cnt_s[e], a.A);
        off_s[e] = row_prefix;
        padpre_s[e] = pad_prefix;
        row_prefix += al;
        pad_prefix += al - cnt_s[e];
    }
    if (tid == 0) {
        off_s[E] = total_rows;
        padpre_s[E] = total_pad;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) base_s[e] += off_s[e];
    if (c == 0) {
        for (int e = tid; e < E; e += kThreads) {
            a.cnt[e] = cnt_s[e];
            a.off[e] = off_s[e];
            a.padpre[e] = padpre_s[e];
        }
        if (tid == 0) {
            a.off[E] = total_rows;
            a.padpre[E] = total_pad;
            a.hdr->num_pad = total_pad;
            uint32_t flags = atomicExch(&a.hdr->pending, 0u);
            if ((int64_t)total_rows > a.capacity) flags |= kDevCapacity;
            if (flags) atomicOr(&a.hdr->status, flags);
        }
    }
    for (int i = tid; i < kWarps * Ep; i += kThreads) wh[i] = 0;
    __syncthreads();

    // ---- 4. assign ----
    const int64_t n = p1 - p0;
    const int64_t per = ((n + kWarps - 1) / kWarps + 31) / 32 * 32;
    const int64_t q0 = min(p0 + w * per, p1), q1 = min(q0 + per, p1);
    int32_t* my = wh + w * Ep;
    for (int64_t qb = q0; qb < q1; qb += 32) {          // pass 1: per-warp counts
        const int64_t i = qb + lane;
        const int key = (i < q1) ? valid_expert(a.topk_idx[i], E) : -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) my[key] += __popc(peers);
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) {           // exclusive scan across warps
        int run = 0;
#pragma unroll
        for (int j = 0; j < kWarps; ++j) {
            const int v = wh[j * Ep + e];
            wh[j * Ep + e] = run;
            run += v;
        }
    }
    __syncthreads();
    const int El = E / a.R;
    const uint32_t lt = lanemask_lt();
    for (int64_t qb = q0; qb < q1; qb += 32) {          // pass 2: ranks, rows, inverse maps
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

    // ---- 5. padding rows of the experts e = c, c + C, ... ----
    for (int e = c; e < E; e += C) {
        const int r0 = off_s[e] + cnt_s[e], r1 = off_s[e + 1];
        const int pp = padpre_s[e];
        for (int r = r0 + tid; r < r1; r += kThreads) {
            a.pad_rows[pp + (r - r0)] = r;
            if ((int64_t)r < a.capacity) {
                a.recv_src[r] = -1;
                a.recv_w[r] = 0.0f;
                a.recv_lexp[r] = -1;
            }
        }
    }
    __syncthreads();
    return true;
}

// Shared memory of layout_body, in ints.
__host__ __device__ inline size_t layout_smem_ints(int E) {
    const int Ep = round4(E);
    return (size_t)2 * Ep + 2 * ((size_t)Ep + 4) + (size_t)kWarps * Ep;
}

// Where layout_body leaves its per-chunk results in shared memory.
struct LayoutSmem {
    int32_t* cnt;      // [E] receive rows per expert
    int32_t* base;     // [E] first row of each expert for this chunk
    int32_t* off;      // [E+1] aligned offsets
    int32_t* padpre;   // [E+1] padding prefix
    __device__ LayoutSmem(int32_t* sm, int E) {
        const int Ep = round4(E);
        cnt = sm;
        base = sm + Ep;
        off = base + Ep;
        padpre = off + Ep + 4;
    }
};

}  // namespace layout_dev
}  // namespace ep
