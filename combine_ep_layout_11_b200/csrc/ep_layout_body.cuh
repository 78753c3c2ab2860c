// Device side of the routing layout, shared by the layout kernel and the fused
// layout + dispatch kernel.  See ep_layout.cu for the algorithm.
#pragma once

#include "ep_internal.h"

namespace ep {
namespace layout_dev {

// Threads per CTA: 512 for up to 1024 experts, 256 beyond (shared memory).
constexpr int kWideThreads = 512;
constexpr int kNarrowThreads = 256;
constexpr int kWideMaxExperts = 1024;
constexpr int kKeyRounds = 4;   // rounds of 32 pairs per warp whose expert ids stay in registers

__host__ __device__ inline int layout_threads(int E) { return E <= kWideMaxExperts ? kWideThreads : kNarrowThreads; }

// Shared memory of layout_body, in ints: per-warp counts [warps][Ep], counts,
// bases, offsets and padding prefix [Ep (+4)], scan partials [8 * threads];
// with per-rank keys also a histogram of the src_E experts.
__host__ __device__ inline size_t layout_smem_ints(int E, int src_E = 0) {
    const int Ep = round4(E), nt = layout_threads(E);
    return (size_t)(nt / 32) * Ep + 4 * (size_t)Ep + 8 + 8 * (size_t)nt + (size_t)round4(src_E);
}

// Where layout_body leaves its per-chunk results in shared memory.
struct LayoutSmem {
    int32_t* wh;       // [warps][Ep] per-warp starting rows (after the assign: ends)
    int32_t* cnt;      // [Ep] receive rows per expert
    int32_t* base;     // [Ep] first row of each expert for this chunk
    int32_t* off;      // [Ep + 4] aligned offsets, off[E] = rows used
    int32_t* padpre;   // [Ep + 4] padding prefix, padpre[E] = padding rows
    int32_t* part;     // [8 * threads] scan partials
    int32_t* ehist;    // [src_E] per-rank keys: pairs per expert in this chunk
    __host__ __device__ LayoutSmem(int32_t* sm, int E) {
        const int Ep = round4(E), nw = layout_threads(E) / 32;
        wh = sm;
        cnt = wh + (size_t)nw * Ep;
        base = cnt + Ep;
        off = base + Ep;
        padpre = off + Ep + 4;
        part = padpre + Ep + 4;
        ehist = part + 8 * layout_threads(E);
    }
};

__device__ __forceinline__ int align_up_i(int x, int a) { return (x + a - 1) / a * a; }

__device__ __forceinline__ int valid_expert(int64_t e, int E) { return (e >= 0 && e < E) ? (int)e : -1; }

// Key of pair i: its expert id (-1 if unselected), or with per-rank keys
// (kRankKeys; pairs are (t, r) of a [T, R] table with R = a.K) the rank r when
// token t has one of its experts there, else -1.  `bad` collects ids outside
// [-1, E).  The token's ids are loaded eight at a time, all eight before any
// is used, so a key costs one memory round trip per eight experts.
template <bool kRankKeys>
__device__ __forceinline__ int pair_key(const LayoutArgs& a, int64_t i, bool& bad, int32_t* hist = nullptr) {
    if (!kRankKeys) {
        const int64_t e = a.topk_idx[i];
        const int key = valid_expert(e, a.E);
        bad |= (key < 0 && e != -1);
        return key;
    }
    const int R = a.K;
    // pair indices stay below 2^31 (T * R <= INT_MAX is checked on the host):
    // 32-bit division
    const int64_t t = (int)i / R;
    const int r = (int)i - (int)t * R;
    // rank r holds the experts [lo, lo + El): a range test, no 64-bit division
    const int El = a.src_E / R;
    const int64_t lo = (int64_t)r * El, hi = lo + El;
    const int64_t* row = a.src_idx + t * a.src_K;
    int key = -1;
    for (int k0 = 0; k0 < a.src_K; k0 += 8) {
        int64_t ev[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) ev[j] = k0 + j < a.src_K ? row[k0 + j] : -1;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t e = ev[j];
            if (e >= lo && e < hi) {
                key = r;
                // each selected (t, k) is local to exactly one rank: counted once
                if (hist) atomicAdd(&hist[e], 1);
            } else if (e != -1 && (e < 0 || e >= a.src_E)) {
                bad = true;
            }
        }
    }
    return key;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// 16-byte load through L2 only (the table rows were written by other CTAs).
__device__ __forceinline__ int4 ld_cg_v4(const int4* p) {
    int4 v;
    asm volatile("ld.global.cg.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_add_release_u32(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Exclusive scan of one 64-bit value per thread across a CTA of NT threads;
// *total gets the sum.  `scratch` holds NT / 32 values.
// Per-rank keys: the rank-local expert ids and weights of receive row `slot`,
// which holds pair i = (t, r).  Entries whose expert is on another rank get -1
// and weight 0.  With K a multiple of 4 and 16-byte aligned arrays a row goes
// out in 16-byte stores (two per four ids, one per four weights).
__device__ __forceinline__ void write_rank_row(const LayoutArgs& a, int64_t i, int slot) {
    if (!a.rank_topk_idx && !a.rank_topk_w) return;
    const int R = a.K, K = a.src_K;
    const int64_t t = (int)i / R;   // 32-bit: T * R <= INT_MAX
    const int r = (int)i - (int)t * R;
    const int El = a.src_E / R;
    const int64_t lo = (int64_t)r * El, hi = lo + El;   // rank r's experts
    const int64_t* row = a.src_idx + t * K;
    int64_t* oi = a.rank_topk_idx ? a.rank_topk_idx + (int64_t)slot * K : nullptr;
    float* ow = a.rank_topk_w ? a.rank_topk_w + (int64_t)slot * K : nullptr;
    const bool vec = (K % 4) == 0 && ((reinterpret_cast<uintptr_t>(a.rank_topk_idx) |
                                       reinterpret_cast<uintptr_t>(a.rank_topk_w)) & 15u) == 0;
    for (int k0 = 0; k0 < K; k0 += 8) {
        int64_t ev[8];
        float wv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const bool in = k0 + j < K;
            ev[j] = in ? row[k0 + j] : -1;
            wv[j] = (in && a.src_w) ? a.src_w[t * K + k0 + j] : 1.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; j += 4) {
            const int k = k0 + j;
            if (k >= K) break;
            long long o[4];
            float w4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t e = ev[j + q];
                const bool local = k + q < K && e >= lo && e < hi;
                o[q] = local ? e - lo : -1;
                w4[q] = local ? wv[j + q] : 0.0f;
            }
            if (vec) {
                if (oi) {
                    reinterpret_cast<longlong2*>(oi + k)[0] = make_longlong2(o[0], o[1]);
                    reinterpret_cast<longlong2*>(oi + k)[1] = make_longlong2(o[2], o[3]);
                }
                if (ow) *reinterpret_cast<float4*>(ow + k) = make_float4(w4[0], w4[1], w4[2], w4[3]);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (k + q >= K) break;
                    if (oi) oi[k + q] = o[q];
                    if (ow) ow[k + q] = w4[q];
                }
            }
        }
    }
}

template <int NT>
__device__ __forceinline__ long long block_exclusive_scan64(long long v, long long* scratch, long long* total) {
    constexpr int kW = NT / 32;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    long long x = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
    }
    if (lane == 31) scratch[wid] = x;
    __syncthreads();
    if (wid == 0) {
        long long t = lane < kW ? scratch[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, t, d);
            if (lane >= d) t += y;
        }
        if (lane < kW) scratch[lane] = t;
    }
    __syncthreads();
    const long long prefix = (wid > 0 ? scratch[wid - 1] : 0) + x - v;
    *total = scratch[kW - 1];
    return prefix;   // `scratch` is read until here: a barrier must come before its next write
}

// One bounded grid barrier over the n co-resident CTAs of this launch.  Two
// arrival counters alternate with the parity of the generation gen0, which
// every CTA read before arriving: each CTA's thread 0 adds one to its counter
// with a release reduction (no round trip to wait for) and polls it with
// acquire loads until all n have arrived; the CTA's writes are ordered before
// that reduction by __syncthreads.  After the barrier CTA 0 zeroes the other
// counter (the previous call used it, the next one will) and advances the
// generation.  The counter of this call keeps the value n until the next call
// zeroes it: a CTA still polling must not see it fall.  Bounded: false if the
// other CTAs have not all arrived within kWaitLimitNs (the workspace must then
// be zeroed again before the next call).
__device__ __forceinline__ bool grid_barrier(WsHeader* hdr, uint32_t n, uint32_t gen0) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t* cnt = (gen0 & 1u) ? &hdr->bar_count_odd : &hdr->bar_count;
        __threadfence();
        red_add_release_u32(cnt, 1u);
        int ok = 1;
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_u32(cnt) < n) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                ok = 0;
                break;
            }
        }
        s_ok = ok;
    }
    __syncthreads();
    const bool ok = s_ok != 0;
    if (ok && blockIdx.x == 0 && threadIdx.x == 0) {
        *((gen0 & 1u) ? &hdr->bar_count : &hdr->bar_count_odd) = 0;
        hdr->bar_gen = gen0 + 1;
    }
    return ok;
}

// The layout work of one CTA: chunk c = blockIdx.x of a.C co-resident CTAs of
// NT threads.  `sm` holds layout_smem_ints(E) ints; on success (true) the
// LayoutSmem arrays hold this chunk's results.  False: the grid barrier timed
// out (reported in the status word) and nothing past the counts was written.
//
//   count   warp w owns a contiguous run of the chunk's pairs; per round of 32
//           pairs, __match_any_sync groups lanes holding the same expert and
//           the group's lowest lane adds the group size to the warp's row
//           wh[w][e]; the expert ids stay in registers for the assign;
//   publish the chunk histogram (sum over warps, which also turns wh into
//           per-warp starting offsets) is row c of table[C][Ep], and is added
//           (red) into row c / kSupChunks of this call's super-chunk sums;
//   barrier one bounded grid barrier;
//   scan    thread groups sum, with 16-byte loads, the super-chunk rows (all
//           of them: the total per expert; those before c's own: part of the
//           prefix) and the chunk rows of c's super-chunk before c (the rest
//           of the prefix): at most kSupRows + kSupChunks - 1 rows;
//           one packed 64-bit block scan gives off[e] and the padding prefix;
//   assign  rank = popc(peers & lanemask_lt) within the round, plus the warp's
//           running offset, plus the chunk base: the stable token-major,
//           k-minor order, equal to the sequential definition bit for bit;
//   pads    receive-row metadata of the padding rows of experts c, c + C, ...
template <int NT, bool kRankKeys = false>
__device__ __forceinline__ bool layout_body(const LayoutArgs& a, int32_t* sm) {
    constexpr int kW = NT / 32;
    __shared__ long long s_scratch[kW];
    __shared__ uint32_t s_gen0;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int c = blockIdx.x, C = a.C, E = a.E, Ep = round4(E), K = a.K;
    LayoutSmem L(sm, E);
    int32_t* my = L.wh + (size_t)w * Ep;

    __shared__ int s_over;
    if (tid == 0) {
        s_gen0 = ld_relaxed_u32(&a.hdr->bar_gen);   // read before arriving at the barrier
        if (c == 0) a.hdr->status = 0;
        s_over = 0;
    }
    for (int e = lane; e < Ep; e += 32) my[e] = 0;
    if (kRankKeys) {
        for (int e = tid; e < a.src_E; e += NT) L.ehist[e] = 0;
        __syncthreads();
    }
    __syncwarp();

    // ---- count ----
    const int64_t p0 = (int64_t)c * a.CT * K;
    const int64_t p1 = min((int64_t)(c + 1) * a.CT, (int64_t)a.T) * K;
    const int64_t per = ((p1 - p0 + kW - 1) / kW + 31) / 32 * 32;
    const int64_t q0 = min(p0 + w * per, p1), q1 = min(q0 + per, p1);
    bool bad = false;
    auto load_key = [&](int64_t i) -> int {
        return i < q1 ? pair_key<kRankKeys>(a, i, bad, kRankKeys ? L.ehist : nullptr) : -1;
    };
    auto count_round = [&](int key) {
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) my[key] += __popc(peers);
        __syncwarp();
    };
    // the first rounds load together and keep their expert ids (and the
    // weights the assign writes) in registers
    int keys[kKeyRounds];
    float wts[kKeyRounds];
#pragma unroll
    for (int r = 0; r < kKeyRounds; ++r) keys[r] = load_key(q0 + 32 * r + lane);
#pragma unroll
    for (int r = 0; r < kKeyRounds; ++r) {
        const int64_t i = q0 + 32 * r + lane;
        wts[r] = (!kRankKeys && a.topk_weights && i < q1) ? a.topk_weights[i] : 1.0f;
    }
#pragma unroll
    for (int r = 0; r < kKeyRounds; ++r)
        if (q0 + 32 * r < q1) count_round(keys[r]);
    for (int64_t qb = q0 + 32 * kKeyRounds; qb < q1; qb += 32) count_round(load_key(qb + lane));
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&a.hdr->pending, kDevBadExpert);
    __syncthreads();
    if (kRankKeys && a.src_counts) {   // this chunk's expert counts, added before the barrier
        for (int e = tid; e < a.src_E; e += NT)
            if (L.ehist[e]) atomicAdd(&a.src_counts[e], L.ehist[e]);
    }
    // chunk histogram; the per-warp counts become per-warp starting offsets
    for (int e = tid; e < Ep; e += NT) {
        int run = 0;
#pragma unroll
        for (int j = 0; j < kW; ++j) {
            const int v = L.wh[j * Ep + e];
            L.wh[j * Ep + e] = run;
            run += v;
        }
        L.cnt[e] = run;
    }
    __syncthreads();
    for (int e4 = tid; e4 < Ep / 4; e4 += NT)
        reinterpret_cast<int4*>(a.table + (size_t)c * Ep)[e4] = reinterpret_cast<const int4*>(L.cnt)[e4];
    // the counts are also added into the super-chunk's row of this call's sum
    // buffer (generation parity); the other buffer, which the previous call
    // used, is zeroed for the next one
    {
        int32_t* sup_now = a.sup + (size_t)(s_gen0 & 1u) * kSupRows * Ep + (size_t)(c / kSupChunks) * Ep;
        for (int e = tid; e < E; e += NT) {
            const int v = L.cnt[e];
            if (v) atomicAdd(&sup_now[e], v);
        }
        int4* sup_next = reinterpret_cast<int4*>(a.sup + (size_t)((s_gen0 + 1u) & 1u) * kSupRows * Ep);
        for (int i = c * NT + tid; i < kSupRows * Ep / 4; i += C * NT) sup_next[i] = make_int4(0, 0, 0, 0);
    }

    // ---- barrier ----
    if (!grid_barrier(a.hdr, (uint32_t)C, s_gen0)) {
        if (tid == 0) atomicOr(&a.hdr->status, kDevTimeout);
        return false;
    }

    // ---- scan ----
    const int cols = Ep / 4;
    int groups = NT / cols;
    if (groups > 8) groups = 8;
    if (groups < 1) groups = 1;
    int32_t* part_tot = L.part;              // [groups][Ep]
    int32_t* part_pre = L.part + 4 * NT;     // [groups][Ep]   (groups * Ep <= 4 * NT)
    // one group: sums go straight to cnt / base (the chunk histogram in cnt
    // is no longer needed once published); several: partials, summed below
    int32_t* dst_tot = groups == 1 ? L.cnt : part_tot;
    int32_t* dst_pre = groups == 1 ? L.base : part_pre;
    {
        // the rows a chunk sums: the G super-chunk rows of this call (all of
        // them for the totals, those before its own super-chunk sg for its
        // prefix), then the chunk rows c0 .. c-1 of its own super-chunk
        const int sg = c / kSupChunks, c0 = sg * kSupChunks;
        const int G = (C + kSupChunks - 1) / kSupChunks;
        const int nv = G + (c - c0);
        const int4* sup_now = reinterpret_cast<const int4*>(a.sup + (size_t)(s_gen0 & 1u) * kSupRows * Ep);
        const int4* tab = reinterpret_cast<const int4*>(a.table);
        const int g = tid / cols;
        if (g < groups) {
            const int v_lo = nv * g / groups, v_hi = nv * (g + 1) / groups;
            for (int q = tid % cols; q < cols; q += (cols < NT ? cols : NT)) {
                int4 tot = make_int4(0, 0, 0, 0), pre = make_int4(0, 0, 0, 0);
                for (int r0 = v_lo; r0 < v_hi; r0 += 8) {
                    // eight unconditional loads (rows past the range re-read the
                    // last row and are dropped), issued back to back
                    int4 v[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = min(r0 + i, v_hi - 1);
                        v[i] = ld_cg_v4((r < G ? sup_now + (size_t)r * cols : tab + (size_t)(c0 + r - G) * cols) + q);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = r0 + i;
                        if (r >= v_hi) continue;
                        if (r < G) {
                            tot.x += v[i].x; tot.y += v[i].y; tot.z += v[i].z; tot.w += v[i].w;
                            if (r >= sg) continue;
                        }
                        pre.x += v[i].x; pre.y += v[i].y; pre.z += v[i].z; pre.w += v[i].w;
                    }
                }
                reinterpret_cast<int4*>(dst_tot + g * Ep)[q] = tot;
                reinterpret_cast<int4*>(dst_pre + g * Ep)[q] = pre;
            }
        }
        __syncthreads();
    }
    // Per expert, each thread owning a run of consecutive experts: its total and
    // its sum over earlier chunks (the thread groups' partials added up), then
    // the aligned offsets (high word) and padding prefix (low word) in one block
    // scan.  Every per-expert value is written and read by its owner only until
    // the barrier before the assign, so no other barrier is needed.
    const int ipt = (E + NT - 1) / NT;
    const int e0 = min(tid * ipt, E), e1 = min(e0 + ipt, E);
    long long loc = 0;
    // rows of expert e: its count aligned up to A, or the fixed slab; padding
    // rows: the rest (none when an expert overflows its slab)
    auto rows_of = [&](int e) { return a.slab > 0 ? a.slab : align_up_i(L.cnt[e], a.A); };
    for (int e = e0; e < e1; ++e) {
        int tot = dst_tot[e], pre = dst_pre[e];
        for (int j = 1; j < groups; ++j) {
            tot += part_tot[j * Ep + e];
            pre += part_pre[j * Ep + e];
        }
        L.cnt[e] = tot;
        L.base[e] = pre;
        const int al = rows_of(e);
        loc += ((long long)al << 32) + max(al - tot, 0);
    }
    long long total = 0;
    long long prefix = block_exclusive_scan64<NT>(loc, s_scratch, &total);
    for (int e = e0; e < e1; ++e) {
        const int al = rows_of(e);
        const int o = (int)(prefix >> 32), pp = (int)(prefix & 0xffffffffll);
        L.off[e] = o;
        L.padpre[e] = pp;
        L.base[e] += o;
        if (c == 0) {   // the per-expert outputs, written once
            a.cnt[e] = L.cnt[e];
            if (a.slab > 0 && L.cnt[e] > a.slab) s_over = 1;   // more pairs than the slab holds
            if (a.stats) a.stats[e] += L.cnt[e];
            a.off[e] = o;
            a.padpre[e] = pp;
        }
        prefix += ((long long)al << 32) + max(al - L.cnt[e], 0);
    }
    const int total_rows = (int)(total >> 32), total_pad = (int)(total & 0xffffffffll);
    if (tid == 0) {
        L.off[E] = total_rows;
        L.padpre[E] = total_pad;
    }
    if (c == 0) {
        if (tid == 0) {
            a.off[E] = total_rows;
            a.padpre[E] = total_pad;
            a.hdr->num_pad = total_pad;
        }
        if (kRankKeys && a.src_counts) {   // every chunk's adds landed before the barrier
            for (int e = tid; e < a.src_E; e += NT) {
                const int32_t n = __ldcg(&a.src_counts[e]);
                if (a.n_exp_out) a.n_exp_out[e] = n;
                if (a.n_recv_out) a.n_recv_out[e] = align_up_i(n, a.src_A);
                a.src_counts[e] = 0;   // ready for the next call; no other CTA reads it after the barrier
            }
        }
    }
    __syncthreads();

    // ---- assign ----
    {
        const int El = E / a.R;
        const uint32_t lt = lanemask_lt();
        auto assign_round = [&](int64_t qb, int key, float wt) {
            const int64_t i = qb + lane;
            const uint32_t peers = __match_any_sync(0xffffffffu, key);
            int slot = -1;
            if (key >= 0) slot = L.base[key] + my[key] + __popc(peers & lt);
            __syncwarp();
            if (key >= 0 && lane == __ffs(peers) - 1) my[key] += __popc(peers);
            __syncwarp();
            if (a.slab > 0 && slot >= 0 && slot - L.off[key] >= a.slab) slot = -1;   // past its slab: dropped
            if (i < q1) {
                if (kRankKeys && a.in_rank) a.in_rank[i] = key >= 0 ? 1 : 0;
                a.pair_slot[i] = slot;
                if (slot >= 0 && (int64_t)slot < a.capacity) {
                    a.recv_src[slot] = (int32_t)(i / K);
                    a.recv_w[slot] = wt;
                    a.recv_lexp[slot] = key % El;
                    if (kRankKeys) write_rank_row(a, i, slot);
                }
            }
        };
#pragma unroll
        for (int r = 0; r < kKeyRounds; ++r)
            if (q0 + 32 * r < q1) assign_round(q0 + 32 * r, keys[r], wts[r]);
        bool unused = false;
        for (int64_t qb = q0 + 32 * kKeyRounds; qb < q1; qb += 32) {
            const int64_t i = qb + lane;
            const float wt = (!kRankKeys && a.topk_weights && i < q1) ? a.topk_weights[i] : 1.0f;
            assign_round(qb, (i < q1) ? pair_key<kRankKeys>(a, i, unused) : -1, wt);
        }
    }

    // ---- padding rows of the experts e = c, c + C, ... ----
    for (int e = c; e < E; e += C) {
        const int r0 = L.off[e] + L.cnt[e], r1 = L.off[e + 1];
        const int pp = L.padpre[e];
        for (int row = r0 + tid; row < r1; row += NT) {
            a.pad_rows[pp + (row - r0)] = row;
            if ((int64_t)row < a.capacity) {
                a.recv_src[row] = -1;
                a.recv_w[row] = 0.0f;
                a.recv_lexp[row] = -1;
            }
        }
    }
    if (c == 0 && tid == 0) {   // fold the flags of this call into the status word
        uint32_t flags = atomicExch(&a.hdr->pending, 0u);
        if ((int64_t)total_rows > a.capacity || s_over) flags |= kDevCapacity;
        if (flags) atomicOr(&a.hdr->status, flags);
    }
    __syncthreads();
    return true;
}

}  // namespace layout_dev
}  // namespace ep
