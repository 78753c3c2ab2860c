// The FP8 cast of dispatch and ep_cast_fp8 ("DeepEP 测试目标 API 系统性参考"
// §4.2 math.py per_token_cast_to_fp8; §3.3 round_scale / use_ue8m0; §2.1
// use_tma_aligned_col_major_sf): bf16 rows are staged in shared memory by TMA,
// cast to e4m3 with their scales by the threads, and the e4m3 rows and
// scale rows leave by TMA bulk stores, K of each per token row.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ep_dispatch_common.cuh"

namespace ep {

namespace {

using namespace dispatch_dev;

constexpr int kCastThreads = 256;
constexpr int kCastOutStages = 2;          // e4m3 rows (and their scales) in flight per cast CTA

// ---------------------------------------------------------------------------
// Cast kernel: bf16 rows in, e4m3 rows and their scales out.  The scale
// variants (EP_SF_* bits): one scale per 128-column block or per row
// (kPerRow), amax / 448 or that rounded up to a power of two (kPow2), stored
// as fp32 or as a UE8M0 exponent byte, row-major or TMA-aligned column-major
// (the last two are runtime fields of DispatchArgs).
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
    return m;
}

// max |x| of one 128-column block: the warp holds it as 32 lanes x 4 values
__device__ __forceinline__ float block_amax(uint2 raw) {
    const float f0 = __uint_as_float(raw.x << 16), f1 = __uint_as_float(raw.x & 0xffff0000u);
    const float f2 = __uint_as_float(raw.y << 16), f3 = __uint_as_float(raw.y & 0xffff0000u);
    return warp_max(fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3))));
}

// The smallest power of two >= s for a positive normal s: clear the mantissa
// and, unless it was already zero, step the exponent up by one.
__device__ __forceinline__ float pow2_ceil(float s) {
    uint32_t u = __float_as_uint(s);
    if (u & 0x7fffffu) u = (u & 0x7f800000u) + 0x800000u;
    return __uint_as_float(u);
}

template <bool kPow2>
__device__ __forceinline__ float make_scale(float amax) {
    const float s = __fdiv_rn(fmaxf(amax, 1e-4f), 448.0f);
    return kPow2 ? pow2_ceil(s) : s;
}

// e4m3 codes of the lane's 4 values under scale s
__device__ __forceinline__ uint32_t quant4(uint2 raw, float s) {
    const float f0 = __uint_as_float(raw.x << 16), f1 = __uint_as_float(raw.x & 0xffff0000u);
    const float f2 = __uint_as_float(raw.y << 16), f3 = __uint_as_float(raw.y & 0xffff0000u);
    const __nv_fp8x2_storage_t lo =
        __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(f0, s), __fdiv_rn(f1, s)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi =
        __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(f2, s), __fdiv_rn(f3, s)), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// Scale g of a row staged in shared memory: fp32, or the UE8M0 byte (the
// biased exponent of a power-of-two scale).
__device__ __forceinline__ void put_scale(uint8_t* row_sf, int g, float s, int elem) {
    if (elem == 4)
        reinterpret_cast<float*>(row_sf)[g] = s;
    else
        row_sf[g] = (uint8_t)((__float_as_uint(s) >> 23) & 0xffu);
}

// Byte offset of scale (row, g) in the scale array.
__device__ __forceinline__ int64_t sf_offset(const DispatchArgs& a, int64_t row, int g) {
    return (a.sf_col_major ? (int64_t)g * a.sf_ld + row : row * a.ng + g) * a.sf_elem;
}

// One scale element from shared memory (src, element g) to global memory.
__device__ __forceinline__ void copy_scale(uint8_t* sf, int64_t off, const uint8_t* src, int g, int elem) {
    if (elem == 4)
        *reinterpret_cast<float*>(sf + off) = reinterpret_cast<const float*>(src)[g];
    else
        sf[off] = src[g];
}

// A row-major scale row that is not a multiple of 16 bytes (so not a TMA
// store) goes out in the widest word dividing its length: 8, 4, 2 or 1 bytes.
__device__ __forceinline__ void copy_word(uint8_t* dst, const uint8_t* src, int w) {
    if (w == 8)
        *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
    else if (w == 4)
        *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(src);
    else if (w == 2)
        *reinterpret_cast<uint16_t*>(dst) = *reinterpret_cast<const uint16_t*>(src);
    else
        *dst = *src;
}

// Barrier 1 over the cast warps only (barrier 0, __syncthreads, also waits
// for the padding warp and is used once, at the end).
__device__ __forceinline__ void cast_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCastThreads) : "memory"); }
__device__ __forceinline__ bool cast_sync_or(bool p) {
    uint32_t r;
    asm volatile(
        "{\n"
        " .reg .pred q, r;\n"
        " setp.ne.u32 q, %1, 0;\n"
        " bar.red.or.pred r, 1, %2, q;\n"
        " selp.u32 %0, 1, 0, r;\n"
        "}\n"
        : "=r"(r)
        : "r"((uint32_t)p), "n"(kCastThreads)
        : "memory");
    return r != 0;
}


// Cast warps 0..7 and one padding warp.  With a handle (a.status_hdr set) the
// token rows come by ticket, as in the copy kernel, and the padding warp
// zero-fills the padding rows and their scales meanwhile; the plain cast
// (ep_cast_fp8: no workspace, no padding) takes rows blockIdx.x, + grid, ...
// Warp 0 draws the items and issues every bulk copy; the item of each input
// stage is published through the stage's mbarrier (a load completing it, or a
// plain arrival with kNoItem when the work has run out).
template <bool kPerRow, bool kPow2>
__global__ void __launch_bounds__(kCastThreads + 32, 4) dispatch_cast_kernel(DispatchArgs a, int stages) {
    constexpr int kWarps = kCastThreads / 32;
    constexpr uint32_t kNoItem = 0xffffffffu;
    extern __shared__ __align__(128) uint8_t smem[];
    const int H = a.H, nb = a.nb, K = a.K, ng = a.ng, elem = a.sf_elem;
    const uint32_t in_stride = round_up_u32(2u * H, 128);
    const uint32_t out_bytes = (uint32_t)H + 4u * nb;       // e4m3 row, then its scales
    const uint32_t out_stride = round_up_u32(out_bytes, 128);
    uint8_t* in = smem;
    uint8_t* out = smem + (size_t)stages * in_stride;
    uint8_t* zero = out + kCastOutStages * (size_t)out_stride;      // kZeroBytes of zeros
    uint64_t* full = reinterpret_cast<uint64_t*>(zero + kZeroBytes);
    int32_t* slots = reinterpret_cast<int32_t*>(full + stages);      // [stages][32]
    uint32_t* stage_item = reinterpret_cast<uint32_t*>(slots + stages * 32);   // [stages]
    int32_t* oslots = reinterpret_cast<int32_t*>(stage_item + stages);   // [kCastOutStages][32] slots per output stage
    float* bmax = reinterpret_cast<float*>(oslots + kCastOutStages * 32);  // per-row scales: block maxima
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint8_t* sf = reinterpret_cast<uint8_t*>(a.recv_scales);
    const uint32_t sf_row_bytes = (uint32_t)ng * (uint32_t)elem;
    const bool bulk_scales = !a.sf_col_major && (sf_row_bytes % 16u) == 0;
    const int sf_word = sf_row_bytes % 8u == 0 ? 8 : sf_row_bytes % 4u == 0 ? 4 : sf_row_bytes % 2u == 0 ? 2 : 1;
    const int sf_words = (int)sf_row_bytes / sf_word;
    WsHeader* h = a.status_hdr;
    const bool tickets = h != nullptr;
    uint8_t* const sf_stage = a.sf_stage;
    const bool scattered_sf = a.sf_col_major && sf_stage == nullptr;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    zero_smem(zero, kZeroBytes, tid, kCastThreads + 32);
    __syncthreads();
    pdl_wait();   // no launch_dependents, as in the copy kernel

    if (warp == kWarps) {
        // ---- padding rows and their scales: pieces of kZeroBytes, 32 per ticket ----
        if (tickets && a.zero_pad) {
            const uint32_t npiece = ((uint32_t)H + kZeroBytes - 1) / kZeroBytes;
            const int64_t pieces = (int64_t)a.hdr->num_pad * npiece;
            const int64_t ntk = (pieces + 31) / 32;
            for (;;) {
                uint32_t tk = 0;
                if (lane == 0) tk = atomicAdd(&h->pad_ticket, 1u);
                tk = __shfl_sync(0xffffffffu, tk, 0);
                if ((int64_t)tk >= ntk) break;
                const int64_t q = (int64_t)tk * 32 + lane;
                if (q < pieces) {
                    const int64_t pr = q / npiece;
                    const uint32_t off = (uint32_t)(q - pr * npiece) * kZeroBytes;
                    const int32_t row = a.pad_rows[pr];
                    if (row >= 0 && (int64_t)row < a.capacity) {
                        bulk_store(a.recv + (int64_t)row * H + off, zero, min(kZeroBytes, (uint32_t)H - off));
                        if (off == 0) {
                            if (bulk_scales)
                                bulk_store(sf + (int64_t)row * sf_row_bytes, zero, sf_row_bytes);
                            else if (a.sf_col_major) {
                                if (scattered_sf)   // staged: the second kernel writes them
                                    for (int g = 0; g < ng; ++g) copy_scale(sf, sf_offset(a, row, g), zero, g, elem);
                            }
                            else
                                for (int wd = 0; wd < sf_words; ++wd)
                                    copy_word(sf + (int64_t)row * sf_row_bytes + wd * sf_word, zero + wd * sf_word,
                                              sf_word);
                        }
                    }
                }
                bulk_commit();
            }
            bulk_wait_all<0>();
        }
        if (tickets) tickets_done(h);
        else __syncthreads();
        return;
    }

    // ---- token rows (cast warps) ----
    const uint32_t items = (uint32_t)a.T;
    const uint32_t G = gridDim.x;
    // warp 0: the CTA's items.  Tickets: the first `stages` in one draw (plus
    // one more, held in `next`), then one drawn ahead of each use.  Without a
    // handle: blockIdx.x, blockIdx.x + G, ...
    uint32_t next = 0, draws = 0;
    auto draw = [&]() -> uint32_t {
        if (!tickets) return blockIdx.x + (draws++) * G;
        const uint32_t t = __shfl_sync(0xffffffffu, next, 0);
        if (lane == 0) next = atomicAdd(&h->tok_ticket, 1u);
        return t;
    };
    // fill stage s with `item`, or mark it the end of this CTA's work
    auto issue = [&](int s, uint32_t item) {
        if (item >= items) {
            if (lane == 0) {
                stage_item[s] = kNoItem;
                mbar_arrive(&full[s]);
            }
            return false;
        }
        if (lane < K) slots[s * 32 + lane] = a.pair_slot ? a.pair_slot[(int64_t)item * K + lane] : (int32_t)item;
        if (lane == 0) {
            stage_item[s] = item;
            mbar_arrive_expect_tx(&full[s], 2u * H);
            bulk_load(in + (size_t)s * in_stride, a.x + (int64_t)item * 2 * H, 2u * H, &full[s]);
        }
        return true;
    };

    bool more = true;   // warp 0: a refill may still find work
    if (warp == 0) {
        uint32_t first = 0;
        if (tickets) {
            if (lane == 0) first = atomicAdd(&h->tok_ticket, (uint32_t)stages + 1u);
            first = __shfl_sync(0xffffffffu, first, 0);
            next = first + (uint32_t)stages;
        }
        for (int s = 0; s < stages && more; ++s) more = issue(s, tickets ? first + (uint32_t)s : draw());
    }

    for (int64_t j = 0;; ++j) {
        const int s = (int)(j % stages);
        const int o = (int)(j % kCastOutStages);
        // output stage o: the stores of item j - kCastOutStages are done reading it
        if (warp == 0) bulk_wait_read<kCastOutStages - 1>();
        const bool landed = mbar_wait(&full[s], (uint32_t)((j / stages) & 1));
        if (cast_sync_or(!landed)) {
            if (tid == 0 && h != nullptr) atomicOr(&h->status, kDevTimeout);
            if (warp == 0) {
                for (int64_t jj = j; jj < j + stages; ++jj)
                    mbar_wait(&full[jj % stages], (uint32_t)((jj / stages) & 1), 100000000ull);
                bulk_wait_all<0>();
            }
            break;
        }
        const uint32_t item = stage_item[s];
        if (item == kNoItem) break;
        const uint8_t* src = in + (size_t)s * in_stride;
        uint8_t* dst = out + (size_t)o * out_stride;
        uint8_t* dst_sf = dst + H;   // this row's ng scales, elem bytes each
        if (kPerRow) {
            for (int b = warp; b < nb; b += kWarps) {
                const float m = block_amax(*reinterpret_cast<const uint2*>(src + (size_t)b * 256 + lane * 8));
                if (lane == 0) bmax[b] = m;
            }
            cast_sync();
            float m = 0.0f;
            for (int b = lane; b < nb; b += 32) m = fmaxf(m, bmax[b]);
            const float sc = make_scale<kPow2>(warp_max(m));
            for (int b = warp; b < nb; b += kWarps) {
                const uint2 raw = *reinterpret_cast<const uint2*>(src + (size_t)b * 256 + lane * 8);
                *reinterpret_cast<uint32_t*>(dst + (size_t)b * 128 + lane * 4) = quant4(raw, sc);
            }
            if (tid == 0) put_scale(dst_sf, 0, sc, elem);
        } else {
            for (int b = warp; b < nb; b += kWarps) {
                const uint2 raw = *reinterpret_cast<const uint2*>(src + (size_t)b * 256 + lane * 8);
                const float sc = make_scale<kPow2>(block_amax(raw));
                *reinterpret_cast<uint32_t*>(dst + (size_t)b * 128 + lane * 4) = quant4(raw, sc);
                if (lane == 0) put_scale(dst_sf, b, sc, elem);
            }
        }
        // unstaged column-major scales are stored by every cast warp below;
        // they read the item's slots from oslots[o], a copy that the refill of
        // input stage s cannot overwrite (it lives as long as output stage o)
        if (scattered_sf && warp == 0 && lane < K) oslots[o * 32 + lane] = slots[s * 32 + lane];
        fence_proxy_async_smem();
        cast_sync();
        if (scattered_sf) {
            for (int q = tid; q < K * ng; q += kCastThreads) {
                const int k = q / ng, g = q - k * ng;
                const int32_t slot = oslots[o * 32 + k];
                if (slot >= 0 && (int64_t)slot < a.capacity) copy_scale(sf, sf_offset(a, slot, g), dst_sf, g, elem);
            }
        }
        if (warp == 0) {
            if (lane < K) {
                const int32_t slot = slots[s * 32 + lane];
                if (slot >= 0 && (int64_t)slot < a.capacity) {
                    bulk_store(a.recv + (int64_t)slot * H, dst, (uint32_t)H);
                    if (bulk_scales) bulk_store(sf + (int64_t)slot * sf_row_bytes, dst_sf, sf_row_bytes);
                }
            }
            // staged column-major scales: the token's scale row, once (the
            // bytes past ng * elem up to the 16-byte stride are not read back)
            // (stage_item[s] still holds the item: the refill comes below)
            if (sf_stage != nullptr && lane == 0)
                bulk_store(sf_stage + (int64_t)stage_item[s] * a.sf_stage_ld, dst_sf, (uint32_t)a.sf_stage_ld);
            if (!a.sf_col_major && !bulk_scales) {
                for (int q = lane; q < K * sf_words; q += 32) {
                    const int k = q / sf_words, wd = q - k * sf_words;
                    const int32_t slot = slots[s * 32 + k];
                    if (slot < 0 || (int64_t)slot >= a.capacity) continue;
                    copy_word(sf + (int64_t)slot * sf_row_bytes + wd * sf_word, dst_sf + wd * sf_word, sf_word);
                }
            }
            bulk_commit();
            if (more) {
                __syncwarp();
                more = issue(s, draw());   // into stage s: every cast thread finished reading it before the barrier
            }
        }
    }
    if (warp == 0) bulk_wait_all<0>();
    if (tickets) tickets_done(h);
    else __syncthreads();
}

// Column-major scales from the staging area: thread i takes receive row i
// (grid-stride) and writes its ng scales, so each store instruction of a warp
// covers 32 consecutive rows of one scale column (128 bytes of fp32, 32 of
// UE8M0) instead of 32 scattered words.  Padding rows (recv_src < 0) get zero
// scales when the dispatch zero-fills padding, and are left alone otherwise.
__global__ void __launch_bounds__(256) scale_colmajor_kernel(DispatchArgs a) {
    pdl_wait();   // the cast kernel's staged rows and the layout's recv_src
    const int64_t n = *a.num_rows;
    const int64_t rows = n < a.capacity ? n : a.capacity;
    const int ng = a.ng, elem = a.sf_elem;
    const int chunks = (int)(a.sf_stage_ld / 16);
    uint8_t* sf = reinterpret_cast<uint8_t*>(a.recv_scales);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; row < rows; row += stride) {
        const int32_t src = a.recv_src[row];
        const bool real = src >= 0 && src < a.T;
        if (!real && !a.zero_pad) continue;
        const uint4* staged = reinterpret_cast<const uint4*>(a.sf_stage + (real ? (int64_t)src * a.sf_stage_ld : 0));
#pragma unroll 2
        for (int c = 0; c < chunks; ++c) {
            const uint4 v = real ? staged[c] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            if (elem == 4) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int g = c * 4 + j;
                    if (g < ng) reinterpret_cast<uint32_t*>(sf)[(int64_t)g * a.sf_ld + row] = w[j];
                }
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int g = c * 16 + j;
                    if (g < ng) sf[(int64_t)g * a.sf_ld + row] = (uint8_t)(w[j >> 2] >> (8 * (j & 3)));
                }
            }
        }
    }
}

template <bool kPerRow, bool kPow2>
cudaError_t launch_cast_variant(const DispatchArgs& a, cudaStream_t s) {
    auto kernel = dispatch_cast_kernel<kPerRow, kPow2>;
    const uint32_t in_stride = round_up_u32(2u * a.H, 128);
    const uint32_t out_stride = round_up_u32((uint32_t)a.H + 4u * a.nb, 128);
    // two input stages (H <= 16384: at most 98 KB of stages), so four CTAs fit
    // an SM at H = 7168: 86.7 against 87.9 us with three (fp8_dispatch);
    // three or four output stages, or two blocks cast per iteration, did not help
    const int stages = 2;
    const size_t smem = (size_t)stages * in_stride + kCastOutStages * (size_t)out_stride + kZeroBytes +
                        (size_t)stages * 8 + (size_t)stages * 33 * 4 + kCastOutStages * 32 * 4 + (size_t)a.nb * 4;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int ctas_per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, kernel, kCastThreads + 32, smem);
    if (err != cudaSuccess) return err;
    if (ctas_per_sm > 4) ctas_per_sm = 4;
    if (ctas_per_sm < 1) ctas_per_sm = 1;
    return launch_pdl(kernel, dim3(a.sms * ctas_per_sm), dim3(kCastThreads + 32), smem, s, false, a, stages);
}

}  // namespace

cudaError_t launch_dispatch_cast(const DispatchArgs& a, cudaStream_t s) {
    const bool per_row = (a.sf_format & EP_SF_PER_ROW) != 0, pow2 = (a.sf_format & EP_SF_POW2) != 0;
    cudaError_t err;
    if (per_row) err = pow2 ? launch_cast_variant<true, true>(a, s) : launch_cast_variant<true, false>(a, s);
    else err = pow2 ? launch_cast_variant<false, true>(a, s) : launch_cast_variant<false, false>(a, s);
    if (err != cudaSuccess || a.sf_stage == nullptr) return err;
    // one thread per receive row, at most eight CTAs of 256 per SM (grid-stride beyond)
    int64_t ctas = (a.capacity + 255) / 256;
    if (ctas > (int64_t)a.sms * 8) ctas = (int64_t)a.sms * 8;
    if (ctas < 1) ctas = 1;
    return launch_pdl(scale_colmajor_kernel, dim3((unsigned)ctas), dim3(256), 0, s, false, a);
}

bool set_scale_format(DispatchArgs* a, int scale_format, int64_t rows) {
    if (scale_format & ~(EP_SF_PER_ROW | EP_SF_POW2 | EP_SF_UE8M0 | EP_SF_COL_MAJOR)) return false;
    if ((scale_format & EP_SF_UE8M0) && !(scale_format & EP_SF_POW2)) return false;
    a->sf_format = scale_format;
    a->ng = (scale_format & EP_SF_PER_ROW) ? 1 : a->nb;
    a->sf_elem = (scale_format & EP_SF_UE8M0) ? 1 : 4;
    a->sf_col_major = (scale_format & EP_SF_COL_MAJOR) ? 1 : 0;
    const int64_t per16 = 16 / a->sf_elem;
    a->sf_ld = (rows + per16 - 1) / per16 * per16;
    return true;
}

}  // namespace ep
