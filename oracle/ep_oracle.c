/*
 * ep_oracle.c - CPU oracle for DeepEP-style MoE expert-parallel token
 * dispatch and combine on R virtual ranks.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, single-threaded
 * statement of what the hot path computes.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg load it; the product library never
 * does, and this file shares no code, header or table with the CUDA sources.
 *
 * Sources, by page title and section:
 *  [API]  "DeepEP 测试目标 API 系统性参考" (DeepEP test-target API reference):
 *         §2.1 dispatch() parameter table (topk_idx with -1 = unselected,
 *         expert_alignment, do_expand, do_zero_padding) and return table;
 *         §2.2 combine() (weighted reduction back to the source order);
 *         §3.2 Buffer.combine() (unweighted: plain sum);
 *         §4.1 refs.py (ordered_accumulate: fixed-order accumulation);
 *         §4.2 math.py (FP8 E4M3 cast: scale = amax / fp8_max,
 *         q = x / scale, dequantisation q * scale; align()).
 *  [RT]   "spark_model/layers/ep_dispatch.rs": build_ep_routing_table, the
 *         token-major / k-minor partition into local and remote pairs.
 *  [URMA] "URMA" tag page: the Ascend full-mesh dispatch ends with count
 *         reconciliation, prefix-sum placement and output reordering.
 *
 * Readings where the pages are silent (all listed in the design notes):
 *  - scales are per 128-column block of a token row, fp32, row-major [T, H/128]
 *    (per row, [T], as a variant); round_scale rounds a scale up to a power
 *    of two; UE8M0 stores such a scale as its biased exponent byte;
 *  - amax is clamped below at 1e-4 so an all-zero block gets a finite scale;
 *  - the quotient x / scale is one correctly rounded binary32 division and the
 *    E4M3 conversion rounds to nearest-even and saturates to +-448;
 *  - combine starts from 0 (or from the output bias: bias0, plus bias1 as one
 *    rounded sum), skips -1 entries, and for k = 0..K-1 in order does
 *    acc = acc + (w * y) with two binary32 roundings (no fused multiply-add),
 *    then rounds acc to bf16 to nearest-even; NULL weights mean w = 1;
 *  - the source rank of token t is t / (T / R); expert e lives on rank e / (E / R).
 *
 * Floating point is binary32 because the method fixes it (fp32 accumulation,
 * fp32 scales).  Build with -O2 -ffp-contract=off and without fast-math so that
 * every operation above is exactly one IEEE-754 binary32 rounding.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_INVALID_ARG 1
#define ORC_ERR_CAPACITY 2
#define ORC_ERR_BAD_EXPERT 3
#define ORC_ERR_INDEX_LEN 10
#define ORC_ERR_WEIGHT_LEN 11

/* ------------------------------------------------------------------ */
/* bf16 <-> binary32                                                    */
/* ------------------------------------------------------------------ */

/* A bf16 value is the upper 16 bits of a binary32 value, so widening is exact. */
static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 value to the nearest bf16 value, ties to the even bf16
 * mantissa.  The 16 dropped bits are compared against the halfway point
 * 0x8000: above rounds up, below truncates, exactly half goes to the even
 * neighbour.  Carries out of the mantissa correctly bump the exponent (and
 * turn the largest finite values into infinity).  NaN stays a quiet NaN. */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------ */
/* FP8 E4M3 ("e4m3fn": no infinities, one NaN pattern per sign)        */
/* ------------------------------------------------------------------ */

/* Format definition: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 *   exponent field 0      : subnormal, value = m/8 * 2^-6
 *   exponent field 1..15  : normal,    value = (1 + m/8) * 2^(E-7)
 *   exponent 15, mantissa 7 (0x7f / 0xff) is NaN; the largest finite is
 *   0x7e = 1.75 * 2^8 = 448.  */
static double e4m3_magnitude(unsigned code7)
{
    unsigned ex = (code7 >> 3) & 0xfu;
    unsigned m = code7 & 0x7u;
    if (ex == 0)
        return ldexp((double)m / 8.0, -6);
    return ldexp(1.0 + (double)m / 8.0, (int)ex - 7);
}

float orc_e4m3_decode(uint8_t code)
{
    unsigned mag = code & 0x7fu;
    if (mag == 0x7fu)
        return NAN;
    double v = e4m3_magnitude(mag);
    return (float)((code & 0x80u) ? -v : v);
}

/* Nearest finite E4M3 value, ties to the even code, saturating: any magnitude
 * at or above 448 encodes as 448.  The non-negative codes 0x00..0x7e are
 * ordered by value, so the search is over that sorted table; the two
 * candidates' distances are binary32 differences, computed exactly in double. */
uint8_t orc_e4m3_encode(float v)
{
    if (isnan(v))
        return 0x7f;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7e);
    /* largest code whose magnitude is <= a */
    unsigned lo = 0, hi = 0x7e;
    while (lo < hi) {
        unsigned mid = (lo + hi + 1) / 2;
        if (e4m3_magnitude(mid) <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    unsigned code = lo;
    if (code < 0x7e) {
        double below = a - e4m3_magnitude(code);
        double above = e4m3_magnitude(code + 1) - a;
        if (above < below || (above == below && ((code + 1) & 1u) == 0))
            code = code + 1;
    }
    return (uint8_t)(sign | code);
}

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_e4m3_encode(v[i]);
}

void orc_e4m3_decode_array(const uint8_t* c, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_e4m3_decode(c[i]);
}

void orc_f32_to_bf16_array(const float* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = f32_to_bf16_rne(v[i]);
}

/* ------------------------------------------------------------------ */
/* Layout: counts, aligned offsets, slots       [API] §2.1, [URMA]      */
/* ------------------------------------------------------------------ */

static int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

/* Expand layout: one receive row per selected (token, k) pair.
 *  cnt[e]       number of pairs that chose expert e
 *  off[e]       sum over e' < e of align(cnt[e'], A); off[E] = rows used
 *  pair_slot    receive row of pair (t, k), -1 when topk_idx[t, k] == -1
 *  recv_src     source token of each receive row, -1 on padding rows
 *  recv_w       topk weight of each receive row (1 when no weights given), 0 on padding
 *  recv_lexp    local expert id e mod (E / R), -1 on padding rows
 * Rows of expert e are [off[e], off[e] + cnt[e]) in token-major, k-minor
 * order of the pairs, followed by align(cnt[e], A) - cnt[e] padding rows.
 * Because each rank owns a contiguous run of experts, this is the order
 * (destination rank, local expert, source token).
 * slab > 0 gives the low-latency form ([API] §3.3 low_latency_dispatch:
 * num_max_dispatch_tokens_per_rank, a receive buffer of
 * [E/R, R * max_tokens, H] per rank): every expert owns a fixed slab of
 * `slab` = R * max_tokens rows, off[e] = e * slab, the rows after its pairs
 * are padding, and more pairs than the slab holds is ORC_ERR_CAPACITY. */
int orc_layout(const int64_t* topk_idx, const float* topk_weights,
               int64_t T, int64_t K, int64_t E, int64_t R, int64_t A,
               int64_t max_tokens_per_rank, int64_t capacity, int64_t slab,
               int32_t* cnt, int32_t* off, int32_t* pair_slot,
               int32_t* recv_src, float* recv_w, int32_t* recv_lexp)
{
    if (T < 0 || K < 1 || E < 1 || R < 1 || A < 1 || E % R != 0 || T % R != 0 || slab < 0)
        return ORC_ERR_INVALID_ARG;
    if (max_tokens_per_rank > 0 && T / R > max_tokens_per_rank)
        return ORC_ERR_CAPACITY;

    /* 1. every entry is either -1 (unselected) or an expert id in [0, E) */
    for (int64_t i = 0; i < T * K; i++)
        if (topk_idx[i] < -1 || topk_idx[i] >= E)
            return ORC_ERR_BAD_EXPERT;

    /* 2. per-expert receive counts */
    for (int64_t e = 0; e < E; e++)
        cnt[e] = 0;
    for (int64_t i = 0; i < T * K; i++)
        if (topk_idx[i] >= 0)
            cnt[topk_idx[i]] += 1;

    /* 3. exclusive prefix sum of the aligned counts; with a fixed slab of
     *    `slab` rows per expert (the low-latency layout) off[e] = e * slab */
    off[0] = 0;
    for (int64_t e = 0; e < E; e++) {
        if (slab > 0) {
            if (cnt[e] > slab)
                return ORC_ERR_CAPACITY;
            off[e + 1] = (int32_t)((e + 1) * slab);
        } else {
            off[e + 1] = (int32_t)(off[e] + align_up(cnt[e], A));
        }
    }
    if (off[E] > capacity)
        return ORC_ERR_CAPACITY;

    /* 4. walk pairs token-major, k-minor; each takes the next row of its expert */
    int64_t experts_per_rank = E / R;
    int64_t* fill = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    if (!fill)
        return ORC_ERR_INVALID_ARG;
    for (int64_t t = 0; t < T; t++) {
        for (int64_t k = 0; k < K; k++) {
            int64_t i = t * K + k;
            int64_t e = topk_idx[i];
            if (e < 0) {
                pair_slot[i] = -1;
                continue;
            }
            int64_t slot = off[e] + fill[e];
            fill[e] += 1;
            pair_slot[i] = (int32_t)slot;
            recv_src[slot] = (int32_t)t;
            recv_w[slot] = topk_weights ? topk_weights[i] : 1.0f;
            recv_lexp[slot] = (int32_t)(e % experts_per_rank);
        }
    }
    free(fill);

    /* 5. alignment padding rows after each expert's real rows */
    for (int64_t e = 0; e < E; e++) {
        for (int64_t slot = off[e] + cnt[e]; slot < off[e + 1]; slot++) {
            recv_src[slot] = -1;
            recv_w[slot] = 0.0f;
            recv_lexp[slot] = -1;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Per-token-per-rank layout                    [API] §2.1, §3.1, §3.2  */
/* ------------------------------------------------------------------ */

/* The default receive form of dispatch (do_expand off, [API] §2.1): one
 * receive row per (token, destination rank) that the token reaches, with the
 * V1 layout quantities of [API] §3.1 (num_tokens_per_rank, is_token_in_rank,
 * num_tokens_per_expert) and the V1 receive outputs (recv_topk_idx,
 * recv_topk_weights, num_recv_tokens_per_expert_list).
 *  is_token_in_rank[t, r]   1 if some k has topk_idx[t, k] on rank r (e / (E/R) == r)
 *  num_tokens_per_rank[r]   number of tokens with is_token_in_rank[t, r]
 *  rank_off[r]              sum over r' < r of num_tokens_per_rank[r']; rank_off[R] = rows used
 *  token_slot[t, r]         receive row of (t, r), -1 if the token does not reach r
 *  num_tokens_per_expert[e] number of pairs (t, k) that chose e
 *  num_recv_per_expert[e]   align(num_tokens_per_expert[e], A) (the aligned list of §3.1)
 *  recv_src[row]            source token of the row
 *  recv_topk_idx[row, k]    topk_idx[t, k] - r*(E/R) if that expert is on the row's rank r, else -1
 *  recv_topk_w[row, k]      topk_weights[t, k] (1 without weights) for those entries, else 0
 * Rows of rank r are [rank_off[r], rank_off[r+1]) in ascending token order
 * (so by source rank, then token).  No padding rows. */
int orc_rank_layout(const int64_t* topk_idx, const float* topk_weights, int64_t T, int64_t K, int64_t E,
                    int64_t R, int64_t A, int64_t capacity, int32_t* num_tokens_per_rank, int32_t* rank_off,
                    uint8_t* is_token_in_rank, int32_t* token_slot, int32_t* num_tokens_per_expert,
                    int32_t* num_recv_per_expert, int32_t* recv_src, int64_t* recv_topk_idx, float* recv_topk_w)
{
    if (T < 0 || K < 1 || E < 1 || R < 1 || A < 1 || E % R != 0 || T % R != 0)
        return ORC_ERR_INVALID_ARG;
    for (int64_t i = 0; i < T * K; i++)
        if (topk_idx[i] < -1 || topk_idx[i] >= E)
            return ORC_ERR_BAD_EXPERT;
    int64_t experts_per_rank = E / R;

    for (int64_t e = 0; e < E; e++)
        num_tokens_per_expert[e] = 0;
    for (int64_t i = 0; i < T * K; i++)
        if (topk_idx[i] >= 0)
            num_tokens_per_expert[topk_idx[i]] += 1;
    for (int64_t e = 0; e < E; e++)
        num_recv_per_expert[e] = (int32_t)align_up(num_tokens_per_expert[e], A);

    for (int64_t t = 0; t < T; t++)
        for (int64_t r = 0; r < R; r++) {
            uint8_t in = 0;
            for (int64_t k = 0; k < K; k++) {
                int64_t e = topk_idx[t * K + k];
                if (e >= 0 && e / experts_per_rank == r)
                    in = 1;
            }
            is_token_in_rank[t * R + r] = in;
        }
    for (int64_t r = 0; r < R; r++) {
        num_tokens_per_rank[r] = 0;
        for (int64_t t = 0; t < T; t++)
            num_tokens_per_rank[r] += is_token_in_rank[t * R + r];
    }
    rank_off[0] = 0;
    for (int64_t r = 0; r < R; r++)
        rank_off[r + 1] = rank_off[r] + num_tokens_per_rank[r];
    if (rank_off[R] > capacity)
        return ORC_ERR_CAPACITY;

    for (int64_t r = 0; r < R; r++) {
        int64_t row = rank_off[r];
        for (int64_t t = 0; t < T; t++) {
            if (!is_token_in_rank[t * R + r]) {
                token_slot[t * R + r] = -1;
                continue;
            }
            token_slot[t * R + r] = (int32_t)row;
            recv_src[row] = (int32_t)t;
            for (int64_t k = 0; k < K; k++) {
                int64_t e = topk_idx[t * K + k];
                int local = e >= 0 && e / experts_per_rank == r;
                recv_topk_idx[row * K + k] = local ? e - r * experts_per_rank : -1;
                recv_topk_w[row * K + k] = local ? (topk_weights ? topk_weights[t * K + k] : 1.0f) : 0.0f;
            }
            row += 1;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Dispatch: row scatter                        [API] §2.1              */
/* ------------------------------------------------------------------ */

/* recv[slot] = x[t] for every selected pair (t, k) with slot = pair_slot[t, k];
 * rows are opaque byte strings (a bf16 row, an fp8 row or a row of scales).
 * With do_zero_padding the alignment padding rows of every expert are zeroed;
 * otherwise they are left untouched. */
void orc_dispatch_rows(const uint8_t* x, int64_t row_bytes, int64_t T, int64_t K,
                       const int32_t* pair_slot, const int32_t* cnt, const int32_t* off,
                       int64_t E, int do_zero_padding, uint8_t* recv)
{
    for (int64_t t = 0; t < T; t++)
        for (int64_t k = 0; k < K; k++) {
            int32_t slot = pair_slot[t * K + k];
            if (slot >= 0)
                memcpy(recv + (int64_t)slot * row_bytes, x + t * row_bytes, (size_t)row_bytes);
        }
    if (do_zero_padding)
        for (int64_t e = 0; e < E; e++)
            for (int64_t slot = off[e] + cnt[e]; slot < off[e + 1]; slot++)
                memset(recv + slot * row_bytes, 0, (size_t)row_bytes);
}

/* ------------------------------------------------------------------ */
/* FP8 cast                                     [API] §4.2              */
/* ------------------------------------------------------------------ */

/* Smallest power of two >= s, for a positive normal s: the round_scale option
 * ([API] §3.3 low_latency_dispatch: round_scale rounds the scale to a power of
 * two; reading: upwards, so that |x / s| <= 448 still holds and nothing
 * saturates).  frexpf writes s = m * 2^e with m in [0.5, 1); s is itself a
 * power of two exactly when m == 0.5. */
static float pow2_ceil(float s)
{
    int e;
    float m = frexpf(s, &e);
    if (m == 0.5f)
        return s;
    return ldexpf(1.0f, e);
}

/* For each token t and each group g of `group` columns (group = 128: one scale
 * per 128-column block; group = H: one scale per row, [API] §4.2
 * per_token_cast_to_fp8):
 *   amax = max |x[t, g*group .. g*group + group - 1]|, clamped below at 1e-4
 *   s    = amax / 448                     (binary32 division)
 *   s    = pow2_ceil(s)                   (only with round_pow2)
 *   q[j] = e4m3(x[t, j] / s)              (binary32 division, RNE, saturating)
 *   scales[t, g] = s                      (row-major [T, H / group])        */
void orc_cast_fp8(const uint16_t* x, int64_t T, int64_t H, int64_t group, int round_pow2, uint8_t* q,
                  float* scales)
{
    int64_t ng = H / group;
    for (int64_t t = 0; t < T; t++) {
        for (int64_t g = 0; g < ng; g++) {
            const uint16_t* blk = x + t * H + g * group;
            float amax = 0.0f;
            for (int64_t j = 0; j < group; j++) {
                float a = fabsf(bf16_to_f32(blk[j]));
                if (a > amax)
                    amax = a;
            }
            if (amax < 1e-4f)
                amax = 1e-4f;
            float s = amax / 448.0f;
            if (round_pow2)
                s = pow2_ceil(s);
            scales[t * ng + g] = s;
            for (int64_t j = 0; j < group; j++) {
                float quotient = bf16_to_f32(blk[j]) / s;
                q[t * H + g * group + j] = orc_e4m3_encode(quotient);
            }
        }
    }
}

/* UE8M0 ([API] §3.3 use_ue8m0): an unsigned 8-bit exponent, value 2^(b - 127),
 * no sign and no mantissa.  A power-of-two scale s = 2^k is stored as
 * b = k + 127; frexpf gives s = 0.5 * 2^e, so k = e - 1.  Returns ORC_OK, or
 * ORC_ERR_INVALID_ARG if some s is not a power of two in [2^-127, 2^127]. */
int orc_ue8m0_encode(const float* s, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++) {
        int e;
        float m = frexpf(s[i], &e);
        if (m != 0.5f || e - 1 < -127 || e - 1 > 127)
            return ORC_ERR_INVALID_ARG;
        out[i] = (uint8_t)(e - 1 + 127);
    }
    return ORC_OK;
}

/* value of a UE8M0 byte: 2^(b - 127) (b = 255 is not produced by the cast). */
void orc_ue8m0_decode(const uint8_t* b, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = ldexpf(1.0f, (int)b[i] - 127);
}

/* Dequantisation: value = float(q) * s, one binary32 multiplication, with the
 * scale of the value's group (group = 128 or H, as in orc_cast_fp8). */
void orc_dequant_fp8(const uint8_t* q, const float* scales, int64_t T, int64_t H, int64_t group, float* out)
{
    int64_t ng = H / group;
    for (int64_t t = 0; t < T; t++)
        for (int64_t j = 0; j < H; j++) {
            float v = orc_e4m3_decode(q[t * H + j]);
            float s = scales[t * ng + j / group];
            out[t * H + j] = v * s;
        }
}

/* ------------------------------------------------------------------ */
/* Combine: ordered weighted reduction          [API] §2.2, §3.2, §4.1 */
/* ------------------------------------------------------------------ */

/* out[t] = bf16( init[t] + sum over k = 0..K-1 with pair_slot[t, k] >= 0 of w[t, k] * y[slot] )
 * accumulated in binary32 in ascending k.  The starting value init[t] is 0,
 * or the output bias ([API] §2.2 combine() bias, §4.1 refs.combine
 * initial_value): float(bias0[t]), and with a second bias
 * float(bias0[t]) + float(bias1[t]) as one rounded sum.  Each term is one
 * rounded product followed by one rounded sum.  NULL weights: w = 1. */
void orc_combine(const uint16_t* y, int64_t H, const int32_t* pair_slot,
                 const float* topk_weights, int64_t T, int64_t K,
                 const uint16_t* bias0, const uint16_t* bias1, uint16_t* out)
{
    float* acc = (float*)malloc((size_t)(H > 0 ? H : 1) * sizeof(float));
    if (!acc)
        return;
    for (int64_t t = 0; t < T; t++) {
        for (int64_t h = 0; h < H; h++) {
            acc[h] = 0.0f;
            if (bias0)
                acc[h] = bf16_to_f32(bias0[t * H + h]);
            if (bias1)
                acc[h] = acc[h] + bf16_to_f32(bias1[t * H + h]);
        }
        for (int64_t k = 0; k < K; k++) {
            int32_t slot = pair_slot[t * K + k];
            if (slot < 0)
                continue;
            float w = topk_weights ? topk_weights[t * K + k] : 1.0f;
            const uint16_t* row = y + (int64_t)slot * H;
            for (int64_t h = 0; h < H; h++) {
                float product = w * bf16_to_f32(row[h]);
                acc[h] = acc[h] + product;
            }
        }
        for (int64_t h = 0; h < H; h++)
            out[t * H + h] = f32_to_bf16_rne(acc[h]);
    }
    free(acc);
}

/* Running per-expert receive counts across calls ([API] §2.1 and §3.3:
 * cumulative_local_expert_recv_stats; rank r's local experts are entries
 * [r*E/R, (r+1)*E/R)): stats[e] += cnt[e]. */
void orc_accumulate_recv_stats(const int32_t* cnt, int64_t E, int32_t* stats)
{
    for (int64_t e = 0; e < E; e++)
        stats[e] += cnt[e];
}

/* ------------------------------------------------------------------ */
/* Local / remote routing table of one rank     [RT]                    */
/* ------------------------------------------------------------------ */

/* Partition the selected pairs of M tokens, token-major then k-minor, into
 * those whose expert lies in [local_start, local_end) and the rest.  Token
 * indices are 0..M-1 within the batch given, expert ids stay absolute.  Length
 * mismatches are reported as errors where the page's function panics; -1
 * entries (unselected) belong to neither bucket. */
int orc_routing_table(const int64_t* gate_indices, int64_t n_indices,
                      const float* gate_weights, int64_t n_weights,
                      int64_t M, int64_t K, int64_t local_start, int64_t local_end,
                      int32_t* local_tok, int32_t* local_eid, float* local_w, int64_t* n_local,
                      int32_t* remote_tok, int32_t* remote_eid, float* remote_w, int64_t* n_remote)
{
    if (n_indices != M * K)
        return ORC_ERR_INDEX_LEN;
    if (n_weights != M * K)
        return ORC_ERR_WEIGHT_LEN;
    int64_t nl = 0, nr = 0;
    for (int64_t t = 0; t < M; t++) {
        for (int64_t k = 0; k < K; k++) {
            int64_t i = t * K + k;
            int64_t e = gate_indices[i];
            if (e < 0)
                continue;
            if (e >= local_start && e < local_end) {
                local_tok[nl] = (int32_t)t;
                local_eid[nl] = (int32_t)e;
                local_w[nl] = gate_weights[i];
                nl++;
            } else {
                remote_tok[nr] = (int32_t)t;
                remote_eid[nr] = (int32_t)e;
                remote_w[nr] = gate_weights[i];
                nr++;
            }
        }
    }
    *n_local = nl;
    *n_remote = nr;
    return ORC_OK;
}
