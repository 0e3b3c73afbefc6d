/*
 * ep_oracle.c -- plain, single-threaded CPU oracle for MoE token routing.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this code.  It shares nothing with
 * the CUDA library (no headers, helpers or tables) and the CUDA library never
 * calls it.
 *
 * What it computes (DeepEP as described on its pages):
 *   A1  get_dispatch_layout      ("GET_DISPATCH_LAYOUT_API", Parameters and
 *                                 Return Values; "Python 接口", Dispatch API
 *                                 inputs num_tokens_per_rank / is_token_in_rank
 *                                 / num_tokens_per_expert)
 *   A2  rank prefix matrix, send positions, receive counts
 *                                ("legacy test analysis": check_data walks
 *                                 recv_gbl_rank_prefix_sum as inclusive block
 *                                 ends; intranode handle tuple)
 *   A3  dispatch scatter         ("Python 接口", Dispatch API outputs recv_x,
 *                                 recv_topk_idx, recv_topk_weights)
 *   A4  combine gather-reduce    ("legacy test analysis", combine_args and the
 *                                 check (combined_x - bias) / is_token_in_rank.sum)
 *   A5  low-latency dispatch with FP8 e4m3 + fp32 scale per 128 channels
 *                                ("legacy test analysis", low_latency_dispatch
 *                                 call and its per-expert checks)
 *   A6  low-latency combine with top-k weights
 *                                ("legacy test analysis", low_latency_combine
 *                                 and x * sum(masked weights) check)
 *
 * Floating point: fp32 everywhere, as the routing method fixes it (fp32
 * accumulation, one final round to bf16).  Build with -ffp-contract=off so
 * that no multiply-add is fused unless written as fmaf().
 *
 * Conventions (readings of the pages, where they are silent):
 *   - expert e lives on rank e / (E/R) (contiguous blocks; the low-latency
 *     test names expert ids rank * num_local_experts + i);
 *   - num_tokens_per_expert counts slots; is_token_in_rank is an OR over slots;
 *   - rank_prefix_matrix P[s][d] = sum over s' <= s of tokens s' sends to d;
 *   - receive order: source rank ascending, then token ascending;
 *   - a non-local slot of a received row: index -1, weight 0.0;
 *   - combine sums the copies in ascending destination rank, in fp32, then
 *     rounds once to bf16 (nearest even);
 *   - low-latency: one slab row per (token, expert); rows ordered by source
 *     rank then token; quantiser amax' = max(amax, 1e-4), inv = 448 / amax',
 *     q = e4m3(x * inv), scale = amax' / 448;
 *   - low-latency combine: acc = fmaf(y, w, acc) over slots in ascending k.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <math.h>

/* ------------------------------------------------------------------------ */
/* bf16 and e4m3 scalar conversions                                         */
/* ------------------------------------------------------------------------ */

/* bf16 bits -> fp32: the bf16 pattern is the top half of the fp32 pattern. */
float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even.  Keep the top 16 bits after
 * adding half an ulp of bf16 (0x7FFF) plus the lsb of the kept part, so that
 * an exact half rounds towards the even pattern.  NaN stays NaN (quiet). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* e4m3 (OCP 8-bit floating point, E4M3 variant) bit layout S.EEEE.MMM,
 * exponent bias 7, no infinities, S.1111.111 is NaN, max finite
 * S.1111.110 = 448, subnormals E=0: (M/8) * 2^-6. */
float orc_e4m3_to_f32(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    float v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexpf((float)m / 8.0f, -6);
    else
        v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -v : v;
}

/* Round a non-negative double q to the nearest integer, ties to even. */
static double round_half_even(double q)
{
    double fl = floor(q);
    double diff = q - fl;
    if (diff > 0.5)
        return fl + 1.0;
    if (diff < 0.5)
        return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* fp32 -> e4m3: round to nearest, ties to even; magnitudes that round beyond
 * 448 saturate to 448 (sign kept); NaN -> S.1111.111.  All arithmetic below is
 * exact in double (scaling a float by a power of two). */
uint8_t orc_f32_to_e4m3(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v))
        return (uint8_t)(sign | 0x7F);
    double a = fabs((double)v);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: steps of 2^-9 */
        double m = round_half_even(a / ldexp(1.0, -9)); /* 0..8 */
        /* m == 8 is 2^-6, the smallest normal: code E=1, M=0 == 8 */
        return (uint8_t)(sign | (uint8_t)m);
    }
    int ex;
    (void)frexp(a, &ex);          /* a = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;               /* a in [2^e, 2^(e+1)) */
    double m8 = round_half_even(a / ldexp(1.0, e - 3)); /* 8..16 */
    if (m8 >= 16.0) {
        m8 = 8.0;
        e += 1;
    }
    int E = e + 7;
    int M = (int)m8 - 8;
    if (E > 15 || (E == 15 && M == 7))
        return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | (uint8_t)(E << 3) | (uint8_t)M);
}

/* Array forms of the conversions above (element by element). */
void orc_f32_to_e4m3_array(const float *v, long n, uint8_t *out)
{
    for (long i = 0; i < n; ++i)
        out[i] = orc_f32_to_e4m3(v[i]);
}

void orc_e4m3_to_f32_array(const uint8_t *c, long n, float *out)
{
    for (long i = 0; i < n; ++i)
        out[i] = orc_e4m3_to_f32(c[i]);
}

void orc_f32_to_bf16_array(const float *v, long n, uint16_t *out)
{
    for (long i = 0; i < n; ++i)
        out[i] = orc_f32_to_bf16(v[i]);
}

/* ------------------------------------------------------------------------ */
/* A1: layout                                                               */
/* ------------------------------------------------------------------------ */

/*
 * topk_idx [S][T][K] int64, -1 = unselected.  Outputs:
 *   ntpr    [S][R] int32  tokens of source s that go to rank d
 *   ntpe    [S][E] int32  slots of source s that select expert e
 *   in_rank [S][T][R] u8  1 iff some slot of (s,t) selects an expert of rank d
 * Returns the number of slots whose id is outside [-1, E) (those are ignored).
 */
long orc_layout(const int64_t *topk_idx, int S, int T, int K, int E, int R,
                int32_t *ntpr, int32_t *ntpe, uint8_t *in_rank)
{
    long bad = 0;
    int El = E / R;
    memset(ntpr, 0, sizeof(int32_t) * (size_t)S * R);
    memset(ntpe, 0, sizeof(int32_t) * (size_t)S * E);
    memset(in_rank, 0, (size_t)S * T * R);
    for (int s = 0; s < S; ++s) {
        for (int t = 0; t < T; ++t) {
            for (int k = 0; k < K; ++k) {
                int64_t e = topk_idx[((size_t)s * T + t) * K + k];
                if (e == -1)
                    continue;
                if (e < -1 || e >= E) {
                    bad++;
                    continue;
                }
                in_rank[((size_t)s * T + t) * R + e / El] = 1;
                ntpe[(size_t)s * E + e] += 1;
            }
        }
        for (int d = 0; d < R; ++d) {
            int32_t n = 0;
            for (int t = 0; t < T; ++t)
                n += in_rank[((size_t)s * T + t) * R + d];
            ntpr[(size_t)s * R + d] = n;
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* A2: rank prefix matrix and positions                                     */
/* ------------------------------------------------------------------------ */

/*
 * in_rank [R][T][R] (source, token, destination).  Outputs:
 *   P            [R][R]   P[s][d] = sum_{s' <= s} ntpr[s'][d]  (inclusive)
 *   recv_count   [R]      P[R-1][d]
 *   send_pos     [R][T][R] row of (s,t) inside destination d, or -1
 *   recv_src_idx [R][cap]  source token index of each received row (rows that
 *                          fit in cap only)
 * Rows are numbered destination by destination, source rank ascending, then
 * token ascending.  Returns the number of copies whose row is >= cap.
 */
long orc_prefix(const uint8_t *in_rank, int R, int T, int cap,
                int32_t *P, int32_t *recv_count, int32_t *send_pos,
                int32_t *recv_src_idx)
{
    long overflow = 0;
    for (int d = 0; d < R; ++d) {
        int32_t run = 0;
        for (int s = 0; s < R; ++s) {
            for (int t = 0; t < T; ++t)
                run += in_rank[((size_t)s * T + t) * R + d];
            P[(size_t)s * R + d] = run;
        }
        recv_count[d] = run;
    }
    for (int d = 0; d < R; ++d) {
        int32_t next_row = 0;
        for (int s = 0; s < R; ++s) {
            for (int t = 0; t < T; ++t) {
                size_t i = ((size_t)s * T + t) * R + d;
                if (!in_rank[i]) {
                    send_pos[i] = -1;
                    continue;
                }
                int32_t row = next_row++;
                send_pos[i] = row;
                if (row < cap)
                    recv_src_idx[(size_t)d * cap + row] = t;
                else
                    overflow++;
            }
        }
    }
    return overflow;
}

/* Receive count per local expert, rounded up to a multiple of `align`:
 * nrte[d][j] = align_up(sum_s ntpe[s][d*El + j], align).  ntpe is [S][E]. */
void orc_expert_recv_counts(const int32_t *ntpe, int S, int E, int R, int align,
                            int32_t *nrte)
{
    int El = E / R;
    for (int d = 0; d < R; ++d) {
        for (int j = 0; j < El; ++j) {
            int64_t n = 0;
            for (int s = 0; s < S; ++s)
                n += ntpe[(size_t)s * E + (size_t)d * El + j];
            if (align > 1)
                n = (n + align - 1) / align * align;
            nrte[(size_t)d * El + j] = (int32_t)n;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* A3: dispatch scatter                                                     */
/* ------------------------------------------------------------------------ */

/*
 * recv_x[d][send_pos[s][t][d]] = x[s][t] for every copy that fits in cap.
 * tokens: optional list of flat token ids s*T+t to copy (NULL = all).
 */
void orc_dispatch_rows(const uint16_t *x, const int32_t *send_pos,
                       int R, int T, int H, int cap,
                       const int64_t *tokens, long ntokens, uint16_t *recv_x)
{
    long n = tokens ? ntokens : (long)R * T;
    for (long i = 0; i < n; ++i) {
        long st = tokens ? tokens[i] : i;
        for (int d = 0; d < R; ++d) {
            int32_t row = send_pos[(size_t)st * R + d];
            if (row < 0 || row >= cap)
                continue;
            memcpy(recv_x + ((size_t)d * cap + row) * H,
                   x + (size_t)st * H, sizeof(uint16_t) * (size_t)H);
        }
    }
}

/*
 * FP8 input: recv_q[d][send_pos[s][t][d]] = x_q[s][t] (H bytes) and the
 * token's H/128 scales to recv_scales[d][row].  x_scales is [R][T][H/128], or
 * [R][H/128][T] when col_major.
 */
void orc_dispatch_rows_fp8(const uint8_t *x_q, const float *x_scales, int col_major,
                           const int32_t *send_pos, int R, int T, int H, int cap,
                           uint8_t *recv_q, float *recv_scales)
{
    int nb = H / 128;
    for (int s = 0; s < R; ++s)
        for (int t = 0; t < T; ++t) {
            size_t st = (size_t)s * T + t;
            for (int d = 0; d < R; ++d) {
                int32_t row = send_pos[st * R + d];
                if (row < 0 || row >= cap)
                    continue;
                size_t o = (size_t)d * cap + row;
                memcpy(recv_q + o * H, x_q + st * H, (size_t)H);
                for (int j = 0; j < nb; ++j)
                    recv_scales[o * nb + j] =
                        col_major ? x_scales[((size_t)s * nb + j) * T + t]
                                  : x_scales[st * nb + j];
            }
        }
}

/*
 * Received metadata.  For the copy of (s,t) held by destination d at row p:
 *   recv_topk_idx[d][p][k]     = idx - d*El if idx / El == d, else -1
 *   recv_topk_weights[d][p][k] = w          if idx / El == d, else 0.0
 * (an unselected slot, idx == -1, is never local).  Either output may be NULL.
 */
void orc_dispatch_meta(const int64_t *topk_idx, const float *topk_weights,
                       const int32_t *send_pos, int R, int T, int K, int E,
                       int cap, int64_t *recv_topk_idx, float *recv_topk_weights)
{
    int El = E / R;
    for (int s = 0; s < R; ++s) {
        for (int t = 0; t < T; ++t) {
            size_t st = (size_t)s * T + t;
            for (int d = 0; d < R; ++d) {
                int32_t row = send_pos[st * R + d];
                if (row < 0 || row >= cap)
                    continue;
                for (int k = 0; k < K; ++k) {
                    int64_t e = topk_idx[st * K + k];
                    int local = (e >= 0 && e < E && e / El == d);
                    size_t o = ((size_t)d * cap + row) * K + k;
                    if (recv_topk_idx)
                        recv_topk_idx[o] = local ? (e - (int64_t)d * El) : -1;
                    if (recv_topk_weights)
                        recv_topk_weights[o] = local ? topk_weights[st * K + k] : 0.0f;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* A4: combine                                                              */
/* ------------------------------------------------------------------------ */

/*
 * out[s][t][h] = bf16( sum over d ascending with send_pos[s][t][d] in [0,cap)
 *                      of float(y[d][send_pos][h]), then + bias0, then +
 *                      bias1 (each optional) ), accumulated in fp32 from +0.0.
 * out_w[s][t][k] = sum over the same d of recv_w[d][send_pos][k] (fp32), when
 * both recv_w and out_w are given.
 * tokens: optional list of flat token ids (NULL = all); out/out_w are indexed
 * by the flat token id in both cases.
 */
void orc_combine(const uint16_t *y, const float *recv_w, const int32_t *send_pos,
                 const uint16_t *bias0, const uint16_t *bias1,
                 int R, int T, int H, int K, int cap,
                 const int64_t *tokens, long ntokens,
                 uint16_t *out, float *out_w)
{
    long n = tokens ? ntokens : (long)R * T;
    for (long i = 0; i < n; ++i) {
        long st = tokens ? tokens[i] : i;
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int d = 0; d < R; ++d) {
                int32_t row = send_pos[(size_t)st * R + d];
                if (row < 0 || row >= cap)
                    continue;
                acc = acc + orc_bf16_to_f32(y[((size_t)d * cap + row) * H + h]);
            }
            if (bias0)
                acc = acc + orc_bf16_to_f32(bias0[(size_t)st * H + h]);
            if (bias1)
                acc = acc + orc_bf16_to_f32(bias1[(size_t)st * H + h]);
            out[(size_t)st * H + h] = orc_f32_to_bf16(acc);
        }
        if (recv_w && out_w) {
            for (int k = 0; k < K; ++k) {
                float acc = 0.0f;
                for (int d = 0; d < R; ++d) {
                    int32_t row = send_pos[(size_t)st * R + d];
                    if (row < 0 || row >= cap)
                        continue;
                    acc = acc + recv_w[((size_t)d * cap + row) * K + k];
                }
                out_w[(size_t)st * K + k] = acc;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* A5: low-latency layout, FP8 quantiser, dispatch                          */
/* ------------------------------------------------------------------------ */

/*
 * Per-expert slab positions.  For each source rank s (ascending) and token t
 * (ascending), every distinct valid expert e of the token gets the next row of
 * expert e's slab; a repeated expert in the same token reuses the row of its
 * first slot.  Outputs:
 *   count        [E]          rows of expert e (= recv count of local expert
 *                             j = e % El on rank e / El)
 *   layout_range [E][R][2]    (first row, number of rows) that source s owns
 *   ll_pos       [R][T][K]    slab row of each slot, -1 if unselected/invalid
 *   recv_src_info[E][R*T]     token index t of each row
 * Returns the number of invalid slots (outside [-1, E)).
 */
long orc_ll_layout_masked(const int64_t *topk_idx, const int32_t *mask, int R, int T,
                          int K, int E, int32_t *count, int32_t *layout_range,
                          int32_t *ll_pos, int32_t *recv_src_info);

long orc_ll_layout(const int64_t *topk_idx, int R, int T, int K, int E,
                   int32_t *count, int32_t *layout_range, int32_t *ll_pos,
                   int32_t *recv_src_info)
{
    return orc_ll_layout_masked(topk_idx, NULL, R, T, K, E, count, layout_range, ll_pos,
                                recv_src_info);
}

/*
 * As orc_ll_layout, with an optional rank mask [R] (non-zero = the rank has
 * failed, the pages' shrink mode): a masked source rank sends nothing and a
 * slot whose expert lives on a masked rank is dropped; both read ll_pos -1.
 */
long orc_ll_layout_masked(const int64_t *topk_idx, const int32_t *mask, int R, int T,
                          int K, int E, int32_t *count, int32_t *layout_range,
                          int32_t *ll_pos, int32_t *recv_src_info)
{
    long bad = 0;
    int cap = R * T;
    int El = E / R;
    for (int e = 0; e < E; ++e)
        count[e] = 0;
    for (int s = 0; s < R; ++s) {
        for (int e = 0; e < E; ++e)
            layout_range[((size_t)e * R + s) * 2 + 0] = count[e];
        for (int t = 0; t < T; ++t) {
            size_t st = (size_t)s * T + t;
            for (int k = 0; k < K; ++k) {
                int64_t e = topk_idx[st * K + k];
                if (e == -1) {
                    ll_pos[st * K + k] = -1;
                    continue;
                }
                if (e < -1 || e >= E) {
                    bad++;
                    ll_pos[st * K + k] = -1;
                    continue;
                }
                if (mask && (mask[s] || mask[e / El])) {
                    ll_pos[st * K + k] = -1;
                    continue;
                }
                int first = -1;
                for (int k2 = 0; k2 < k; ++k2)
                    if (topk_idx[st * K + k2] == e) {
                        first = k2;
                        break;
                    }
                if (first >= 0) {
                    ll_pos[st * K + k] = ll_pos[st * K + first];
                    continue;
                }
                int32_t row = count[e]++;
                ll_pos[st * K + k] = row;
                recv_src_info[(size_t)e * cap + row] = t;
            }
        }
        for (int e = 0; e < E; ++e)
            layout_range[((size_t)e * R + s) * 2 + 1] =
                count[e] - layout_range[((size_t)e * R + s) * 2 + 0];
    }
    return bad;
}

/*
 * Quantise one token row of H bf16 values (H % 128 == 0) to e4m3 with one
 * fp32 scale per 128 channels:
 *   amax  = max |x| over the block, raised to at least 1e-4
 *   inv   = 448 / amax          (fp32 division)
 *   q[i]  = e4m3(x[i] * inv)    (fp32 multiply, then nearest-even, saturate)
 *   scale = amax / 448          (fp32 division)
 */
/*
 * Variants of the per-128-channel cast:
 *   round_scale = 0: as orc_quantize_row;
 *   round_scale = 1: the scale amax' / 448 is rounded UP to a power of two
 *                    2^e (so |x| / scale <= 448), and x is multiplied by the
 *                    exact reciprocal 2^-e;
 * scales_f32 (fp32 scale per block) and/or scales_ue8m0 (the scale's biased
 * exponent byte, value 2^(byte - 127); only with round_scale) may be NULL.
 */
void orc_quantize_row_ex(const uint16_t *x, int H, int round_scale, uint8_t *q,
                         float *scales_f32, uint8_t *scales_ue8m0)
{
    for (int b = 0; b < H / 128; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 128; ++i) {
            float a = fabsf(orc_bf16_to_f32(x[b * 128 + i]));
            if (a > amax)
                amax = a;
        }
        if (amax < 1e-4f)
            amax = 1e-4f;
        float scale, inv;
        if (round_scale) {
            /* smallest power of two >= amax / 448 (a normal float here) */
            double sf = (double)(amax / 448.0f);
            int ex;
            double fr = frexp(sf, &ex);            /* sf = fr * 2^ex, fr in [0.5,1) */
            int e = (fr == 0.5) ? ex - 1 : ex;     /* 2^e >= sf, 2^(e-1) < sf */
            scale = (float)ldexp(1.0, e);
            inv = (float)ldexp(1.0, -e);
            if (scales_ue8m0)
                scales_ue8m0[b] = (uint8_t)(e + 127);
        } else {
            inv = 448.0f / amax;
            scale = amax / 448.0f;
        }
        for (int i = 0; i < 128; ++i)
            q[b * 128 + i] = orc_f32_to_e4m3(orc_bf16_to_f32(x[b * 128 + i]) * inv);
        if (scales_f32)
            scales_f32[b] = scale;
    }
}

void orc_quantize_row(const uint16_t *x, int H, uint8_t *q, float *scales)
{
    orc_quantize_row_ex(x, H, 0, q, scales, NULL);
}

/*
 * Place token rows into per-expert slabs using ll_pos.
 *   use_fp8 = 1: recv_q [E][R*T][H] e4m3 bytes, recv_scales [E][R*T][H/128]
 *   use_fp8 = 0: recv_q is [E][R*T][H] bf16 bits (uint16), scales unused
 * tokens: optional flat token list (NULL = all).
 */
void orc_ll_dispatch_rows(const uint16_t *x, const int64_t *topk_idx,
                          const int32_t *ll_pos, int R, int T, int H, int K,
                          int E, int use_fp8, const int64_t *tokens,
                          long ntokens, void *recv_q, float *recv_scales)
{
    int cap = R * T;
    long n = tokens ? ntokens : (long)R * T;
    uint8_t qrow[65536];
    float srow[512];
    for (long i = 0; i < n; ++i) {
        long st = tokens ? tokens[i] : i;
        if (use_fp8)
            orc_quantize_row(x + (size_t)st * H, H, qrow, srow);
        for (int k = 0; k < K; ++k) {
            int64_t e = topk_idx[(size_t)st * K + k];
            int32_t row = ll_pos[(size_t)st * K + k];
            if (e < 0 || e >= E || row < 0 || row >= cap)
                continue;
            size_t slot = (size_t)e * cap + row;
            if (use_fp8) {
                memcpy((uint8_t *)recv_q + slot * H, qrow, (size_t)H);
                memcpy(recv_scales + slot * (H / 128), srow,
                       sizeof(float) * (size_t)(H / 128));
            } else {
                memcpy((uint16_t *)recv_q + slot * H, x + (size_t)st * H,
                       sizeof(uint16_t) * (size_t)H);
            }
        }
    }
}

/* Dequantise e4m3 rows back to bf16: bf16(float(q) * scale). This is the
 * identity "expert" that the tests put between LL dispatch and LL combine.
 * rows: number of consecutive rows. */
void orc_dequant_rows(const uint8_t *q, const float *scales, long rows, int H,
                      uint16_t *y)
{
    for (long r = 0; r < rows; ++r)
        for (int h = 0; h < H; ++h) {
            float v = orc_e4m3_to_f32(q[(size_t)r * H + h]) *
                      scales[(size_t)r * (H / 128) + h / 128];
            y[(size_t)r * H + h] = orc_f32_to_bf16(v);
        }
}

/* ------------------------------------------------------------------------ */
/* A6: low-latency combine                                                  */
/* ------------------------------------------------------------------------ */

/*
 * out[s][t][h] = bf16(acc), acc = +0.0 then, for k ascending over valid slots
 * (0 <= idx < E and 0 <= ll_pos < R*T):
 *     acc = fmaf(float(y[idx][ll_pos][h]), w[s][t][k], acc)
 * y is [E][R*T][H] bf16 bits.  tokens: optional flat token list.
 */
void orc_ll_combine_masked(const uint16_t *y, const int64_t *topk_idx,
                           const float *topk_weights, const int32_t *ll_pos,
                           const int32_t *mask, int R, int T, int H, int K, int E,
                           const int64_t *tokens, long ntokens, uint16_t *out);

void orc_ll_combine(const uint16_t *y, const int64_t *topk_idx,
                    const float *topk_weights, const int32_t *ll_pos,
                    int R, int T, int H, int K, int E,
                    const int64_t *tokens, long ntokens, uint16_t *out)
{
    orc_ll_combine_masked(y, topk_idx, topk_weights, ll_pos, NULL, R, T, H, K, E, tokens,
                          ntokens, out);
}

/* As orc_ll_combine; with a rank mask, slots of masked source ranks and slots
 * whose expert lives on a masked rank contribute nothing. */
void orc_ll_combine_masked(const uint16_t *y, const int64_t *topk_idx,
                           const float *topk_weights, const int32_t *ll_pos,
                           const int32_t *mask, int R, int T, int H, int K, int E,
                           const int64_t *tokens, long ntokens, uint16_t *out)
{
    int cap = R * T;
    int El = E / R;
    long n = tokens ? ntokens : (long)R * T;
    for (long i = 0; i < n; ++i) {
        long st = tokens ? tokens[i] : i;
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int64_t e = topk_idx[(size_t)st * K + k];
                int32_t row = ll_pos[(size_t)st * K + k];
                if (e < 0 || e >= E || row < 0 || row >= cap)
                    continue;
                if (mask && (mask[st / T] || mask[e / El]))
                    continue;
                float v = orc_bf16_to_f32(y[((size_t)e * cap + row) * H + h]);
                acc = fmaf(v, topk_weights[(size_t)st * K + k], acc);
            }
            out[(size_t)st * H + h] = orc_f32_to_bf16(acc);
        }
    }
}
