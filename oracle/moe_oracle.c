/*
 * moe_oracle.c -- the oracle: a plain, slow, single-threaded CPU statement of
 * the Mixture-of-Experts route -> layout -> dispatch -> combine path.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check of
 * the package entry file and the CPU-baseline leg of bench.py may load it.
 * It shares no source, header, table or helper with the CUDA library; the
 * two meet only through the seeded synthetic inputs of the harness package.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (no FMA contraction, no flush-to-zero: every float operation below is one
 * IEEE-754 binary32 or binary64 operation with round-to-nearest-even).
 *
 * Sources followed (page title, then section):
 *  [EPMC] "Efficient and portable mixture-of-experts communication"
 *         (Perplexity, 2025-04-02): "Introdução" (router -> probability
 *         distribution -> top-K -> weighted average), "Despacho" (count per
 *         destination expert, contiguous per-expert buffers, source indices
 *         kept for combine), "Combinação" (gather 16-bit expert outputs,
 *         router-weighted sum at the receiver).
 *  [EFA]  "Enabling trillion-parameter models on AWS EFA" (Perplexity,
 *         2025-11-04): "Gönderme ve Alma Arabellekleri" (counts first, then
 *         offsets, contiguous sender writes, receive bound), "Dağıtım ve
 *         Birleştirme" (per-expert counts -> cumulative sums -> offsets ->
 *         pack), "Dağıtım/Birleştirme Gecikmesi" (block-scaled fp8 dispatch,
 *         bf16 combine, accumulation only at the combine receiver).
 *  [DSV3] DeepSeek-V3 report fragments quoted on the third to fifth pages:
 *         activations quantised on 1x128 tiles ("per token per 128
 *         channels"); gating kept in original precision; combine in BF16.
 *  [OFP8] OCP 8-bit Floating Point Specification (OFP8) v1.0, E4M3 format
 *         (bias 7, no infinities, S.1111.111 is NaN, max finite 448), and
 *         Micikevicius et al. 2022, "FP8 Formats for Deep Learning".
 *
 * Readings where the pages are silent (each is restated in the design notes):
 *  - top-k order and ties: sort by (logit descending, expert index ascending)
 *    with ordinary float comparison (-0 == +0).
 *  - weights: softmax over all E logits, weight = probability of the chosen
 *    expert, no renormalisation unless asked; evaluated in binary64 with libm
 *    exp and rounded once to binary32.
 *  - slot order inside an expert's receive region: ascending flat index
 *    i = g*k + j (ascending source rank, then token).
 *  - fp8 scale: s = amax / 448 (one binary32 division), s = 1 for an all-zero
 *    block; codes q = e4m3_rne_satfinite(x / s) (one binary32 division each).
 *  - combine: acc = 0; for j ascending: acc = acc + (w_j * y_j), a separate
 *    binary32 multiply and add; the output is acc rounded to bf16 (RNE).
 *
 * Parity status: every function here is pinned by the CPU tests (hand-worked
 * fixtures, brute force, torch library routines, closed-form error bounds).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_INVALID 1
#define ORACLE_ERR_CAPACITY 3

/* ------------------------------------------------------------------------ */
/* bf16 <-> binary32, written from the formats' definitions                  */
/* ------------------------------------------------------------------------ */

/* bf16 is the upper half of a binary32: widening is exact. */
static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 to bf16, nearest, ties to even.  The two candidates are
 * the value truncated to 16 bits and the next bf16 above it in magnitude; the
 * 16 dropped bits decide which is nearer, an exact half goes to the candidate
 * with an even last bit.  A carry out of the mantissa raises the exponent,
 * which is the correct next value (up to infinity). */
static uint16_t float_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) /* NaN: a quiet NaN, sign kept */
        return (uint16_t)(((u >> 16) & 0x8000u) | 0x7fc0u);
    uint32_t kept = u & 0xffff0000u;
    uint32_t dropped = u & 0x0000ffffu;
    int odd = (kept & 0x00010000u) != 0;
    if (dropped > 0x8000u || (dropped == 0x8000u && odd))
        kept += 0x00010000u;
    return (uint16_t)(kept >> 16);
}

uint16_t oracle_float_to_bf16(float f) { return float_to_bf16_rne(f); }
float oracle_bf16_to_float(uint16_t b) { return bf16_to_float(b); }

/* ------------------------------------------------------------------------ */
/* OCP E4M3 ("e4m3fn") encode / decode [OFP8]                                */
/* ------------------------------------------------------------------------ */

/* Round a non-negative double q to an integer, ties to even. */
static double round_half_even(double q)
{
    double fl = floor(q);
    double frac = q - fl; /* exact: q has few significant bits here */
    if (frac > 0.5)
        return fl + 1.0;
    if (frac < 0.5)
        return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* Encode one binary32 value as an E4M3 byte: round to nearest, ties to even,
 * saturating to the largest finite magnitude (448) instead of producing NaN.
 * E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Normal
 * values (1 + m/8) * 2^(e-7) for exponent field e in 1..15 (but S.1111.111 is
 * NaN, so the largest is 1.75 * 2^8 = 448); subnormals m/8 * 2^-6 = m * 2^-9.
 * NaN encodes as 0x7F.  The sign of zero is kept (-0 -> 0x80). */
static uint8_t e4m3_encode(float v)
{
    if (isnan(v))
        return 0x7f;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v); /* exact widening */
    if (a > 448.0)              /* includes +inf: satfinite */
        return (uint8_t)(sign | 0x7e);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: value = n * 2^-9, n in 0..8 (8 is the smallest
         * normal, whose code 0x08 continues the sequence) */
        double n = round_half_even(a * 512.0); /* exact scaling */
        return (uint8_t)(sign | (uint8_t)n);
    }
    int ex;
    double m = frexp(a, &ex); /* a = m * 2^ex, m in [0.5, 1) */
    int e = ex - 1;            /* a = (2m) * 2^e, 2m in [1, 2) */
    double n = round_half_even((2.0 * m - 1.0) * 8.0);
    if (n == 8.0) { /* mantissa rounded up to the next binade */
        n = 0.0;
        e += 1;
    }
    /* a <= 448 keeps e <= 8 and (e == 8 => n <= 6): no overflow here */
    return (uint8_t)(sign | (uint8_t)((e + 7) << 3) | (uint8_t)n);
}

/* Decode an E4M3 byte to binary32 (exact). */
static float e4m3_decode(uint8_t c)
{
    int sign = (c & 0x80) != 0;
    int ef = (c >> 3) & 0x0f;
    int mf = c & 0x07;
    double a;
    if (ef == 0x0f && mf == 0x07)
        return NAN;
    if (ef == 0)
        a = ldexp((double)mf, -9);
    else
        a = ldexp(1.0 + mf / 8.0, ef - 7);
    return (float)(sign ? -a : a);
}

uint8_t oracle_e4m3_encode(float v) { return e4m3_encode(v); }
float oracle_e4m3_decode(uint8_t c) { return e4m3_decode(c); }

void oracle_e4m3_encode_array(const float *v, int64_t n, uint8_t *q)
{
    for (int64_t i = 0; i < n; ++i)
        q[i] = e4m3_encode(v[i]);
}

/* Exhaustive-check helper: encode the binary32 whose bit pattern is
 * first_bits + i, for i in [0, n), and count the codes that differ from
 * codes[i].  The index of the first mismatch goes to *first_bad (or -1). */
int64_t oracle_e4m3_count_mismatch(uint32_t first_bits, int64_t n,
                                   const uint8_t *codes, int64_t *first_bad)
{
    int64_t bad = 0;
    *first_bad = -1;
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u = first_bits + (uint32_t)i;
        float f;
        memcpy(&f, &u, sizeof f);
        if (e4m3_encode(f) != codes[i]) {
            if (bad == 0)
                *first_bad = i;
            ++bad;
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* Route: softmax over router logits, top-k [EPMC "Introdução"; DSV3 gating  */
/* precision]                                                                */
/* ------------------------------------------------------------------------ */

typedef struct {
    float v;
    int32_t e;
} scored_t;

/* (logit descending, expert index ascending) */
static int cmp_scored(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa;
    const scored_t *b = (const scored_t *)pb;
    if (a->v > b->v)
        return -1;
    if (a->v < b->v)
        return 1;
    return (a->e < b->e) ? -1 : (a->e > b->e);
}

/* logits: [T][E] binary32.  Outputs topk_idx [T][k], topk_w [T][k].
 * For each token: the k experts first in (logit desc, index asc) order;
 * p_e = exp(l_e - m) / sum_e' exp(l_e' - m) with m = max_e l_e, in binary64,
 * the sum taken over e ascending; w_j = p_{idx_j} rounded to binary32.  With
 * renormalize: w_j = exp(l_j - m) / sum_{j'} exp(l_j' - m) over the chosen k
 * (sum in j order), i.e. the softmax restricted to the chosen experts. */
int oracle_route(const float *logits, int T, int E, int k, int renormalize,
                 int32_t *topk_idx, float *topk_w)
{
    if (T < 0 || E < 1 || k < 1 || k > E)
        return ORACLE_ERR_INVALID;
    scored_t *s = (scored_t *)malloc(sizeof(scored_t) * (size_t)E);
    if (!s)
        return ORACLE_ERR_INVALID;
    for (int g = 0; g < T; ++g) {
        const float *l = logits + (size_t)g * E;
        for (int e = 0; e < E; ++e) {
            s[e].v = l[e];
            s[e].e = e;
        }
        qsort(s, (size_t)E, sizeof(scored_t), cmp_scored);

        double m = (double)l[0];
        for (int e = 1; e < E; ++e)
            if ((double)l[e] > m)
                m = (double)l[e];
        double denom = 0.0;
        for (int e = 0; e < E; ++e)
            denom += exp((double)l[e] - m);

        double chosen_sum = 0.0;
        for (int j = 0; j < k; ++j)
            chosen_sum += exp((double)s[j].v - m);

        for (int j = 0; j < k; ++j) {
            double num = exp((double)s[j].v - m);
            topk_idx[(size_t)g * k + j] = s[j].e;
            topk_w[(size_t)g * k + j] =
                (float)(num / (renormalize ? chosen_sum : denom));
        }
    }
    free(s);
    return ORACLE_OK;
}

/* Route with shared experts and expert replicas [DSV3: during decoding the
 * shared expert is treated as a routed one that every token selects, so a
 * token selects 9 experts; redundant experts replicate heavily loaded ones].
 *
 * Routed part: exactly oracle_route over the E routed logits (top-k and
 * softmax weights, optionally renormalised over the chosen k).  Shared part:
 * the n_shared logical experts E .. E + n_shared - 1 follow in slot order,
 * each with weight shared_weight.  Every chosen logical expert l is then
 * mapped to one of its physical replicas
 *     replica_ids[replica_offsets[l] + (g / T_r) % n_rep(l)],
 *     n_rep(l) = replica_offsets[l + 1] - replica_offsets[l],
 * i.e. tokens of source rank r use replica r mod n_rep.  With no table
 * (replica_offsets == NULL) the physical id is the logical one.  A replica
 * id outside [0, E_phys) or an expert without replicas gives slot -1 and
 * ORACLE_ERR_INVALID.  Outputs are [T][k + n_shared]. */
int oracle_route_ex(const float *logits, int T, int E, int k, int renormalize,
                    int n_shared, float shared_weight,
                    const int32_t *replica_offsets, const int32_t *replica_ids,
                    int E_phys, int T_r, int32_t *topk_idx, float *topk_w)
{
    if (n_shared < 0 || T_r < 1)
        return ORACLE_ERR_INVALID;
    const int kk = k + n_shared;
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1) * k);
    float *w = (float *)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * k);
    if (!idx || !w) {
        free(idx);
        free(w);
        return ORACLE_ERR_INVALID;
    }
    int status = oracle_route(logits, T, E, k, renormalize, idx, w);
    if (status != ORACLE_OK) {
        free(idx);
        free(w);
        return status;
    }
    for (int g = 0; g < T; ++g) {
        for (int j = 0; j < kk; ++j) {
            int32_t l = (j < k) ? idx[(size_t)g * k + j] : E + (j - k);
            float wt = (j < k) ? w[(size_t)g * k + j] : shared_weight;
            int32_t phys = l;
            if (replica_offsets) {
                int32_t a = replica_offsets[l], b = replica_offsets[l + 1];
                if (b <= a) {
                    phys = -1;
                } else {
                    int32_t r = (g / T_r) % (b - a);
                    phys = replica_ids[a + r];
                }
            }
            if (phys < 0 || phys >= E_phys) {
                phys = -1;
                status = ORACLE_ERR_INVALID;
            }
            topk_idx[(size_t)g * kk + j] = phys;
            topk_w[(size_t)g * kk + j] = wt;
        }
    }
    free(idx);
    free(w);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Layout: counts -> offsets -> slots [EFA "Gönderme ve Alma Arabellekleri", */
/* "Dağıtım ve Birleştirme"; EPMC "Despacho"]                                */
/* ------------------------------------------------------------------------ */

/* topk_idx: [T][k] expert ids.  Tokens belong to R logical source ranks of
 * T/R tokens each (token g on rank g / (T/R)); experts to R logical
 * destination ranks of L = E/R experts each (expert e on rank e / L).
 *
 * capacity == 0 (packed): expert e owns rows [off_e, off_e + count_e) with
 *   off = exclusive prefix sum of the counts in expert order; rank r's region
 *   is experts [r*L, (r+1)*L).
 * capacity  > 0 (padded): expert e owns rows [e*cap, (e+1)*cap); a slot whose
 *   position within the expert reaches cap is dropped (dispatch_pos = -1)
 *   and ORACLE_ERR_CAPACITY is returned.
 * A slot holding -1 is a masked (empty) slot: skipped, not counted.  Any other
 * id outside [0, E) is skipped too and makes the call return
 * ORACLE_ERR_INVALID.
 *
 * Outputs: expert_counts[E] (slots routed to e, dropped ones included),
 * expert_src_counts[E][R], rank_counts[R] (slots routed to the rank's
 * experts), expert_offsets[E+1] (row base of e; [E] = packed total or E*cap),
 * dispatch_pos[T*k] (row of slot i = g*k+j, or -1), recv_src[rows] (i, or -1
 * for a row no slot fills). */
int oracle_layout(const int32_t *topk_idx, int T, int k, int E, int R,
                  int capacity, int64_t rows, int32_t *expert_counts,
                  int32_t *expert_src_counts, int32_t *rank_counts,
                  int32_t *expert_offsets, int32_t *dispatch_pos,
                  int32_t *recv_src)
{
    if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0 || (T > 0 && T % R != 0) ||
        capacity < 0)
        return ORACLE_ERR_INVALID;
    const int L = E / R;
    const int Tr = (T > 0) ? T / R : 1;
    int status = ORACLE_OK;

    memset(expert_counts, 0, sizeof(int32_t) * (size_t)E);
    memset(expert_src_counts, 0, sizeof(int32_t) * (size_t)E * R);
    memset(rank_counts, 0, sizeof(int32_t) * (size_t)R);

    /* pass 1: counts */
    for (int64_t i = 0; i < (int64_t)T * k; ++i) {
        int32_t e = topk_idx[i];
        if (e < 0 || e >= E) {
            if (e != -1)
                status = ORACLE_ERR_INVALID;
            continue;
        }
        int g = (int)(i / k);
        expert_counts[e] += 1;
        expert_src_counts[(size_t)e * R + g / Tr] += 1;
        rank_counts[e / L] += 1;
    }

    /* offsets */
    if (capacity == 0) {
        int32_t run = 0;
        for (int e = 0; e < E; ++e) {
            expert_offsets[e] = run;
            run += expert_counts[e];
        }
        expert_offsets[E] = run;
    } else {
        for (int e = 0; e <= E; ++e)
            expert_offsets[e] = (int32_t)((int64_t)e * capacity);
    }
    int64_t needed = (int64_t)expert_offsets[E];
    if (rows < needed)
        return ORACLE_ERR_INVALID;

    for (int64_t r = 0; r < rows; ++r)
        recv_src[r] = -1;

    /* pass 2: slots in ascending flat index */
    int32_t *seen = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (!seen)
        return ORACLE_ERR_INVALID;
    for (int64_t i = 0; i < (int64_t)T * k; ++i) {
        int32_t e = topk_idx[i];
        if (e < 0 || e >= E) {
            dispatch_pos[i] = -1;
            continue;
        }
        int32_t pos = seen[e]++;
        if (capacity > 0 && pos >= capacity) {
            dispatch_pos[i] = -1;
            if (status == ORACLE_OK)
                status = ORACLE_ERR_CAPACITY;
            continue;
        }
        int32_t row = expert_offsets[e] + pos;
        dispatch_pos[i] = row;
        recv_src[row] = (int32_t)i;
    }
    free(seen);
    return status;
}

/* Two-phase form [EPMC "Kernels portáteis": each rank keeps private storage
 * to receive from every other rank; the number of tokens a DP group may
 * dispatch is fixed, which bounds what a rank receives for each local
 * expert from each source rank, so senders derive unique addresses without
 * synchronising; after receiving, tokens are reorganised into the layout the
 * expert kernels need.  EFA "Dağıtım ve Birleştirme": the receiver computes
 * the offsets once all counts are known].
 *
 * Private region of (expert e, source rank r): rows
 * [(e*R + r)*max_m, (e*R + r + 1)*max_m).  A slot's position p in it is the
 * number of earlier slots (smaller flat index) of the same source rank
 * routed to the same expert; p >= max_m drops the slot (-1,
 * ORACLE_ERR_CAPACITY).  region_base[e][r] is the row, in the packed layout
 * of oracle_layout, of the first slot of that region:
 *   expert_offsets[e] + sum_{r' < r} expert_src_counts[e][r'].
 * recv_src_private[rows] (rows = E*R*max_m) holds the slot of each private
 * row, -1 elsewhere.  Masked (-1) and invalid ids as in oracle_layout. */
int oracle_private_layout(const int32_t *topk_idx, int T, int k, int E, int R,
                          int max_m, int32_t *private_pos, int32_t *region_base,
                          int32_t *recv_src_private)
{
    if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0 || (T > 0 && T % R != 0) ||
        max_m < 1)
        return ORACLE_ERR_INVALID;
    const int Tr = (T > 0) ? T / R : 1;
    int status = ORACLE_OK;
    int32_t *src = (int32_t *)calloc((size_t)E * R, sizeof(int32_t));
    int32_t *seen = (int32_t *)calloc((size_t)E * R, sizeof(int32_t));
    if (!src || !seen) {
        free(src);
        free(seen);
        return ORACLE_ERR_INVALID;
    }
    for (int64_t i = 0; i < (int64_t)T * k; ++i) {
        int32_t e = topk_idx[i];
        if (e >= 0 && e < E)
            src[(size_t)e * R + (i / k) / Tr] += 1;
    }
    /* packed offsets, then the base of each (expert, rank) region in them */
    int32_t run = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < R; ++r) {
            region_base[(size_t)e * R + r] = run;
            run += src[(size_t)e * R + r];
        }
    const int64_t rows = (int64_t)E * R * max_m;
    for (int64_t x = 0; x < rows; ++x)
        recv_src_private[x] = -1;
    for (int64_t i = 0; i < (int64_t)T * k; ++i) {
        int32_t e = topk_idx[i];
        if (e < 0 || e >= E) {
            if (e != -1)
                status = ORACLE_ERR_INVALID;
            private_pos[i] = -1;
            continue;
        }
        int r = (int)((i / k) / Tr);
        int32_t p = seen[(size_t)e * R + r]++;
        if (p >= max_m) {
            private_pos[i] = -1;
            if (status == ORACLE_OK)
                status = ORACLE_ERR_CAPACITY;
            continue;
        }
        int64_t row = ((int64_t)e * R + r) * max_m + p;
        private_pos[i] = (int32_t)row;
        recv_src_private[row] = (int32_t)i;
    }
    free(src);
    free(seen);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Dispatch [EFA "Dağıtım ve Birleştirme"; EPMC "Despacho"; DSV3 1x128]      */
/* ------------------------------------------------------------------------ */

/* recv_x[dispatch_pos[g*k+j]] = x[g] for every slot that has a row. */
int oracle_dispatch_bf16(const uint16_t *x, int T, int H, int k,
                         const int32_t *dispatch_pos, uint16_t *recv_x,
                         int64_t rows)
{
    int status = ORACLE_OK;
    for (int g = 0; g < T; ++g)
        for (int j = 0; j < k; ++j) {
            int32_t row = dispatch_pos[(size_t)g * k + j];
            if (row < 0)
                continue;
            if (row >= rows) {
                status = ORACLE_ERR_INVALID;
                continue;
            }
            for (int h = 0; h < H; ++h)
                recv_x[(size_t)row * H + h] = x[(size_t)g * H + h];
        }
    return status;
}

/* Quantise one token row of H bf16 values on 1x128 blocks:
 *   amax_b = max |x| over the block's 128 channels (exact in binary32),
 *   s_b    = amax_b / 448   (s_b = 1 when amax_b == 0),
 *   q      = e4m3_rne_satfinite(x / s_b). */
static void quantize_row(const uint16_t *xrow, int H, uint8_t *q, float *s)
{
    for (int b = 0; b < H / 128; ++b) {
        float amax = 0.0f;
        for (int c = 0; c < 128; ++c) {
            float a = fabsf(bf16_to_float(xrow[b * 128 + c]));
            if (a > amax)
                amax = a;
        }
        float scale = (amax == 0.0f) ? 1.0f : amax / 448.0f;
        for (int c = 0; c < 128; ++c) {
            float v = bf16_to_float(xrow[b * 128 + c]) / scale;
            q[b * 128 + c] = e4m3_encode(v);
        }
        s[b] = scale;
    }
}

/* FP8 dispatch: each token is quantised once and its codes and scales are
 * written to each of its k rows: recv_q [rows][H], recv_scale [rows][H/128]. */
int oracle_dispatch_fp8(const uint16_t *x, int T, int H, int k,
                        const int32_t *dispatch_pos, uint8_t *recv_q,
                        float *recv_scale, int64_t rows)
{
    if (H % 128 != 0)
        return ORACLE_ERR_INVALID;
    const int S = H / 128;
    int status = ORACLE_OK;
    uint8_t *q = (uint8_t *)malloc((size_t)H);
    float *s = (float *)malloc(sizeof(float) * (size_t)S);
    if (!q || !s) {
        free(q);
        free(s);
        return ORACLE_ERR_INVALID;
    }
    for (int g = 0; g < T; ++g) {
        quantize_row(x + (size_t)g * H, H, q, s);
        for (int j = 0; j < k; ++j) {
            int32_t row = dispatch_pos[(size_t)g * k + j];
            if (row < 0)
                continue;
            if (row >= rows) {
                status = ORACLE_ERR_INVALID;
                continue;
            }
            memcpy(recv_q + (size_t)row * H, q, (size_t)H);
            memcpy(recv_scale + (size_t)row * S, s, sizeof(float) * (size_t)S);
        }
    }
    free(q);
    free(s);
    return status;
}

/* Sampled form: the codes and scales of the listed tokens only,
 * q_out [n][H], s_out [n][H/128] (the bytes each of the token's rows gets). */
int oracle_quantize_tokens(const uint16_t *x, int T, int H,
                           const int32_t *tokens, int n, uint8_t *q_out,
                           float *s_out)
{
    if (H % 128 != 0)
        return ORACLE_ERR_INVALID;
    for (int i = 0; i < n; ++i) {
        int g = tokens[i];
        if (g < 0 || g >= T)
            return ORACLE_ERR_INVALID;
        quantize_row(x + (size_t)g * H, H, q_out + (size_t)i * H,
                     s_out + (size_t)i * (H / 128));
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Combine [EPMC "Combinação"; EFA "Dağıtım/Birleştirme Gecikmesi"; DSV3     */
/* combine in BF16]                                                          */
/* ------------------------------------------------------------------------ */

/* For the listed tokens (all T when tokens == NULL, n ignored):
 *   acc = 0; for j = 0..k-1 (slots with dispatch_pos = -1 skipped):
 *       acc = acc + (topk_w[g][j] * y[dispatch_pos[g][j]][h])
 * one binary32 multiply and one binary32 add per term; acc_out receives acc
 * and out its bf16 rounding.  Outputs are [n][H] in list order. */
int oracle_combine(const uint16_t *y, const int32_t *dispatch_pos,
                   const float *topk_w, int T, int H, int k, int64_t rows,
                   const int32_t *tokens, int n, float *acc_out,
                   uint16_t *out)
{
    int count = tokens ? n : T;
    for (int i = 0; i < count; ++i) {
        int g = tokens ? tokens[i] : i;
        if (g < 0 || g >= T)
            return ORACLE_ERR_INVALID;
        for (int j = 0; j < k; ++j) {
            int32_t row = dispatch_pos[(size_t)g * k + j];
            if (row >= rows)
                return ORACLE_ERR_INVALID;
        }
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int32_t row = dispatch_pos[(size_t)g * k + j];
                if (row < 0)
                    continue;
                float prod = topk_w[(size_t)g * k + j] *
                             bf16_to_float(y[(size_t)row * H + h]);
                acc = acc + prod;
            }
            if (acc_out)
                acc_out[(size_t)i * H + h] = acc;
            out[(size_t)i * H + h] = float_to_bf16_rne(acc);
        }
    }
    return ORACLE_OK;
}

/*
 * Combine with an FP8 payload: the expert rows arrive as E4M3 codes with one
 * binary32 scale per 1x128 block (the dispatch format, DeepSeek-V3
 * fragments: activations scaled per token per 128 channels).  Each element
 * is first restored as one binary32 product, v = decode(q) * s (decode is
 * exact in binary32), then summed as in oracle_combine: acc = acc + w_j * v
 * over j ascending, one multiply and one add per term, -1 slots skipped.
 *   yq [rows][H] codes, ys [rows][H/128] scales.
 */
int oracle_combine_fp8(const uint8_t *yq, const float *ys, const int32_t *dispatch_pos,
                       const float *topk_w, int T, int H, int k, int64_t rows,
                       const int32_t *tokens, int n, float *acc_out, uint16_t *out)
{
    if (H % 128 != 0)
        return ORACLE_ERR_INVALID;
    int S = H / 128;
    int count = tokens ? n : T;
    for (int i = 0; i < count; ++i) {
        int g = tokens ? tokens[i] : i;
        if (g < 0 || g >= T)
            return ORACLE_ERR_INVALID;
        for (int j = 0; j < k; ++j) {
            int32_t row = dispatch_pos[(size_t)g * k + j];
            if (row >= rows)
                return ORACLE_ERR_INVALID;
        }
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int32_t row = dispatch_pos[(size_t)g * k + j];
                if (row < 0)
                    continue;
                float v = e4m3_decode(yq[(size_t)row * H + h]) * ys[(size_t)row * S + h / 128];
                float prod = topk_w[(size_t)g * k + j] * v;
                acc = acc + prod;
            }
            if (acc_out)
                acc_out[(size_t)i * H + h] = acc;
            out[(size_t)i * H + h] = float_to_bf16_rne(acc);
        }
    }
    return ORACLE_OK;
}
