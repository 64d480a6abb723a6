/*
 * moe_oracle.c -- CPU oracle for MoE token dispatch and combine.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this file's library.  The product path never does;
 * it shares no code, header or table with this file.
 *
 * This is a plain, slow, single-threaded statement of what the path computes,
 * written from the pages, with no blocking, fusion or reordering:
 *
 *   Dispatch ("Enabling trillion-parameter models on AWS EFA", sections
 *   "Introdução" and "MoE all-to-all sobre EFA"): take the tokens and each
 *   token's experts and group the tokens by expert.  Section "Buffers de Envio e
 *   Recebimento" and section "Despacho e Combinação" fix how: count the tokens
 *   per expert, take the cumulative sum of the counts as offsets, and pack each
 *   expert's tokens contiguously from its offset.  Inside an expert's segment the
 *   tokens are kept in (token, k) order, so the dispatch is a stable counting
 *   sort of the T*k routing entries by expert id.
 *
 *   Block fp8 ("Lower latency and higher throughput with multi-node DeepSeek
 *   deployment", section "Quantização"; the EFA article, section "Avaliação":
 *   "block-scaled fp8 dispatch"): one fp32 scale per 128-element activation
 *   vector, computed from that vector.  Scale = amax / 448 (448 is the largest
 *   finite e4m3 value), codes = e4m3(x / scale), rounded to nearest with ties to
 *   even and saturated to +-448.
 *
 *   Combine (EFA article, sections "Introdução", "Buffers de Envio e
 *   Recebimento" and "Despacho e Combinação"; DeepSeek article, section
 *   "Paralelismo de Especialistas"): gather each token's processed rows back and
 *   form the routing-weighted sum.  Evaluated here in fp64.
 *
 * Readings where the pages are silent:
 *   - weights are used as given (weighted sum, no division by their total);
 *   - an expert id outside [0, E) is dropped and flagged (error bit 1);
 *   - an entry whose slot would fall at or beyond the receive capacity is
 *     dropped and flagged (error bit 2); its slot is -1;
 *   - receive rows that hold no entry (padding, unused capacity) have
 *     recv_src = -1, and their payload is left untouched;
 *   - an all-zero 128-block gets scale 0 and all codes +0.
 */
#include <math.h>
#include <quadmath.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define ORACLE_BAD_INDEX 1
#define ORACLE_CAPACITY 2

/* A bf16 value is the upper 16 bits of an IEEE binary32. */
static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * e4m3 ("E4M3", OCP 8-bit floating point specification): 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits.  No infinities; S.1111.111 is NaN, so the
 * largest finite magnitude is S.1111.110 = 1.75 * 2^8 = 448.  Exponent field 0
 * holds the subnormals m * 2^-9 (m = 0..7); field f >= 1 holds (1 + m/8) * 2^(f-7).
 *
 * Conversion of a finite float v: round |v| to the nearest point of that grid
 * (ties to the point whose mantissa is even), clamp the result to 448, keep the
 * sign of v.
 */
uint8_t oracle_e4m3_from_float(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);

    /* Spacing of the grid around a: 2^-9 below the smallest normal 2^-6,
     * else 2^(floor(log2 a) - 3) (three mantissa bits). */
    double step;
    if (a < 0x1p-6) {
        step = 0x1p-9;
    } else {
        int e;
        frexp(a, &e);              /* a = f * 2^e with f in [0.5, 1) */
        step = ldexp(1.0, (e - 1) - 3);
    }
    /* a/step is exact (step is a power of two); nearbyint rounds ties to even
     * in the default rounding mode, and an even multiple of the step is a code
     * with an even mantissa. */
    double q = nearbyint(a / step) * step;
    if (q > 448.0)
        q = 448.0;

    uint8_t bits;
    if (q < 0x1p-6) {
        bits = (uint8_t)(q / 0x1p-9);          /* field 0, mantissa q/2^-9 */
    } else {
        int e;
        frexp(q, &e);
        int unbiased = e - 1;                  /* q = (1 + m/8) * 2^unbiased */
        int m = (int)((q / ldexp(1.0, unbiased) - 1.0) * 8.0);
        bits = (uint8_t)(((unbiased + 7) << 3) | m);
    }
    return (uint8_t)(sign | bits);
}

/*
 * Quantise one token's hidden vector (H bf16 values, H a multiple of 128) to
 * e4m3 codes with one fp32 scale per 128-element block.
 */
static void quantise_row_fp8(const uint16_t *x, int32_t H, uint8_t *codes, float *scales)
{
    for (int32_t b = 0; b < H / 128; ++b) {
        float amax = 0.0f;
        for (int32_t i = 0; i < 128; ++i) {
            float v = fabsf(bf16_to_float(x[b * 128 + i]));
            if (v > amax)
                amax = v;
        }
        if (amax == 0.0f) {
            scales[b] = 0.0f;
            for (int32_t i = 0; i < 128; ++i)
                codes[b * 128 + i] = 0x00;
            continue;
        }
        float scale = amax / 448.0f;                     /* binary32, round to nearest */
        scales[b] = scale;
        for (int32_t i = 0; i < 128; ++i) {
            float q = bf16_to_float(x[b * 128 + i]) / scale;  /* binary32, round to nearest */
            codes[b * 128 + i] = oracle_e4m3_from_float(q);
        }
    }
}

/* Rows an expert segment takes: its count, rounded up to a multiple of 128
 * when padding is on. */
static int64_t padded(int64_t count, int32_t pad128)
{
    return pad128 ? (count + 127) / 128 * 128 : count;
}

/*
 * Dispatch.  Inputs: x[T,H] bf16 bits, topk_idx[T,k].  Outputs (all written):
 *   expert_count[E], expert_offset[E+1], rank_offset[R+1], slot[T,k],
 *   recv_src[rows_cap]; payload rows recv_x[slot] (bf16 bits, or e4m3 codes
 *   with recv_scale[slot, H/128]) for every kept entry.
 * Returns the OR of the error bits.
 */
/*
 * Steps 1-4 of the dispatch (counts, offsets, rank offsets, slots and
 * recv_src); returns the error bits.
 */
int32_t oracle_dispatch_layout(int32_t T, int32_t k, int32_t E, int32_t R, int32_t pad128,
                               int64_t rows_cap, const int32_t *topk_idx,
                               int32_t *expert_count, int32_t *expert_offset,
                               int32_t *rank_offset, int32_t *recv_src, int32_t *slot)
{
    int32_t err = 0;

    /* 1. Per-expert token counts. */
    for (int32_t e = 0; e < E; ++e)
        expert_count[e] = 0;
    for (int32_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) {
            int32_t e = topk_idx[(int64_t)t * k + j];
            if (e < 0 || e >= E)
                err |= ORACLE_BAD_INDEX;
            else
                expert_count[e] += 1;
        }

    /* 2. Offsets: cumulative sum of the (optionally padded) counts. */
    expert_offset[0] = 0;
    for (int32_t e = 0; e < E; ++e)
        expert_offset[e + 1] = (int32_t)(expert_offset[e] + padded(expert_count[e], pad128));

    /* 3. Rank r hosts experts [r*E/R, (r+1)*E/R); its buffer starts where its
     *    first expert's segment starts. */
    for (int32_t r = 0; r <= R; ++r)
        rank_offset[r] = expert_offset[(int64_t)r * (E / R)];

    /* 4. Slots: walk the entries in (token, k) order; each expert hands out the
     *    next row of its segment. */
    for (int64_t i = 0; i < rows_cap; ++i)
        recv_src[i] = -1;
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int32_t e = 0; e < E; ++e)
        cursor[e] = expert_offset[e];
    for (int32_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) {
            int64_t i = (int64_t)t * k + j;
            int32_t e = topk_idx[i];
            if (e < 0 || e >= E) {
                slot[i] = -1;
                continue;
            }
            int32_t s = cursor[e]++;
            if (s >= rows_cap) {
                err |= ORACLE_CAPACITY;
                slot[i] = -1;
                continue;
            }
            slot[i] = s;
            recv_src[s] = (int32_t)i;
        }
    free(cursor);
    return err;
}

/*
 * Step 5 of the dispatch for tokens [t0, t1): the token's row (or its e4m3
 * codes and scales) to every slot.
 */
void oracle_dispatch_payload_rows(int32_t t0, int32_t t1, int32_t H, int32_t k, int32_t fp8,
                                  const uint16_t *x, const int32_t *slot, void *recv_x,
                                  float *recv_scale)
{
    int32_t nb = H / 128;
    uint8_t *codes = NULL;
    float *scales = NULL;
    if (fp8) {
        codes = (uint8_t *)malloc((size_t)(H > 0 ? H : 1));
        scales = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    }
    for (int32_t t = t0; t < t1; ++t) {
        const uint16_t *xt = x + (int64_t)t * H;
        if (fp8)
            quantise_row_fp8(xt, H, codes, scales);
        for (int32_t j = 0; j < k; ++j) {
            int32_t s = slot[(int64_t)t * k + j];
            if (s < 0)
                continue;
            if (fp8) {
                memcpy((uint8_t *)recv_x + (int64_t)s * H, codes, (size_t)H);
                memcpy(recv_scale + (int64_t)s * nb, scales, sizeof(float) * (size_t)nb);
            } else {
                memcpy((uint16_t *)recv_x + (int64_t)s * H, xt, sizeof(uint16_t) * (size_t)H);
            }
        }
    }
    free(codes);
    free(scales);
}

int32_t oracle_dispatch(int32_t T, int32_t H, int32_t k, int32_t E, int32_t R,
                        int32_t fp8, int32_t pad128, int64_t rows_cap,
                        const uint16_t *x, const int32_t *topk_idx,
                        void *recv_x, float *recv_scale,
                        int32_t *expert_count, int32_t *expert_offset,
                        int32_t *rank_offset, int32_t *recv_src, int32_t *slot)
{
    const int32_t err = oracle_dispatch_layout(T, k, E, R, pad128, rows_cap, topk_idx, expert_count,
                                               expert_offset, rank_offset, recv_src, slot);
    oracle_dispatch_payload_rows(0, T, H, k, fp8, x, slot, recv_x, recv_scale);
    return err;
}

/*
 * Combine: y[t,h] = sum_j topk_w[t,j] * expert_out[slot[t,j], h], in fp64,
 * j ascending.  Entries with slot -1 (dropped at dispatch) contribute nothing.
 */
void oracle_combine(int32_t T, int32_t H, int32_t k, const int32_t *slot,
                    const float *topk_w, const uint16_t *expert_out, double *y)
{
    for (int32_t t = 0; t < T; ++t)
        for (int32_t h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int32_t j = 0; j < k; ++j) {
                int32_t s = slot[(int64_t)t * k + j];
                if (s < 0)
                    continue;
                acc += (double)topk_w[(int64_t)t * k + j] *
                       (double)bf16_to_float(expert_out[(int64_t)s * H + h]);
            }
            y[(int64_t)t * H + h] = acc;
        }
}

/* The block quantiser alone, for one row: exposed for the tests' pins. */
void oracle_quantise_row_fp8(const uint16_t *x, int32_t H, uint8_t *codes, float *scales)
{
    quantise_row_fp8(x, H, codes, scales);
}

/* The nearest bf16 (8 significant bits, ties to even) to a double, rounded
 * once and directly, as bf16 bits.  Inputs here are finite and far from the
 * bf16 range limits. */
static uint16_t double_to_bf16(double v)
{
    if (v == 0.0)
        return signbit(v) ? 0x8000 : 0x0000;
    int e;
    double f = frexp(fabs(v), &e); /* |v| = f * 2^e, f in [0.5, 1) */
    /* 8 significant bits: units of 2^(e-8) */
    double units = nearbyint(ldexp(f, 8));
    double q = ldexp(units, e - 8);
    float qf = (float)q; /* exact: q has at most 9 significant bits */
    uint32_t u;
    memcpy(&u, &qf, sizeof u);
    uint16_t b = (uint16_t)(u >> 16);
    return (uint16_t)(signbit(v) ? (b | 0x8000) : b);
}

/*
 * Sender-side (per-rank) partial accumulation of combine.  "Enabling
 * trillion-parameter models on AWS EFA", section "Avaliação": DeepEP
 * accumulates on the sending side to move less data, which may change
 * precision.  Each rank r sums, for token t, the weighted rows of t's entries
 * whose experts it hosts (rank of expert e: e / (E/R)), and sends that partial
 * as one bf16 row; the token's home then sums the partials.
 *
 * Outputs: partial[t, q, :] (bf16 bits, q-th distinct rank of token t in order
 * of first appearance over j), partial_rank[t, q], npart[t]; and y[t, :] =
 * sum_q partial[t, q] (fp64).  Entries with slot -1 are skipped; a token with
 * no kept entry has npart 0 and y 0.
 */
void oracle_combine_rank_partial(int32_t T, int32_t H, int32_t k, int32_t E, int32_t R,
                                 const int32_t *topk_idx, const int32_t *slot,
                                 const float *topk_w, const uint16_t *expert_out,
                                 uint16_t *partial, int32_t *partial_rank, int32_t *npart,
                                 double *y)
{
    const int32_t per_rank = E / R;
    double *acc = (double *)malloc(sizeof(double) * (size_t)(H > 0 ? H : 1));
    for (int32_t t = 0; t < T; ++t) {
        int32_t n = 0;
        for (int32_t j = 0; j < k; ++j) {
            int32_t s = slot[(int64_t)t * k + j];
            if (s < 0)
                continue;
            int32_t r = topk_idx[(int64_t)t * k + j] / per_rank;
            int seen = 0;
            for (int32_t q = 0; q < n; ++q)
                if (partial_rank[(int64_t)t * k + q] == r)
                    seen = 1;
            if (seen)
                continue; /* this rank's partial was formed at its first entry */
            for (int32_t h = 0; h < H; ++h)
                acc[h] = 0.0;
            for (int32_t jj = j; jj < k; ++jj) {
                int32_t s2 = slot[(int64_t)t * k + jj];
                if (s2 < 0 || topk_idx[(int64_t)t * k + jj] / per_rank != r)
                    continue;
                for (int32_t h = 0; h < H; ++h)
                    acc[h] += (double)topk_w[(int64_t)t * k + jj] *
                              (double)bf16_to_float(expert_out[(int64_t)s2 * H + h]);
            }
            for (int32_t h = 0; h < H; ++h)
                partial[((int64_t)t * k + n) * H + h] = double_to_bf16(acc[h]);
            partial_rank[(int64_t)t * k + n] = r;
            ++n;
        }
        npart[t] = n;
        for (int32_t h = 0; h < H; ++h) {
            double sum = 0.0;
            for (int32_t q = 0; q < n; ++q)
                sum += (double)bf16_to_float(partial[((int64_t)t * k + q) * H + h]);
            y[(int64_t)t * H + h] = sum;
        }
    }
    free(acc);
}

/*
 * The activation of one (gate, up) pair: SiLU of the gate times the up value
 * ("Lower latency and higher throughput with multi-node DeepSeek deployment",
 * section "Quantização", where the SiLU kernel feeds the block quantiser).
 * Its value is the binary32 number nearest to the real number
 *
 *     silu(g) * u = g * u / (1 + e^-g),
 *
 * ties to even, with g and u the exact values of the bf16 inputs; a zero result
 * carries the sign of g * u, as an IEEE product does.  This is the plain
 * definition, written out: the quotient is evaluated in binary128 (113-bit
 * significands; g * u is exact there, e^-g comes from libquadmath's expq and
 * overflows to +inf only where the result is a signed zero anyway) and
 * converted to binary32 once.  The binary128 value is within a few units of
 * 2^-112 (relative) of the real one, so the single conversion gives the
 * nearest binary32 unless the real value lies closer than that to a point
 * halfway between two binary32 numbers; silu(g) * u is transcendental for
 * g, u != 0, so it is never exactly halfway, and the tests check the result
 * against 50-digit decimal arithmetic.  Results beyond the binary32 range
 * (|g * u| near 2^128) are out of contract.
 */
float oracle_silu_mul(float g, float u)
{
    const __float128 G = g, U = u;
    return (float)(G * U / ((__float128)1 + expq(-G)));
}

/* oracle_silu_mul over n pairs given as bf16 bits. */
void oracle_silu_mul_many(int64_t n, const uint16_t *g, const uint16_t *u, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_silu_mul(bf16_to_float(g[i]), bf16_to_float(u[i]));
}

/*
 * Expert-side activation and block quantiser ("Lower latency and higher
 * throughput with multi-node DeepSeek deployment", section "Quantização": the
 * SiLU kernel splits activations along the hidden dimension and takes the
 * largest magnitude of every 128-element block for its scale; it reads the
 * routing counts to know which rows are populated).
 *   gate_up [rows_cap, 2I] bf16: gate = columns [0, I), up = [I, 2I).
 *   a = silu(gate) * up (oracle_silu_mul), then per 128-block: scale = amax/448,
 *   codes e4m3(a/scale) as in the dispatch quantiser.
 * Only rows r < rows_in_use with recv_src[r] >= 0 are written.  Scales are
 * row-major [rows_cap, I/128] or, with col_major, [I/128, rows_cap].
 */
void oracle_silu_quant(int64_t rows_cap, int32_t I, const uint16_t *gate_up,
                       const int32_t *recv_src, int64_t rows_in_use, uint8_t *act,
                       float *act_scale, int32_t col_major)
{
    const int32_t nb = I / 128;
    float *a = (float *)malloc(sizeof(float) * (size_t)(I > 0 ? I : 1));
    if (rows_in_use > rows_cap)
        rows_in_use = rows_cap;
    for (int64_t r = 0; r < rows_in_use; ++r) {
        if (recv_src[r] < 0)
            continue;
        const uint16_t *g = gate_up + r * 2 * (int64_t)I;
        const uint16_t *u = g + I;
        for (int32_t i = 0; i < I; ++i)
            a[i] = oracle_silu_mul(bf16_to_float(g[i]), bf16_to_float(u[i]));
        for (int32_t b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int32_t i = 0; i < 128; ++i) {
                float v = fabsf(a[b * 128 + i]);
                if (v > amax)
                    amax = v;
            }
            float scale = 0.0f;
            if (amax > 0.0f)
                scale = amax / 448.0f;
            for (int32_t i = 0; i < 128; ++i)
                act[r * I + b * 128 + i] =
                    amax > 0.0f ? oracle_e4m3_from_float(a[b * 128 + i] / scale) : 0x00;
            if (col_major)
                act_scale[(int64_t)b * rows_cap + r] = scale;
            else
                act_scale[r * nb + b] = scale;
        }
    }
    free(a);
}

/*
 * Router top-k ("Lower latency and higher throughput with multi-node DeepSeek
 * deployment", section "Roteador MoE": one top-k with index tracking serves all
 * MoE models; plain top-k is the special case of group-limited top-k with a
 * single group).  For each token's logits l[0..E):
 *   - experts form n_group contiguous groups of E/n_group; a group's score is
 *     its largest logit; the topk_group best groups are kept (ties: lower
 *     group id);
 *   - the k largest logits among the kept groups' experts are chosen, best
 *     first (ties: lower expert id);
 *   - weights: score_fn 0 = softmax: exp(l_j - m) / sum, the sum over the k
 *     chosen (renormalize) or over all E logits; score_fn 1 = sigmoid:
 *     s_j = 1/(1+exp(-l_j)), divided by the sum of the chosen s (renormalize)
 *     or as is.
 * Selection compares logits only (softmax and sigmoid are increasing), so it
 * is exact; the weights are computed in fp64.
 */
void oracle_router_topk(int32_t T, int32_t E, int32_t k, const float *logits, int32_t score_fn,
                        int32_t n_group, int32_t topk_group, int32_t renormalize,
                        int32_t *topk_idx, float *topk_w)
{
    const int32_t gsize = E / n_group;
    char *group_kept = (char *)malloc((size_t)n_group);
    char *taken = (char *)malloc((size_t)E);
    for (int32_t t = 0; t < T; ++t) {
        const float *l = logits + (int64_t)t * E;
        for (int32_t g = 0; g < n_group; ++g)
            group_kept[g] = 0;
        for (int32_t pick = 0; pick < topk_group; ++pick) {
            int32_t best = -1;
            float best_score = 0.0f;
            for (int32_t g = 0; g < n_group; ++g) {
                if (group_kept[g])
                    continue;
                float gmax = l[g * gsize];
                for (int32_t i = 1; i < gsize; ++i)
                    if (l[g * gsize + i] > gmax)
                        gmax = l[g * gsize + i];
                if (best < 0 || gmax > best_score) {
                    best = g;
                    best_score = gmax;
                }
            }
            group_kept[best] = 1;
        }
        for (int32_t e = 0; e < E; ++e)
            taken[e] = 0;
        for (int32_t j = 0; j < k; ++j) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e] || !group_kept[e / gsize])
                    continue;
                if (best < 0 || l[e] > l[best])
                    best = e;
            }
            taken[best] = 1;
            topk_idx[(int64_t)t * k + j] = best;
        }
        double w[64];
        double sum = 0.0;
        if (score_fn == 0) {
            double m = l[topk_idx[(int64_t)t * k]]; /* the largest chosen logit */
            if (!renormalize)
                for (int32_t e = 0; e < E; ++e)
                    if (l[e] > m)
                        m = l[e];
            for (int32_t j = 0; j < k; ++j)
                w[j] = exp((double)l[topk_idx[(int64_t)t * k + j]] - m);
            if (renormalize)
                for (int32_t j = 0; j < k; ++j)
                    sum += w[j];
            else
                for (int32_t e = 0; e < E; ++e)
                    sum += exp((double)l[e] - m);
            for (int32_t j = 0; j < k; ++j)
                w[j] /= sum;
        } else {
            for (int32_t j = 0; j < k; ++j) {
                w[j] = 1.0 / (1.0 + exp(-(double)l[topk_idx[(int64_t)t * k + j]]));
                sum += w[j];
            }
            if (renormalize)
                for (int32_t j = 0; j < k; ++j)
                    w[j] /= sum;
        }
        for (int32_t j = 0; j < k; ++j)
            topk_w[(int64_t)t * k + j] = (float)w[j];
    }
    free(group_kept);
    free(taken);
}
