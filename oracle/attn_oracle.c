/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link,
 * load or call this file: only the tests, the smoke check and the bench's
 * CPU-baseline leg use it. It shares no code, header, table or constant with
 * the CUDA library.
 *
 * What it computes is the plain definition of attention, the "naive" three
 * steps that every page describes as the thing FlashAttention reproduces
 * exactly:
 *   - "Describe Flash Attention at a high level" (mantramindai), section
 *     "What naive attention does": S = Q K^T / sqrt(d), P = softmax(S), O = P V,
 *     each written out in full;
 *   - "How FlashAttention Speeds Up the Attention Layer" (hassanahmed.net), the
 *     three-step standard attention (S = Q K^T, P = softmax(S), O = P V);
 *   - "flashattention-memory-bound" (appliedaiprep), "A strong answer".
 * The pages insist the fast method gives the same numbers up to floating-point
 * rounding (mantramindai, "Follow-up questions to expect"; zenaique, table
 * "Output: Exact, identical"), so this definition is the oracle.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - the scale is an argument (the pages use 1/sqrt(d); one page omits it);
 *   - causal visibility is bottom-right aligned: key j is visible to query i
 *     iff j <= i + (Nkv - Nq); with Nq == Nkv this is the usual j <= i;
 *   - LSE is the natural log of the sum of exp over the visible scaled scores;
 *   - a row with no visible key has O = 0 and LSE = -inf;
 *   - the softmax subtracts the row maximum before exponentiating (the stable
 *     form in the worked example of "The two ideas", mantramindai);
 *   - split-KV partials are normalised per chunk (O_c, lse_c), and the merge is
 *     the max-and-sum trick of "Follow-up questions to expect" (mantramindai,
 *     the decode question): LSE = ln sum_c exp(lse_c), O = sum_c
 *     exp(lse_c - LSE) O_c, computed with the maximum lse_c subtracted first.
 *
 * All arithmetic is in double. bf16 inputs are widened exactly (the 16 bits
 * become the top half of an IEEE single, which converts to double exactly).
 *
 * Built with -DORACLE_MUTANT=<n> it plants one known mistake; the tests build
 * those variants to show that the pins catch each of them. The normal build
 * has ORACLE_MUTANT undefined and none of those branches.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* exact widening of a bfloat16 bit pattern */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double *widen_bf16(const uint16_t *src, size_t n) {
    double *dst = (double *)malloc(n * sizeof(double));
    if (!dst) return NULL;
    for (size_t i = 0; i < n; ++i) dst[i] = bf16_to_double(src[i]);
    return dst;
}

/* Is key j visible to query row i? (bottom-right aligned causal mask) */
static int visible(long i, long j, long Nq, long Nkv, int causal) {
    if (!causal) return 1;
#if ORACLE_MUTANT == 3 /* off-by-one: strict inequality */
    return j < i + (Nkv - Nq);
#elif ORACLE_MUTANT == 4 /* top-left aligned mask */
    (void)Nq; (void)Nkv;
    return j <= i;
#else
    return j <= i + (Nkv - Nq);
#endif
}

/*
 * Step 1 for one query row: s_j = scale * sum_c q_c k_jc for visible j,
 * -inf for masked j.
 */
static void score_row(const double *q_row, const double *k, long Nkv, long d,
                      long i, long Nq, int causal, double scale, double *s_row) {
    for (long j = 0; j < Nkv; ++j) {
        if (!visible(i, j, Nq, Nkv, causal)) {
            s_row[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (long c = 0; c < d; ++c) {
#if ORACLE_MUTANT == 2 /* wrong key row: mirrored index */
            acc += q_row[c] * k[(Nkv - 1 - j) * d + c];
#else
            acc += q_row[c] * k[j * d + c];
#endif
        }
#if ORACLE_MUTANT == 1 /* dropped scale */
        s_row[j] = acc;
#else
        s_row[j] = scale * acc;
#endif
    }
}

/*
 * Step 2 for one row: p_j = exp(s_j - m) / sum_j exp(s_j - m), m = max_j s_j.
 * Writes P over S in place and returns LSE = m + ln sum_j exp(s_j - m).
 */
static double softmax_row(double *row, long Nkv) {
    double m = -INFINITY;
    for (long j = 0; j < Nkv; ++j)
        if (row[j] > m) m = row[j];
    if (m == -INFINITY) { /* no visible key */
        for (long j = 0; j < Nkv; ++j) row[j] = 0.0;
        return -INFINITY;
    }
    double sum = 0.0;
    for (long j = 0; j < Nkv; ++j) {
#if ORACLE_MUTANT == 5 /* sign error in the exponent */
        double e = (row[j] == -INFINITY) ? 0.0 : exp(m - row[j]);
#else
        double e = exp(row[j] - m);
#endif
        row[j] = e;
        sum += e;
    }
#if ORACLE_MUTANT == 6 /* dropped normalisation */
    (void)0;
#else
    for (long j = 0; j < Nkv; ++j) row[j] /= sum;
#endif
#if ORACLE_MUTANT == 7 /* LSE without the max term */
    return log(sum);
#else
    return m + log(sum);
#endif
}

/* Step 3 for one row: o_c = sum_j p_j v_jc. */
static void pv_row(const double *p_row, const double *v, long Nkv, long d,
                   double *o_row) {
    for (long c = 0; c < d; ++c) o_row[c] = 0.0;
    for (long j = 0; j < Nkv; ++j) {
        double p = p_row[j];
        if (p == 0.0) continue;
        for (long c = 0; c < d; ++c) {
#if ORACLE_MUTANT == 8 /* transposed V operand (index read as [c, j] of a square tile) */
            o_row[c] += p * v[(c % Nkv) * d + (j % d)];
#else
            o_row[c] += p * v[j * d + c];
#endif
        }
    }
}

/*
 * Exact attention for one head in double, with S and P materialised as the
 * naive definition does (Nq x Nkv doubles; P overwrites S).
 *   q [Nq, d], k [Nkv, d], v [Nkv, d] row-major; o [Nq, d]; lse [Nq].
 *   p_out, if not NULL, receives P [Nq, Nkv].
 * Returns 0, or -1 if memory ran out or a size is invalid.
 */
int oracle_attn_head_f64(const double *q, const double *k, const double *v,
                         long Nq, long Nkv, long d, int causal, double scale,
                         double *o, double *lse, double *p_out) {
    if (Nq < 0 || Nkv < 0 || d <= 0) return -1;
    if (Nq == 0) return 0;
    double *S = (double *)malloc((size_t)Nq * (size_t)(Nkv > 0 ? Nkv : 1) * sizeof(double));
    if (!S) return -1;
    /* step 1: S = scale * Q K^T, masked */
#pragma omp parallel for schedule(dynamic, 4)
    for (long i = 0; i < Nq; ++i)
        score_row(q + i * d, k, Nkv, d, i, Nq, causal, scale, S + i * Nkv);
    /* step 2: P = softmax(S) row by row, LSE alongside */
#pragma omp parallel for schedule(dynamic, 4)
    for (long i = 0; i < Nq; ++i) lse[i] = softmax_row(S + i * Nkv, Nkv);
    /* step 3: O = P V */
#pragma omp parallel for schedule(dynamic, 4)
    for (long i = 0; i < Nq; ++i) pv_row(S + i * Nkv, v, Nkv, d, o + i * d);
    if (p_out) memcpy(p_out, S, (size_t)Nq * (size_t)Nkv * sizeof(double));
    free(S);
    return 0;
}

/*
 * Same definition on bf16 inputs [B, H, N, d] (all heads, one after another).
 * o [B, H, Nq, d] and lse [B, H, Nq] are double.
 */
int oracle_attn_fwd_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         long B, long H, long Nq, long Nkv, long d, int causal,
                         double scale, double *o, double *lse) {
    if (B < 0 || H < 0 || Nq < 0 || Nkv < 0 || d <= 0) return -1;
    for (long bh = 0; bh < B * H; ++bh) {
        double *qh = widen_bf16(q + bh * Nq * d, (size_t)(Nq * d));
        double *kh = widen_bf16(k + bh * Nkv * d, (size_t)(Nkv * d));
        double *vh = widen_bf16(v + bh * Nkv * d, (size_t)(Nkv * d));
        int rc = (qh && kh && vh) ? 0 : -1;
        if (rc == 0)
            rc = oracle_attn_head_f64(qh, kh, vh, Nq, Nkv, d, causal, scale,
                                      o + bh * Nq * d, lse + bh * Nq, NULL);
        free(qh); free(kh); free(vh);
        if (rc) return rc;
    }
    return 0;
}

/*
 * The same definition evaluated only at selected query rows of one head
 * (used where a full head would be too large to materialise). For each listed
 * row i: its row of S, its row of P, its row of O and its LSE.
 *   q_head [Nq, d], k_head/v_head [Nkv, d] as bf16 bits; rows[nrows] in [0, Nq);
 *   o [nrows, d], lse [nrows].
 */
int oracle_attn_rows_bf16(const uint16_t *q_head, const uint16_t *k_head,
                          const uint16_t *v_head, long Nq, long Nkv, long d,
                          int causal, double scale, const int64_t *rows,
                          long nrows, double *o, double *lse) {
    if (Nq <= 0 || Nkv < 0 || d <= 0 || nrows < 0) return -1;
    for (long r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= Nq) return -1;
    double *kh = widen_bf16(k_head, (size_t)(Nkv * d));
    double *vh = widen_bf16(v_head, (size_t)(Nkv * d));
    int rc = (kh && vh) ? 0 : -1;
    if (rc == 0) {
#pragma omp parallel
        {
            double *srow = (double *)malloc((size_t)(Nkv > 0 ? Nkv : 1) * sizeof(double));
            double *qrow = (double *)malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 1)
            for (long r = 0; r < nrows; ++r) {
                if (!srow || !qrow) continue;
                long i = (long)rows[r];
                for (long c = 0; c < d; ++c) qrow[c] = bf16_to_double(q_head[i * d + c]);
                score_row(qrow, kh, Nkv, d, i, Nq, causal, scale, srow);
                lse[r] = softmax_row(srow, Nkv);
                pv_row(srow, vh, Nkv, d, o + r * d);
            }
            if (!srow || !qrow) rc = -1;
            free(srow); free(qrow);
        }
    }
    free(kh); free(vh);
    return rc;
}

/*
 * Split-KV partials for one decode row (Nq = 1, no mask), the decode method of
 * "Follow-up questions to expect" (mantramindai): the keys are cut into
 * num_splits chunks of L = ceil(Nkv / num_splits) consecutive keys (the last
 * one shorter, trailing ones possibly empty); each chunk gets the exact
 * attention of the row restricted to its keys, normalised within the chunk.
 *   q_row [d], k_head/v_head [Nkv, d] bf16 bits;
 *   o_part [num_splits, d], lse_part [num_splits] (empty chunk: 0 and -inf).
 */
int oracle_decode_partials_bf16(const uint16_t *q_row, const uint16_t *k_head,
                                const uint16_t *v_head, long Nkv, long d,
                                double scale, long num_splits, double *o_part,
                                double *lse_part) {
    if (Nkv < 0 || d <= 0 || num_splits <= 0) return -1;
    long L = (Nkv + num_splits - 1) / num_splits;
    double *q = widen_bf16(q_row, (size_t)d);
    double *kh = widen_bf16(k_head, (size_t)(Nkv * d));
    double *vh = widen_bf16(v_head, (size_t)(Nkv * d));
    int rc = (q && kh && vh) ? 0 : -1;
    for (long c = 0; rc == 0 && c < num_splits; ++c) {
        long j0 = c * L, j1 = (c + 1) * L;
        if (j0 > Nkv) j0 = Nkv;
        if (j1 > Nkv) j1 = Nkv;
        long n = j1 - j0;
        if (n <= 0) {
            for (long x = 0; x < d; ++x) o_part[c * d + x] = 0.0;
            lse_part[c] = -INFINITY;
            continue;
        }
        rc = oracle_attn_head_f64(q, kh + j0 * d, vh + j0 * d, 1, n, d, 0, scale,
                                  o_part + c * d, lse_part + c, NULL);
    }
    free(q); free(kh); free(vh);
    return rc;
}

/*
 * The max-and-sum merge of normalised partials (O_c, lse_c), c < S:
 *   M = max_c lse_c;  w_c = exp(lse_c - M);  LSE = M + ln sum_c w_c;
 *   O = sum_c (w_c / sum_c w_c) O_c.
 * All chunks empty (M = -inf): O = 0, LSE = -inf.
 */
int oracle_lse_merge_f64(const double *o_part, const double *lse_part, long S,
                         long d, double *o, double *lse) {
    if (S <= 0 || d <= 0) return -1;
    double M = -INFINITY;
    for (long c = 0; c < S; ++c)
        if (lse_part[c] > M) M = lse_part[c];
    for (long x = 0; x < d; ++x) o[x] = 0.0;
    if (M == -INFINITY) {
        *lse = -INFINITY;
        return 0;
    }
    double W = 0.0;
    for (long c = 0; c < S; ++c) W += exp(lse_part[c] - M);
    for (long c = 0; c < S; ++c) {
#if ORACLE_MUTANT == 9 /* weights not normalised by their sum */
        double w = exp(lse_part[c] - M);
#else
        double w = exp(lse_part[c] - M) / W;
#endif
        if (w == 0.0) continue;
        for (long x = 0; x < d; ++x) o[x] += w * o_part[c * d + x];
    }
    *lse = M + log(W);
    return 0;
}

/* Batched merge over [B, H]: o_part [B,H,S,d], lse_part [B,H,S] as float. */
int oracle_lse_merge_f32in(const float *o_part, const float *lse_part, long BH,
                           long S, long d, double *o, double *lse) {
    if (BH < 0 || S <= 0 || d <= 0) return -1;
    int rc = 0;
#pragma omp parallel
    {
        double *op = (double *)malloc((size_t)(S * d) * sizeof(double));
        double *lp = (double *)malloc((size_t)S * sizeof(double));
#pragma omp for schedule(static)
        for (long bh = 0; bh < BH; ++bh) {
            if (!op || !lp) continue;
            for (long x = 0; x < S * d; ++x) op[x] = (double)o_part[bh * S * d + x];
            for (long c = 0; c < S; ++c) lp[c] = (double)lse_part[bh * S + c];
            oracle_lse_merge_f64(op, lp, S, d, o + bh * d, lse + bh);
        }
        if (!op || !lp) rc = -1;
        free(op); free(lp);
    }
    return rc;
}

/*
 * Paged-KV decode: one query row per (b, h) attends to the seq_lens[b] cached
 * tokens of sequence b, stored in fixed-size pages. Token j of sequence b lives
 * in physical page block_table[b][j / page_size], slot j % page_size; a page
 * holds page_size tokens of every head, laid out [num_pages][H][page_size][d].
 * (The serving variant of split-KV decode, "paged variants for decode",
 * mantramindai "Versions"; the layout is this library's reading: the pages give
 * none.) The result is the plain definition over the gathered keys; a
 * sequence with no token gives O = 0, LSE = -inf.
 *   q [B, H, d]; k_cache, v_cache [num_pages, H, page_size, d] (bf16 bits);
 *   block_table [B, max_pages]; seq_lens [B]; o [B, H, d]; lse [B, H].
 * Returns -1 on an invalid size or a table entry outside [0, num_pages).
 */
int oracle_decode_paged_bf16(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                             const int32_t *block_table, const int32_t *seq_lens, long B, long H,
                             long d, long page_size, long max_pages, long num_pages,
                             double scale, double *o, double *lse) {
    if (B < 0 || H < 0 || d <= 0 || page_size <= 0 || max_pages <= 0 || num_pages <= 0) return -1;
    for (long b = 0; b < B; ++b) {
        long n = seq_lens[b];
        if (n < 0 || n > max_pages * page_size) return -1;
#if ORACLE_MUTANT == 11 /* reads one token past the sequence */
        if (n < max_pages * page_size) n += 1;
#endif
        double *kh = (double *)malloc((size_t)((n > 0 ? n : 1) * d) * sizeof(double));
        double *vh = (double *)malloc((size_t)((n > 0 ? n : 1) * d) * sizeof(double));
        double *qh = (double *)malloc((size_t)d * sizeof(double));
        int rc = (kh && vh && qh) ? 0 : -1;
        for (long h = 0; rc == 0 && h < H; ++h) {
            for (long j = 0; j < n; ++j) {
#if ORACLE_MUTANT == 10 /* ignores the block table (logical page = physical page) */
                long page = j / page_size;
#else
                long page = block_table[b * max_pages + j / page_size];
#endif
                if (page < 0 || page >= num_pages) { rc = -1; break; }
                const uint16_t *kr = k_cache + ((page * H + h) * page_size + j % page_size) * d;
                const uint16_t *vr = v_cache + ((page * H + h) * page_size + j % page_size) * d;
                for (long c = 0; c < d; ++c) {
                    kh[j * d + c] = bf16_to_double(kr[c]);
                    vh[j * d + c] = bf16_to_double(vr[c]);
                }
            }
            if (rc) break;
            for (long c = 0; c < d; ++c) qh[c] = bf16_to_double(q[(b * H + h) * d + c]);
            if (n == 0) {
                for (long c = 0; c < d; ++c) o[(b * H + h) * d + c] = 0.0;
                lse[b * H + h] = -INFINITY;
                continue;
            }
            rc = oracle_attn_head_f64(qh, kh, vh, 1, n, d, 0, scale, o + (b * H + h) * d,
                                      lse + b * H + h, NULL);
        }
        free(kh); free(vh); free(qh);
        if (rc) return rc;
    }
    return 0;
}

/*
 * Backward pass: gradients of L = sum(dO * O) for one head, the gradients the
 * pages say FlashAttention recomputes from Q, K and V instead of storing P
 * ("Describe Flash Attention at a high level" (mantramindai), "The two ideas",
 * item 3, and "Follow-up questions to expect": outputs and gradients match
 * standard attention; "How FlashAttention Speeds Up the Attention Layer"
 * (hassanahmed.net), the backward-pass paragraph). The pages print no
 * formulas; these are the chain rule applied to the definition above, with S
 * and P materialised:
 *   dV = P^T dO;  dP = dO V^T;  D_i = sum_j P_ij dP_ij (= sum_c dO_ic O_ic);
 *   dS = P o (dP - D);  dQ = scale dS K;  dK = scale dS^T Q.
 *   q, dq [Nq, d]; k, v, dk, dv [Nkv, d]; dout [Nq, d].
 */
int oracle_attn_bwd_head_f64(const double *q, const double *k, const double *v,
                             const double *dout, long Nq, long Nkv, long d, int causal,
                             double scale, double *dq, double *dk, double *dv) {
    if (Nq < 0 || Nkv < 0 || d <= 0) return -1;
    size_t nn = (size_t)(Nq > 0 ? Nq : 1) * (size_t)(Nkv > 0 ? Nkv : 1);
    double *P = (double *)malloc(nn * sizeof(double));
    double *dS = (double *)malloc(nn * sizeof(double));
    if (!P || !dS) { free(P); free(dS); return -1; }
    /* recompute S and P */
#pragma omp parallel for schedule(dynamic, 4)
    for (long i = 0; i < Nq; ++i) {
        score_row(q + i * d, k, Nkv, d, i, Nq, causal, scale, P + i * Nkv);
        softmax_row(P + i * Nkv, Nkv);
    }
    /* dP, D and dS, row by row */
#pragma omp parallel for schedule(dynamic, 4)
    for (long i = 0; i < Nq; ++i) {
        double D = 0.0;
        for (long j = 0; j < Nkv; ++j) {
            double dp = 0.0;
            for (long c = 0; c < d; ++c) dp += dout[i * d + c] * v[j * d + c];
            dS[i * Nkv + j] = dp;
            D += P[i * Nkv + j] * dp;
        }
        for (long j = 0; j < Nkv; ++j) {
#if ORACLE_MUTANT == 12 /* dropped the D term */
            dS[i * Nkv + j] = P[i * Nkv + j] * dS[i * Nkv + j];
#else
            dS[i * Nkv + j] = P[i * Nkv + j] * (dS[i * Nkv + j] - D);
#endif
        }
    }
    /* dQ = scale dS K */
#pragma omp parallel for schedule(static)
    for (long i = 0; i < Nq; ++i)
        for (long c = 0; c < d; ++c) {
            double acc = 0.0;
            for (long j = 0; j < Nkv; ++j) acc += dS[i * Nkv + j] * k[j * d + c];
            dq[i * d + c] = scale * acc;
        }
    /* dK = scale dS^T Q, dV = P^T dO */
#pragma omp parallel for schedule(static)
    for (long j = 0; j < Nkv; ++j)
        for (long c = 0; c < d; ++c) {
            double ak = 0.0, av = 0.0;
            for (long i = 0; i < Nq; ++i) {
                ak += dS[i * Nkv + j] * q[i * d + c];
                av += P[i * Nkv + j] * dout[i * d + c];
            }
#if ORACLE_MUTANT == 13 /* dK without the scale */
            dk[j * d + c] = ak;
#else
            dk[j * d + c] = scale * ak;
#endif
            dv[j * d + c] = av;
        }
    free(P); free(dS);
    return 0;
}

/* Backward on bf16 inputs [B, H, N, d]; dq [B,H,Nq,d], dk and dv [B,H,Nkv,d] double. */
int oracle_attn_bwd_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const uint16_t *dout, long B, long H, long Nq, long Nkv, long d,
                         int causal, double scale, double *dq, double *dk, double *dv) {
    if (B < 0 || H < 0 || Nq < 0 || Nkv < 0 || d <= 0) return -1;
    for (long bh = 0; bh < B * H; ++bh) {
        double *qh = widen_bf16(q + bh * Nq * d, (size_t)(Nq * d));
        double *kh = widen_bf16(k + bh * Nkv * d, (size_t)(Nkv * d));
        double *vh = widen_bf16(v + bh * Nkv * d, (size_t)(Nkv * d));
        double *oh = widen_bf16(dout + bh * Nq * d, (size_t)(Nq * d));
        int rc = (qh && kh && vh && oh) ? 0 : -1;
        if (rc == 0)
            rc = oracle_attn_bwd_head_f64(qh, kh, vh, oh, Nq, Nkv, d, causal, scale,
                                          dq + bh * Nq * d, dk + bh * Nkv * d, dv + bh * Nkv * d);
        free(qh); free(kh); free(vh); free(oh);
        if (rc) return rc;
    }
    return 0;
}

/*
 * 8-bit inputs. The pages name an FP8 path (mantramindai "Versions";
 * hassanahmed.net, the FlashAttention-3 paragraph) but no format; the reading
 * used here: OCP FP8 E4M3 codes with one descale factor per (b, h) and
 * tensor, a code c standing for descale * value(c). The oracle decodes each
 * code from the format's definition and evaluates the same exact attention
 * on the decoded values; how a kernel rounds P internally is not its concern.
 *
 * E4M3: bit 7 sign, bits 3-6 exponent with bias 7, bits 0-2 mantissa. An
 * exponent field of 0 is subnormal (mantissa/8 * 2^-6); exponent 15 with
 * mantissa 7 is NaN; there are no infinities (so 0x7E = 448 is the largest).
 */
static double e4m3_to_double(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
#if ORACLE_MUTANT == 14 /* exponent bias 8 instead of 7 */
    const int bias = 8;
#else
    const int bias = 7;
#endif
    const double mag = (e == 0) ? ldexp((double)m / 8.0, 1 - bias)
                                : ldexp(1.0 + (double)m / 8.0, e - bias);
    return sign ? -mag : mag;
}

/* decoded values of n codes (for the pins) */
void oracle_e4m3_decode(const uint8_t *codes, long n, double *out) {
    for (long i = 0; i < n; ++i) out[i] = e4m3_to_double(codes[i]);
}

static double *widen_e4m3(const uint8_t *src, size_t n, double descale) {
    double *dst = (double *)malloc(n * sizeof(double));
    if (!dst) return NULL;
    for (size_t i = 0; i < n; ++i) dst[i] = descale * e4m3_to_double(src[i]);
    return dst;
}

/*
 * Exact attention on e4m3 inputs [B, H, N, d] with descale factors [B, H]
 * (fp32, widened exactly). o [B, H, Nq, d] and lse [B, H, Nq] are double.
 */
int oracle_attn_fwd_fp8(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                        const float *q_descale, const float *k_descale,
                        const float *v_descale, long B, long H, long Nq, long Nkv, long d,
                        int causal, double scale, double *o, double *lse) {
    if (B < 0 || H < 0 || Nq < 0 || Nkv < 0 || d <= 0) return -1;
    for (long bh = 0; bh < B * H; ++bh) {
#if ORACLE_MUTANT == 15 /* V's descale factor ignored */
        const double dv = 1.0;
#else
        const double dv = (double)v_descale[bh];
#endif
        double *qh = widen_e4m3(q + bh * Nq * d, (size_t)(Nq * d), (double)q_descale[bh]);
        double *kh = widen_e4m3(k + bh * Nkv * d, (size_t)(Nkv * d), (double)k_descale[bh]);
        double *vh = widen_e4m3(v + bh * Nkv * d, (size_t)(Nkv * d), dv);
        int rc = (qh && kh && vh) ? 0 : -1;
        if (rc == 0)
            rc = oracle_attn_head_f64(qh, kh, vh, Nq, Nkv, d, causal, scale,
                                      o + bh * Nq * d, lse + bh * Nq, NULL);
        free(qh); free(kh); free(vh);
        if (rc) return rc;
    }
    return 0;
}

/* number of OpenMP threads the oracle will use (1 without OpenMP) */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
