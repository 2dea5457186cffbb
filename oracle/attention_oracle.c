/*
 * attention_oracle.c -- plain, slow fp64 CPU attention used ONLY as test
 * infrastructure.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs may load it.  It shares no code, header,
 * table or helper with the CUDA library and never touches a GPU.
 *
 * What it computes is the plain definition of scaled dot-product attention
 * as the pages state it:
 *
 *   "注意力机制基础" (standard-attention tutorial), section 2.1:
 *     S = Q K^T scaled by 1/sqrt(d); upper triangle set to -inf for
 *     autoregressive use; P = row softmax(S); O = P V.
 *   "FlashAttention优化", section 2.2: the softmax in three passes -- a max
 *     pass, an exp-and-sum pass, a normalise pass.  This oracle materialises
 *     a block of S rows and runs exactly those three passes per row.
 *   "FlashAttention: Fast and Memory-Efficient Exact Attention with
 *     IO-Awareness" (paper review), 方法 item 3: the backward needs S and P,
 *     which the fast method recomputes; here they are simply recomputed by
 *     the same three-pass definition.  The backward formulas are not printed
 *     on the pages; they are the textbook derivative of the definition:
 *       dV_j = sum_i P_ij dO_i
 *       dP_ij = dO_i . V_j
 *       D_i  = sum_j P_ij dP_ij
 *       dS_ij = P_ij (dP_ij - D_i)
 *       dQ_i = scale * sum_j dS_ij K_j
 *       dK_j = scale * sum_i dS_ij Q_i
 *     with dK/dV of a key/value head summed over the query heads that share
 *     it (grouped-query attention, "FlashAttention优化" section 5.3; reading:
 *     query head h uses key/value head floor(h / (Hq/Hkv))).
 *   LSE_i = m_i + ln(l_i), natural log, in the scaled-logit domain.
 *
 * oracle_softmax_rows is the middle step of standard attention alone -- the
 * row softmax of score rows given as input -- for checking the standard-
 * attention comparator, which materialises S and P in device memory.
 *
 * The streaming variant (oracle_attention_fwd_streaming) follows the online
 * softmax recurrence of "FlashAttention优化" section 3.2.1 (running max m and
 * sum l, l_i = e^(m_{i-1}-m_i) l_{i-1} + sum exp(x_j - m_i)) together with the
 * output rescale by exp(m_old - m_new) of the paper review, 方法 item 2.  It
 * exists only so that tests can check the recurrence against the three-pass
 * definition for arbitrary tile sizes and tile orders ("FlashAttention优化"
 * section 3.2.2: any block order gives the same result).
 *
 * Layouts (all row-major, innermost dimension d):
 *   dense  (cu_seqlens == NULL): q/o/dq [B][N][Hq][d], k/v/dk/dv [B][N][Hkv][d],
 *                                lse/D [B][Hq][N]
 *   varlen (cu_seqlens != NULL): sequence s owns token rows
 *                                [cu_seqlens[s], cu_seqlens[s+1]); q/o/dq
 *                                [total][Hq][d], k/v [total][Hkv][d],
 *                                lse/D [Hq][total]
 * All arrays are double.  Masked logits are -inf; a row with no allowed key
 * (only possible for an empty sequence, which has no rows) cannot occur.
 *
 * Return value: 0 on success, -1 on invalid arguments, -2 on allocation
 * failure.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_ROW_BLOCK 64
#define ORACLE_MASK_TILE 128   /* block-mask granularity: 128 x 128 (query, key) tiles */

typedef struct {
    int B, Hq, Hkv, N, d, causal, g;
    double scale;
    const int* cu;
    /* optional block mask (dense layout only): tile (ti, tj) of sequence b
       and key/value head hk is allowed iff
       bm[b * bm_sb + hk * bm_sh + ti * bm_nt + tj] != 0 */
    const unsigned char* bm;
    long bm_sb, bm_sh;
    int bm_nt;
} shape_t;

/* number of sequences and the token range of sequence s */
static void seq_range(const shape_t* sh, int s, long* start, int* len) {
    if (sh->cu) {
        *start = sh->cu[s];
        *len = sh->cu[s + 1] - sh->cu[s];
    } else {
        *start = (long)s * sh->N;
        *len = sh->N;
    }
}

/* element offset of token row t (global token index) of head h in a tensor
   with H heads */
static long tok_off(const shape_t* sh, long t, int h, int H) {
    return (t * H + h) * (long)sh->d;
}

/* offset of the per-row statistic (lse, D) of head h, token index within
   sequence i, sequence start `start` */
static long stat_off(const shape_t* sh, int s, long start, int h, int i) {
    if (sh->cu) {
        long total = sh->cu[sh->B];
        return (long)h * total + start + i;
    }
    return ((long)s * sh->Hq + h) * sh->N + i;
}

static int check_args(const shape_t* sh) {
    if (sh->B < 0 || sh->Hq <= 0 || sh->Hkv <= 0 || sh->d <= 0 || sh->N < 0)
        return -1;
    if (sh->Hq % sh->Hkv != 0) return -1;
    if (sh->cu) {
        for (int s = 0; s < sh->B; ++s)
            if (sh->cu[s + 1] < sh->cu[s]) return -1;
        if (sh->cu[0] != 0) return -1;
    }
    return 0;
}

/* S row i of one (sequence, head): S_ij = scale * q_i . k_j, -inf where the
   causal mask removes key j > i ("注意力机制基础" 2.1). */
static void score_row(const shape_t* sh, const double* q, const double* k,
                      long start, int len, int h, int i, double* srow) {
    const int d = sh->d;
    const int hk = h / sh->g;
    const double* qi = q + tok_off(sh, start + i, h, sh->Hq);
    for (int j = 0; j < len; ++j) {
        if (sh->causal && j > i) {
            srow[j] = -INFINITY;
            continue;
        }
        if (sh->bm) {
            const long b = start / sh->N;
            if (!sh->bm[b * sh->bm_sb + hk * sh->bm_sh + (long)(i / ORACLE_MASK_TILE) * sh->bm_nt +
                        j / ORACLE_MASK_TILE]) {
                srow[j] = -INFINITY;
                continue;
            }
        }
        const double* kj = k + tok_off(sh, start + j, hk, sh->Hkv);
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
        srow[j] = sh->scale * acc;
    }
}

/* Three-pass softmax of one materialised row ("FlashAttention优化" 2.2):
   pass 1 max, pass 2 exp and sum, pass 3 normalise.  Returns the LSE. */
static double softmax_row_three_pass(const double* srow, int len, double* prow) {
    double m = -INFINITY;
    for (int j = 0; j < len; ++j)
        if (srow[j] > m) m = srow[j];
    if (m == -INFINITY) {
        /* no allowed key (a block mask can remove them all): P = 0, and the
           log of the empty sum is -inf */
        for (int j = 0; j < len; ++j) prow[j] = 0.0;
        return -INFINITY;
    }
    double l = 0.0;
    for (int j = 0; j < len; ++j) {
        double e = (srow[j] == -INFINITY) ? 0.0 : exp(srow[j] - m);
        prow[j] = e;
        l += e;
    }
    for (int j = 0; j < len; ++j) prow[j] /= l;
    return m + log(l);
}

static int nseq(const shape_t* sh) { return sh->B; }

static int attention_fwd_sh(shape_t sh, const double* q, const double* k, const double* v,
                            double* o, double* lse, int nthreads) {
    const int Hq = sh.Hq, Hkv = sh.Hkv, d = sh.d;
    if (check_args(&sh)) return -1;
    sh.g = Hq / Hkv;
    int maxlen = 0;
    for (int s = 0; s < nseq(&sh); ++s) {
        long st; int len;
        seq_range(&sh, s, &st, &len);
        if (len > maxlen) maxlen = len;
    }
    if (maxlen == 0) return 0;
    const int nrb = (maxlen + ORACLE_ROW_BLOCK - 1) / ORACLE_ROW_BLOCK;
    const long units = (long)nseq(&sh) * Hq * nrb;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        /* one materialised block of S and P rows per thread */
        double* S = (double*)malloc(sizeof(double) * ORACLE_ROW_BLOCK * (size_t)maxlen);
        double* P = (double*)malloc(sizeof(double) * ORACLE_ROW_BLOCK * (size_t)maxlen);
        if (!S || !P) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long u = 0; u < units; ++u) {
            if (!S || !P) continue;
            const int rb = (int)(u % nrb);
            const int h = (int)((u / nrb) % Hq);
            const int s = (int)(u / ((long)nrb * Hq));
            long st; int len;
            seq_range(&sh, s, &st, &len);
            const int r0 = rb * ORACLE_ROW_BLOCK;
            if (r0 >= len) continue;
            const int r1 = (r0 + ORACLE_ROW_BLOCK < len) ? r0 + ORACLE_ROW_BLOCK : len;
            const int hk = h / sh.g;
            for (int i = r0; i < r1; ++i)
                score_row(&sh, q, k, st, len, h, i, S + (size_t)(i - r0) * maxlen);
            for (int i = r0; i < r1; ++i) {
                double* srow = S + (size_t)(i - r0) * maxlen;
                double* prow = P + (size_t)(i - r0) * maxlen;
                lse[stat_off(&sh, s, st, h, i)] = softmax_row_three_pass(srow, len, prow);
                /* O_i = sum_j P_ij V_j ("注意力机制基础" 2.1, step 4) */
                double* oi = o + tok_off(&sh, st + i, h, Hq);
                for (int c = 0; c < d; ++c) oi[c] = 0.0;
                for (int j = 0; j < len; ++j) {
                    const double p = prow[j];
                    if (p == 0.0) continue;
                    const double* vj = v + tok_off(&sh, st + j, hk, Hkv);
                    for (int c = 0; c < d; ++c) oi[c] += p * vj[c];
                }
            }
        }
        free(S);
        free(P);
    }
    return err;
}

static int attention_bwd_sh(shape_t sh, const double* q, const double* k, const double* v,
                            const double* dout, double* dq, double* dk, double* dv,
                            double* o, double* lse, double* Dout, int nthreads) {
    const int Hq = sh.Hq, Hkv = sh.Hkv, d = sh.d;
    const double scale = sh.scale;
    if (check_args(&sh)) return -1;
    sh.g = Hq / Hkv;
    int maxlen = 0;
    for (int s = 0; s < nseq(&sh); ++s) {
        long st; int len;
        seq_range(&sh, s, &st, &len);
        if (len > maxlen) maxlen = len;
    }
    if (maxlen == 0) return 0;
    /* a unit is one (sequence, key/value head): it owns dK and dV of that
       head, so no two units write the same output element */
    const long units = (long)nseq(&sh) * Hkv;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* S = (double*)malloc(sizeof(double) * ORACLE_ROW_BLOCK * (size_t)maxlen);
        double* P = (double*)malloc(sizeof(double) * ORACLE_ROW_BLOCK * (size_t)maxlen);
        double* dP = (double*)malloc(sizeof(double) * (size_t)maxlen);
        if (!S || !P || !dP) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long u = 0; u < units; ++u) {
            if (!S || !P || !dP) continue;
            const int hk = (int)(u % Hkv);
            const int s = (int)(u / Hkv);
            long st; int len;
            seq_range(&sh, s, &st, &len);
            for (int j = 0; j < len; ++j) {
                double* dkj = dk + tok_off(&sh, st + j, hk, Hkv);
                double* dvj = dv + tok_off(&sh, st + j, hk, Hkv);
                for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
            }
            for (int h = hk * sh.g; h < (hk + 1) * sh.g; ++h) {
                for (int r0 = 0; r0 < len; r0 += ORACLE_ROW_BLOCK) {
                    const int r1 = (r0 + ORACLE_ROW_BLOCK < len) ? r0 + ORACLE_ROW_BLOCK : len;
                    for (int i = r0; i < r1; ++i)
                        score_row(&sh, q, k, st, len, h, i, S + (size_t)(i - r0) * maxlen);
                    for (int i = r0; i < r1; ++i) {
                        const double* srow = S + (size_t)(i - r0) * maxlen;
                        double* prow = P + (size_t)(i - r0) * maxlen;
                        const double L = softmax_row_three_pass(srow, len, prow);
                        const long so = stat_off(&sh, s, st, h, i);
                        if (lse) lse[so] = L;
                        const double* qi = q + tok_off(&sh, st + i, h, Hq);
                        const double* doi = dout + tok_off(&sh, st + i, h, Hq);
                        /* O_i, kept only as a by-product for the tests */
                        if (o) {
                            double* oi = o + tok_off(&sh, st + i, h, Hq);
                            for (int c = 0; c < d; ++c) oi[c] = 0.0;
                            for (int j = 0; j < len; ++j) {
                                if (prow[j] == 0.0) continue;
                                const double* vj = v + tok_off(&sh, st + j, hk, Hkv);
                                for (int c = 0; c < d; ++c) oi[c] += prow[j] * vj[c];
                            }
                        }
                        /* dP_ij = dO_i . V_j and D_i = sum_j P_ij dP_ij */
                        double Di = 0.0;
                        for (int j = 0; j < len; ++j) {
                            const double* vj = v + tok_off(&sh, st + j, hk, Hkv);
                            double acc = 0.0;
                            for (int c = 0; c < d; ++c) acc += doi[c] * vj[c];
                            dP[j] = acc;
                            Di += prow[j] * acc;
                        }
                        if (Dout) Dout[so] = Di;
                        double* dqi = dq + tok_off(&sh, st + i, h, Hq);
                        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
                        for (int j = 0; j < len; ++j) {
                            const double p = prow[j];
                            if (p == 0.0) continue;
                            const double ds = p * (dP[j] - Di);
                            const double* kj = k + tok_off(&sh, st + j, hk, Hkv);
                            double* dkj = dk + tok_off(&sh, st + j, hk, Hkv);
                            double* dvj = dv + tok_off(&sh, st + j, hk, Hkv);
                            for (int c = 0; c < d; ++c) {
                                dqi[c] += scale * ds * kj[c];
                                dkj[c] += scale * ds * qi[c];
                                dvj[c] += p * doi[c];
                            }
                        }
                    }
                }
            }
        }
        free(S);
        free(P);
        free(dP);
    }
    return err;
}

int oracle_attention_fwd(const double* q, const double* k, const double* v,
                         double* o, double* lse,
                         int B, int Hq, int Hkv, int N, int d, double scale,
                         int causal, const int* cu_seqlens, int nthreads) {
    shape_t sh = {B, Hq, Hkv, N, d, causal, 0, scale, cu_seqlens, NULL, 0, 0, 0};
    return attention_fwd_sh(sh, q, k, v, o, lse, nthreads);
}

int oracle_attention_bwd(const double* q, const double* k, const double* v,
                         const double* dout,
                         double* dq, double* dk, double* dv,
                         double* o, double* lse, double* Dout,
                         int B, int Hq, int Hkv, int N, int d, double scale,
                         int causal, const int* cu_seqlens, int nthreads) {
    shape_t sh = {B, Hq, Hkv, N, d, causal, 0, scale, cu_seqlens, NULL, 0, 0, 0};
    return attention_bwd_sh(sh, q, k, v, dout, dq, dk, dv, o, lse, Dout, nthreads);
}

/* Block-sparse attention (dense layout only): the same definition with S_ij
   also set to -inf when the 128 x 128 tile that holds (i, j) is not allowed
   by the block mask of the key/value head (a generalisation of the causal
   tile skipping, "FlashAttention优化" 7.2 and the paper review's block-
   sparse variant; exact on the allowed entries).  bm is
   [*][*][ceil(N/128)][ceil(N/128)] bytes with strides bm_sb per sequence
   and bm_sh per key/value head (0 broadcasts).  A row with no allowed key
   gets P = 0, O = 0 and LSE = -inf. */
int oracle_attention_fwd_blockmask(const double* q, const double* k, const double* v,
                                   double* o, double* lse,
                                   int B, int Hq, int Hkv, int N, int d, double scale,
                                   int causal, const unsigned char* bm, long bm_sb,
                                   long bm_sh, int nthreads) {
    if (!bm) return -1;
    shape_t sh = {B, Hq, Hkv, N, d, causal, 0, scale, NULL, bm, bm_sb, bm_sh,
                  (N + ORACLE_MASK_TILE - 1) / ORACLE_MASK_TILE};
    return attention_fwd_sh(sh, q, k, v, o, lse, nthreads);
}

int oracle_attention_bwd_blockmask(const double* q, const double* k, const double* v,
                                   const double* dout,
                                   double* dq, double* dk, double* dv,
                                   double* o, double* lse, double* Dout,
                                   int B, int Hq, int Hkv, int N, int d, double scale,
                                   int causal, const unsigned char* bm, long bm_sb,
                                   long bm_sh, int nthreads) {
    if (!bm) return -1;
    shape_t sh = {B, Hq, Hkv, N, d, causal, 0, scale, NULL, bm, bm_sb, bm_sh,
                  (N + ORACLE_MASK_TILE - 1) / ORACLE_MASK_TILE};
    return attention_bwd_sh(sh, q, k, v, dout, dq, dk, dv, o, lse, Dout, nthreads);
}

/* Query-row sample: O, LSE, D and dQ of the listed rows only.  Each row is
   computed from its own full S row, so the cost is O(len * d) per row.
   rows[3*r .. 3*r+2] = (sequence s, query head h, row i within sequence). */
int oracle_attention_rows(const double* q, const double* k, const double* v,
                          const double* dout, const long* rows, long nrows,
                          double* o_rows, double* lse_rows, double* D_rows,
                          double* dq_rows,
                          int B, int Hq, int Hkv, int N, int d, double scale,
                          int causal, const int* cu_seqlens, int nthreads) {
    shape_t sh = {B, Hq, Hkv, N, d, causal, 0, scale, cu_seqlens, NULL, 0, 0, 0};
    if (check_args(&sh)) return -1;
    sh.g = Hq / Hkv;
    for (long r = 0; r < nrows; ++r) {
        const long s = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        long st; int len;
        if (s < 0 || s >= B || h < 0 || h >= Hq) return -1;
        seq_range(&sh, (int)s, &st, &len);
        if (i < 0 || i >= len) return -1;
    }
    int maxlen = 0;
    for (int s = 0; s < nseq(&sh); ++s) {
        long st; int len;
        seq_range(&sh, s, &st, &len);
        if (len > maxlen) maxlen = len;
    }
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* srow = (double*)malloc(sizeof(double) * (size_t)(maxlen + 1));
        double* prow = (double*)malloc(sizeof(double) * (size_t)(maxlen + 1));
        if (!srow || !prow) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
        for (long r = 0; r < nrows; ++r) {
            if (!srow || !prow) continue;
            const int s = (int)rows[3 * r], h = (int)rows[3 * r + 1], i = (int)rows[3 * r + 2];
            const int hk = h / sh.g;
            long st; int len;
            seq_range(&sh, s, &st, &len);
            score_row(&sh, q, k, st, len, h, i, srow);
            lse_rows[r] = softmax_row_three_pass(srow, len, prow);
            double* oi = o_rows + r * d;
            for (int c = 0; c < d; ++c) oi[c] = 0.0;
            for (int j = 0; j < len; ++j) {
                if (prow[j] == 0.0) continue;
                const double* vj = v + tok_off(&sh, st + j, hk, Hkv);
                for (int c = 0; c < d; ++c) oi[c] += prow[j] * vj[c];
            }
            if (!dout) continue;
            const double* doi = dout + tok_off(&sh, st + i, h, Hq);
            double Di = 0.0;
            /* reuse srow for dP */
            for (int j = 0; j < len; ++j) {
                const double* vj = v + tok_off(&sh, st + j, hk, Hkv);
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += doi[c] * vj[c];
                srow[j] = acc;
                Di += prow[j] * acc;
            }
            D_rows[r] = Di;
            double* dqi = dq_rows + r * d;
            for (int c = 0; c < d; ++c) dqi[c] = 0.0;
            for (int j = 0; j < len; ++j) {
                if (prow[j] == 0.0) continue;
                const double ds = prow[j] * (srow[j] - Di);
                const double* kj = k + tok_off(&sh, st + j, hk, Hkv);
                for (int c = 0; c < d; ++c) dqi[c] += scale * ds * kj[c];
            }
        }
        free(srow);
        free(prow);
    }
    return err;
}

/* Online-softmax forward for ONE (sequence, head) problem given as dense
   row-major matrices q [n][d], k [n][d], v [n][d].  Keys are consumed in
   tiles of `tile` columns, in the order given by tile_order (a permutation of
   0..ntiles-1).  Per query row:
     m = -inf, l = 0, acc = 0
     for each tile: mt = tile max; m' = max(m, mt);
                    l = e^(m - m') l + sum_j exp(x_j - m');
                    acc = e^(m - m') acc + sum_j exp(x_j - m') v_j;  m = m'
     O = acc / l,  LSE = m + ln l
   ("FlashAttention优化" 3.2.1; paper review 方法 item 2). */
int oracle_attention_fwd_streaming(const double* q, const double* k, const double* v,
                                   double* o, double* lse, int n, int d,
                                   double scale, int causal, int tile,
                                   const int* tile_order) {
    if (n < 0 || d <= 0 || tile <= 0) return -1;
    const int ntiles = (n + tile - 1) / tile;
    double* x = (double*)malloc(sizeof(double) * (size_t)(tile + 1));
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    if (!x || !acc) { free(x); free(acc); return -2; }
    for (int i = 0; i < n; ++i) {
        double m = -INFINITY, l = 0.0;
        for (int c = 0; c < d; ++c) acc[c] = 0.0;
        for (int t = 0; t < ntiles; ++t) {
            const int tb = tile_order ? tile_order[t] : t;
            const int j0 = tb * tile;
            const int j1 = (j0 + tile < n) ? j0 + tile : n;
            double mt = -INFINITY;
            for (int j = j0; j < j1; ++j) {
                double s;
                if (causal && j > i) {
                    s = -INFINITY;
                } else {
                    s = 0.0;
                    for (int c = 0; c < d; ++c) s += q[(long)i * d + c] * k[(long)j * d + c];
                    s *= scale;
                }
                x[j - j0] = s;
                if (s > mt) mt = s;
            }
            const double mnew = (mt > m) ? mt : m;
            if (mnew == -INFINITY) continue; /* nothing allowed seen yet */
            const double alpha = (m == -INFINITY) ? 0.0 : exp(m - mnew);
            l *= alpha;
            for (int c = 0; c < d; ++c) acc[c] *= alpha;
            for (int j = j0; j < j1; ++j) {
                if (x[j - j0] == -INFINITY) continue;
                const double p = exp(x[j - j0] - mnew);
                l += p;
                for (int c = 0; c < d; ++c) acc[c] += p * v[(long)j * d + c];
            }
            m = mnew;
        }
        for (int c = 0; c < d; ++c) o[(long)i * d + c] = acc[c] / l;
        lse[i] = m + log(l);
    }
    free(x);
    free(acc);
    return 0;
}

/* The softmax step of standard attention on given score rows
   ("注意力机制基础" 2.1 step 3; 2.2.2: S is read back and P written):
   s holds rows of n raw scores q_i . k_j, row r belonging to query
   i = r mod n of its head; the logit is scale * s_rj, -inf for j > i when
   causal; each row then takes the three passes of softmax_row_three_pass.
   p gets P (same layout as s), lse the natural-log LSE of each row. */
int oracle_softmax_rows(const double* s, long rows, int n, double scale, int causal,
                        double* p, double* lse, int nthreads) {
    if (rows < 0 || n < 1 || !(scale > 0.0)) return -1;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)n);
        if (!x) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
        for (long r = 0; r < rows; ++r) {
            if (!x) continue;
            const long i = r % n;
            const double* srow = s + (size_t)r * n;
            for (int j = 0; j < n; ++j)
                x[j] = (causal && j > i) ? -INFINITY : scale * srow[j];
            lse[r] = softmax_row_three_pass(x, n, p + (size_t)r * n);
        }
        free(x);
    }
    return err;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
