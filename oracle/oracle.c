/*
 * oracle.c -- plain fp64 CPU oracle for block-sparse and index-sparse softmax
 * attention (forward O and LSE, backward dQ, dK and dV) and for the conversion of
 * token-level top-k indices or block masks into per-tile block lists.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code, header,
 * table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes.  The pages this project follows print no formulas for the
 * attention itself; they name the operation ("IndexSparse / BlockSparse
 * attention", MagiAttention PR #334, Summary and section 2) and describe the
 * online-softmax recurrence a kernel uses to reach it (nvfp4-megamoe-kernel commit
 * log, multi-row softmax notes).  The result that recurrence reaches is the
 * textbook softmax attention restricted to an allowed key set, written out here
 * directly, row by row, with no tiling and no online rescaling:
 *
 *   s_ij   = scale * <q_i, k_j>                      for j in A_i
 *   LSE_i  = log sum_{j in A_i} exp(s_ij)            (natural log; -inf if A_i empty)
 *   P_ij   = exp(s_ij - LSE_i)
 *   O_i    = sum_{j in A_i} P_ij v_j                 (0 if A_i empty)
 *   Delta_i = <dO_i, O_i>
 *   dP_ij  = <dO_i, v_j>
 *   dS_ij  = P_ij (dP_ij - Delta_i)
 *   dq_i   = scale * sum_j dS_ij k_j
 *   dk_j   = scale * sum_{h in group(g)} sum_i dS_ij q_i
 *   dv_j   = sum_{h in group(g)} sum_i P_ij dO_i
 *
 * Query head h reads key/value head g = h / (HQ / HK) (grouped-query attention).
 *
 * The allowed set A_i for query i of batch b under KV head g:
 *   dense       : every key j < Sk
 *   block mask  : mask[b][g][i / bs][j / bs] != 0                (block granularity bs)
 *   index       : { idx[b][i][g][t] : t < topk, idx != -1 }      (a set: duplicates collapse,
 *                 as the "presence matrix" built with scatter_ in MagiAttention PR #334,
 *                 section 2, implies; -1 is padding as in xtuner PR #2096, Main Changes 1)
 *   and, when causal, additionally j <= i (top-left alignment).
 *
 * Block lists.  For the tile size T (128), tile (mt, nt) of (b, g) is
 *   FULL     if every (i, j) in it with i < Sq, j < Sk is allowed and the tile lies
 *            wholly inside [0, Sk) along j,
 *   PARTIAL  if some but not all such (i, j) are allowed (or the FULL test fails only
 *            because the tile crosses Sk),
 *   absent   if none is allowed.
 * Forward lists: per (b, g, mt) the FULL n-tiles ascending, then the PARTIAL n-tiles
 * ascending, then -1 fill; counts (n_full, n_partial).  Backward lists: the same per
 * (b, g, nt) over m-tiles (the transposed, key-to-query lists of MagiAttention PR #331,
 * "CSR Tile Mapping").  Index mode also returns the presence bitmap
 * [b][g][i][ceil(Sk/32)] with bit j%32 of word j/32 set iff j is one of row i's indices.
 *
 * Inputs and outputs are fp64 (the benchmark's inputs are bf16 values, widened exactly).
 * Layouts: q [B][Sq][HQ][Dqk], k [B][Sk][HK][Dqk], v [B][Sk][HK][Dv],
 * o / dO [B][Sq][HQ][Dv], LSE / Delta [B][HQ][Sq].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_DENSE 0
#define OR_BLOCK 1
#define OR_INDEX 2

#define OR_OK 0
#define OR_ERR_ARG (-1)
#define OR_ERR_INDEX (-3)
#define OR_ERR_NOMEM (-4)

typedef struct {
    int64_t B, Sq, Sk, HQ, HK, Dqk, Dv;
    double scale;
    int64_t causal;
    int64_t mode;
    const uint8_t *mask; /* block mode: [B][HK][Mb][Nb] */
    int64_t bs, Mb, Nb;
    const int32_t *idx; /* index mode: [B][Sq][HK][topk] */
    int64_t topk;
} or_problem;

static int check_problem(const or_problem *p)
{
    if (p->B < 0 || p->Sq < 0 || p->Sk < 0 || p->HQ <= 0 || p->HK <= 0) return OR_ERR_ARG;
    if (p->HQ % p->HK != 0) return OR_ERR_ARG;
    if (p->mode == OR_BLOCK) {
        if (!p->mask || p->bs <= 0) return OR_ERR_ARG;
        if (p->Mb * p->bs < p->Sq || p->Nb * p->bs < p->Sk) return OR_ERR_ARG;
    } else if (p->mode == OR_INDEX) {
        if (!p->idx || p->topk < 0) return OR_ERR_ARG;
        for (int64_t e = 0; e < p->B * p->Sq * p->HK * p->topk; ++e)
            if (p->idx[e] < -1 || p->idx[e] >= p->Sk) return OR_ERR_INDEX;
    } else if (p->mode != OR_DENSE) {
        return OR_ERR_ARG;
    }
    return OR_OK;
}

/* Point membership test: is key j in A_i for (b, g)?  Index mode scans the row. */
static int is_allowed(const or_problem *p, int64_t b, int64_t g, int64_t i, int64_t j)
{
    if (i < 0 || i >= p->Sq || j < 0 || j >= p->Sk) return 0;
    if (p->causal && j > i) return 0;
    if (p->mode == OR_BLOCK)
        return p->mask[((b * p->HK + g) * p->Mb + i / p->bs) * p->Nb + j / p->bs] != 0;
    if (p->mode == OR_INDEX) {
        const int32_t *row = p->idx + ((b * p->Sq + i) * p->HK + g) * p->topk;
        for (int64_t t = 0; t < p->topk; ++t)
            if (row[t] == j) return 1;
        return 0;
    }
    return 1;
}

/* The allowed keys of query i, ascending, written to keys[]; returns how many.
 * flag[] is Sk bytes of scratch (index mode builds the row's set in it). */
static int64_t allowed_keys(const or_problem *p, int64_t b, int64_t g, int64_t i,
                            int64_t *keys, uint8_t *flag)
{
    int64_t n = 0;
    if (p->mode == OR_INDEX) {
        memset(flag, 0, (size_t)p->Sk);
        const int32_t *row = p->idx + ((b * p->Sq + i) * p->HK + g) * p->topk;
        for (int64_t t = 0; t < p->topk; ++t)
            if (row[t] >= 0) flag[row[t]] = 1;
        for (int64_t j = 0; j < p->Sk; ++j)
            if (flag[j] && (!p->causal || j <= i)) keys[n++] = j;
        return n;
    }
    for (int64_t j = 0; j < p->Sk; ++j)
        if (is_allowed(p, b, g, i, j)) keys[n++] = j;
    return n;
}

static double dot(const double *a, const double *b, int64_t n)
{
    double acc = 0.0;
    for (int64_t d = 0; d < n; ++d) acc += a[d] * b[d];
    return acc;
}

static const double *q_row(const or_problem *p, const double *q, int64_t b, int64_t h, int64_t i)
{
    return q + ((b * p->Sq + i) * p->HQ + h) * p->Dqk;
}
static const double *k_row(const or_problem *p, const double *k, int64_t b, int64_t g, int64_t j)
{
    return k + ((b * p->Sk + j) * p->HK + g) * p->Dqk;
}
static const double *v_row(const or_problem *p, const double *v, int64_t b, int64_t g, int64_t j)
{
    return v + ((b * p->Sk + j) * p->HK + g) * p->Dv;
}
static const double *do_row(const or_problem *p, const double *dout, int64_t b, int64_t h, int64_t i)
{
    return dout + ((b * p->Sq + i) * p->HQ + h) * p->Dv;
}

/*
 * Forward for a list of query rows.  rows holds n_rows triplets (b, h, i); o receives
 * n_rows x Dv values and lse n_rows values.  LSE = max + log(sum exp(s - max)), the
 * same number as log(sum exp(s)) without overflow.
 */
int oracle_fwd_rows(const or_problem *p, const double *q, const double *k, const double *v,
                    int64_t n_rows, const int64_t *rows, double *o, double *lse)
{
    int rc = check_problem(p);
    if (rc) return rc;
    const int64_t G = p->HQ / p->HK;
    int failed = 0;
#pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(p->Sk + 1));
        uint8_t *flag = (uint8_t *)malloc((size_t)p->Sk + 1);
        double *s = (double *)malloc(sizeof(double) * (size_t)(p->Sk + 1));
        if (!keys || !flag || !s) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            if (failed) continue;
            const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            const int64_t g = h / G;
            double *orow = o + r * p->Dv;
            for (int64_t d = 0; d < p->Dv; ++d) orow[d] = 0.0;
            const int64_t n = allowed_keys(p, b, g, i, keys, flag);
            if (n == 0) {
                lse[r] = -INFINITY;
                continue;
            }
            const double *qi = q_row(p, q, b, h, i);
            double m = -INFINITY;
            for (int64_t t = 0; t < n; ++t) {
                s[t] = p->scale * dot(qi, k_row(p, k, b, g, keys[t]), p->Dqk);
                if (s[t] > m) m = s[t];
            }
            double sum = 0.0;
            for (int64_t t = 0; t < n; ++t) sum += exp(s[t] - m);
            const double L = m + log(sum);
            lse[r] = L;
            for (int64_t t = 0; t < n; ++t) {
                const double pij = exp(s[t] - L);
                const double *vj = v_row(p, v, b, g, keys[t]);
                for (int64_t d = 0; d < p->Dv; ++d) orow[d] += pij * vj[d];
            }
        }
        free(keys);
        free(flag);
        free(s);
    }
    return failed ? OR_ERR_NOMEM : OR_OK;
}

/* Delta_i = <dO_i, O_i> for a list of rows, O given per row (n_rows x Dv, fp64). */
int oracle_delta_rows(const or_problem *p, const double *dout, int64_t n_rows, const int64_t *rows,
                      const double *o, double *delta)
{
    for (int64_t r = 0; r < n_rows; ++r) {
        const double *dorow = do_row(p, dout, rows[3 * r], rows[3 * r + 1], rows[3 * r + 2]);
        double acc = 0.0;
        for (int64_t d = 0; d < p->Dv; ++d) acc += dorow[d] * o[r * p->Dv + d];
        delta[r] = acc;
    }
    return OR_OK;
}

/*
 * dQ for a list of query rows (b, h, i).  lse and delta are full [B][HQ][Sq] arrays
 * (fp64, as returned by the oracle's forward and delta); dq receives n_rows x Dqk.
 */
int oracle_bwd_rows(const or_problem *p, const double *q, const double *k, const double *v,
                    const double *dout, const double *lse, const double *delta,
                    int64_t n_rows, const int64_t *rows, double *dq)
{
    int rc = check_problem(p);
    if (rc) return rc;
    const int64_t G = p->HQ / p->HK;
    int failed = 0;
#pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(p->Sk + 1));
        uint8_t *flag = (uint8_t *)malloc((size_t)p->Sk + 1);
        if (!keys || !flag) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            if (failed) continue;
            const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            const int64_t g = h / G;
            double *dqrow = dq + r * p->Dqk;
            for (int64_t d = 0; d < p->Dqk; ++d) dqrow[d] = 0.0;
            const int64_t n = allowed_keys(p, b, g, i, keys, flag);
            if (n == 0) continue;
            const double L = lse[(b * p->HQ + h) * p->Sq + i];
            const double Di = delta[(b * p->HQ + h) * p->Sq + i];
            const double *qi = q_row(p, q, b, h, i);
            const double *doi = do_row(p, dout, b, h, i);
            for (int64_t t = 0; t < n; ++t) {
                const double *kj = k_row(p, k, b, g, keys[t]);
                const double pij = exp(p->scale * dot(qi, kj, p->Dqk) - L);
                const double dpij = dot(doi, v_row(p, v, b, g, keys[t]), p->Dv);
                const double dsij = pij * (dpij - Di);
                for (int64_t d = 0; d < p->Dqk; ++d) dqrow[d] += p->scale * dsij * kj[d];
            }
        }
        free(keys);
        free(flag);
    }
    return failed ? OR_ERR_NOMEM : OR_OK;
}

/*
 * dK and dV for a list of keys (b, g, j): sums over every query head of the group and
 * every query i whose allowed set holds j.  dk receives n_keys x Dqk, dv n_keys x Dv.
 */
int oracle_bwd_keys(const or_problem *p, const double *q, const double *k, const double *v,
                    const double *dout, const double *lse, const double *delta,
                    int64_t n_keys, const int64_t *keys, double *dk, double *dv)
{
    int rc = check_problem(p);
    if (rc) return rc;
    const int64_t G = p->HQ / p->HK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_keys; ++r) {
        const int64_t b = keys[3 * r], g = keys[3 * r + 1], j = keys[3 * r + 2];
        double *dkrow = dk + r * p->Dqk;
        double *dvrow = dv + r * p->Dv;
        for (int64_t d = 0; d < p->Dqk; ++d) dkrow[d] = 0.0;
        for (int64_t d = 0; d < p->Dv; ++d) dvrow[d] = 0.0;
        const double *kj = k_row(p, k, b, g, j);
        const double *vj = v_row(p, v, b, g, j);
        for (int64_t h = g * G; h < (g + 1) * G; ++h) {
            for (int64_t i = 0; i < p->Sq; ++i) {
                if (!is_allowed(p, b, g, i, j)) continue;
                const double L = lse[(b * p->HQ + h) * p->Sq + i];
                const double Di = delta[(b * p->HQ + h) * p->Sq + i];
                const double *qi = q_row(p, q, b, h, i);
                const double *doi = do_row(p, dout, b, h, i);
                const double pij = exp(p->scale * dot(qi, kj, p->Dqk) - L);
                const double dpij = dot(doi, vj, p->Dv);
                const double dsij = pij * (dpij - Di);
                for (int64_t d = 0; d < p->Dqk; ++d) dkrow[d] += p->scale * dsij * qi[d];
                for (int64_t d = 0; d < p->Dv; ++d) dvrow[d] += pij * doi[d];
            }
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------------ */
/* Block lists                                                                     */
/* ------------------------------------------------------------------------------ */

/*
 * Presence bitmap of index mode: bitmap[b][g][i][w], w < ceil(Sk/32); bit j%32 of
 * word j/32 is set iff j is one of row (b, i, g)'s indices.  Causality is not folded
 * in: the bitmap is the index set only.
 */
int oracle_presence_bitmap(const or_problem *p, uint32_t *bitmap)
{
    if (p->mode != OR_INDEX) return OR_ERR_ARG;
    int rc = check_problem(p);
    if (rc) return rc;
    const int64_t W = (p->Sk + 31) / 32;
    memset(bitmap, 0, sizeof(uint32_t) * (size_t)(p->B * p->HK * p->Sq * W));
    for (int64_t b = 0; b < p->B; ++b)
        for (int64_t i = 0; i < p->Sq; ++i)
            for (int64_t g = 0; g < p->HK; ++g)
                for (int64_t t = 0; t < p->topk; ++t) {
                    const int32_t j = p->idx[((b * p->Sq + i) * p->HK + g) * p->topk + t];
                    if (j == -1) continue;
                    bitmap[((b * p->HK + g) * p->Sq + i) * W + j / 32] |= 1u << (j % 32);
                }
    return OR_OK;
}

/* 0 = absent, 1 = partial, 2 = full: the tile classification stated in the header. */
static int classify_tile(const or_problem *p, const uint32_t *bitmap, int64_t T,
                         int64_t b, int64_t g, int64_t mt, int64_t nt)
{
    const int64_t W = (p->Sk + 31) / 32;
    int any = 0, all = 1;
    for (int64_t i = mt * T; i < (mt + 1) * T && i < p->Sq; ++i) {
        for (int64_t j = nt * T; j < (nt + 1) * T && j < p->Sk; ++j) {
            int a;
            if (p->mode == OR_INDEX)
                a = ((bitmap[((b * p->HK + g) * p->Sq + i) * W + j / 32] >> (j % 32)) & 1u) &&
                    (!p->causal || j <= i);
            else
                a = is_allowed(p, b, g, i, j);
            any |= a;
            all &= a;
        }
    }
    if ((nt + 1) * T > p->Sk) all = 0;
    return any ? (all ? 2 : 1) : 0;
}

/*
 * Forward and backward tile lists.  With Tm = ceil(Sq/T), Tn = ceil(Sk/T):
 *   cnt  [B][HK][Tm][2]   (n_full, n_partial)      idx  [B][HK][Tm][Tn]
 *   tcnt [B][HK][Tn][2]                             tidx [B][HK][Tn][Tm]
 * bitmap: index mode only, [B][HK][Sq][ceil(Sk/32)], filled here (may be NULL
 * otherwise).
 */
int oracle_block_lists(const or_problem *p, int64_t T, uint32_t *bitmap,
                       int32_t *cnt, int32_t *idx, int32_t *tcnt, int32_t *tidx)
{
    int rc = check_problem(p);
    if (rc) return rc;
    if (T <= 0) return OR_ERR_ARG;
    if (p->mode == OR_INDEX) {
        if (!bitmap) return OR_ERR_ARG;
        rc = oracle_presence_bitmap(p, bitmap);
        if (rc) return rc;
    }
    const int64_t Tm = (p->Sq + T - 1) / T, Tn = (p->Sk + T - 1) / T;
    uint8_t *cls = (uint8_t *)malloc((size_t)(p->B * p->HK * Tm * Tn) + 1);
    if (!cls) return OR_ERR_NOMEM;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t bg = 0; bg < p->B * p->HK; ++bg)
        for (int64_t mt = 0; mt < Tm; ++mt)
            for (int64_t nt = 0; nt < Tn; ++nt)
                cls[(bg * Tm + mt) * Tn + nt] =
                    (uint8_t)classify_tile(p, bitmap, T, bg / p->HK, bg % p->HK, mt, nt);

    for (int64_t bg = 0; bg < p->B * p->HK; ++bg) {
        for (int64_t mt = 0; mt < Tm; ++mt) {
            int32_t *out = idx + (bg * Tm + mt) * Tn;
            int32_t nf = 0, np = 0;
            for (int64_t nt = 0; nt < Tn; ++nt)
                if (cls[(bg * Tm + mt) * Tn + nt] == 2) out[nf++] = (int32_t)nt;
            for (int64_t nt = 0; nt < Tn; ++nt)
                if (cls[(bg * Tm + mt) * Tn + nt] == 1) out[nf + np++] = (int32_t)nt;
            for (int64_t e = nf + np; e < Tn; ++e) out[e] = -1;
            cnt[(bg * Tm + mt) * 2] = nf;
            cnt[(bg * Tm + mt) * 2 + 1] = np;
        }
        for (int64_t nt = 0; nt < Tn; ++nt) {
            int32_t *out = tidx + (bg * Tn + nt) * Tm;
            int32_t nf = 0, np = 0;
            for (int64_t mt = 0; mt < Tm; ++mt)
                if (cls[(bg * Tm + mt) * Tn + nt] == 2) out[nf++] = (int32_t)mt;
            for (int64_t mt = 0; mt < Tm; ++mt)
                if (cls[(bg * Tm + mt) * Tn + nt] == 1) out[nf + np++] = (int32_t)mt;
            for (int64_t e = nf + np; e < Tm; ++e) out[e] = -1;
            tcnt[(bg * Tn + nt) * 2] = nf;
            tcnt[(bg * Tn + nt) * 2 + 1] = np;
        }
    }
    free(cls);
    return OR_OK;
}

/* Point membership, exported so that tests can compare it with independent checks. */
int oracle_is_allowed(const or_problem *p, int64_t b, int64_t g, int64_t i, int64_t j)
{
    return is_allowed(p, b, g, i, j);
}
