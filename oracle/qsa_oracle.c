/*
 * QSA reference oracle: plain, slow, fp64 CPU implementation of the Qwen
 * Sparse Attention hot path (compress -> score -> top-k select -> attend).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path and must never serve as a
 * fallback for it.
 *
 * Sources (web pages on the method):
 *  - "Qwen4 architecture: QSA, GR, PLE" (codebridge-ai.com), section
 *    "1. QSA: not looking at every token equally": keys are compressed into
 *    small blocks, the blocks are scored, the most relevant contiguous token
 *    blocks are selected, and attention runs closely over those regions only.
 *  - "Qwen4 in llama.cpp: Dissecting PR #27742" (ramgpt.org), section
 *    "QSA Is an Address-Selection Problem, Not a New Attention Equation":
 *    compressed-block representation -> indexer scoring -> top-k selection ->
 *    visible cache cells -> ordinary softmax attention over those cells.
 *
 * The pages give no formulas for the compression, the score or the
 * aggregation; this file uses the fixed parameterization of the build:
 * mean-pooled keys per block, scores = <mean pooled query, key summary>
 * scaled by sm_scale, selection shared by one query block and all query
 * heads of a KV group, block 0 (sink) and the causal diagonal block always
 * kept, ties broken by the lower block index.  Two further ways of
 * combining the query block's tokens and the group's heads (max over
 * tokens; sum of per-(head, token) softmaxes) are scored by
 * qsa_oracle_block_scores for the selection variants.
 *
 * Every floating-point quantity is fp64.  bf16 inputs are widened exactly.
 * OpenMP only splits independent rows/tokens; no step is reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact widening of a bf16 bit pattern: bf16 is the top half of an fp32. */
static double bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int qsa_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Step 1 -- compress keys ("compress into small blocks", page
 * "Qwen4 architecture: QSA, GR, PLE", section 1; "compressed-block
 * representation", page "Qwen4 in llama.cpp", section "QSA Is an
 * Address-Selection Problem").
 *
 * K  : [B][H][T][d] bf16 bits.  Kc : [B][H][T/blk][d] fp64.
 * For every complete block j in [jb, je):
 *     Kc[b][h][j][c] = (1/blk) * sum_{r=0}^{blk-1} K[b][h][j*blk + r][c]
 */
void qsa_oracle_compress_keys(const uint16_t *K, int B, int H, int T, int d,
                              int blk, int jb, int je, double *Kc)
{
    const int64_t NB = T / blk;
#pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < B * H; bh++) {
        for (int j = jb; j < je; j++) {
            const uint16_t *base = K + ((int64_t)bh * T + (int64_t)j * blk) * d;
            double *out = Kc + ((int64_t)bh * NB + j) * d;
            for (int c = 0; c < d; c++) {
                double s = 0.0;
                for (int r = 0; r < blk; r++)
                    s += bf16_to_f64(base[(int64_t)r * d + c]);
                out[c] = s / (double)blk;
            }
        }
    }
}

/*
 * bf16-summary option of step 1: each summary rounded to the nearest bf16
 * value, ties to even.  bf16 keeps 8 significant bits (an implicit 1 and 7
 * stored) and fp32's exponent range, so the values representable near x
 * are the multiples of 2^(max(e, -126) - 7), e = floor(log2 |x|) (the
 * max() gives the evenly spaced subnormals below 2^-126).  x / q is exact (q
 * is a power of two), and rint() in the default rounding mode rounds it to
 * the nearest integer with ties to even; an integer just past 2^8 * 2^e
 * lands on the next binade's grid, which is also the right bf16 value.
 * |x| >= 2^128 (never met by means of bf16 keys) is not handled.
 */
void qsa_oracle_round_bf16(const double *x, int64_t n, double *y)
{
    for (int64_t i = 0; i < n; i++) {
        if (x[i] == 0.0 || !isfinite(x[i])) {
            y[i] = x[i];
            continue;
        }
        int E;
        frexp(x[i], &E);              /* |x| in [2^(E-1), 2^E) */
        int e = E - 1;
        if (e < -126) e = -126;
        const double q = ldexp(1.0, e - 7);
        y[i] = rint(x[i] / q) * q;
    }
}

/*
 * Quantized-KV option (page "Qwen4 in llama.cpp: Dissecting PR #27742",
 * section "Quantized KV Exposed a Backend Storage Invariant": K/V stored in
 * a Hadamard-rotated basis to spread channel outliers before quantization,
 * attention in the rotated basis, the output returned to the original basis
 * by the same transform, H^2 = I).  The kernels take every decision that
 * produces a code in fp32, so these steps are written in fp32 with the same
 * operations in the same order; the attention itself is fp64 (oracle.py).
 *
 * Unnormalised n-point Walsh-Hadamard transform (Sylvester order) of rows of
 * n fp32 values, in place: for len = 1, 2, 4, ..., n/2, every pair
 * (j, j + len) with j mod 2 len < len becomes (x_j + x_{j+len},
 * x_j - x_{j+len}).  Applying it twice multiplies by n.
 */
void qsa_oracle_fwht_f32(float *x, int64_t rows, int n)
{
    for (int64_t r = 0; r < rows; r++) {
        float *v = x + r * n;
        for (int len = 1; len < n; len <<= 1)
            for (int i = 0; i < n; i += 2 * len)
                for (int j = i; j < i + len; j++) {
                    const float a = v[j], b = v[j + len];
                    v[j] = a + b;
                    v[j + len] = a - b;
                }
    }
}

/*
 * fp32 -> fp8 e4m3 code (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; no infinities; largest finite 448 = 1.75 * 2^8; subnormals are the
 * multiples of 2^-9 below 2^-6): the nearest representable value, ties to
 * even, saturating to +-448.  Near v the representable values are the
 * multiples of 2^(max(e, -6) - 3), e = floor(log2 |v|); a / q is exact.
 */
static uint8_t e4m3_rn_sat(float v)
{
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a == 0.0) return sign;
    int E;
    frexp(a, &E);
    int e = E - 1;
    if (e < -6) e = -6;
    double r = rint(a / ldexp(1.0, e - 3)) * ldexp(1.0, e - 3);
    if (r > 448.0) r = 448.0;
    if (r < ldexp(1.0, -6)) return sign | (uint8_t)(r / ldexp(1.0, -9));   /* subnormal (or zero) */
    frexp(r, &E);
    e = E - 1;
    const int mant = (int)((r / ldexp(1.0, e) - 1.0) * 8.0);
    return sign | (uint8_t)((e + 7) << 3) | (uint8_t)mant;
}

void qsa_oracle_e4m3(const float *x, int64_t n, uint8_t *codes)
{
    for (int64_t i = 0; i < n; i++) codes[i] = e4m3_rn_sat(x[i]);
}

/*
 * Quantized, rotated cache rows: for each row of n bf16 values x,
 * u = WHT(x) in fp32 (qsa_oracle_fwht_f32), a = max |u|, s = a / 448 (0 when
 * a = 0), codes = e4m3(u / s) (0 when s = 0).  u ~= s * code; the
 * normalised rotation is u / sqrt(n).
 */
void qsa_oracle_quantize_rows_fp8(const uint16_t *X, int64_t rows, int n, uint8_t *codes, float *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        float u[256];
        for (int c = 0; c < n; c++) u[c] = (float)bf16_to_f64(X[r * n + c]);
        qsa_oracle_fwht_f32(u, 1, n);
        float a = 0.0f;
        for (int c = 0; c < n; c++) a = fmaxf(a, fabsf(u[c]));
        const float sc = a > 0.0f ? a / 448.0f : 0.0f;
        scales[r] = sc;
        for (int c = 0; c < n; c++) codes[r * n + c] = sc > 0.0f ? e4m3_rn_sat(u[c] / sc) : 0;
    }
}

/*
 * Step 2 -- pooled query of a selection row.  One selection row is one
 * query block (qblk consecutive query tokens; 1 in decode) of one KV group;
 * the selection is shared by all query heads of the group.  The row's query
 * is the mean over the group's G heads and the block's valid tokens, so its
 * score equals the mean of the per-(head, token) block scores.
 *
 * Q : [B][Tq][Hq][d] bf16 bits.  Qbar : [B][Hkv][NR][d] fp64, NR = ceil(Tq/qblk).
 * Query head h belongs to group h / (Hq/Hkv).
 */
void qsa_oracle_pool_queries(const uint16_t *Q, int B, int Tq, int Hq, int Hkv,
                             int d, int qblk, double *Qbar)
{
    const int G = Hq / Hkv;
    const int NR = (Tq + qblk - 1) / qblk;
#pragma omp parallel for collapse(3) schedule(static)
    for (int b = 0; b < B; b++) {
        for (int g = 0; g < Hkv; g++) {
            for (int i = 0; i < NR; i++) {
                const int t0 = i * qblk;
                const int t1 = (t0 + qblk < Tq) ? t0 + qblk : Tq;
                const double n = (double)(t1 - t0) * (double)G;
                double *out = Qbar + (((int64_t)b * Hkv + g) * NR + i) * d;
                for (int c = 0; c < d; c++) {
                    double s = 0.0;
                    for (int t = t0; t < t1; t++)
                        for (int h = g * G; h < (g + 1) * G; h++)
                            s += bf16_to_f64(Q[(((int64_t)b * Tq + t) * Hq + h) * d + c]);
                    out[c] = s / n;
                }
            }
        }
    }
}

typedef struct {
    double s;
    int j;
} scored_block;

/* Total order of the top-k: higher score first, then the lower block index. */
static int by_score_then_index(const void *pa, const void *pb)
{
    const scored_block *a = (const scored_block *)pa;
    const scored_block *b = (const scored_block *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

/* The causal diagonal block of selection row i: the block holding the row's
 * last query position. */
static int diagonal_block(int i, int Tq, int q_pos0, int qblk, int blk)
{
    int t_last = (i + 1) * qblk - 1;
    if (t_last > Tq - 1) t_last = Tq - 1;
    return (q_pos0 + t_last) / blk;
}

/*
 * Steps 3 and 4 -- score the compressed key blocks against the row's pooled
 * query ("indexer scoring") and keep the top-k blocks ("top-k selection"),
 * page "Qwen4 in llama.cpp", section "QSA Is an Address-Selection Problem".
 *
 * For selection row (b, g, i) with diagonal block D:
 *   candidates C = {1, ..., D-1}  (complete blocks strictly before D; the
 *                                  diagonal's summary would see the future)
 *   s_j = sm_scale * <Qbar[b][g][i], Kc[b][g][j]>
 *   F   = {0} plus {D} if D > 0   (sink and diagonal, always kept; they
 *                                  count toward topk)
 *   m   = min(topk - |F|, |C|) candidates taken in the order
 *         (s descending, j ascending)
 *   out = F plus the chosen, ascending, padded with -1 to topk entries.
 *
 * rows    : list of flat row ids ((b*Hkv + g)*NR + i), or NULL for all rows
 * idx     : [nrows][topk] int32
 * gap     : [nrows] s_(m) - s_(m+1) among the candidates, +inf when the set
 *           does not depend on the scores (m == 0 or m == |C|)
 * m_out   : [nrows] number of chosen candidates
 * scores  : optional [nrows][NB] -- s_j for candidates, NaN elsewhere
 * Qbar    : [B][Hkv][NR][d]; Kc : [B][Hkv][NB][d]
 * Returns 0, or -1 if topk < 2.
 */
/* The selection rule of step 4 for one row: cand[0..ncand) are the scored
 * candidates {1, ..., D-1}; writes the row's indices, gap and m. */
static void select_row(scored_block *cand, int ncand, int D, int topk, int32_t *out, double *gap,
                       int32_t *m_out)
{
    qsort(cand, (size_t)ncand, sizeof(scored_block), by_score_then_index);
    const int nforced = D > 0 ? 2 : 1;
    int m = topk - nforced;
    if (m > ncand) m = ncand;
    *gap = (m == 0 || m == ncand) ? INFINITY : cand[m - 1].s - cand[m].s;
    *m_out = m;
    /* ascending output: 0, chosen blocks in increasing index, D */
    int n = 0;
    out[n++] = 0;
    for (int j = 1; j < D; j++) {
        int chosen = 0;
        for (int c = 0; c < m; c++)
            if (cand[c].j == j) { chosen = 1; break; }
        if (chosen) out[n++] = j;
    }
    if (D > 0) out[n++] = D;
    while (n < topk) out[n++] = -1;
}

int qsa_oracle_select(const double *Qbar, const double *Kc, int B, int Hkv, int NR,
                      int NB, int d, int Tq, int q_pos0, int qblk, int blk, int topk,
                      double sm_scale, const int32_t *rows, int nrows, int32_t *idx,
                      double *gap, int32_t *m_out, double *scores)
{
    if (topk < 2) return -1;
    const int total = B * Hkv * NR;
    if (!rows) nrows = total;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; r++) {
        const int row = rows ? rows[r] : r;
        const int i = row % NR;
        const int bg = row / NR;
        const int D = diagonal_block(i, Tq, q_pos0, qblk, blk);
        const int ncand = D > 1 ? D - 1 : 0;
        const double *q = Qbar + (int64_t)row * d;
        scored_block *cand = (scored_block *)malloc(sizeof(scored_block) * (ncand > 0 ? ncand : 1));
        for (int j = 1; j < D; j++) {
            const double *kc = Kc + ((int64_t)bg * NB + j) * d;
            double dot = 0.0;
            for (int c = 0; c < d; c++) dot += q[c] * kc[c];
            cand[j - 1].s = sm_scale * dot;
            cand[j - 1].j = j;
        }
        if (scores) {
            double *srow = scores + (int64_t)r * NB;
            for (int j = 0; j < NB; j++) srow[j] = NAN;
            for (int n = 0; n < ncand; n++) srow[cand[n].j] = cand[n].s;
        }
        select_row(cand, ncand, D, topk, idx + (int64_t)r * topk, &gap[r], &m_out[r]);
        free(cand);
    }
    return 0;
}

/*
 * Step 3 with the row's tokens and heads combined in other ways than the
 * pooled query.  The pages have the selector score compressed keys against
 * the queries (page "Qwen4 in llama.cpp: Dissecting PR #27742", section "QSA
 * Is an Address-Selection Problem, Not a New Attention Equation") and leave
 * open how the query block's tokens and the group's heads are combined.
 * For row (b, g, i) with diagonal block D, tokens t of the row's query
 * block (the valid ones) and heads h of group g:
 *   z[h][t][j] = sm_scale * <Q[b][t][h], Kc[b][g][j]>   for j in {0, ..., D-1}
 *   aggregator 0 (mean):        s_j = mean over (h, t) of z[h][t][j]
 *   aggregator 1 (max):         s_j = max over t of (mean over h of z[h][t][j])
 *   aggregator 2 (softmax-sum): s_j = sum over (h, t) of softmax over
 *                               j' in {0, ..., D-1} of z[h][t][j'], at j
 * (the normalisation set of the softmax-sum is every complete block before
 * the diagonal, the sink included).
 * Q : [B][Tq][Hq][d] bf16 bits; Kc : [B][Hkv][NB][d]
 * rows : flat row ids ((b*Hkv + g)*NR + i) or NULL for all
 * scores : [nrows][NB] -- s_j for j < D, NaN elsewhere
 * Returns 0, or -1 for an unknown aggregator.
 */
int qsa_oracle_block_scores(const uint16_t *Q, const double *Kc, int B, int Tq, int Hq, int Hkv, int NB,
                            int d, int q_pos0, int qblk, int blk, double sm_scale, int aggregator,
                            const int32_t *rows, int nrows, double *scores)
{
    if (aggregator < 0 || aggregator > 2) return -1;
    const int G = Hq / Hkv;
    const int NR = (Tq + qblk - 1) / qblk;
    if (!rows) nrows = B * Hkv * NR;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; r++) {
        const int row = rows ? rows[r] : r;
        const int i = row % NR, bg = row / NR, b = bg / Hkv, g = bg % Hkv;
        const int D = diagonal_block(i, Tq, q_pos0, qblk, blk);
        const int t0 = i * qblk, t1 = (t0 + qblk < Tq) ? t0 + qblk : Tq;
        double *srow = scores + (int64_t)r * NB;
        for (int j = 0; j < NB; j++) srow[j] = NAN;
        if (D < 1) continue;
        /* z[(t - t0) * G + (h - g*G)][j] */
        const int nq = (t1 - t0) * G;
        double *z = (double *)malloc(sizeof(double) * (size_t)nq * D);
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
        for (int t = t0; t < t1; t++)
            for (int hh = 0; hh < G; hh++) {
                const uint16_t *qrow = Q + (((int64_t)b * Tq + t) * Hq + g * G + hh) * d;
                for (int c = 0; c < d; c++) qv[c] = bf16_to_f64(qrow[c]);
                double *zr = z + (int64_t)((t - t0) * G + hh) * D;
                for (int j = 0; j < D; j++) {
                    const double *kc = Kc + ((int64_t)bg * NB + j) * d;
                    double dot = 0.0;
                    for (int c = 0; c < d; c++) dot += qv[c] * kc[c];
                    zr[j] = sm_scale * dot;
                }
            }
        for (int j = 0; j < D; j++) {
            double s = 0.0;
            if (aggregator == 0) {
                for (int n = 0; n < nq; n++) s += z[(int64_t)n * D + j];
                s /= (double)nq;
            } else if (aggregator == 1) {
                s = -INFINITY;
                for (int t = 0; t < t1 - t0; t++) {
                    double m = 0.0;
                    for (int hh = 0; hh < G; hh++) m += z[(int64_t)(t * G + hh) * D + j];
                    m /= (double)G;
                    if (m > s) s = m;
                }
            }
            srow[j] = s;
        }
        if (aggregator == 2) {
            for (int j = 0; j < D; j++) srow[j] = 0.0;
            for (int n = 0; n < nq; n++) {
                const double *zr = z + (int64_t)n * D;
                double mx = -INFINITY, sum = 0.0;
                for (int j = 0; j < D; j++) if (zr[j] > mx) mx = zr[j];
                for (int j = 0; j < D; j++) sum += exp(zr[j] - mx);
                for (int j = 0; j < D; j++) srow[j] += exp(zr[j] - mx) / sum;
            }
        }
        free(qv);
        free(z);
    }
    return 0;
}

/*
 * Step 4 on a given score table: the selection rule of qsa_oracle_select
 * with s_j = scores[r][j] for the candidates j in {1, ..., D-1}.
 */
int qsa_oracle_select_scores(const double *scores, int B, int Hkv, int NR, int NB, int Tq, int q_pos0,
                             int qblk, int blk, int topk, const int32_t *rows, int nrows, int32_t *idx,
                             double *gap, int32_t *m_out)
{
    if (topk < 2) return -1;
    if (!rows) nrows = B * Hkv * NR;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; r++) {
        const int row = rows ? rows[r] : r;
        const int D = diagonal_block(row % NR, Tq, q_pos0, qblk, blk);
        const int ncand = D > 1 ? D - 1 : 0;
        scored_block *cand = (scored_block *)malloc(sizeof(scored_block) * (ncand > 0 ? ncand : 1));
        for (int j = 1; j < D; j++) {
            cand[j - 1].s = scores[(int64_t)r * NB + j];
            cand[j - 1].j = j;
        }
        select_row(cand, ncand, D, topk, idx + (int64_t)r * topk, &gap[r], &m_out[r]);
        free(cand);
    }
    return 0;
}

/*
 * Step 5 -- exact softmax attention over the selected blocks only ("attend
 * closely to the selected regions", page "Qwen4 architecture: QSA, GR,
 * PLE", section 1; "attention over those cells", page "Qwen4 in llama.cpp",
 * section "QSA Is an Address-Selection Problem").
 *
 * Query token t of batch b sits at absolute position p = q_pos0 + t and
 * uses the selection of its row i = t / qblk in its head's group.  Visible
 * keys: u in the selected blocks with u <= p.
 *   z_u = sm_scale * <q, k_u>,  O = sum_u exp(z_u - max z) v_u / sum_u exp(z_u - max z)
 *   lse = max z + log(sum_u exp(z_u - max z))
 *
 * Q : [B][Tq][Hq][d]; K, V : [B][Hkv][T_kv][d] (bf16 bits)
 * idx : [B][Hkv][NR][topk] int32, -1 = unused slot
 * tokens : list of flat tokens (b*Tq + t), or NULL for all
 * O : [ntok][Hq][d] fp64; lse : optional [ntok][Hq]
 * Returns 0, or -1 if an index lies outside the cache or after the token.
 */
int qsa_oracle_attend(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                      const int32_t *idx, int B, int Tq, int Hq, int Hkv, int T_kv,
                      int d, int q_pos0, int qblk, int blk, int topk, double sm_scale,
                      const int32_t *tokens, int ntok, double *O, double *lse)
{
    const int G = Hq / Hkv;
    const int NR = (Tq + qblk - 1) / qblk;
    if (!tokens) ntok = B * Tq;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int n = 0; n < ntok; n++) {
        const int flat = tokens ? tokens[n] : n;
        const int b = flat / Tq, t = flat % Tq;
        const int64_t p = (int64_t)q_pos0 + t;
        const int i = t / qblk;
        double *z = (double *)malloc(sizeof(double) * (size_t)topk * blk);
        int64_t *u_of = (int64_t *)malloc(sizeof(int64_t) * (size_t)topk * blk);
        for (int h = 0; h < Hq; h++) {
            const int g = h / G;
            const int32_t *sel = idx + (((int64_t)b * Hkv + g) * NR + i) * topk;
            const uint16_t *q = Q + (((int64_t)b * Tq + t) * Hq + h) * d;
            const uint16_t *Kbg = K + ((int64_t)b * Hkv + g) * (int64_t)T_kv * d;
            const uint16_t *Vbg = V + ((int64_t)b * Hkv + g) * (int64_t)T_kv * d;
            int nvis = 0;
            for (int s = 0; s < topk; s++) {
                const int j = sel[s];
                if (j < 0) continue;
                if ((int64_t)j * blk > p || p >= T_kv) { bad = 1; continue; }
                for (int r = 0; r < blk; r++) {
                    const int64_t u = (int64_t)j * blk + r;
                    if (u > p) break;
                    double dot = 0.0;
                    for (int c = 0; c < d; c++)
                        dot += bf16_to_f64(q[c]) * bf16_to_f64(Kbg[u * d + c]);
                    z[nvis] = sm_scale * dot;
                    u_of[nvis] = u;
                    nvis++;
                }
            }
            double *o = O + ((int64_t)n * Hq + h) * d;
            double zmax = -INFINITY;
            for (int e = 0; e < nvis; e++)
                if (z[e] > zmax) zmax = z[e];
            double l = 0.0;
            for (int c = 0; c < d; c++) o[c] = 0.0;
            for (int e = 0; e < nvis; e++) {
                const double w = exp(z[e] - zmax);
                l += w;
                for (int c = 0; c < d; c++) o[c] += w * bf16_to_f64(Vbg[u_of[e] * d + c]);
            }
            for (int c = 0; c < d; c++) o[c] = nvis ? o[c] / l : 0.0;
            if (lse) lse[(int64_t)n * Hq + h] = nvis ? zmax + log(l) : -INFINITY;
        }
        free(z);
        free(u_of);
    }
    return bad ? -1 : 0;
}
