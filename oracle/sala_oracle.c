/*
 * sala_oracle.c -- plain fp64 CPU oracle for the SALA hybrid-attention hot path.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
 * and the benchmark's CPU-baseline leg load this library.  It shares no code,
 * header, table or helper with the CUDA library; it is written from the method
 * description alone, in double precision, as plain loops that can be checked
 * against the text by eye.  OpenMP only splits independent (batch, head) or
 * (batch, row) iterations across cores; no blocking or reordering of any sum.
 *
 * Sources (web pages on MiniCPM-SALA):
 *   - "MiniCPM-SALA: Hybridizing Sparse and Linear Attention..." summary page,
 *     section "Prerequisites / Linear Attention": the Lightning state update
 *     S_t = S_{t-1} + k_t v_t^T, with S_t the accumulated state.
 *   - AI-tech-review tech-report mirror, section 02 (2): InfLLM-V2 sparse layers,
 *     each query attends to a small set of selected key/value blocks, dense at
 *     standard length, output gate on the sparse layers too.
 *   - same page, section 02 (3): Lightning layers with QK-normalisation,
 *     GQA-to-MHA and an output gate.
 *   - same page, section 02 (4): HyPE -- RoPE in the linear layers, NoPE in the
 *     sparse layers.
 *   - summary page, "Prerequisites / Sparse Attention": sliding window plus
 *     global anchors.
 * Readings where the pages are silent (all stated where used):
 *   no decay in the recurrence; readout o_t = q_t^T S_t with S_t inclusive of
 *   token t; no normaliser; QK-norm = per-head RMSNorm over the head dimension
 *   (eps, optional weight) followed by rotate-half RoPE with inverse frequency
 *   base^(-2i/D); gate y = sigmoid(g) * o elementwise; block representative =
 *   mean of the block's keys; block score = (1/sqrt(D)) * sum over the GQA
 *   group's query heads of q_h . Kbar_j; candidates = complete blocks that are
 *   neither init nor local; ties go to the smaller block index.
 *
 * Layouts: every activation array is contiguous [B, rows, heads, D] in double.
 * States are [B, H, D, D], S[i][j] with i the key dimension, j the value one.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define IDX4(a, b, c, d, B1, C1, D1) ((((int64_t)(a) * (B1) + (b)) * (C1) + (c)) * (D1) + (d))

/* ------------------------------------------------------------------------ */
/* QK-normalisation and rotary position embedding (Lightning layers only).   */
/* ------------------------------------------------------------------------ */

/* Per-head RMSNorm over the head dimension: x / sqrt(mean(x^2) + eps) * w.
 * (tech-report mirror, section 02 (3): QK-normalization in the linear layers;
 * RMSNorm is the reading adopted for "QK-normalization".) */
static void rms_normalise(const double *x, const double *w, int D, double eps, double *y)
{
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    double r = 1.0 / sqrt(ss / (double)D + eps);
    for (int d = 0; d < D; ++d) y[d] = x[d] * r * (w ? w[d] : 1.0);
}

/* Rotate-half RoPE at position pos: for i < D/2 the pair (x_i, x_{i+D/2}) is
 * rotated by angle pos * base^(-2i/D).  (tech-report mirror, section 02 (4):
 * HyPE keeps RoPE in the linear layers.) */
static void rotate_half(double *x, int D, double pos, double base)
{
    int h = D / 2;
    for (int i = 0; i < h; ++i) {
        double inv_freq = pow(base, -2.0 * (double)i / (double)D);
        double a = pos * inv_freq;
        double c = cos(a), s = sin(a);
        double x0 = x[i], x1 = x[i + h];
        x[i] = x0 * c - x1 * s;
        x[i + h] = x1 * c + x0 * s;
    }
}

/* Normalise then rotate one head vector (exported for the pins). */
void oracle_qk_prep(const double *x, const double *w, int D, double eps,
                    double pos, double base, double *y)
{
    rms_normalise(x, w, D, eps, y);
    rotate_half(y, D, pos, base);
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* ------------------------------------------------------------------------ */
/* Lightning attention, three independent formulations.                      */
/* ------------------------------------------------------------------------ */

/*
 * Recurrent form -- the definition on the summary page ("Prerequisites /
 * Linear Attention"): S_t = S_{t-1} + k_t v_t^T, read out as o_t = q_t^T S_t.
 *
 * q, k, v, g: [B, T, H, D]; g may be NULL (no gate).  S0: [B, H, D, D] or NULL
 * (zero initial state).  qw, kw: [D] norm weights or NULL (weight 1).
 * rows (ascending) / nrows: the token positions whose output is wanted, or
 * NULL for all T (then nrows must equal T).  y: [B, nrows, H, D].
 * S_out: [B, H, D, D] final state after token T-1, may be NULL.
 */
void oracle_lightning_recurrent(const double *q, const double *k, const double *v,
                                const double *g, const double *S0,
                                const double *qw, const double *kw,
                                int B, int T, int H, int D, int64_t pos0,
                                double base, double eps,
                                const int64_t *rows, int nrows,
                                double *y, double *S_out)
{
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * D * D);
            double *qh = (double *)malloc(sizeof(double) * D);
            double *kh = (double *)malloc(sizeof(double) * D);
            if (S0)
                memcpy(S, S0 + ((int64_t)b * H + h) * D * D, sizeof(double) * D * D);
            else
                memset(S, 0, sizeof(double) * D * D);
            int r = 0;
            for (int t = 0; t < T; ++t) {
                int64_t base_in = IDX4(b, t, h, 0, T, H, D);
                double pos = (double)(pos0 + t);
                oracle_qk_prep(k + base_in, kw, D, eps, pos, base, kh);
                const double *vt = v + base_in;
                for (int i = 0; i < D; ++i)
                    for (int j = 0; j < D; ++j) S[i * D + j] += kh[i] * vt[j];
                int want = rows ? (r < nrows && rows[r] == t) : 1;
                if (!want) continue;
                int orow = rows ? r : t;
                oracle_qk_prep(q + base_in, qw, D, eps, pos, base, qh);
                double *yo = y + IDX4(b, orow, h, 0, nrows, H, D);
                for (int j = 0; j < D; ++j) {
                    double o = 0.0;
                    for (int i = 0; i < D; ++i) o += qh[i] * S[i * D + j];
                    yo[j] = g ? sigmoid(g[base_in + j]) * o : o;
                }
                if (rows) ++r;
            }
            if (S_out) memcpy(S_out + ((int64_t)b * H + h) * D * D, S, sizeof(double) * D * D);
            free(S); free(qh); free(kh);
        }
    }
}

/*
 * The same recurrence on operands that are already prepared: qh, kh normalised and
 * rotated, and the gate given as its multiplier (sigmoid(g) already applied):
 *   S_t = S_{t-1} + kh_t v_t^T,   y_t = gate_t * (qh_t^T S_t)   (gate NULL: y_t = o_t).
 * qh, kh, v, gate: [B, T, H, D]; S0 as above (NULL = zero); y: [B, T, H, D];
 * S_out: [B, H, D, D] or NULL.
 */
void oracle_lightning_recurrent_prepared(const double *qh, const double *kh, const double *v,
                                         const double *gate, const double *S0, int B, int T,
                                         int H, int D, double *y, double *S_out)
{
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * D * D);
            if (S0)
                memcpy(S, S0 + ((int64_t)b * H + h) * D * D, sizeof(double) * D * D);
            else
                memset(S, 0, sizeof(double) * D * D);
            for (int t = 0; t < T; ++t) {
                int64_t at = IDX4(b, t, h, 0, T, H, D);
                for (int i = 0; i < D; ++i)
                    for (int j = 0; j < D; ++j) S[i * D + j] += kh[at + i] * v[at + j];
                for (int j = 0; j < D; ++j) {
                    double o = 0.0;
                    for (int i = 0; i < D; ++i) o += qh[at + i] * S[i * D + j];
                    y[at + j] = gate ? gate[at + j] * o : o;
                }
            }
            if (S_out) memcpy(S_out + ((int64_t)b * H + h) * D * D, S, sizeof(double) * D * D);
            free(S);
        }
    }
}

/*
 * Quadratic (parallel) form of the same recurrence: unrolling
 * S_t = S0 + sum_{s<=t} k_s v_s^T gives
 *   o_t = q_t^T S0 + sum_{s<=t} (q_t . k_s) v_s,
 * i.e. (Q K^T masked to s <= t, diagonal included) V plus the initial-state term.
 * Written independently of the recurrent routine (no running state).
 */
void oracle_lightning_quadratic(const double *q, const double *k, const double *v,
                                const double *g, const double *S0,
                                const double *qw, const double *kw,
                                int B, int T, int H, int D, int64_t pos0,
                                double base, double eps, double *y)
{
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *Qh = (double *)malloc(sizeof(double) * (size_t)T * D);
            double *Kh = (double *)malloc(sizeof(double) * (size_t)T * D);
            for (int t = 0; t < T; ++t) {
                int64_t o = IDX4(b, t, h, 0, T, H, D);
                oracle_qk_prep(q + o, qw, D, eps, (double)(pos0 + t), base, Qh + (int64_t)t * D);
                oracle_qk_prep(k + o, kw, D, eps, (double)(pos0 + t), base, Kh + (int64_t)t * D);
            }
            const double *S = S0 ? S0 + ((int64_t)b * H + h) * D * D : NULL;
            for (int t = 0; t < T; ++t) {
                const double *qt = Qh + (int64_t)t * D;
                double *yo = y + IDX4(b, t, h, 0, T, H, D);
                for (int j = 0; j < D; ++j) yo[j] = 0.0;
                if (S)
                    for (int j = 0; j < D; ++j) {
                        double acc = 0.0;
                        for (int i = 0; i < D; ++i) acc += qt[i] * S[i * D + j];
                        yo[j] = acc;
                    }
                for (int s = 0; s <= t; ++s) {
                    const double *ks = Kh + (int64_t)s * D;
                    double a = 0.0;
                    for (int i = 0; i < D; ++i) a += qt[i] * ks[i];
                    const double *vs = v + IDX4(b, s, h, 0, T, H, D);
                    for (int j = 0; j < D; ++j) yo[j] += a * vs[j];
                }
                if (g) {
                    const double *gt = g + IDX4(b, t, h, 0, T, H, D);
                    for (int j = 0; j < D; ++j) yo[j] *= sigmoid(gt[j]);
                }
            }
            free(Qh); free(Kh);
        }
    }
}

/*
 * Chunked form with chunk length C (any C >= 1; the last chunk may be short):
 *   O_c = (Q_c K_c^T, masked to s <= t inclusive) V_c + Q_c S_{c-1}
 *   S_c = S_{c-1} + K_c^T V_c
 * An exact regrouping of the recurrence's sums (same terms, summed by chunk).
 * S_out may be NULL.
 */
void oracle_lightning_chunked(const double *q, const double *k, const double *v,
                              const double *g, const double *S0,
                              const double *qw, const double *kw,
                              int B, int T, int H, int D, int64_t pos0,
                              double base, double eps, int C,
                              double *y, double *S_out)
{
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * D * D);
            double *Qc = (double *)malloc(sizeof(double) * (size_t)C * D);
            double *Kc = (double *)malloc(sizeof(double) * (size_t)C * D);
            double *A = (double *)malloc(sizeof(double) * (size_t)C * C);
            if (S0)
                memcpy(S, S0 + ((int64_t)b * H + h) * D * D, sizeof(double) * D * D);
            else
                memset(S, 0, sizeof(double) * D * D);
            for (int t0 = 0; t0 < T; t0 += C) {
                int n = (T - t0 < C) ? (T - t0) : C;
                for (int r = 0; r < n; ++r) {
                    int64_t o = IDX4(b, t0 + r, h, 0, T, H, D);
                    oracle_qk_prep(q + o, qw, D, eps, (double)(pos0 + t0 + r), base, Qc + (int64_t)r * D);
                    oracle_qk_prep(k + o, kw, D, eps, (double)(pos0 + t0 + r), base, Kc + (int64_t)r * D);
                }
                /* intra-chunk scores, lower-triangular inclusive mask */
                for (int r = 0; r < n; ++r)
                    for (int s = 0; s < n; ++s) {
                        double a = 0.0;
                        if (s <= r)
                            for (int i = 0; i < D; ++i) a += Qc[r * D + i] * Kc[s * D + i];
                        A[r * C + s] = a;
                    }
                for (int r = 0; r < n; ++r) {
                    double *yo = y + IDX4(b, t0 + r, h, 0, T, H, D);
                    for (int j = 0; j < D; ++j) {
                        double inter = 0.0, intra = 0.0;
                        for (int i = 0; i < D; ++i) inter += Qc[r * D + i] * S[i * D + j];
                        for (int s = 0; s < n; ++s)
                            intra += A[r * C + s] * v[IDX4(b, t0 + s, h, j, T, H, D)];
                        double o = inter + intra;
                        yo[j] = g ? sigmoid(g[IDX4(b, t0 + r, h, j, T, H, D)]) * o : o;
                    }
                }
                /* state update with the whole chunk */
                for (int i = 0; i < D; ++i)
                    for (int j = 0; j < D; ++j) {
                        double acc = 0.0;
                        for (int s = 0; s < n; ++s)
                            acc += Kc[s * D + i] * v[IDX4(b, t0 + s, h, j, T, H, D)];
                        S[i * D + j] += acc;
                    }
            }
            if (S_out) memcpy(S_out + ((int64_t)b * H + h) * D * D, S, sizeof(double) * D * D);
            free(S); free(Qc); free(Kc); free(A);
        }
    }
}

/*
 * One decode step per batch entry: one new token at position pos[b].
 * q, k, v, g: [B, H, D] (g may be NULL); S: [B, H, D, D] updated in place;
 * y: [B, H, D].  S <- S + k v^T, then o = q^T S (new state, token included).
 */
void oracle_lightning_decode(const double *q, const double *k, const double *v,
                             const double *g, double *S,
                             const double *qw, const double *kw,
                             const int64_t *pos, int B, int H, int D,
                             double base, double eps, double *y)
{
#pragma omp parallel for collapse(2)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *qh = (double *)malloc(sizeof(double) * D);
            double *kh = (double *)malloc(sizeof(double) * D);
            int64_t o = ((int64_t)b * H + h) * D;
            double *Sbh = S + ((int64_t)b * H + h) * D * D;
            oracle_qk_prep(q + o, qw, D, eps, (double)pos[b], base, qh);
            oracle_qk_prep(k + o, kw, D, eps, (double)pos[b], base, kh);
            for (int i = 0; i < D; ++i)
                for (int j = 0; j < D; ++j) Sbh[i * D + j] += kh[i] * v[o + j];
            for (int j = 0; j < D; ++j) {
                double acc = 0.0;
                for (int i = 0; i < D; ++i) acc += qh[i] * Sbh[i * D + j];
                y[o + j] = g ? sigmoid(g[o + j]) * acc : acc;
            }
            free(qh); free(kh);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* InfLLM-v2-style block selection and block-sparse attention (NoPE).         */
/* ------------------------------------------------------------------------ */

/* Mean of each complete block of `blk` keys: kbar[b, j, hk, :] for
 * j < floor(T / blk).  k: [B, T, Hkv, D]; kbar: [B, T/blk, Hkv, D]. */
void oracle_block_means(const double *k, int B, int T, int Hkv, int D, int blk, double *kbar)
{
    int nb = T / blk;
#pragma omp parallel for collapse(2)
    for (int b = 0; b < B; ++b)
        for (int j = 0; j < nb; ++j)
            for (int hk = 0; hk < Hkv; ++hk)
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int s = 0; s < blk; ++s) acc += k[IDX4(b, j * blk + s, hk, d, T, Hkv, D)];
                    kbar[IDX4(b, j, hk, d, nb, Hkv, D)] = acc / (double)blk;
                }
}

typedef struct { double score; int j; } cand_t;

/* Larger score first; equal scores -> smaller block index first. */
static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

static int int_cmp(const void *pa, const void *pb)
{
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

/*
 * Block scores of one query row t for KV head hk, for candidate blocks
 * j in [n_init, c - n_local] (c = floor(t / blk)):
 *   score_j = (1/sqrt(D)) * sum_{h in group(hk)} sum_d q[t, h, d] * kbar[j, hk, d].
 * q_row points at q[b, row, 0, 0] ([Hq, D]); kbar_b at kbar[b, 0, 0, 0].
 * Returns the number of candidates written to `out`.
 */
static int block_scores(const double *q_row, const double *kbar_b, int nb, int Hq, int Hkv,
                        int D, int blk, int n_init, int n_local, int64_t t, int hk,
                        cand_t *out)
{
    int grp = Hq / Hkv;
    int64_t c = t / blk;
    int64_t lo = n_init, hi = c - n_local; /* inclusive range of candidates */
    int n = 0;
    double scale = 1.0 / sqrt((double)D);
    for (int64_t j = lo; j <= hi; ++j) {
        if (j >= nb) break; /* only complete blocks have a representative */
        double acc = 0.0;
        for (int h = hk * grp; h < (hk + 1) * grp; ++h)
            for (int d = 0; d < D; ++d)
                acc += q_row[(int64_t)h * D + d] * kbar_b[((int64_t)j * Hkv + hk) * D + d];
        out[n].score = acc * scale;
        out[n].j = (int)j;
        ++n;
    }
    return n;
}

/*
 * Per-head softmax-normalised block scores (the selection variant that scores a
 * block by how much of each head's attention it would draw): for each query head h
 * of the group, s_{h,j} = (1/sqrt(D)) q[t, h] . kbar[j, hk] over the same candidate
 * set as block_scores, p_{h,j} = exp(s_{h,j}) / sum_{j'} exp(s_{h,j'}) (softmax over
 * the candidates, computed with the per-head maximum subtracted), and
 *   score_j = sum_{h in group(hk)} p_{h,j}.
 * Each head's p sums to 1, so a row's scores sum to the group size.
 */
static int block_scores_head_softmax(const double *q_row, const double *kbar_b, int nb, int Hq,
                                     int Hkv, int D, int blk, int n_init, int n_local, int64_t t,
                                     int hk, cand_t *out)
{
    int grp = Hq / Hkv;
    int64_t c = t / blk;
    int64_t lo = n_init, hi = c - n_local;
    if (hi > nb - 1) hi = nb - 1; /* only complete blocks have a representative */
    int n = hi >= lo ? (int)(hi - lo + 1) : 0;
    double scale = 1.0 / sqrt((double)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int e = 0; e < n; ++e) {
        out[e].j = (int)(lo + e);
        out[e].score = 0.0;
    }
    for (int h = hk * grp; h < (hk + 1) * grp; ++h) {
        double m = -INFINITY, l = 0.0;
        for (int e = 0; e < n; ++e) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += q_row[(int64_t)h * D + d] * kbar_b[((int64_t)(lo + e) * Hkv + hk) * D + d];
            s[e] = acc * scale;
            if (s[e] > m) m = s[e];
        }
        for (int e = 0; e < n; ++e) l += exp(s[e] - m);
        for (int e = 0; e < n; ++e) out[e].score += exp(s[e] - m) / l;
    }
    free(s);
    return n;
}

/*
 * Block selection for query rows: top-`topk` candidates by score (ties -> smaller
 * block index), united with the init blocks {0..n_init-1} and the local window
 * {c-n_local+1..c} (clipped to [0, c]), sorted ascending, padded with -1 to
 * n_sel = n_init + topk + n_local entries.
 *
 * q: [B, nrows, Hq, D] (the rows listed in `rows`, or all T rows when rows is
 * NULL).  k: [B, T, Hkv, D].  idx: [B, Hkv, nrows, n_sel] int32.
 * gap: [B, Hkv, nrows], score of the topk-th minus the (topk+1)-th candidate
 * (+inf when every candidate is selected), or NULL.
 * scores_out: [B, Hkv, nrows, max_cand] or NULL -- candidate scores by block
 * index offset (entry j - n_init), NaN where not a candidate.
 */
void oracle_sparse_select_mode(const double *q, const double *k, int B, int T, int Hq, int Hkv,
                               int D, int blk, int topk, int n_init, int n_local,
                               const int64_t *rows, int nrows, int32_t *idx, double *gap,
                               double *scores_out, int max_cand, int mode);

void oracle_sparse_select(const double *q, const double *k, int B, int T, int Hq, int Hkv,
                          int D, int blk, int topk, int n_init, int n_local,
                          const int64_t *rows, int nrows, int32_t *idx, double *gap,
                          double *scores_out, int max_cand)
{
    oracle_sparse_select_mode(q, k, B, T, Hq, Hkv, D, blk, topk, n_init, n_local, rows, nrows,
                              idx, gap, scores_out, max_cand, 0);
}

/* mode 0: group-summed scores (block_scores); mode 1: per-head softmax-normalised
 * scores summed over the group (block_scores_head_softmax). */
void oracle_sparse_select_mode(const double *q, const double *k, int B, int T, int Hq, int Hkv,
                               int D, int blk, int topk, int n_init, int n_local,
                               const int64_t *rows, int nrows, int32_t *idx, double *gap,
                               double *scores_out, int max_cand, int mode)
{
    int nb = T / blk;
    int n_sel = n_init + topk + n_local;
    double *kbar = (double *)malloc(sizeof(double) * (size_t)B * (nb > 0 ? nb : 1) * Hkv * D);
    oracle_block_means(k, B, T, Hkv, D, blk, kbar);
#pragma omp parallel for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk)
            for (int r = 0; r < nrows; ++r) {
                int64_t t = rows ? rows[r] : r;
                int64_t c = t / blk;
                cand_t *cands = (cand_t *)malloc(sizeof(cand_t) * (size_t)(c + 1));
                int *sel = (int *)malloc(sizeof(int) * (size_t)(n_sel + 1));
                int n = mode == 1
                            ? block_scores_head_softmax(q + IDX4(b, r, 0, 0, nrows, Hq, D),
                                                        kbar + (int64_t)b * nb * Hkv * D, nb, Hq,
                                                        Hkv, D, blk, n_init, n_local, t, hk, cands)
                            : block_scores(q + IDX4(b, r, 0, 0, nrows, Hq, D),
                                           kbar + (int64_t)b * nb * Hkv * D, nb, Hq, Hkv, D, blk,
                                           n_init, n_local, t, hk, cands);
                if (scores_out) {
                    double *so = scores_out + (((int64_t)b * Hkv + hk) * nrows + r) * max_cand;
                    for (int e = 0; e < max_cand; ++e) so[e] = NAN;
                    for (int e = 0; e < n && e < max_cand; ++e) so[cands[e].j - n_init] = cands[e].score;
                }
                qsort(cands, (size_t)n, sizeof(cand_t), cand_cmp);
                int m = 0;
                /* init blocks, then chosen candidates, then the local window */
                for (int64_t j = 0; j < n_init && j <= c; ++j) sel[m++] = (int)j;
                int take = n < topk ? n : topk;
                for (int e = 0; e < take; ++e) sel[m++] = cands[e].j;
                for (int64_t j = c - n_local + 1; j <= c; ++j)
                    if (j >= n_init) sel[m++] = (int)j; /* j < n_init already listed */
                qsort(sel, (size_t)m, sizeof(int), int_cmp);
                int32_t *io = idx + (((int64_t)b * Hkv + hk) * nrows + r) * n_sel;
                int w = 0;
                for (int e = 0; e < m; ++e)
                    if (w == 0 || io[w - 1] != sel[e]) io[w++] = sel[e];
                for (; w < n_sel; ++w) io[w] = -1;
                if (gap) {
                    double gv = INFINITY;
                    if (n > topk) gv = cands[topk - 1].score - cands[topk].score;
                    gap[((int64_t)b * Hkv + hk) * nrows + r] = gv;
                }
                free(cands); free(sel);
            }
    free(kbar);
}

/*
 * Softmax attention of query rows over a key set.  For each (b, row, h) with
 * hk = h / (Hq / Hkv): keys = union over the listed blocks j >= 0 of
 * [j*blk, min((j+1)*blk, T)), restricted to s <= t; NoPE (no rotation);
 *   o = sum_s softmax_s(scale * q . k_s) v_s,   y = sigmoid(g) * o if g.
 * An empty key set gives o = 0.
 *
 * q, g: [B, nrows, Hq, D] (rows listed in `rows`, or all T when NULL);
 * k, v: [B, T, Hkv, D]; idx: [B, Hkv, nrows, n_sel] or NULL for dense causal
 * attention (all s <= t); y: [B, nrows, Hq, D].
 */
void oracle_attention(const double *q, const double *k, const double *v, const double *g,
                      const int32_t *idx, int n_sel, int B, int T, int Hq, int Hkv, int D,
                      int blk, double scale, const int64_t *rows, int nrows, double *y)
{
    int grp = Hq / Hkv;
#pragma omp parallel for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < nrows; ++r)
            for (int h = 0; h < Hq; ++h) {
                int64_t t = rows ? rows[r] : r;
                int hk = h / grp;
                char *mark = (char *)calloc((size_t)(t + 1), 1);
                if (idx) {
                    const int32_t *ir = idx + (((int64_t)b * Hkv + hk) * nrows + r) * n_sel;
                    for (int e = 0; e < n_sel; ++e) {
                        int64_t j = ir[e];
                        if (j < 0) continue;
                        for (int64_t s = j * blk; s < (j + 1) * blk && s <= t && s < T; ++s) mark[s] = 1;
                    }
                } else {
                    for (int64_t s = 0; s <= t; ++s) mark[s] = 1;
                }
                const double *qr = q + IDX4(b, r, h, 0, nrows, Hq, D);
                double *yo = y + IDX4(b, r, h, 0, nrows, Hq, D);
                double m = -INFINITY;
                int64_t cnt = 0;
                for (int64_t s = 0; s <= t; ++s) {
                    if (!mark[s]) continue;
                    const double *ks = k + IDX4(b, s, hk, 0, T, Hkv, D);
                    double a = 0.0;
                    for (int d = 0; d < D; ++d) a += qr[d] * ks[d];
                    a *= scale;
                    if (a > m) m = a;
                    ++cnt;
                }
                for (int d = 0; d < D; ++d) yo[d] = 0.0;
                if (cnt > 0) {
                    double l = 0.0;
                    for (int64_t s = 0; s <= t; ++s) {
                        if (!mark[s]) continue;
                        const double *ks = k + IDX4(b, s, hk, 0, T, Hkv, D);
                        const double *vs = v + IDX4(b, s, hk, 0, T, Hkv, D);
                        double a = 0.0;
                        for (int d = 0; d < D; ++d) a += qr[d] * ks[d];
                        double p = exp(a * scale - m);
                        l += p;
                        for (int d = 0; d < D; ++d) yo[d] += p * vs[d];
                    }
                    for (int d = 0; d < D; ++d) yo[d] /= l;
                }
                if (g) {
                    const double *gr = g + IDX4(b, r, h, 0, nrows, Hq, D);
                    for (int d = 0; d < D; ++d) yo[d] *= sigmoid(gr[d]);
                }
                free(mark);
            }
}

/* ------------------------------------------------------------------------ */
/* Input projection of a Lightning layer with its preparation fused in.      */
/* ------------------------------------------------------------------------ */

/*
 * Plain matrix product y = x W^T: x [M, K] (rows = tokens), W [N, K] (rows =
 * output features, the layout of a linear layer's weight), y [M, N].
 */
void oracle_matmul_nt(const double *x, const double *w, int64_t M, int K, int N, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += x[m * K + k] * w[(int64_t)n * K + k];
            y[m * N + n] = acc;
        }
}

/*
 * Lightning-layer inputs from hidden states x [B, T, hidden] (tech-report mirror,
 * section 02 (3): QK-normalisation and an output gate in the linear layers; section
 * 02 (4): RoPE in the linear layers):
 *   [q | k | v | g] = x W^T, W [4 H D, hidden] with the q rows first, then k, v, g
 *   (head h of a section = its rows h D .. h D + D - 1);
 *   qh = RoPE(RMSNorm(q) * qw), kh = RoPE(RMSNorm(k) * kw) at position pos0 + t;
 *   v unchanged; gate = sigmoid(g), the output gate's multiplier.
 * qw, kw: [D] or NULL (weight 1).  Outputs qh, kh, v, gate: [B, T, H, D].
 */
void oracle_lightning_projection(const double *x, const double *w, const double *qw,
                                 const double *kw, int B, int T, int hidden, int H, int D,
                                 int64_t pos0, double base, double eps, double *qh, double *kh,
                                 double *v, double *gate)
{
    int N = 4 * H * D;
    int64_t M = (int64_t)B * T;
    double *y = (double *)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * N);
    oracle_matmul_nt(x, w, M, hidden, N, y);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int h = 0; h < H; ++h) {
            int64_t t = m % T;
            const double *row = y + m * N;
            int64_t o = (m * H + h) * D;
            oracle_qk_prep(row + (int64_t)(0 * H + h) * D, qw, D, eps, (double)(pos0 + t), base,
                           qh + o);
            oracle_qk_prep(row + (int64_t)(1 * H + h) * D, kw, D, eps, (double)(pos0 + t), base,
                           kh + o);
            for (int d = 0; d < D; ++d) {
                v[o + d] = row[(int64_t)(2 * H + h) * D + d];
                gate[o + d] = sigmoid(row[(int64_t)(3 * H + h) * D + d]);
            }
        }
    free(y);
}
