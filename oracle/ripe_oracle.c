/*
 * ripe_oracle.c -- plain fp64 CPU oracle for RIPE verify-attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product calls this file: only the
 * tests, the smoke check and the benchmark's CPU-baseline leg load it.  It shares
 * no code, header or constant with the CUDA library.
 *
 * What it computes.  The RIPE abstract (zhuanzhiai.com mirror, the sentences
 * on R planes per recurrent layer and on the RIPE store): a looped LM keeps R KV planes per
 * recurrent layer, one per loop; RIPE stores the deepest plane R for every
 * position and all R planes only for a window of recent positions.  Verification
 * of a draft block reads, for a query at loop depth r:
 *   - committed positions p in [0, T) at plane r if p is still inside the window
 *     (p >= ws, the store's window start), otherwise at the deepest plane R;
 *   - the draft-block tokens j' = 0..j of its own branch at plane r (causal).
 * Branches at different recurrent depths are verified in one batched call
 * (LoopSpec article on rit.work, section on the early draft branch).
 *
 * For row j of a branch (sequence b, depth r) and head h, with keys k_p and
 * values v_p drawn as above:
 *   s_p = scale * <q, k_p>,  o = sum_p softmax(s)_p v_p,  lse = ln sum_p e^{s_p}.
 * Everything is fp64; inputs arrive as fp64 copies of the exact bf16/fp32 values.
 *
 * Two evaluations of the same definition are provided:
 *   mode 0 (naive):  gather every score of the row, subtract the max, normalise;
 *   mode 1 (region): partial softmax sums over the deep region [0, min(ws,T)),
 *                    the window region [min(ws,T), T) and the draft block, then
 *                    merged by their maxima -- the two-region split of the
 *                    method, written out in three steps.
 *
 * Input layout (logical, not the GPU store's):
 *   Kd/Vd  + deep_off[b]: [H][T_b][d]           plane R of positions 0..T_b-1
 *   Kw/Vw  + win_off[b] : [H][R-1][T_b-lo_b][d] planes 1..R-1 of positions
 *                          lo_b..T_b-1, lo_b = min(ws_b, T_b)
 *   branches            : nbranch x {seq, depth (1..R), ntok, row0, row_stride}
 *   Q, Kb, Vb, O        : [nrows][H][d]; row of token j = row0 + j*row_stride
 *   lse                 : [nrows][H] (natural log)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t T, lo, ws;
    const double *kd, *vd, *kw, *vw;
} seq_view;

typedef struct {
    int H, d, R;
    const seq_view* seqs;
    const int32_t* br;
    const double *Q, *Kb, *Vb;
    double scale;
} problem;

/* Key / value row of committed position p read at depth r, head h. */
static const double* committed_row(const problem* P, const seq_view* s, int h, int64_t p, int r,
                                   int want_v) {
    const int d = P->d, R = P->R;
    if (r < R && p >= s->ws) {
        int64_t nw = s->T - s->lo;
        const double* base = want_v ? s->vw : s->kw;
        return base + (((int64_t)h * (R - 1) + (r - 1)) * nw + (p - s->lo)) * d;
    }
    const double* base = want_v ? s->vd : s->kd;
    return base + ((int64_t)h * s->T + p) * d;
}

static double dot(const double* a, const double* b, int d) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += a[c] * b[c];
    return acc;
}

/* mode 0: every score of the row, then one max-subtracted softmax. */
static void row_naive(const problem* P, int i, int j, int h, double* out, double* lse_out,
                      double* scores) {
    const int32_t* b = P->br + 5 * i;
    const seq_view* s = P->seqs + b[0];
    const int r = b[1], row0 = b[3], stride = b[4], H = P->H, d = P->d;
    const double* q = P->Q + ((int64_t)(row0 + j * stride) * H + h) * d;
    int64_t n = 0;
    for (int64_t p = 0; p < s->T; ++p)
        scores[n++] = P->scale * dot(q, committed_row(P, s, h, p, r, 0), d);
    for (int jj = 0; jj <= j; ++jj)
        scores[n++] = P->scale * dot(q, P->Kb + ((int64_t)(row0 + jj * stride) * H + h) * d, d);
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) m = scores[t] > m ? scores[t] : m;
    double sum = 0.0;
    for (int64_t t = 0; t < n; ++t) { scores[t] = exp(scores[t] - m); sum += scores[t]; }
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    n = 0;
    for (int64_t p = 0; p < s->T; ++p) {
        const double* v = committed_row(P, s, h, p, r, 1);
        double w = scores[n++] / sum;
        for (int c = 0; c < d; ++c) out[c] += w * v[c];
    }
    for (int jj = 0; jj <= j; ++jj) {
        const double* v = P->Vb + ((int64_t)(row0 + jj * stride) * H + h) * d;
        double w = scores[n++] / sum;
        for (int c = 0; c < d; ++c) out[c] += w * v[c];
    }
    *lse_out = m + log(sum);
}

/* A partial softmax sum over one region: max m, sum l of e^{s-m}, o = sum e^{s-m} v. */
typedef struct { double m, l; double* o; } partial;

static void partial_reset(partial* pt, int d) {
    pt->m = -INFINITY; pt->l = 0.0;
    for (int c = 0; c < d; ++c) pt->o[c] = 0.0;
}

/* Two passes over the region's keys: the max, then the sums. */
static void partial_committed(const problem* P, const seq_view* s, int h, int r, const double* q,
                              int64_t p0, int64_t p1, partial* pt) {
    const int d = P->d;
    partial_reset(pt, d);
    for (int64_t p = p0; p < p1; ++p) {
        double sc = P->scale * dot(q, committed_row(P, s, h, p, r, 0), d);
        if (sc > pt->m) pt->m = sc;
    }
    for (int64_t p = p0; p < p1; ++p) {
        double w = exp(P->scale * dot(q, committed_row(P, s, h, p, r, 0), d) - pt->m);
        const double* v = committed_row(P, s, h, p, r, 1);
        pt->l += w;
        for (int c = 0; c < d; ++c) pt->o[c] += w * v[c];
    }
}

static void partial_block(const problem* P, int i, int j, int h, const double* q, partial* pt) {
    const int32_t* b = P->br + 5 * i;
    const int row0 = b[3], stride = b[4], H = P->H, d = P->d;
    partial_reset(pt, d);
    for (int jj = 0; jj <= j; ++jj) {
        double sc = P->scale * dot(q, P->Kb + ((int64_t)(row0 + jj * stride) * H + h) * d, d);
        if (sc > pt->m) pt->m = sc;
    }
    for (int jj = 0; jj <= j; ++jj) {
        int64_t rr = ((int64_t)(row0 + jj * stride) * H + h) * d;
        double w = exp(P->scale * dot(q, P->Kb + rr, d) - pt->m);
        pt->l += w;
        for (int c = 0; c < d; ++c) pt->o[c] += w * P->Vb[rr + c];
    }
}

/* mode 1: deep region, window region and block, each a partial, then merged:
 * M = max_i m_i, L = sum_i l_i e^{m_i-M}, o = sum_i e^{m_i-M} o_i / L, lse = M + ln L. */
static void row_region(const problem* P, int i, int j, int h, double* out, double* lse_out,
                       double* work) {
    const int32_t* b = P->br + 5 * i;
    const seq_view* s = P->seqs + b[0];
    const int r = b[1], row0 = b[3], stride = b[4], H = P->H, d = P->d;
    const double* q = P->Q + ((int64_t)(row0 + j * stride) * H + h) * d;
    partial pts[3];
    for (int t = 0; t < 3; ++t) pts[t].o = work + (int64_t)t * d;
    partial_committed(P, s, h, P->R, q, 0, s->lo, &pts[0]);
    partial_committed(P, s, h, r, q, s->lo, s->T, &pts[1]);
    partial_block(P, i, j, h, q, &pts[2]);
    double M = -INFINITY;
    for (int t = 0; t < 3; ++t)
        if (pts[t].l > 0.0 && pts[t].m > M) M = pts[t].m;
    double L = 0.0;
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int t = 0; t < 3; ++t) {
        if (pts[t].l == 0.0) continue;
        double a = exp(pts[t].m - M);
        L += a * pts[t].l;
        for (int c = 0; c < d; ++c) out[c] += a * pts[t].o[c];
    }
    for (int c = 0; c < d; ++c) out[c] /= L;
    *lse_out = M + log(L);
}

int oracle_verify(int nseq, int H, int d, int R,
                  const int64_t* T, const int64_t* ws,
                  const int64_t* deep_off, const double* Kd, const double* Vd,
                  const int64_t* win_off, const double* Kw, const double* Vw,
                  int nbranch, const int32_t* branches,
                  int nrows, const double* Q, const double* Kb, const double* Vb,
                  double scale, int mode, double* O, double* lse) {
    if (nseq < 0 || H <= 0 || d <= 0 || R <= 0 || nbranch < 0 || nrows < 0) return 1;
    seq_view* seqs = (seq_view*)calloc(nseq > 0 ? nseq : 1, sizeof(seq_view));
    if (!seqs) return 2;
    int64_t maxT = 0;
    for (int b = 0; b < nseq; ++b) {
        seqs[b].T = T[b];
        seqs[b].ws = ws[b];
        seqs[b].lo = ws[b] < T[b] ? ws[b] : T[b];
        seqs[b].kd = Kd + deep_off[b];
        seqs[b].vd = Vd + deep_off[b];
        seqs[b].kw = Kw ? Kw + win_off[b] : NULL;
        seqs[b].vw = Vw ? Vw + win_off[b] : NULL;
        if (T[b] > maxT) maxT = T[b];
    }
    int maxn = 0;
    for (int i = 0; i < nbranch; ++i) {
        const int32_t* b = branches + 5 * i;
        if (b[0] < 0 || b[0] >= nseq || b[1] < 1 || b[1] > R || b[2] < 0) { free(seqs); return 1; }
        if (b[2] > maxn) maxn = b[2];
        if (b[2] > 0 && (b[3] < 0 || b[3] + (int64_t)(b[2] - 1) * b[4] >= nrows)) { free(seqs); return 1; }
    }
    problem P = {H, d, R, seqs, branches, Q, Kb, Vb, scale};
    int64_t nunits = (int64_t)nbranch * H;
#pragma omp parallel
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)(maxT + maxn + 1));
        double* work = (double*)malloc(sizeof(double) * (size_t)(3 * d));
#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < nunits; ++u) {
            int i = (int)(u / H), h = (int)(u % H);
            const int32_t* b = branches + 5 * i;
            for (int j = 0; j < b[2]; ++j) {
                int64_t row = b[3] + (int64_t)j * b[4];
                double* out = O + (row * H + h) * d;
                double* l = lse + row * H + h;
                if (mode == 0) row_naive(&P, i, j, h, out, l, scores);
                else row_region(&P, i, j, h, out, l, work);
            }
        }
        free(scores);
        free(work);
    }
    free(seqs);
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Sliding-window reading (the RIPE abstract's fifth sentence, read per query):
 * the query of draft token j sits at position T + j and sees the W most recent
 * positions T+j-W+1 .. T+j at its own depth r, everything older at the deepest
 * plane R.  Committed position p is read at plane r if p >= T + j - W + 1 and the
 * store still holds its planes (p >= ws), else at plane R; draft token j' <= j at
 * plane r if j' >= j - W + 1, else at plane R.  The plane-R key and value of draft
 * token j' are those of the same token's depth-R row, so the branches must be the
 * all-depths form of one sequence each: branch (s, r) has row0 = s*k*R + r - 1 and
 * row_stride R.  Every score of a row is gathered, then one max-subtracted softmax
 * (the definition written out, as mode 0).
 */
int oracle_verify_sliding(int nseq, int H, int d, int R, int W,
                          const int64_t* T, const int64_t* ws,
                          const int64_t* deep_off, const double* Kd, const double* Vd,
                          const int64_t* win_off, const double* Kw, const double* Vw,
                          int nbranch, const int32_t* branches,
                          int nrows, const double* Q, const double* Kb, const double* Vb,
                          double scale, double* O, double* lse) {
    if (nseq < 0 || H <= 0 || d <= 0 || R <= 0 || W < 0 || nbranch < 0 || nrows < 0) return 1;
    seq_view* seqs = (seq_view*)calloc(nseq > 0 ? nseq : 1, sizeof(seq_view));
    if (!seqs) return 2;
    int64_t maxT = 0;
    for (int b = 0; b < nseq; ++b) {
        seqs[b].T = T[b];
        seqs[b].ws = ws[b];
        seqs[b].lo = ws[b] < T[b] ? ws[b] : T[b];
        seqs[b].kd = Kd + deep_off[b];
        seqs[b].vd = Vd + deep_off[b];
        seqs[b].kw = Kw ? Kw + win_off[b] : NULL;
        seqs[b].vw = Vw ? Vw + win_off[b] : NULL;
        if (T[b] > maxT) maxT = T[b];
    }
    int maxn = 0;
    for (int i = 0; i < nbranch; ++i) {
        const int32_t* b = branches + 5 * i;
        if (b[0] < 0 || b[0] >= nseq || b[1] < 1 || b[1] > R || b[2] < 0 || b[4] != R) { free(seqs); return 1; }
        if (b[2] > maxn) maxn = b[2];
        const int64_t rowR0 = (int64_t)b[3] - (b[1] - 1) + (R - 1);
        if (b[2] > 0 && (b[3] < 0 || rowR0 + (int64_t)(b[2] - 1) * R >= nrows)) { free(seqs); return 1; }
    }
    problem P = {H, d, R, seqs, branches, Q, Kb, Vb, scale};
    int64_t nunits = (int64_t)nbranch * H;
#pragma omp parallel
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)(maxT + maxn + 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < nunits; ++u) {
            const int i = (int)(u / H), h = (int)(u % H);
            const int32_t* b = branches + 5 * i;
            const seq_view* s = seqs + b[0];
            const int r = b[1], row0 = b[3];
            const int64_t rowR0 = (int64_t)row0 - (r - 1) + (R - 1);
            for (int j = 0; j < b[2]; ++j) {
                const int64_t row = row0 + (int64_t)j * R;
                const double* q = Q + (row * H + h) * d;
                const int64_t start = s->T + j - W + 1;   /* first position of the row's window */
                int64_t n = 0;
                for (int64_t p = 0; p < s->T; ++p) {
                    const int plane = (p >= start && p >= s->ws) ? r : R;
                    scores[n++] = scale * dot(q, committed_row(&P, s, h, p, plane, 0), d);
                }
                for (int jj = 0; jj <= j; ++jj) {
                    const int64_t kr = (jj >= j - W + 1) ? row0 + (int64_t)jj * R : rowR0 + (int64_t)jj * R;
                    scores[n++] = scale * dot(q, Kb + (kr * H + h) * d, d);
                }
                double m = -INFINITY;
                for (int64_t t = 0; t < n; ++t) m = scores[t] > m ? scores[t] : m;
                double sum = 0.0;
                for (int64_t t = 0; t < n; ++t) { scores[t] = exp(scores[t] - m); sum += scores[t]; }
                double* out = O + (row * H + h) * d;
                for (int c = 0; c < d; ++c) out[c] = 0.0;
                n = 0;
                for (int64_t p = 0; p < s->T; ++p) {
                    const int plane = (p >= start && p >= s->ws) ? r : R;
                    const double* v = committed_row(&P, s, h, p, plane, 1);
                    const double w = scores[n++] / sum;
                    for (int c = 0; c < d; ++c) out[c] += w * v[c];
                }
                for (int jj = 0; jj <= j; ++jj) {
                    const int64_t kr = (jj >= j - W + 1) ? row0 + (int64_t)jj * R : rowR0 + (int64_t)jj * R;
                    const double* v = Vb + (kr * H + h) * d;
                    const double w = scores[n++] / sum;
                    for (int c = 0; c < d; ++c) out[c] += w * v[c];
                }
                lse[row * H + h] = m + log(sum);
            }
        }
        free(scores);
    }
    free(seqs);
    return 0;
}
