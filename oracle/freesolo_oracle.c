/*
 * FreeSolo sparse-attention forward pass: plain float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this code.  The CUDA library never links, calls or
 * includes it, and this file includes nothing from the CUDA library.
 *
 * Source: "FreeSolo" technical summary, section "Methodology":
 *   §3.1 Range Separation  eq. (2)   o_i = o_i^sr + alpha_h o_i^lr
 *   §3.2 Local Branch      eq. (3)   RoPE logits inside the look-back radius w
 *                          eq. (4)   softmax readout over the local set L_i
 *   §3.3 Long-Range Branch eq. (5)   cell summaries kbar_c, p_c, a_c over s-token cells
 *                          eq. (7)   cell score r_ic with the erf position prior
 *                          eq. (8)   FS-L pruning A_i = Recent_W(C_i) u TopP(a_c)
 *                          eq. (9)   NoPE token readout over the selected cells, RMSNorm
 *   §3.4                   eqs. (10)-(11) FS-B: beam search over two causal forests of
 *                                    balanced trees (all candidates; cells with a_c >= tau_h)
 *                          eq. (12)  token-level rerank: a cell scored by the log-sum-exp
 *                                    of its tokens' NoPE logits plus the prior term
 * "Introduction and Theoretical Foundation": RoPE (Su et al.) is applied only inside the
 * local window; the long-range branch selects and reads cells without rotation.
 *
 * Readings where the page is silent or garbled (each is also listed in the design notes):
 *   - L_i = { j : max(0, i-w) <= j <= i }            ("look-back radius w", §3.2)
 *   - C_i = { c : (c+1)s <= i-w }, full cells only    (eq. (6) is missing from the page)
 *   - RoPE: interleaved pairs (2m, 2m+1), theta_m = base^(-2m/d) (Su et al.)
 *   - RMSNorm(u) = u / sqrt(mean(u^2) + eps), no learned gain
 *   - ties in TopP and top-K: larger value first, then the lower cell index
 *   - |A_i| < K: all of A_i is selected; S_i empty gives o^lr = 0
 *   - W < 0 and P < 0 together mean "no pruning" (base FS: A_i = C_i)
 *   - backward pass: the selection (a top-K, piecewise constant in Q and K) is held
 *     fixed, and the summaries, which only feed the selection, get no gradient
 *   - eq. (12) reranks a shortlist: the `shortlist` best cells of A_i by eq. (7)
 *     (shortlist <= 0: all of A_i) are rescored by eq. (12) and the K best kept; its
 *     g_h is eq. (7)'s erf((i - p_c) / (2 sigma_h)) (eq. (11) uses the same name)
 *   - FS-B (eqs. (10)-(11)): the forests, leaf order, node statistics and beam rules
 *     are stated above orc_tree_select_rows
 *
 * Every quantity is computed in double from the float32 inputs (bf16 inputs are
 * passed as their exact float32 values).  No tiling, fusion or reordering beyond
 * what the equations state; the only memo is that the rotated keys and the cell
 * summaries of a (batch, head) are computed once and reused by its rows.
 *
 * Parity status: pinned (brute force, closed forms, invariants); see the tests.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, H, Nq, Nk, d;     /* Q is [B,H,Nq,d]; K,V are [B,H,Nk,d]; row-major */
    int w, s, K;             /* look-back radius, cell size, cells kept per query */
    int W, P;                /* FS-L recent / norm budgets; both < 0 => no pruning */
    double rope_base;        /* RoPE base (10000) */
    double rms_eps;          /* RMSNorm epsilon */
    long long pos0;          /* absolute position of key index 0 (shift checks) */
    const double *alpha;     /* [H] range-combination weights, eq. (2) */
    const double *lambda;    /* [H] prior weights, eq. (7); NULL => 0 */
    const double *sigma;     /* [H] prior widths, eq. (7); NULL => unused */
    int mutation;            /* 0 always, except tests that plant a known mistake */
} orc_params;

/* Planted mistakes, used only by the pin-sensitivity tests. */
enum {
    MUT_NONE = 0,
    MUT_ROPE_KEY_SIGN = 1,   /* keys rotated by R(-j): breaks eq. (3) */
    MUT_DROP_PRIOR = 2,      /* eq. (7) without the erf term */
    MUT_WINDOW_SHORT = 3,    /* L_i starts at i-w+1 */
    MUT_CAND_LOOSE = 4,      /* C_i takes cells with c*s <= i-w (overlapping the window) */
    MUT_AMAX_MEAN = 5,       /* a_c = mean norm instead of max (eq. (5)) */
    MUT_NO_EPS = 6,          /* RMSNorm without eps */
    MUT_ALPHA_ON_SR = 7,     /* o = alpha*o^sr + o^lr (eq. (2) transposed) */
    MUT_ROPE_IN_READOUT = 8, /* long-range readout uses rotated vectors */
    MUT_SCALE_D = 9,         /* logits scaled by 1/d instead of 1/sqrt(d) */
    MUT_TIE_HIGH_INDEX = 10, /* ties broken toward the higher cell index */
    MUT_RERANK_MEAN = 11,    /* eq. (12) with the mean logit instead of the log-sum-exp */
    MUT_RERANK_ROPE = 12,    /* eq. (12) with rotated query and keys */
    MUT_BWD_NO_RMS = 13,     /* backward: RMSNorm treated as a constant scale */
    MUT_TREE_NO_RHO = 14,    /* eq. (11) without the c ||q|| rho_v term */
    MUT_TREE_PMAX = 15,      /* eq. (11) prior at the latest cell of v instead of p_v^min */
    MUT_TREE_SORT_DESC = 16, /* tree leaves in descending code order */
};

int orc_num_cells(const orc_params *p) { return p->s > 0 ? p->Nk / p->s : 0; }

static int pruning_on(const orc_params *p) { return !(p->W < 0 && p->P < 0); }

/* |C_i| for the key-index position i of a query: cells c with (c+1)s <= i-w. */
int orc_candidate_count(const orc_params *p, long long i)
{
    long long lim = i - p->w;                 /* (c+1)s <= lim */
    if (p->mutation == MUT_CAND_LOOSE) lim += p->s;
    if (lim < p->s) return 0;
    long long n = lim / p->s;
    int C = orc_num_cells(p);
    return (int)(n < C ? n : C);
}

/* ---- small deterministic sort: by value descending, then index ascending ---- */
typedef struct { double v; int idx; } vi_pair;

static int beats(const vi_pair *a, const vi_pair *b, int tie_high)
{
    if (a->v > b->v) return 1;
    if (a->v < b->v) return 0;
    return tie_high ? (a->idx > b->idx) : (a->idx < b->idx);
}

static void sort_desc(vi_pair *x, int n, vi_pair *tmp, int tie_high)
{   /* bottom-up merge sort; stable and O(n log n) */
    for (int width = 1; width < n; width *= 2) {
        for (int lo = 0; lo < n; lo += 2 * width) {
            int mid = lo + width < n ? lo + width : n;
            int hi = lo + 2 * width < n ? lo + 2 * width : n;
            int a = lo, b = mid, o = lo;
            while (a < mid && b < hi) tmp[o++] = beats(&x[b], &x[a], tie_high) ? x[b++] : x[a++];
            while (a < mid) tmp[o++] = x[a++];
            while (b < hi) tmp[o++] = x[b++];
        }
        memcpy(x, tmp, sizeof(vi_pair) * (size_t)n);
    }
}

static int cmp_int(const void *a, const void *b)
{
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* ---- eq. (5): cell summaries of one (b,h) head ---- */
static void summaries_bh(const orc_params *p, const float *Kbh, double *kbar, double *amax)
{
    const int C = orc_num_cells(p), d = p->d, s = p->s;
    for (int c = 0; c < C; c++) {
        double *kb = kbar + (size_t)c * d;
        for (int m = 0; m < d; m++) kb[m] = 0.0;
        double best = 0.0, normsum = 0.0;
        for (int t = 0; t < s; t++) {
            const float *k = Kbh + ((size_t)c * s + t) * d;
            double sq = 0.0;
            for (int m = 0; m < d; m++) {
                kb[m] += (double)k[m];
                sq += (double)k[m] * (double)k[m];
            }
            double nrm = sqrt(sq);
            normsum += nrm;
            if (t == 0 || nrm > best) best = nrm;
        }
        for (int m = 0; m < d; m++) kb[m] /= (double)s;
        amax[c] = (p->mutation == MUT_AMAX_MEAN) ? normsum / s : best;
    }
}

/* Summaries for every (b,h): kbar [B,H,C,d], amax [B,H,C]. */
void orc_cell_summaries(const orc_params *p, const float *K, double *kbar, double *amax)
{
    const int C = orc_num_cells(p);
    #pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < p->B * p->H; bh++)
        summaries_bh(p, K + (size_t)bh * p->Nk * p->d, kbar + (size_t)bh * C * p->d,
                     amax + (size_t)bh * C);
}

/* ---- eq. (8): admitted cells A for a candidate prefix of n cells (ascending) ---- */
int orc_admitted(const orc_params *p, const double *amax_bh, int n, int *out)
{
    if (n <= 0) return 0;
    if (!pruning_on(p)) {
        for (int c = 0; c < n; c++) out[c] = c;
        return n;
    }
    char *in = (char *)calloc((size_t)n, 1);
    int W = p->W < 0 ? 0 : p->W, P = p->P < 0 ? 0 : p->P;
    for (int c = n - W; c < n; c++)                     /* Recent_W(C_i) */
        if (c >= 0) in[c] = 1;
    if (P > 0) {                                        /* TopP over C_i by a_c */
        vi_pair *x = (vi_pair *)malloc(sizeof(vi_pair) * (size_t)n);
        vi_pair *tmp = (vi_pair *)malloc(sizeof(vi_pair) * (size_t)n);
        for (int c = 0; c < n; c++) { x[c].v = amax_bh[c]; x[c].idx = c; }
        sort_desc(x, n, tmp, p->mutation == MUT_TIE_HIGH_INDEX);
        for (int t = 0; t < P && t < n; t++) in[x[t].idx] = 1;
        free(x); free(tmp);
    }
    int cnt = 0;
    for (int c = 0; c < n; c++) if (in[c]) out[cnt++] = c;
    free(in);
    return cnt;
}

/* ---- RoPE (Su et al.): interleaved pairs rotated by pos * theta_m ---- */
static void rope_rotate(const orc_params *p, const float *x, long long pos, double *out)
{
    const int d = p->d;
    for (int m = 0; m < d / 2; m++) {
        double theta = pow(p->rope_base, -2.0 * m / (double)d);
        double ang = (double)pos * theta;
        double cs = cos(ang), sn = sin(ang);
        double x0 = x[2 * m], x1 = x[2 * m + 1];
        out[2 * m] = x0 * cs - x1 * sn;
        out[2 * m + 1] = x0 * sn + x1 * cs;
    }
}

static double logit_scale(const orc_params *p)
{
    return p->mutation == MUT_SCALE_D ? 1.0 / p->d : 1.0 / sqrt((double)p->d);
}

/* ---- eq. (7) + top-K for one query row ----
 * idx_out[K]: selected cells ascending, -1 padded.  If acells/ascores are given they
 * receive A_i and the scores r_ic (in A_i's ascending order).  Returns |A_i|. */
static int select_row(const orc_params *p, const float *qrow, long long i, int h,
                      const double *kbar_bh, const double *amax_bh,
                      int *idx_out, int *acells, double *ascores)
{
    const int d = p->d, Kc = p->K;
    int n = orc_candidate_count(p, i);
    int *A = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
    int nA = orc_admitted(p, amax_bh, n, A);
    vi_pair *x = (vi_pair *)malloc(sizeof(vi_pair) * (size_t)(nA > 0 ? nA : 1));
    vi_pair *tmp = (vi_pair *)malloc(sizeof(vi_pair) * (size_t)(nA > 0 ? nA : 1));
    double lam = p->lambda ? p->lambda[h] : 0.0;
    if (p->mutation == MUT_DROP_PRIOR) lam = 0.0;
    double sig = p->sigma ? p->sigma[h] : 1.0;
    double pos_i = (double)(p->pos0 + i);
    for (int t = 0; t < nA; t++) {
        int c = A[t];
        const double *kb = kbar_bh + (size_t)c * d;
        double dot = 0.0;
        for (int m = 0; m < d; m++) dot += (double)qrow[m] * kb[m];
        double r = dot * logit_scale(p);
        if (lam != 0.0) {
            double p_c = (double)p->pos0 + (c + 0.5) * p->s;
            r += lam * amax_bh[c] * erf((pos_i - p_c) / (2.0 * sig));
        }
        x[t].v = r; x[t].idx = c;
        if (acells) acells[t] = c;
        if (ascores) ascores[t] = r;
    }
    sort_desc(x, nA, tmp, p->mutation == MUT_TIE_HIGH_INDEX);
    int keep = nA < Kc ? nA : Kc;
    for (int t = 0; t < keep; t++) idx_out[t] = x[t].idx;
    qsort(idx_out, (size_t)keep, sizeof(int), cmp_int);
    for (int t = keep; t < Kc; t++) idx_out[t] = -1;
    free(A); free(x); free(tmp);
    return nA;
}

/* ---- eq. (9): NoPE token readout over the selected cells, then RMSNorm ---- */
static void readout_row(const orc_params *p, const float *qrow, long long i,
                        const float *Kbh, const float *Vbh, const int *idx,
                        double *u_out, double *olr_out)
{
    const int d = p->d, s = p->s, Kc = p->K;
    int ncell = 0;
    for (int t = 0; t < Kc; t++) if (idx[t] >= 0) ncell++;
    double *u = (double *)calloc((size_t)d, sizeof(double));
    if (ncell > 0) {
        int ntok = ncell * s;
        double *lg = (double *)malloc(sizeof(double) * (size_t)ntok);
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
        double *kv = (double *)malloc(sizeof(double) * (size_t)d);
        if (p->mutation == MUT_ROPE_IN_READOUT) rope_rotate(p, qrow, p->pos0 + i, qv);
        else for (int m = 0; m < d; m++) qv[m] = qrow[m];
        int t = 0;
        double mx = -INFINITY;
        for (int e = 0; e < Kc; e++) {
            if (idx[e] < 0) continue;
            for (int j = idx[e] * s; j < (idx[e] + 1) * s; j++, t++) {
                const float *k = Kbh + (size_t)j * d;
                if (p->mutation == MUT_ROPE_IN_READOUT) rope_rotate(p, k, p->pos0 + j, kv);
                else for (int m = 0; m < d; m++) kv[m] = k[m];
                double dot = 0.0;
                for (int m = 0; m < d; m++) dot += qv[m] * kv[m];
                lg[t] = dot * logit_scale(p);
                if (lg[t] > mx) mx = lg[t];
            }
        }
        double den = 0.0;
        t = 0;
        for (int e = 0; e < Kc; e++) {
            if (idx[e] < 0) continue;
            for (int j = idx[e] * s; j < (idx[e] + 1) * s; j++, t++) {
                double pj = exp(lg[t] - mx);
                den += pj;
                const float *v = Vbh + (size_t)j * d;
                for (int m = 0; m < d; m++) u[m] += pj * (double)v[m];
            }
        }
        for (int m = 0; m < d; m++) u[m] /= den;
        free(lg); free(qv); free(kv);
    }
    double ms = 0.0;
    for (int m = 0; m < d; m++) ms += u[m] * u[m];
    ms /= d;
    double eps = p->mutation == MUT_NO_EPS ? 0.0 : p->rms_eps;
    double inv = (ncell > 0 && ms + eps > 0.0) ? 1.0 / sqrt(ms + eps) : 0.0;
    for (int m = 0; m < d; m++) {
        if (u_out) u_out[m] = u[m];
        olr_out[m] = u[m] * inv;
    }
    free(u);
}

/* ---- eqs. (3)-(4): RoPE attention over L_i = [max(0,i-w), i] ---- */
static void window_row(const orc_params *p, const double *qrot, long long i,
                       const double *krot_bh, const float *Vbh, double *osr)
{
    const int d = p->d;
    long long lo = i - p->w;
    if (p->mutation == MUT_WINDOW_SHORT) lo += 1;
    if (lo < 0) lo = 0;
    long long n = i - lo + 1;
    double *lg = (double *)malloc(sizeof(double) * (size_t)n);
    double mx = -INFINITY;
    for (long long j = lo; j <= i; j++) {
        const double *k = krot_bh + (size_t)j * d;
        double dot = 0.0;
        for (int m = 0; m < d; m++) dot += qrot[m] * k[m];
        lg[j - lo] = dot * logit_scale(p);
        if (lg[j - lo] > mx) mx = lg[j - lo];
    }
    double den = 0.0;
    for (int m = 0; m < d; m++) osr[m] = 0.0;
    for (long long j = lo; j <= i; j++) {
        double pj = exp(lg[j - lo] - mx);
        den += pj;
        const float *v = Vbh + (size_t)j * d;
        for (int m = 0; m < d; m++) osr[m] += pj * (double)v[m];
    }
    for (int m = 0; m < d; m++) osr[m] /= den;
    free(lg);
}

/* Per-(b,h) state shared by that head's rows. */
typedef struct { double *kbar, *amax, *krot; } head_state;

static void head_prepare(const orc_params *p, const float *Kbh, head_state *st)
{
    const int C = orc_num_cells(p), d = p->d;
    st->kbar = (double *)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1) * d);
    st->amax = (double *)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
    st->krot = (double *)malloc(sizeof(double) * (size_t)p->Nk * d);
    summaries_bh(p, Kbh, st->kbar, st->amax);
    #pragma omp parallel for schedule(static)
    for (int j = 0; j < p->Nk; j++) {
        long long pos = p->pos0 + j;
        if (p->mutation == MUT_ROPE_KEY_SIGN) pos = -pos;
        rope_rotate(p, Kbh + (size_t)j * d, pos, st->krot + (size_t)j * d);
    }
}

static void head_release(head_state *st) { free(st->kbar); free(st->amax); free(st->krot); }

/* ---- eq. (2) for a list of rows ----
 * rows: flat indices (b*H + h)*Nq + r, or NULL for all B*H*Nq rows in order.
 * O [nrows, d]; idx_out [nrows, K] (may be NULL); olr_out/osr_out [nrows, d] (may be NULL).
 * Returns 0, or -1 on invalid arguments. */
int orc_forward(const orc_params *p, const float *Q, const float *K, const float *V,
                long long nrows, const long long *rows,
                double *O, int *idx_out, double *olr_out, double *osr_out)
{
    if (p->d <= 0 || (p->d & 1) || p->s <= 0 || p->K < 0 || p->w < 0) return -1;
    if (p->Nq > p->Nk) return -1;
    const int d = p->d, BH = p->B * p->H;
    const long long total = (long long)BH * p->Nq;
    if (!rows) nrows = total;
    /* bucket the requested rows by head so that each head is prepared once */
    long long *order = (long long *)malloc(sizeof(long long) * (size_t)(nrows > 0 ? nrows : 1));
    long long *start = (long long *)calloc((size_t)BH + 1, sizeof(long long));
    for (long long t = 0; t < nrows; t++) {
        long long f = rows ? rows[t] : t;
        if (f < 0 || f >= total) { free(order); free(start); return -1; }
        start[f / p->Nq + 1]++;
    }
    for (int bh = 0; bh < BH; bh++) start[bh + 1] += start[bh];
    long long *fill = (long long *)malloc(sizeof(long long) * (size_t)BH);
    for (int bh = 0; bh < BH; bh++) fill[bh] = start[bh];
    for (long long t = 0; t < nrows; t++) {
        long long f = rows ? rows[t] : t;
        order[fill[f / p->Nq]++] = t;
    }
    free(fill);

    for (int bh = 0; bh < BH; bh++) {
        if (start[bh] == start[bh + 1]) continue;
        const int h = bh % p->H;
        const float *Kbh = K + (size_t)bh * p->Nk * d;
        const float *Vbh = V + (size_t)bh * p->Nk * d;
        head_state st;
        head_prepare(p, Kbh, &st);
        #pragma omp parallel for schedule(dynamic, 4)
        for (long long e = start[bh]; e < start[bh + 1]; e++) {
            long long t = order[e];
            long long f = rows ? rows[t] : t;
            int r = (int)(f % p->Nq);
            long long i = (long long)(p->Nk - p->Nq) + r;   /* key-index position of row r */
            const float *qrow = Q + (size_t)f * d;
            double *qrot = (double *)malloc(sizeof(double) * (size_t)d);
            double *osr = (double *)malloc(sizeof(double) * (size_t)d);
            double *olr = (double *)malloc(sizeof(double) * (size_t)d);
            int *idx = (int *)malloc(sizeof(int) * (size_t)(p->K > 0 ? p->K : 1));
            rope_rotate(p, qrow, p->pos0 + i, qrot);
            window_row(p, qrot, i, st.krot, Vbh, osr);
            select_row(p, qrow, i, h, st.kbar, st.amax, idx, NULL, NULL);
            readout_row(p, qrow, i, Kbh, Vbh, idx, NULL, olr);
            double a = p->alpha ? p->alpha[h] : 0.0;
            for (int m = 0; m < d; m++) {
                O[(size_t)t * d + m] = (p->mutation == MUT_ALPHA_ON_SR)
                                           ? a * osr[m] + olr[m] : osr[m] + a * olr[m];
                if (olr_out) olr_out[(size_t)t * d + m] = olr[m];
                if (osr_out) osr_out[(size_t)t * d + m] = osr[m];
            }
            if (idx_out) memcpy(idx_out + (size_t)t * p->K, idx, sizeof(int) * (size_t)p->K);
            free(qrot); free(osr); free(olr); free(idx);
        }
        head_release(&st);
    }
    free(order); free(start);
    return 0;
}

/* ---- eq. (12): token-level rerank for one query row ----
 * The shortlist (the `shortlist` best cells of A_i by eq. (7); all of A_i if
 * shortlist <= 0) is rescored by
 *     rt_ic = log sum_{j in I_c} exp(q_i . k_j / sqrt(d)) + lambda_h a_c erf((i - p_c)/(2 sigma_h))
 * over the raw (unrotated) keys of the cell's tokens I_c, and the K best form S_i (ties:
 * lower cell).  idx_out[K] ascending, -1 padded; cells/scores (capacity >= |A_i|) receive
 * the shortlist (ascending) and its rt.  Returns the shortlist size. */
int orc_rerank_row(const orc_params *p, const float *Q, const float *K, const double *kbar,
                   const double *amax, int b, int h, int r, int shortlist, int *idx_out,
                   int *cells, double *scores)
{
    const int C = orc_num_cells(p), d = p->d, s = p->s;
    size_t bh = (size_t)b * p->H + h;
    long long i = (long long)(p->Nk - p->Nq) + r;
    const float *qrow = Q + (bh * p->Nq + r) * d;
    const float *Kbh = K + bh * (size_t)p->Nk * d;
    /* shortlist by eq. (7): select_row with K = shortlist (or |C_i| for all of A_i) */
    orc_params ps = *p;
    int n = orc_candidate_count(p, i);
    ps.K = shortlist > 0 ? shortlist : (n > 0 ? n : 1);
    int *sl = (int *)malloc(sizeof(int) * (size_t)ps.K);
    select_row(&ps, qrow, i, h, kbar + bh * C * d, amax + bh * C, sl, NULL, NULL);
    int ns = 0;
    while (ns < ps.K && sl[ns] >= 0) ns++;
    vi_pair *x = (vi_pair *)malloc(sizeof(vi_pair) * (size_t)(ns > 0 ? ns : 1));
    vi_pair *tmp = (vi_pair *)malloc(sizeof(vi_pair) * (size_t)(ns > 0 ? ns : 1));
    double lam = p->lambda ? p->lambda[h] : 0.0;
    double sig = p->sigma ? p->sigma[h] : 1.0;
    double pos_i = (double)(p->pos0 + i);
    double *lg = (double *)malloc(sizeof(double) * (size_t)s);
    double qv[512], kv[512];
    for (int t = 0; t < ns; t++) {
        int c = sl[t];
        double mx = -INFINITY, acc = 0.0;
        for (int j = 0; j < s; j++) {            /* the cell's token logits */
            long long jj = (long long)c * s + j;
            const float *k = Kbh + (size_t)jj * d;
            double dot = 0.0;
            if (p->mutation == MUT_RERANK_ROPE) {
                rope_rotate(p, qrow, p->pos0 + i, qv);
                rope_rotate(p, k, p->pos0 + jj, kv);
                for (int m = 0; m < d; m++) dot += qv[m] * kv[m];
            } else {
                for (int m = 0; m < d; m++) dot += (double)qrow[m] * k[m];
            }
            lg[j] = dot * logit_scale(p);
            if (lg[j] > mx) mx = lg[j];
            acc += lg[j];
        }
        double rt;
        if (p->mutation == MUT_RERANK_MEAN) {
            rt = acc / s;
        } else {                                  /* log-sum-exp, shifted by the max */
            double se = 0.0;
            for (int j = 0; j < s; j++) se += exp(lg[j] - mx);
            rt = mx + log(se);
        }
        if (lam != 0.0) {
            double p_c = (double)p->pos0 + (c + 0.5) * s;
            rt += lam * amax[bh * C + c] * erf((pos_i - p_c) / (2.0 * sig));
        }
        x[t].v = rt; x[t].idx = c;
        if (cells) cells[t] = c;
        if (scores) scores[t] = rt;
    }
    sort_desc(x, ns, tmp, p->mutation == MUT_TIE_HIGH_INDEX);
    int keep = ns < p->K ? ns : p->K;
    for (int t = 0; t < keep; t++) idx_out[t] = x[t].idx;
    qsort(idx_out, (size_t)keep, sizeof(int), cmp_int);
    for (int t = keep; t < p->K; t++) idx_out[t] = -1;
    free(sl); free(x); free(tmp); free(lg);
    return ns;
}

/* x rotated by R(pos)^T = R(-pos) (double vectors): the adjoint of the RoPE rotation */
static void rope_rotate_back(const orc_params *p, const double *x, long long pos, double *out)
{
    const int d = p->d;
    for (int m = 0; m < d / 2; m++) {
        double theta = pow(p->rope_base, -2.0 * m / (double)d);
        double ang = (double)pos * theta;
        double cs = cos(ang), sn = sin(ang);
        out[2 * m] = x[2 * m] * cs + x[2 * m + 1] * sn;
        out[2 * m + 1] = -x[2 * m] * sn + x[2 * m + 1] * cs;
    }
}

/* ---- backward of eq. (2) with the selection held fixed ----
 * O_i = o_i^sr + alpha_h RMSNorm(u_i):
 *   window (eqs. (3)-(4)):  o^sr = sum_j p_j v_j, p = softmax(l), l_j = (R_i q).(R_j k_j)/sqrt(d)
 *   readout (eq. (9)):      u = sum_t pi_t v_t, pi = softmax(lambda), lambda_t = q.k_t/sqrt(d)
 * For an upstream gradient dO, each softmax branch o = sum_j p_j v_j with output gradient
 * g gives dv_j += p_j g, dl_j = p_j (g.v_j - g.o), and dl flows to q and k through the dot
 * products (for the window, through the rotations and back by R^T).  RMSNorm y = u r,
 * r = (mean(u^2) + eps)^(-1/2): du = r (dy - y (dy.y)/d).  dalpha_h = sum_i dO_i.y_i.
 * idx [B,H,Nq,K] are the cells the forward pass selected.  Outputs are overwritten:
 * dQ [B,H,Nq,d], dK, dV [B,H,Nk,d], dalpha [H].  Returns 0. */
int orc_backward(const orc_params *p, const float *Q, const float *K, const float *V, const int *idx,
                 const double *dO, double *dQ, double *dK, double *dV, double *dalpha)
{
    const int d = p->d, s = p->s, Kc = p->K, BH = p->B * p->H;
    const double sc = logit_scale(p);
    memset(dQ, 0, sizeof(double) * (size_t)BH * p->Nq * d);
    memset(dK, 0, sizeof(double) * (size_t)BH * p->Nk * d);
    memset(dV, 0, sizeof(double) * (size_t)BH * p->Nk * d);
    memset(dalpha, 0, sizeof(double) * (size_t)p->H);
    double *krot = (double *)malloc(sizeof(double) * (size_t)p->Nk * d);
    double *lg = (double *)malloc(sizeof(double) * (size_t)(p->Nk > 0 ? p->Nk : 1));
    double qrot[512], dqrot[512], dk[512], tmp[512], o[512], u[512], y[512], du[512];
    for (int bh = 0; bh < BH; bh++) {
        const int h = bh % p->H;
        const double a = p->alpha ? p->alpha[h] : 0.0;
        const float *Kbh = K + (size_t)bh * p->Nk * d, *Vbh = V + (size_t)bh * p->Nk * d;
        double *dKbh = dK + (size_t)bh * p->Nk * d, *dVbh = dV + (size_t)bh * p->Nk * d;
        for (int j = 0; j < p->Nk; j++) rope_rotate(p, Kbh + (size_t)j * d, p->pos0 + j, krot + (size_t)j * d);
        for (int r = 0; r < p->Nq; r++) {
            const long long i = (long long)(p->Nk - p->Nq) + r;
            const float *q = Q + ((size_t)bh * p->Nq + r) * d;
            const double *g = dO + ((size_t)bh * p->Nq + r) * d;
            double *dq = dQ + ((size_t)bh * p->Nq + r) * d;
            /* window branch */
            rope_rotate(p, q, p->pos0 + i, qrot);
            long long j0 = i - p->w < 0 ? 0 : i - p->w;
            double mx = -INFINITY, den = 0.0;
            for (long long j = j0; j <= i; j++) {
                double dot = 0.0;
                for (int m = 0; m < d; m++) dot += qrot[m] * krot[(size_t)j * d + m];
                lg[j - j0] = dot * sc;
                if (lg[j - j0] > mx) mx = lg[j - j0];
            }
            for (int m = 0; m < d; m++) o[m] = 0.0;
            for (long long j = j0; j <= i; j++) {
                lg[j - j0] = exp(lg[j - j0] - mx);
                den += lg[j - j0];
            }
            for (long long j = j0; j <= i; j++) {
                lg[j - j0] /= den;
                for (int m = 0; m < d; m++) o[m] += lg[j - j0] * Vbh[(size_t)j * d + m];
            }
            double D = 0.0;
            for (int m = 0; m < d; m++) D += g[m] * o[m];
            for (int m = 0; m < d; m++) dqrot[m] = 0.0;
            for (long long j = j0; j <= i; j++) {
                const double pj = lg[j - j0];
                double dp = 0.0;
                for (int m = 0; m < d; m++) dp += g[m] * Vbh[(size_t)j * d + m];
                const double ds = pj * (dp - D) * sc;
                for (int m = 0; m < d; m++) {
                    dVbh[(size_t)j * d + m] += pj * g[m];
                    dqrot[m] += ds * krot[(size_t)j * d + m];
                    dk[m] = ds * qrot[m];
                }
                rope_rotate_back(p, dk, p->pos0 + j, tmp);
                for (int m = 0; m < d; m++) dKbh[(size_t)j * d + m] += tmp[m];
            }
            rope_rotate_back(p, dqrot, p->pos0 + i, tmp);
            for (int m = 0; m < d; m++) dq[m] += tmp[m];
            /* readout branch */
            const int *sel = idx + ((size_t)bh * p->Nq + r) * Kc;
            int ncell = 0;
            for (int e = 0; e < Kc; e++) ncell += sel[e] >= 0;
            if (ncell == 0) continue;
            mx = -INFINITY;
            int t = 0;
            for (int e = 0; e < Kc; e++) {
                if (sel[e] < 0) continue;
                for (int j = sel[e] * s; j < (sel[e] + 1) * s; j++, t++) {
                    double dot = 0.0;
                    for (int m = 0; m < d; m++) dot += (double)q[m] * Kbh[(size_t)j * d + m];
                    lg[t] = dot * sc;
                    if (lg[t] > mx) mx = lg[t];
                }
            }
            const int ntok = t;
            den = 0.0;
            for (t = 0; t < ntok; t++) { lg[t] = exp(lg[t] - mx); den += lg[t]; }
            for (int m = 0; m < d; m++) u[m] = 0.0;
            t = 0;
            for (int e = 0; e < Kc; e++) {
                if (sel[e] < 0) continue;
                for (int j = sel[e] * s; j < (sel[e] + 1) * s; j++, t++) {
                    lg[t] /= den;
                    for (int m = 0; m < d; m++) u[m] += lg[t] * Vbh[(size_t)j * d + m];
                }
            }
            double ms = 0.0;
            for (int m = 0; m < d; m++) ms += u[m] * u[m];
            const double rin = 1.0 / sqrt(ms / d + p->rms_eps);
            double dyy = 0.0, gy = 0.0;
            for (int m = 0; m < d; m++) {
                y[m] = u[m] * rin;
                dyy += a * g[m] * y[m];
                gy += g[m] * y[m];
            }
            dalpha[h] += gy;
            for (int m = 0; m < d; m++)
                du[m] = p->mutation == MUT_BWD_NO_RMS ? rin * a * g[m] : rin * (a * g[m] - y[m] * dyy / d);
            D = 0.0;
            for (int m = 0; m < d; m++) D += du[m] * u[m];
            t = 0;
            for (int e = 0; e < Kc; e++) {
                if (sel[e] < 0) continue;
                for (int j = sel[e] * s; j < (sel[e] + 1) * s; j++, t++) {
                    double dp = 0.0;
                    for (int m = 0; m < d; m++) dp += du[m] * Vbh[(size_t)j * d + m];
                    const double ds = lg[t] * (dp - D) * sc;
                    for (int m = 0; m < d; m++) {
                        dVbh[(size_t)j * d + m] += lg[t] * du[m];
                        dq[m] += ds * Kbh[(size_t)j * d + m];
                        dKbh[(size_t)j * d + m] += ds * q[m];
                    }
                }
            }
        }
    }
    free(krot); free(lg);
    return 0;
}

/* ---- backward on samples (full-size checks) ----
 * One row's contribution to the gradients of eq. (2), the same arithmetic as orc_backward:
 * adds the row's dq (if dq) and its contribution to key `key` (dk, dv; key < 0: none).
 * krot holds the head's keys rotated by their positions. */
static void row_grad(const orc_params *p, const float *Kbh, const float *Vbh, const double *krot,
                     const float *q, long long i, const int *sel, const double *g, double a,
                     double *dq, int key, double *dk, double *dv)
{
    const int d = p->d, s = p->s, Kc = p->K;
    const double sc = logit_scale(p);
    double qrot[512], dqrot[512], tmp[512], o[512], u[512], y[512], du[512], kk[512];
    memset(dqrot, 0, sizeof(dqrot));
    /* window branch */
    rope_rotate(p, q, p->pos0 + i, qrot);
    const long long j0 = i - p->w < 0 ? 0 : i - p->w;
    const int n = (int)(i - j0 + 1);
    double *lg = (double *)malloc(sizeof(double) * (size_t)(n > Kc * s ? n : Kc * s + 1));
    double mx = -INFINITY, den = 0.0;
    for (long long j = j0; j <= i; j++) {
        double dot = 0.0;
        for (int m = 0; m < d; m++) dot += qrot[m] * krot[(size_t)j * d + m];
        lg[j - j0] = dot * sc;
        if (lg[j - j0] > mx) mx = lg[j - j0];
    }
    for (int m = 0; m < d; m++) o[m] = 0.0;
    for (long long j = j0; j <= i; j++) { lg[j - j0] = exp(lg[j - j0] - mx); den += lg[j - j0]; }
    for (long long j = j0; j <= i; j++) {
        lg[j - j0] /= den;
        for (int m = 0; m < d; m++) o[m] += lg[j - j0] * Vbh[(size_t)j * d + m];
    }
    double D = 0.0;
    for (int m = 0; m < d; m++) { D += g[m] * o[m]; dqrot[m] = 0.0; }
    for (long long j = j0; j <= i; j++) {
        double dp = 0.0;
        for (int m = 0; m < d; m++) dp += g[m] * Vbh[(size_t)j * d + m];
        const double ds = lg[j - j0] * (dp - D) * sc;
        if (dq) for (int m = 0; m < d; m++) dqrot[m] += ds * krot[(size_t)j * d + m];
        if (j == key) {
            for (int m = 0; m < d; m++) { dv[m] += lg[j - j0] * g[m]; kk[m] = ds * qrot[m]; }
            rope_rotate_back(p, kk, p->pos0 + j, tmp);
            for (int m = 0; m < d; m++) dk[m] += tmp[m];
        }
    }
    if (dq) {
        rope_rotate_back(p, dqrot, p->pos0 + i, tmp);
        for (int m = 0; m < d; m++) dq[m] += tmp[m];
    }
    /* readout branch */
    int ncell = 0;
    for (int e = 0; e < Kc; e++) ncell += sel[e] >= 0;
    if (ncell == 0) { free(lg); return; }
    mx = -INFINITY;
    int t = 0;
    for (int e = 0; e < Kc; e++) {
        if (sel[e] < 0) continue;
        for (int j = sel[e] * s; j < (sel[e] + 1) * s; j++, t++) {
            double dot = 0.0;
            for (int m = 0; m < d; m++) dot += (double)q[m] * Kbh[(size_t)j * d + m];
            lg[t] = dot * sc;
            if (lg[t] > mx) mx = lg[t];
        }
    }
    const int ntok = t;
    den = 0.0;
    for (t = 0; t < ntok; t++) { lg[t] = exp(lg[t] - mx); den += lg[t]; }
    for (int m = 0; m < d; m++) u[m] = 0.0;
    t = 0;
    for (int e = 0; e < Kc; e++) {
        if (sel[e] < 0) continue;
        for (int j = sel[e] * s; j < (sel[e] + 1) * s; j++, t++) {
            lg[t] /= den;
            for (int m = 0; m < d; m++) u[m] += lg[t] * Vbh[(size_t)j * d + m];
        }
    }
    double ms = 0.0;
    for (int m = 0; m < d; m++) ms += u[m] * u[m];
    const double rin = 1.0 / sqrt(ms / d + p->rms_eps);
    double dyy = 0.0;
    for (int m = 0; m < d; m++) { y[m] = u[m] * rin; dyy += a * g[m] * y[m]; }
    for (int m = 0; m < d; m++) du[m] = rin * (a * g[m] - y[m] * dyy / d);
    D = 0.0;
    for (int m = 0; m < d; m++) D += du[m] * u[m];
    t = 0;
    for (int e = 0; e < Kc; e++) {
        if (sel[e] < 0) continue;
        for (int j = sel[e] * s; j < (sel[e] + 1) * s; j++, t++) {
            double dp = 0.0;
            for (int m = 0; m < d; m++) dp += du[m] * Vbh[(size_t)j * d + m];
            const double ds = lg[t] * (dp - D) * sc;
            if (dq) for (int m = 0; m < d; m++) dq[m] += ds * Kbh[(size_t)j * d + m];
            if (j == key) for (int m = 0; m < d; m++) { dv[m] += lg[t] * du[m]; dk[m] += ds * q[m]; }
        }
    }
    free(lg);
}

/* Gradients of eq. (2) on samples of a (possibly full-size) problem: dQ of the given rows
 * (flat (b*H + h)*Nq + r) and dK, dV of the given keys (flat (b*H + h)*Nk + j), with every
 * row's cells idx [B,H,Nq,K] and upstream gradient dO [B,H,Nq,d] given.  A key gathers
 * every row whose window holds it and every row whose cells hold it. */
int orc_backward_sampled(const orc_params *p, const float *Q, const float *K, const float *V, const int *idx,
                         const double *dO, long long nrows, const long long *rows, double *dQ,
                         long long nkeys, const long long *keys, double *dK, double *dV)
{
    const int d = p->d, s = p->s, Kc = p->K, BH = p->B * p->H;
    const long long q0 = (long long)(p->Nk - p->Nq);
    memset(dQ, 0, sizeof(double) * (size_t)(nrows > 0 ? nrows : 0) * d);
    memset(dK, 0, sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 0) * d);
    memset(dV, 0, sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 0) * d);
    for (int bh = 0; bh < BH; bh++) {
        int used = 0;
        for (long long t = 0; t < nrows && !used; t++) used = rows[t] / p->Nq == bh;
        for (long long t = 0; t < nkeys && !used; t++) used = keys[t] / p->Nk == bh;
        if (!used) continue;
        const int h = bh % p->H;
        const double a = p->alpha ? p->alpha[h] : 0.0;
        const float *Kbh = K + (size_t)bh * p->Nk * d, *Vbh = V + (size_t)bh * p->Nk * d;
        double *krot = (double *)malloc(sizeof(double) * (size_t)p->Nk * d);
        #pragma omp parallel for schedule(static)
        for (int j = 0; j < p->Nk; j++) rope_rotate(p, Kbh + (size_t)j * d, p->pos0 + j, krot + (size_t)j * d);
        #pragma omp parallel for schedule(dynamic, 1)
        for (long long t = 0; t < nrows; t++) {
            if (rows[t] / p->Nq != bh) continue;
            const int r = (int)(rows[t] % p->Nq);
            row_grad(p, Kbh, Vbh, krot, Q + ((size_t)bh * p->Nq + r) * d, q0 + r,
                     idx + ((size_t)bh * p->Nq + r) * Kc, dO + ((size_t)bh * p->Nq + r) * d, a,
                     dQ + (size_t)t * d, -1, NULL, NULL);
        }
        #pragma omp parallel for schedule(dynamic, 1)
        for (long long t = 0; t < nkeys; t++) {
            if (keys[t] / p->Nk != bh) continue;
            const int j = (int)(keys[t] % p->Nk);
            const int cj = j / s;
            for (int r = 0; r < p->Nq; r++) {
                const long long i = q0 + r;
                const int *sel = idx + ((size_t)bh * p->Nq + r) * Kc;
                int in = j <= i && j >= i - p->w;
                for (int e = 0; e < Kc && !in; e++) in = sel[e] == cj && cj < orc_num_cells(p);
                if (!in) continue;
                row_grad(p, Kbh, Vbh, krot, Q + ((size_t)bh * p->Nq + r) * d, i, sel,
                         dO + ((size_t)bh * p->Nq + r) * d, a, NULL, j, dK + (size_t)t * d, dV + (size_t)t * d);
            }
        }
        free(krot);
    }
    return 0;
}

/* eq. (7) selection (steps 3-6) for every row, no outputs: idx [B,H,Nq,K]. */
int orc_select_all(const orc_params *p, const float *Q, const double *kbar, const double *amax, int *idx)
{
    const int C = orc_num_cells(p), BH = p->B * p->H;
    #pragma omp parallel for schedule(dynamic, 64)
    for (long long f = 0; f < (long long)BH * p->Nq; f++) {
        const int bh = (int)(f / p->Nq), r = (int)(f % p->Nq);
        const long long i = (long long)(p->Nk - p->Nq) + r;
        select_row(p, Q + (size_t)f * p->d, i, bh % p->H, kbar + (size_t)bh * C * p->d, amax + (size_t)bh * C,
                   idx + (size_t)f * p->K, NULL, NULL);
    }
    return 0;
}

/* ---- single-step entry points for the tests ---- */

/* Selection for one row (b,h,r) given its head's summaries.  Writes idx_out[K];
 * acells/ascores (capacity >= |C_i|) receive A_i and its scores.  Returns |A_i|. */
int orc_select_row(const orc_params *p, const float *Q, const double *kbar, const double *amax,
                   int b, int h, int r, int *idx_out, int *acells, double *ascores)
{
    const int C = orc_num_cells(p);
    size_t bh = (size_t)b * p->H + h;
    long long i = (long long)(p->Nk - p->Nq) + r;
    return select_row(p, Q + (bh * p->Nq + r) * p->d, i, h, kbar + bh * C * p->d,
                      amax + bh * C, idx_out, acells, ascores);
}

/* Readout for one row on caller-given cells idx[K] (ascending, -1 padded). */
void orc_readout_row(const orc_params *p, const float *Q, const float *K, const float *V,
                     int b, int h, int r, const int *idx, double *u_out, double *olr_out)
{
    size_t bh = (size_t)b * p->H + h;
    long long i = (long long)(p->Nk - p->Nq) + r;
    readout_row(p, Q + (bh * p->Nq + r) * p->d, i, K + bh * p->Nk * p->d,
                V + bh * p->Nk * p->d, idx, u_out, olr_out);
}

/* Readout for many rows, each on its own caller-given cells (rows as in orc_forward). */
void orc_readout_rows(const orc_params *p, const float *Q, const float *K, const float *V,
                      long long nrows, const long long *rows, const int *idx,
                      double *u_out, double *olr_out)
{
    #pragma omp parallel for schedule(dynamic, 8)
    for (long long t = 0; t < nrows; t++) {
        long long f = rows[t];
        int r = (int)(f % p->Nq);
        long long bh = f / p->Nq;
        orc_readout_row(p, Q, K, V, (int)(bh / p->H), (int)(bh % p->H), r,
                        idx + (size_t)t * p->K, u_out ? u_out + (size_t)t * p->d : NULL,
                        olr_out + (size_t)t * p->d);
    }
}

/* RoPE rotation of one vector at an absolute position (exposed for the eq. (3) check). */
void orc_rope(const orc_params *p, const float *x, long long pos, double *out)
{
    rope_rotate(p, x, pos, out);
}

/* ==== FS-B: balanced-tree search over two causal forests (§3.4 eqs. (10)-(11)) ====
 * The summary prints the admitted sets (10) and the node score (11) only; the rest is
 * read as follows (the "growing archive" with radix-sort-built balanced trees, §3.4, §5):
 *  - a forest is built over a sequence of cells: forest 0 over all cells in time order
 *    (A^0_i = C_i), forest tau over the cells with a_c >= tau_h in time order (A^tau_i);
 *  - for every k and every aligned block of 2^k consecutive sequence entries there is one
 *    balanced binary tree over the block's cells; a prefix of n entries is covered by the
 *    trees of the set bits of n (those a binary counter holds after n insertions), so a
 *    query only reaches cells of its prefix (causal);
 *  - a tree's leaves are its cells radix-sorted by a 16-bit code, the signs of the first
 *    16 coordinates of kbar_c (coordinate 0 most significant), ties by time; node v of the
 *    complete binary tree over that order holds a run of consecutive leaves;
 *  - mu_v = mean of kbar_c, rho_v = max ||kbar_c - mu_v||, A_v = max a_c, p_v^min =
 *    min p_c over the leaves of v; c of eq. (11) is a parameter; g_h is eq. (7)'s;
 *  - beam search of width beta on each forest: the beam starts as the prefix's roots (the
 *    beta best); then every internal node of the beam is replaced by its two children and
 *    the beta best kept (by U_v, ties to the lower p_v^min), until only leaves remain;
 *  - S_i = the K best cells by eq. (7) among the leaves both beams end on (a leaf's U_v
 *    is its eq. (7) score), ascending, -1 padded.
 * With c >= 1 and lambda_h >= 0, U_v bounds the eq. (7) score of every leaf below v
 * (Cauchy-Schwarz for the dot product; erf increasing for the prior). */

typedef struct {
    int n, L;          /* sequence length; levels k = 0 .. L-1 (2^k <= n) */
    int *seq;          /* [n] cell of each sequence entry */
    int **ord;         /* ord[k][(blk << k) + j]: leaf j (code order) of block blk */
    double **mu;       /* mu[k][((blk << (k+1)) + v) * d], heap index v in [1, 2^(k+1)) */
    double **rho, **A;
    int **pmin;
} orc_forest;

static unsigned cell_code(const orc_params *p, const double *kb)
{
    int nb = p->d < 16 ? p->d : 16;
    unsigned code = 0;
    for (int b = 0; b < nb; b++) code = (code << 1) | (kb[b] > 0.0 ? 1u : 0u);
    return code;
}

/* stable LSD radix sort of cells by their code, two 8-bit digits */
static void radix_sort_cells(int *cells, int n, const unsigned *code, int *tmp)
{
    for (int shift = 0; shift < 16; shift += 8) {
        int cnt[257];
        memset(cnt, 0, sizeof(cnt));
        for (int t = 0; t < n; t++) cnt[((code[cells[t]] >> shift) & 255u) + 1]++;
        for (int b = 0; b < 256; b++) cnt[b + 1] += cnt[b];
        for (int t = 0; t < n; t++) tmp[cnt[(code[cells[t]] >> shift) & 255u]++] = cells[t];
        memcpy(cells, tmp, sizeof(int) * (size_t)n);
    }
}

static void forest_build(const orc_params *p, const double *kbar_bh, const double *amax_bh,
                         const double *tau_h, orc_forest *F)
{
    const int C = orc_num_cells(p), d = p->d;
    memset(F, 0, sizeof(*F));
    F->seq = (int *)malloc(sizeof(int) * (size_t)(C > 0 ? C : 1));
    for (int c = 0; c < C; c++)
        if (!tau_h || amax_bh[c] >= *tau_h) F->seq[F->n++] = c;
    while (F->L < 31 && (1 << F->L) <= F->n) F->L++;
    unsigned *code = (unsigned *)malloc(sizeof(unsigned) * (size_t)(C > 0 ? C : 1));
    for (int c = 0; c < C; c++) code[c] = cell_code(p, kbar_bh + (size_t)c * d);
    int *tmp = (int *)malloc(sizeof(int) * (size_t)(F->n > 0 ? F->n : 1));
    F->ord = (int **)calloc((size_t)(F->L + 1), sizeof(int *));
    F->mu = (double **)calloc((size_t)(F->L + 1), sizeof(double *));
    F->rho = (double **)calloc((size_t)(F->L + 1), sizeof(double *));
    F->A = (double **)calloc((size_t)(F->L + 1), sizeof(double *));
    F->pmin = (int **)calloc((size_t)(F->L + 1), sizeof(int *));
    for (int k = 0; k < F->L; k++) {
        const int nblk = F->n >> k, nleaf = 1 << k, nnode = 2 << k;
        F->ord[k] = (int *)malloc(sizeof(int) * (size_t)nblk * nleaf);
        F->mu[k] = (double *)calloc((size_t)nblk * nnode * d, sizeof(double));
        F->rho[k] = (double *)calloc((size_t)nblk * nnode, sizeof(double));
        F->A[k] = (double *)calloc((size_t)nblk * nnode, sizeof(double));
        F->pmin[k] = (int *)calloc((size_t)nblk * nnode, sizeof(int));
        for (int blk = 0; blk < nblk; blk++) {
            int *o = F->ord[k] + (size_t)blk * nleaf;
            memcpy(o, F->seq + (size_t)blk * nleaf, sizeof(int) * (size_t)nleaf);
            radix_sort_cells(o, nleaf, code, tmp);
            if (p->mutation == MUT_TREE_SORT_DESC)
                for (int a = 0, b = nleaf - 1; a < b; a++, b--) { int x = o[a]; o[a] = o[b]; o[b] = x; }
            for (int v = 1; v < nnode; v++) {
                int t = 0;
                while ((2 << t) <= v) t++;                  /* depth of v */
                const int first = (v - (1 << t)) << (k - t), cnt = 1 << (k - t);
                const size_t nv = (size_t)blk * nnode + v;
                double *mu = F->mu[k] + nv * d;
                double Av = -INFINITY;
                int pm = o[first];
                for (int j = first; j < first + cnt; j++) {
                    const double *kb = kbar_bh + (size_t)o[j] * d;
                    for (int m = 0; m < d; m++) mu[m] += kb[m];
                    if (amax_bh[o[j]] > Av) Av = amax_bh[o[j]];
                    if (p->mutation == MUT_TREE_PMAX ? o[j] > pm : o[j] < pm) pm = o[j];
                }
                for (int m = 0; m < d; m++) mu[m] /= cnt;
                double rho = 0.0;
                for (int j = first; j < first + cnt; j++) {
                    const double *kb = kbar_bh + (size_t)o[j] * d;
                    double sq = 0.0;
                    for (int m = 0; m < d; m++) sq += (kb[m] - mu[m]) * (kb[m] - mu[m]);
                    if (sqrt(sq) > rho) rho = sqrt(sq);
                }
                F->rho[k][nv] = rho;
                F->A[k][nv] = Av;
                F->pmin[k][nv] = pm;
            }
        }
    }
    free(code);
    free(tmp);
}

static void forest_free(orc_forest *F)
{
    for (int k = 0; k < F->L; k++) {
        free(F->ord[k]); free(F->mu[k]); free(F->rho[k]); free(F->A[k]); free(F->pmin[k]);
    }
    free(F->ord); free(F->mu); free(F->rho); free(F->A); free(F->pmin); free(F->seq);
    memset(F, 0, sizeof(*F));
}

/* eq. (11) for node (k, blk, v) and the query q at position i of head h */
static double node_U(const orc_params *p, const orc_forest *F, int k, int blk, int v,
                     const float *qrow, long long i, int h, double c_explore)
{
    const int d = p->d;
    const size_t nv = (size_t)blk * (2 << k) + v;
    const double *mu = F->mu[k] + nv * d;
    double dot = 0.0, qq = 0.0;
    for (int m = 0; m < d; m++) {
        dot += (double)qrow[m] * mu[m];
        qq += (double)qrow[m] * qrow[m];
    }
    const double rho_term = p->mutation == MUT_TREE_NO_RHO ? 0.0 : c_explore * sqrt(qq) * F->rho[k][nv];
    double U = (dot + rho_term) * logit_scale(p);
    const double lam = p->lambda ? p->lambda[h] : 0.0;
    if (lam != 0.0) {
        const double pv = (double)p->pos0 + (F->pmin[k][nv] + 0.5) * p->s;
        U += lam * F->A[k][nv] * erf(((double)(p->pos0 + i) - pv) / (2.0 * p->sigma[h]));
    }
    return U;
}

/* eq. (7) for one cell */
static double eq7_score(const orc_params *p, const float *qrow, long long i, int h,
                        const double *kbar_bh, const double *amax_bh, int c)
{
    const double *kb = kbar_bh + (size_t)c * p->d;
    double dot = 0.0;
    for (int m = 0; m < p->d; m++) dot += (double)qrow[m] * kb[m];
    double r = dot * logit_scale(p);
    const double lam = p->lambda ? p->lambda[h] : 0.0;
    if (lam != 0.0) {
        const double pc = (double)p->pos0 + (c + 0.5) * p->s;
        r += lam * amax_bh[c] * erf(((double)(p->pos0 + i) - pc) / (2.0 * p->sigma[h]));
    }
    return r;
}

typedef struct { double U; int k, blk, v, pmin; } beam_node;

static int beam_before(const beam_node *a, const beam_node *b)
{
    if (a->U != b->U) return a->U > b->U;
    return a->pmin < b->pmin;
}

/* keep the beta best of x[0..n) (sorted, best first); returns the new count and lowers
 * *margin to the cut's relative gap when something is cut */
static int beam_cut(beam_node *x, int n, int beta, double *margin)
{
    for (int a = 1; a < n; a++) {                      /* insertion sort, best first */
        beam_node t = x[a];
        int b = a - 1;
        while (b >= 0 && beam_before(&t, &x[b])) { x[b + 1] = x[b]; b--; }
        x[b + 1] = t;
    }
    if (n <= beta) return n;
    const double gap = (x[beta - 1].U - x[beta].U) / fmax(1.0, fabs(x[beta - 1].U));
    if (gap < *margin) *margin = gap;
    return beta;
}

/* beam search on one forest for the prefix of m sequence entries: the leaf cells it ends on */
static int forest_search(const orc_params *p, const orc_forest *F, int m, const float *qrow,
                         long long i, int h, int beta, double c_explore, int *cells, double *margin)
{
    beam_node *cur = (beam_node *)malloc(sizeof(beam_node) * (size_t)(2 * beta + 64));
    int n = 0;
    for (int k = F->L - 1; k >= 0; k--) {              /* roots: the set bits of m */
        if (!((m >> k) & 1)) continue;
        beam_node r;
        r.k = k; r.blk = (m >> k) - 1; r.v = 1;
        r.U = node_U(p, F, k, r.blk, 1, qrow, i, h, c_explore);
        r.pmin = F->pmin[k][(size_t)r.blk * (2 << k) + 1];
        cur[n++] = r;
    }
    n = beam_cut(cur, n, beta, margin);
    for (;;) {
        beam_node *next = (beam_node *)malloc(sizeof(beam_node) * (size_t)(2 * beta + 64));
        int nn = 0, expanded = 0;
        for (int t = 0; t < n; t++) {
            const beam_node e = cur[t];
            if (e.v >= (1 << e.k)) { next[nn++] = e; continue; }      /* a leaf */
            expanded = 1;
            for (int ch = 0; ch < 2; ch++) {
                beam_node c = e;
                c.v = 2 * e.v + ch;
                c.U = node_U(p, F, e.k, e.blk, c.v, qrow, i, h, c_explore);
                c.pmin = F->pmin[e.k][(size_t)e.blk * (2 << e.k) + c.v];
                next[nn++] = c;
            }
        }
        free(cur);
        cur = next;
        n = nn;
        if (!expanded) break;
        n = beam_cut(cur, n, beta, margin);
    }
    for (int t = 0; t < n; t++) {
        const beam_node e = cur[t];
        cells[t] = F->ord[e.k][((size_t)e.blk << e.k) + (e.v - (1 << e.k))];
    }
    free(cur);
    return n;
}

/* FS-B selection for a list of rows (flat (b*H + h)*Nq + r; NULL = all rows in order).
 * tau: [H] thresholds of forest tau, or NULL for forest 0 alone.  idx_out [nrows, K];
 * margin_out (or NULL): per row, the smallest relative gap at any beam cut (1 if none).
 * Returns 0, or -1 for bad arguments. */
int orc_tree_select_rows(const orc_params *p, const float *Q, const double *kbar, const double *amax,
                         const double *tau, int beta, double c_explore, long long nrows,
                         const long long *rows, int *idx_out, double *margin_out)
{
    const int C = orc_num_cells(p), BH = p->B * p->H, Kc = p->K;
    if (beta < 1 || (p->lambda && !p->sigma)) return -1;
    if (!rows) nrows = (long long)BH * p->Nq;
    for (int bh = 0; bh < BH; bh++) {
        int any = 0;
        for (long long t = 0; t < nrows && !any; t++) any = (rows ? rows[t] : t) / p->Nq == bh;
        if (!any) continue;
        const int h = bh % p->H;
        const double *kb = kbar + (size_t)bh * C * p->d, *am = amax + (size_t)bh * C;
        orc_forest F0, Ft;
        forest_build(p, kb, am, NULL, &F0);
        if (tau) forest_build(p, kb, am, tau + h, &Ft);
        #pragma omp parallel for schedule(dynamic, 16)
        for (long long t = 0; t < nrows; t++) {
            const long long f = rows ? rows[t] : t;
            if (f / p->Nq != bh) continue;
            const int r = (int)(f % p->Nq);
            const long long i = (long long)(p->Nk - p->Nq) + r;
            const float *q = Q + (size_t)f * p->d;
            const int n = orc_candidate_count(p, i);
            double margin = 1.0;
            int *cells = (int *)malloc(sizeof(int) * (size_t)(4 * beta + 128));
            int nc = forest_search(p, &F0, n, q, i, h, beta, c_explore, cells, &margin);
            if (tau) {
                int m = 0;
                while (m < Ft.n && Ft.seq[m] < n) m++;          /* admitted cells of C_i */
                nc += forest_search(p, &Ft, m, q, i, h, beta, c_explore, cells + nc, &margin);
            }
            vi_pair *x = (vi_pair *)malloc(sizeof(vi_pair) * (size_t)(nc > 0 ? nc : 1));
            vi_pair *tmp = (vi_pair *)malloc(sizeof(vi_pair) * (size_t)(nc > 0 ? nc : 1));
            int nx = 0;
            for (int a = 0; a < nc; a++) {                      /* the union (a cell once) */
                int dup = 0;
                for (int b = 0; b < a && !dup; b++) dup = cells[b] == cells[a];
                if (dup) continue;
                x[nx].v = eq7_score(p, q, i, h, kb, am, cells[a]);
                x[nx].idx = cells[a];
                nx++;
            }
            sort_desc(x, nx, tmp, 0);
            int *out = idx_out + (size_t)t * Kc;
            const int keep = nx < Kc ? nx : Kc;
            for (int a = 0; a < keep; a++) out[a] = x[a].idx;
            qsort(out, (size_t)keep, sizeof(int), cmp_int);
            for (int a = keep; a < Kc; a++) out[a] = -1;
            if (margin_out) margin_out[t] = margin;
            free(cells); free(x); free(tmp);
        }
        forest_free(&F0);
        if (tau) forest_free(&Ft);
    }
    return 0;
}

/* One node of one (b,h) forest (0: all cells; 1: cells with a_c >= tau[h]): its leaves in
 * code order into `leaves` (capacity >= 2^k) and eq. (11) for query row r into *U.
 * *nseq receives the forest's sequence length.  Returns the leaf count, or -1 if the node
 * does not exist. */
int orc_tree_node(const orc_params *p, const float *Q, const double *kbar, const double *amax,
                  const double *tau, int b, int h, int forest, int k, int blk, int v, int r,
                  double c_explore, int *leaves, double *U, int *nseq)
{
    const int C = orc_num_cells(p);
    const size_t bh = (size_t)b * p->H + h;
    orc_forest F;
    forest_build(p, kbar + bh * C * p->d, amax + bh * C, forest ? tau + h : NULL, &F);
    *nseq = F.n;
    int cnt = -1;
    if (k >= 0 && k < F.L && blk >= 0 && blk < (F.n >> k) && v >= 1 && v < (2 << k)) {
        int t = 0;
        while ((2 << t) <= v) t++;
        const int first = (v - (1 << t)) << (k - t);
        cnt = 1 << (k - t);
        for (int j = 0; j < cnt; j++) leaves[j] = F.ord[k][((size_t)blk << k) + first + j];
        const long long i = (long long)(p->Nk - p->Nq) + r;
        *U = node_U(p, &F, k, blk, v, Q + (bh * p->Nq + r) * p->d, i, h, c_explore);
    }
    forest_free(&F);
    return cnt;
}
