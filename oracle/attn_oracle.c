/*
 * attn_oracle.c -- plain fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA library is compared
 * against.  Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * load it; the product path (the CUDA library and its Python binding) never does, and
 * the two share no code, headers, tables or helpers.
 *
 * What it computes is the plain definition of attention, written out row by row in
 * double precision, with no tiling, no online softmax and no reordering:
 *
 *   Step 1  S = scale * Q K^T, with S_ij = -inf where the causal mask hides key j > i.
 *   Step 2  P = softmax(S) per row: m_i = max_j S_ij, l_i = sum_j exp(S_ij - m_i),
 *           P_ij = exp(S_ij - m_i) / l_i; the saved statistic is LSE_i = m_i + ln l_i.
 *   Step 3  O = P V.
 *
 * Sources: "FlashAttention 与高效注意力内核：IO 感知与分块计算" (plumephp.com tutorial),
 * section "标准注意力三步" (S = Q K^T, P = softmax(S), O = P V) and section "前向" (only O
 * and the softmax statistics m, l are kept); "Flash-Attention" concept page
 * (awesome-system-papers), section "核心思想" (the 1/sqrt(d) scale inside the softmax).
 *
 * Backward: the standard analytic chain rule through the softmax, with the gradient of
 * the scaled scores S = scale * Q K^T:
 *   D_i   = sum_c dO_ic O_ic
 *   dP_ij = dO_i . V_j
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij K_j
 *   dK_j  = scale * sum_i dS_ij Q_i      (summed over the query heads that share K_j)
 *   dV_j  = sum_i P_ij dO_i              (summed likewise)
 * The tutorial's section "反向" says only that the backward recomputes S and P from
 * Q/K/V and the saved statistics and then forms dQ/dK/dV from dO; the formulas above are
 * the plain derivative of the forward definition.  Here P_ij is re-formed from the saved
 * LSE as exp(S_ij - LSE_i), which equals exp(S_ij - m_i) / l_i by definition.
 *
 * Grouped-query attention ("相关工作" page, paper 6 "Grouped-Query Attention"): query
 * head h reads key/value head floor(h * hkv / hq), i.e. contiguous groups of hq/hkv
 * query heads share one K/V head.  Variable-length packing ("验证清单": 变长序列打包):
 * sequences are concatenated along the token axis, described by cu_seqlens (prefix sums,
 * cu_seqlens[0] = 0), and attention never crosses a sequence boundary.
 *
 * Layouts (all row-major, double):  q, o, dout, dq : [T, hq, d]
 *                                   k, v, dk, dv   : [T, hkv, d]
 *                                   lse            : [hq, T]
 * A query row with no visible key (impossible for causal self-attention with length >= 1)
 * gets O = 0 and LSE = -inf.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEM 2

typedef struct {
    const double *q, *k, *v, *dout;
    const int32_t *cu;
    int32_t nseq, hq, hkv, d, causal;
    double scale;
    const uint8_t *row_sel;  /* optional: only rows with row_sel[t] != 0 are produced */
    const uint8_t *key_sel;  /* optional: only keys with key_sel[t] != 0 get dK/dV */
    double *o, *lse, *dd;    /* forward results (and D for the backward) */
    double *dq, *dk, *dv;
} problem;

/* ---- the three steps, for one query row -------------------------------------------- */

/* Number of keys row i (0-based inside its sequence of length n) may look at. */
static int visible_keys(int i, int n, int causal) { return causal ? i + 1 : n; }

/* Step 1: s_j = scale * <q_i, k_j> for visible keys, -inf for hidden ones. */
static void score_row(const problem *P, int64_t row, int64_t key0, int n, int vis, int h, double *s)
{
    const int d = P->d;
    const int g = (int)(((int64_t)h * P->hkv) / P->hq);
    const double *qi = P->q + (row * P->hq + h) * d;
    for (int j = 0; j < n; ++j) {
        if (j >= vis) { s[j] = -INFINITY; continue; }
        const double *kj = P->k + ((key0 + j) * P->hkv + g) * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
        s[j] = P->scale * acc;
    }
}

/* Step 2: p_j = exp(s_j - m) / l with m = max s, l = sum exp(s_j - m); returns LSE = m + ln l. */
static double softmax_row(const double *s, int n, double *p)
{
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) if (s[j] > m) m = s[j];
    if (m == -INFINITY) { for (int j = 0; j < n; ++j) p[j] = 0.0; return -INFINITY; }
    double l = 0.0;
    for (int j = 0; j < n; ++j) { p[j] = exp(s[j] - m); l += p[j]; }
    for (int j = 0; j < n; ++j) p[j] /= l;
    return m + log(l);
}

/* Step 3: o_i = sum_j p_j v_j. */
static void output_row(const problem *P, int64_t key0, int n, int h, const double *p, double *oi)
{
    const int d = P->d;
    const int g = (int)(((int64_t)h * P->hkv) / P->hq);
    for (int c = 0; c < d; ++c) oi[c] = 0.0;
    for (int j = 0; j < n; ++j) {
        if (p[j] == 0.0) continue;
        const double *vj = P->v + ((key0 + j) * P->hkv + g) * d;
        for (int c = 0; c < d; ++c) oi[c] += p[j] * vj[c];
    }
}

/* ---- work items and threads -------------------------------------------------------- */

#define ROWS_PER_ITEM 32

typedef struct {
    problem *P;
    int kind;            /* 0: forward rows, 1: dQ rows, 2: dK/dV keys */
    int64_t nitems;
    int64_t *item_seq;   /* item -> sequence */
    int64_t *item_head;  /* item -> head (query head for kinds 0/1, kv head for kind 2) */
    int64_t *item_row0;  /* item -> first row (inside the sequence) */
    int64_t next;
    pthread_mutex_t lock;
    int failed;
} workset;

static void do_forward_rows(problem *P, int64_t seq, int h, int r0, int r1, double *s, double *p)
{
    const int64_t t0 = P->cu[seq];
    const int n = (int)(P->cu[seq + 1] - t0);
    for (int i = r0; i < r1; ++i) {
        const int64_t row = t0 + i;
        if (P->row_sel && !P->row_sel[row]) continue;
        const int vis = visible_keys(i, n, P->causal);
        score_row(P, row, t0, n, vis, h, s);
        const double lse = softmax_row(s, n, p);
        double *oi = P->o + (row * P->hq + h) * P->d;
        output_row(P, t0, n, h, p, oi);
        P->lse[(int64_t)h * P->cu[P->nseq] + row] = lse;
        if (P->dd) {  /* D_i = sum_c dO_ic O_ic, needed by the backward */
            const double *doi = P->dout + (row * P->hq + h) * P->d;
            double acc = 0.0;
            for (int c = 0; c < P->d; ++c) acc += doi[c] * oi[c];
            P->dd[(int64_t)h * P->cu[P->nseq] + row] = acc;
        }
    }
}

/* dS_ij for keys j in [j0, j1) of one row (all visible), given the saved LSE_i and D_i:
 * P_ij = exp(S_ij - LSE_i), dS_ij = P_ij (dP_ij - D_i).  p[j] and ds[j] are written for
 * j in [j0, j1) only. */
static void ds_row(const problem *P, int64_t row, int64_t key0, int j0, int j1, int h,
                   double *ds, double *p)
{
    const int d = P->d;
    const int g = (int)(((int64_t)h * P->hkv) / P->hq);
    const int64_t T = P->cu[P->nseq];
    const double lse = P->lse[(int64_t)h * T + row];
    const double Di = P->dd[(int64_t)h * T + row];
    const double *qi = P->q + (row * P->hq + h) * d;
    const double *doi = P->dout + (row * P->hq + h) * d;
    for (int j = j0; j < j1; ++j) {
        const double *kj = P->k + ((key0 + j) * P->hkv + g) * d;
        const double *vj = P->v + ((key0 + j) * P->hkv + g) * d;
        double sc = 0.0, dp = 0.0;
        for (int c = 0; c < d; ++c) { sc += qi[c] * kj[c]; dp += doi[c] * vj[c]; }
        p[j] = exp(P->scale * sc - lse);
        ds[j] = p[j] * (dp - Di);
    }
}

static void do_dq_rows(problem *P, int64_t seq, int h, int r0, int r1, double *s, double *p)
{
    const int64_t t0 = P->cu[seq];
    const int n = (int)(P->cu[seq + 1] - t0);
    const int d = P->d;
    const int g = (int)(((int64_t)h * P->hkv) / P->hq);
    for (int i = r0; i < r1; ++i) {
        const int64_t row = t0 + i;
        if (P->row_sel && !P->row_sel[row]) continue;
        const int vis = visible_keys(i, n, P->causal);
        ds_row(P, row, t0, 0, vis, h, s, p);
        double *dqi = P->dq + (row * P->hq + h) * d;
        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
        for (int j = 0; j < vis; ++j) {
            const double *kj = P->k + ((t0 + j) * P->hkv + g) * d;
            for (int c = 0; c < d; ++c) dqi[c] += s[j] * kj[c];
        }
        for (int c = 0; c < d; ++c) dqi[c] *= P->scale;
    }
}

/* dK_j, dV_j for keys j in [r0, r1) of one kv head: sum over the query heads of its
 * group and over every query row that sees key j. */
static void do_dkdv_keys(problem *P, int64_t seq, int g, int r0, int r1, double *s, double *p)
{
    const int64_t t0 = P->cu[seq];
    const int n = (int)(P->cu[seq + 1] - t0);
    const int d = P->d;
    const int G = P->hq / P->hkv;
    double *acck = (double *)calloc((size_t)(r1 - r0) * d, sizeof(double));
    double *accv = (double *)calloc((size_t)(r1 - r0) * d, sizeof(double));
    if (!acck || !accv) { free(acck); free(accv); return; }
    int any = 0;
    for (int j = r0; j < r1; ++j) if (!P->key_sel || P->key_sel[t0 + j]) any = 1;
    if (any) {
        for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            for (int i = 0; i < n; ++i) {
                const int vis = visible_keys(i, n, P->causal);
                if (vis <= r0) continue;  /* row i sees none of these keys */
                const int64_t row = t0 + i;
                const int j1 = r1 < vis ? r1 : vis;
                ds_row(P, row, t0, r0, j1, h, s, p);
                const double *qi = P->q + (row * P->hq + h) * d;
                const double *doi = P->dout + (row * P->hq + h) * d;
                for (int j = r0; j < j1; ++j) {
                    double *ak = acck + (size_t)(j - r0) * d;
                    double *av = accv + (size_t)(j - r0) * d;
                    for (int c = 0; c < d; ++c) { ak[c] += s[j] * qi[c]; av[c] += p[j] * doi[c]; }
                }
            }
        }
    }
    for (int j = r0; j < r1; ++j) {
        const int64_t key = t0 + j;
        if (P->key_sel && !P->key_sel[key]) continue;
        double *dkj = P->dk + (key * P->hkv + g) * d;
        double *dvj = P->dv + (key * P->hkv + g) * d;
        for (int c = 0; c < d; ++c) {
            dkj[c] = P->scale * acck[(size_t)(j - r0) * d + c];
            dvj[c] = accv[(size_t)(j - r0) * d + c];
        }
    }
    free(acck);
    free(accv);
}

static void *worker(void *arg)
{
    workset *W = (workset *)arg;
    problem *P = W->P;
    int64_t maxn = 0;
    for (int b = 0; b < P->nseq; ++b) {
        const int64_t n = P->cu[b + 1] - P->cu[b];
        if (n > maxn) maxn = n;
    }
    double *s = (double *)malloc((size_t)(maxn > 0 ? maxn : 1) * sizeof(double));
    double *p = (double *)malloc((size_t)(maxn > 0 ? maxn : 1) * sizeof(double));
    if (!s || !p) {
        pthread_mutex_lock(&W->lock); W->failed = 1; pthread_mutex_unlock(&W->lock);
        free(s); free(p);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&W->lock);
        const int64_t it = W->next++;
        pthread_mutex_unlock(&W->lock);
        if (it >= W->nitems) break;
        const int64_t seq = W->item_seq[it];
        const int h = (int)W->item_head[it];
        const int r0 = (int)W->item_row0[it];
        const int n = (int)(P->cu[seq + 1] - P->cu[seq]);
        const int r1 = r0 + ROWS_PER_ITEM < n ? r0 + ROWS_PER_ITEM : n;
        if (W->kind == 0) do_forward_rows(P, seq, h, r0, r1, s, p);
        else if (W->kind == 1) do_dq_rows(P, seq, h, r0, r1, s, p);
        else do_dkdv_keys(P, seq, h, r0, r1, s, p);
    }
    free(s);
    free(p);
    return NULL;
}

static int run_items(problem *P, int kind, int nheads, int nthreads)
{
    int64_t nitems = 0;
    for (int b = 0; b < P->nseq; ++b) {
        const int64_t n = P->cu[b + 1] - P->cu[b];
        nitems += (int64_t)nheads * ((n + ROWS_PER_ITEM - 1) / ROWS_PER_ITEM);
    }
    workset W;
    memset(&W, 0, sizeof W);
    W.P = P;
    W.kind = kind;
    W.nitems = nitems;
    W.item_seq = (int64_t *)malloc((size_t)(nitems > 0 ? nitems : 1) * sizeof(int64_t));
    W.item_head = (int64_t *)malloc((size_t)(nitems > 0 ? nitems : 1) * sizeof(int64_t));
    W.item_row0 = (int64_t *)malloc((size_t)(nitems > 0 ? nitems : 1) * sizeof(int64_t));
    if (!W.item_seq || !W.item_head || !W.item_row0) {
        free(W.item_seq); free(W.item_head); free(W.item_row0);
        return ORACLE_NO_MEM;
    }
    int64_t it = 0;
    for (int b = 0; b < P->nseq; ++b) {
        const int64_t n = P->cu[b + 1] - P->cu[b];
        for (int h = 0; h < nheads; ++h)
            for (int64_t r = 0; r < n; r += ROWS_PER_ITEM) {
                W.item_seq[it] = b; W.item_head[it] = h; W.item_row0[it] = r; ++it;
            }
    }
    pthread_mutex_init(&W.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    pthread_t *tid = (pthread_t *)malloc((size_t)nthreads * sizeof(pthread_t));
    int started = 0;
    if (tid) {
        for (; started < nthreads; ++started)
            if (pthread_create(&tid[started], NULL, worker, &W) != 0) break;
    }
    if (started == 0) worker(&W);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    pthread_mutex_destroy(&W.lock);
    free(W.item_seq); free(W.item_head); free(W.item_row0);
    return W.failed ? ORACLE_NO_MEM : ORACLE_OK;
}

static int check_args(const int32_t *cu, int32_t nseq, int32_t hq, int32_t hkv, int32_t d)
{
    if (!cu || nseq < 0 || hq <= 0 || hkv <= 0 || d <= 0 || hq % hkv != 0) return ORACLE_BAD_ARG;
    if (cu[0] != 0) return ORACLE_BAD_ARG;
    for (int b = 0; b < nseq; ++b) if (cu[b + 1] < cu[b]) return ORACLE_BAD_ARG;
    return ORACLE_OK;
}

/* ---- decoding forward: fewer query rows than keys ----------------------------------
 * "FlashAttention 与高效注意力内核" tutorial, section "FlashAttention 变体族谱": the decode
 * variant (FlashDecoding) serves "one query against a long KV".  What it computes is the
 * same three steps as above; only the shapes differ.  Sequence b has
 * Lq = cu_q[b+1] - cu_q[b] query rows and Lk = cu_k[b+1] - cu_k[b] keys, and the query
 * rows are the LAST Lq positions of the sequence (the tokens being decoded), so under the
 * causal mask query row i (0-based inside its sequence) sees keys j <= Lk - Lq + i, none
 * when that is negative.  With Lq = Lk this is the self-attention mask above.
 * Layouts: q, o [Tq, hq, d]; k, v [Tk, hkv, d]; lse [hq, Tq] with Tq = cu_q[nseq]. */
typedef struct {
    problem P;                  /* q, k, v, hq, hkv, d, scale, causal, o, lse */
    const int32_t *cu_q, *cu_k;
    int32_t nseq;
    int64_t tq;
    int64_t next, nitems;       /* items: (sequence, query head) */
    pthread_mutex_t lock;
    int failed;
} cross_work;

static int cross_visible(int i, int lq, int lk, int causal)
{
    if (!causal) return lk;
    const int v = lk - lq + i + 1;
    return v < 0 ? 0 : (v > lk ? lk : v);
}

static void *cross_worker(void *arg)
{
    cross_work *W = (cross_work *)arg;
    problem *P = &W->P;
    int64_t maxk = 1;
    for (int b = 0; b < W->nseq; ++b) {
        const int64_t n = W->cu_k[b + 1] - W->cu_k[b];
        if (n > maxk) maxk = n;
    }
    double *s = (double *)malloc((size_t)maxk * sizeof(double));
    double *p = (double *)malloc((size_t)maxk * sizeof(double));
    if (!s || !p) {
        pthread_mutex_lock(&W->lock); W->failed = 1; pthread_mutex_unlock(&W->lock);
        free(s); free(p);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&W->lock);
        const int64_t it = W->next++;
        pthread_mutex_unlock(&W->lock);
        if (it >= W->nitems) break;
        const int b = (int)(it / P->hq);
        const int h = (int)(it % P->hq);
        const int64_t q0 = W->cu_q[b], k0 = W->cu_k[b];
        const int lq = (int)(W->cu_q[b + 1] - q0), lk = (int)(W->cu_k[b + 1] - k0);
        for (int i = 0; i < lq; ++i) {
            const int64_t row = q0 + i;
            const int vis = cross_visible(i, lq, lk, P->causal);
            score_row(P, row, k0, lk, vis, h, s);
            const double lse = softmax_row(s, lk, p);
            output_row(P, k0, lk, h, p, P->o + (row * P->hq + h) * P->d);
            P->lse[(int64_t)h * W->tq + row] = lse;
        }
    }
    free(s);
    free(p);
    return NULL;
}

int oracle_attn_fwd_cross(const double *q, const double *k, const double *v,
                          const int32_t *cu_q, const int32_t *cu_k, int32_t nseq,
                          int32_t hq, int32_t hkv, int32_t d, double scale, int32_t causal,
                          double *o, double *lse, int32_t nthreads)
{
    int rc = check_args(cu_q, nseq, hq, hkv, d);
    if (rc) return rc;
    rc = check_args(cu_k, nseq, hq, hkv, d);
    if (rc) return rc;
    cross_work W;
    memset(&W, 0, sizeof W);
    W.P.q = q; W.P.k = k; W.P.v = v; W.P.hq = hq; W.P.hkv = hkv; W.P.d = d;
    W.P.scale = scale; W.P.causal = causal; W.P.o = o; W.P.lse = lse;
    W.cu_q = cu_q; W.cu_k = cu_k; W.nseq = nseq; W.tq = cu_q[nseq];
    W.nitems = (int64_t)nseq * hq;
    pthread_mutex_init(&W.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    pthread_t *tid = (pthread_t *)malloc((size_t)nthreads * sizeof(pthread_t));
    int started = 0;
    if (tid) {
        for (; started < nthreads; ++started)
            if (pthread_create(&tid[started], NULL, cross_worker, &W) != 0) break;
    }
    if (started == 0) cross_worker(&W);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    pthread_mutex_destroy(&W.lock);
    return W.failed ? ORACLE_NO_MEM : ORACLE_OK;
}

/* ---- FP8 forward: the steps of the quantised method -------------------------------
 * The "Flash-Attention" concept page names FP8 attention (FlashAttention-3 on H100,
 * 观察 2; quantised attention, 设计空间 路线 4) and conditional rescaling (已知局限)
 * without a recipe, so this oracle follows the steps of the quantised forward rather than a
 * closed form: Q, K, V are the dequantised e4m3 values (passed in as doubles); each row
 * runs the online softmax of the "FlashAttention 与高效注意力内核" tutorial (sections
 * Online Softmax 技巧 / 修正公式) over 128-key blocks, the running max moving only when a
 * block's max exceeds it by more than 8 in log2 units, and the probabilities that multiply
 * V are rounded to e4m3 (round to nearest even, saturating at 448) while the row sum l
 * uses them unrounded:
 *     m_new = max(m, blockmax) if blockmax > m + 8 else m        (log2 units)
 *     p_j   = 2^(s_j log2 e - m_new),  l = l 2^(m - m_new) + sum_j p_j
 *     O     = O 2^(m - m_new) + sum_j e4m3(p_j) v_j
 * and finally O / l, LSE = m ln 2 + ln l.  With round_p = 0 this is the exact forward
 * (the online softmax reaches the plain definition up to rounding). */
double oracle_round_e4m3(double x)
{
    if (x != x) return x;
    const double a = fabs(x);
    if (a >= 448.0) return copysign(448.0, x);
    double q;                                  /* spacing of e4m3 values around a */
    if (a < 0.015625) {
        q = 0.001953125;                       /* subnormals (and the lowest binade): 2^-9 */
    } else {
        int e;
        (void)frexp(a, &e);                    /* a = f 2^e, f in [0.5, 1): 3 mantissa bits */
        q = ldexp(1.0, e - 4);
    }
    const double r = nearbyint(a / q) * q;     /* default rounding mode: nearest, ties to even */
    return copysign(r > 448.0 ? 448.0 : r, x);
}

typedef struct {
    problem P;                  /* q, k, v (dequantised), hq, hkv, d, scale, causal, o, lse, cu */
    int32_t round_p;
    int64_t T;
    int64_t next, nitems;       /* items: (sequence, query head) */
    pthread_mutex_t lock;
    int failed;
} fp8_work;

#define FP8_KEYS_PER_BLOCK 128
#define FP8_RESCALE_SKIP 8.0

static void *fp8_worker(void *arg)
{
    fp8_work *W = (fp8_work *)arg;
    problem *P = &W->P;
    int64_t maxn = 1;
    for (int b = 0; b < P->nseq; ++b) {
        const int64_t n = P->cu[b + 1] - P->cu[b];
        if (n > maxn) maxn = n;
    }
    double *s = (double *)malloc((size_t)maxn * sizeof(double));
    double *acc = (double *)malloc((size_t)P->d * sizeof(double));
    if (!s || !acc) {
        pthread_mutex_lock(&W->lock); W->failed = 1; pthread_mutex_unlock(&W->lock);
        free(s); free(acc);
        return NULL;
    }
    const double log2e = 1.4426950408889634, ln2 = 0.6931471805599453;
    for (;;) {
        pthread_mutex_lock(&W->lock);
        const int64_t it = W->next++;
        pthread_mutex_unlock(&W->lock);
        if (it >= W->nitems) break;
        const int b = (int)(it / P->hq);
        const int h = (int)(it % P->hq);
        const int g = (int)(((int64_t)h * P->hkv) / P->hq);
        const int64_t t0 = P->cu[b];
        const int n = (int)(P->cu[b + 1] - t0);
        for (int i = 0; i < n; ++i) {
            const int64_t row = t0 + i;
            score_row(P, row, t0, n, visible_keys(i, n, P->causal), h, s);
            double m = -INFINITY, l = 0.0;
            for (int c = 0; c < P->d; ++c) acc[c] = 0.0;
            for (int j0 = 0; j0 < n; j0 += FP8_KEYS_PER_BLOCK) {
                const int j1 = j0 + FP8_KEYS_PER_BLOCK < n ? j0 + FP8_KEYS_PER_BLOCK : n;
                double mx = -INFINITY;
                for (int j = j0; j < j1; ++j) if (s[j] > mx) mx = s[j];
                const double cand = mx * log2e;
                const double m_new = cand > m + FP8_RESCALE_SKIP ? cand : m;
                if (m_new == -INFINITY) continue;             /* nothing visible yet */
                const double alpha = m == -INFINITY ? 0.0 : exp2(m - m_new);
                l *= alpha;
                for (int c = 0; c < P->d; ++c) acc[c] *= alpha;
                for (int j = j0; j < j1; ++j) {
                    if (s[j] == -INFINITY) continue;
                    const double pj = exp2(s[j] * log2e - m_new);
                    l += pj;
                    const double pv = W->round_p ? oracle_round_e4m3(pj) : pj;
                    const double *vj = P->v + ((t0 + j) * P->hkv + g) * P->d;
                    for (int c = 0; c < P->d; ++c) acc[c] += pv * vj[c];
                }
                m = m_new;
            }
            double *oi = P->o + (row * P->hq + h) * P->d;
            for (int c = 0; c < P->d; ++c) oi[c] = l > 0.0 ? acc[c] / l : 0.0;
            P->lse[(int64_t)h * W->T + row] = l > 0.0 ? m * ln2 + log(l) : -INFINITY;
        }
    }
    free(s);
    free(acc);
    return NULL;
}

int oracle_attn_fwd_fp8sim(const double *q, const double *k, const double *v,
                           const int32_t *cu_seqlens, int32_t nseq,
                           int32_t hq, int32_t hkv, int32_t d, double scale, int32_t causal,
                           int32_t round_p, double *o, double *lse, int32_t nthreads)
{
    int rc = check_args(cu_seqlens, nseq, hq, hkv, d);
    if (rc) return rc;
    fp8_work W;
    memset(&W, 0, sizeof W);
    W.P.q = q; W.P.k = k; W.P.v = v; W.P.cu = cu_seqlens; W.P.nseq = nseq;
    W.P.hq = hq; W.P.hkv = hkv; W.P.d = d; W.P.scale = scale; W.P.causal = causal;
    W.P.o = o; W.P.lse = lse;
    W.round_p = round_p;
    W.T = cu_seqlens[nseq];
    W.nitems = (int64_t)nseq * hq;
    pthread_mutex_init(&W.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    pthread_t *tid = (pthread_t *)malloc((size_t)nthreads * sizeof(pthread_t));
    int started = 0;
    if (tid) {
        for (; started < nthreads; ++started)
            if (pthread_create(&tid[started], NULL, fp8_worker, &W) != 0) break;
    }
    if (started == 0) fp8_worker(&W);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    pthread_mutex_destroy(&W.lock);
    return W.failed ? ORACLE_NO_MEM : ORACLE_OK;
}

/* Forward: o [T,hq,d], lse [hq,T].  row_sel (optional, [T]) restricts which rows are
 * written; other entries of o and lse are left untouched. */
int oracle_attn_fwd(const double *q, const double *k, const double *v,
                    const int32_t *cu_seqlens, int32_t nseq,
                    int32_t hq, int32_t hkv, int32_t d, double scale, int32_t causal,
                    const uint8_t *row_sel, double *o, double *lse, int32_t nthreads)
{
    int rc = check_args(cu_seqlens, nseq, hq, hkv, d);
    if (rc) return rc;
    problem P;
    memset(&P, 0, sizeof P);
    P.q = q; P.k = k; P.v = v; P.cu = cu_seqlens; P.nseq = nseq;
    P.hq = hq; P.hkv = hkv; P.d = d; P.scale = scale; P.causal = causal;
    P.row_sel = row_sel; P.o = o; P.lse = lse;
    return run_items(&P, 0, hq, nthreads);
}

/* Backward: dq [T,hq,d], dk/dv [T,hkv,d].  The oracle forms its own O, LSE and D from
 * the definition first (all rows of every head).  row_sel / key_sel (optional, [T])
 * restrict which dQ rows and which dK/dV keys are produced; others stay untouched.
 * o_out / lse_out (optional) receive the forward results.
 *
 * o_in / lse_in (optional) make this the backward *as a function of its inputs*: the
 * backward takes the forward's saved O and statistics ("前向: 只保存输出 O 与每块的
 * softmax 统计量"; "反向重算流程": recompute S and P from Q/K/V and those statistics).
 * When o_in is given, D_i = sum_c dO_ic o_in_ic; when lse_in is given,
 * P_ij = exp(S_ij - lse_in_i).  Without them the oracle's own O and LSE are used, which
 * is the exact gradient of the forward definition. */
int oracle_attn_bwd_ex(const double *q, const double *k, const double *v, const double *dout,
                       const int32_t *cu_seqlens, int32_t nseq,
                       int32_t hq, int32_t hkv, int32_t d, double scale, int32_t causal,
                       const uint8_t *row_sel, const uint8_t *key_sel,
                       const double *o_in, const double *lse_in,
                       double *dq, double *dk, double *dv,
                       double *o_out, double *lse_out, int32_t nthreads)
{
    int rc = check_args(cu_seqlens, nseq, hq, hkv, d);
    if (rc) return rc;
    const int64_t T = cu_seqlens[nseq];
    double *o = o_out ? o_out : (double *)malloc((size_t)(T > 0 ? T : 1) * hq * d * sizeof(double));
    double *lse = lse_out ? lse_out : (double *)malloc((size_t)(T > 0 ? T : 1) * hq * sizeof(double));
    double *dd = (double *)malloc((size_t)(T > 0 ? T : 1) * hq * sizeof(double));
    if (!o || !lse || !dd) {
        if (!o_out) free(o);
        if (!lse_out) free(lse);
        free(dd);
        return ORACLE_NO_MEM;
    }
    problem P;
    memset(&P, 0, sizeof P);
    P.q = q; P.k = k; P.v = v; P.dout = dout; P.cu = cu_seqlens; P.nseq = nseq;
    P.hq = hq; P.hkv = hkv; P.d = d; P.scale = scale; P.causal = causal;
    P.o = o; P.lse = lse; P.dd = dd;
    P.dq = dq; P.dk = dk; P.dv = dv;
    rc = run_items(&P, 0, hq, nthreads);          /* O, LSE, D for every row */
    if (!rc && (o_in || lse_in)) {                 /* the given O / LSE replace the oracle's */
        for (int64_t t = 0; t < T; ++t)
            for (int h = 0; h < hq; ++h) {
                if (lse_in) lse[(int64_t)h * T + t] = lse_in[(int64_t)h * T + t];
                if (o_in) {
                    const double *og = o_in + (t * hq + h) * d;
                    const double *dog = dout + (t * hq + h) * d;
                    double dsum = 0.0;
                    for (int c = 0; c < d; ++c) dsum += dog[c] * og[c];
                    dd[(int64_t)h * T + t] = dsum;
                }
            }
    }
    if (!rc) { P.row_sel = row_sel; rc = run_items(&P, 1, hq, nthreads); }   /* dQ rows */
    if (!rc) { P.row_sel = NULL; P.key_sel = key_sel; rc = run_items(&P, 2, hkv, nthreads); } /* dK, dV */
    if (!o_out) free(o);
    if (!lse_out) free(lse);
    free(dd);
    return rc;
}

/* The exact gradient of the forward definition (the oracle's own O and LSE). */
int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                    const int32_t *cu_seqlens, int32_t nseq,
                    int32_t hq, int32_t hkv, int32_t d, double scale, int32_t causal,
                    const uint8_t *row_sel, const uint8_t *key_sel,
                    double *dq, double *dk, double *dv,
                    double *o_out, double *lse_out, int32_t nthreads)
{
    return oracle_attn_bwd_ex(q, k, v, dout, cu_seqlens, nseq, hq, hkv, d, scale, causal, row_sel, key_sel,
                              NULL, NULL, dq, dk, dv, o_out, lse_out, nthreads);
}

/* The probability matrix of one (sequence, head) problem, materialised: p [n, n].
 * q [n,d], k [n,d].  Used by the tests for the row-sum / mask invariants. */
int oracle_attn_probs(const double *q, const double *k, int32_t n, int32_t d,
                      double scale, int32_t causal, double *p, double *lse)
{
    if (n < 0 || d <= 0) return ORACLE_BAD_ARG;
    int32_t cu[2] = {0, n};
    problem P;
    memset(&P, 0, sizeof P);
    P.q = q; P.k = k; P.cu = cu; P.nseq = 1; P.hq = 1; P.hkv = 1; P.d = d;
    P.scale = scale; P.causal = causal;
    double *s = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    if (!s) return ORACLE_NO_MEM;
    for (int i = 0; i < n; ++i) {
        score_row(&P, i, 0, n, visible_keys(i, n, causal), 0, s);
        const double l = softmax_row(s, n, p + (size_t)i * n);
        if (lse) lse[i] = l;
    }
    free(s);
    return ORACLE_OK;
}
