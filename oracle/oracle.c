/*
 * oracle.c -- exact softmax attention on the CPU, in fp64.
 *
 * TEST INFRASTRUCTURE.  This file is the correctness oracle for the GPU
 * attention forward pass.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load it.  It shares no code, header, table or
 * helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes is the plain definition of the result the tiled method
 * reaches exactly ("FlashAttention 2: Three Places the Chip Was Still
 * Waiting", section 1 "New here?": the answer is exact, not approximate;
 * "FlashAttention-2 and -3: From Algebra to GPU Scheduling", "Keep the
 * unchanged mathematical target in view"):
 *
 *   for every batch b, query head hq and query row i
 *     hk   = hq / (Hq / Hkv)                       (consecutive GQA groups)
 *     g_i  = i + Nk - Nq                           (the row's diagonal key)
 *     J_i  = { j in [k_begin, k_end) : not causal or j <= g_i,
 *                                      wl < 0 or j >= g_i - wl,
 *                                      wr < 0 or j <= g_i + wr }
 *     s_j  = scale * sum_c q[b,i,hq,c] * k[b,j,hk,c]     for j in J_i
 *     m    = max_j s_j
 *     w_j  = exp(s_j - m),   l = sum_j w_j
 *     O[b,i,hq,:] = sum_j w_j * v[b,j,hk,:] / l
 *     LSE[b,hq,i] = m + ln l
 *
 * The full score row is materialised (standard attention, the thing the
 * tiled method avoids); there is no tiling, no running max, no rescaling.
 * A row with an empty J_i gets O = 0 and LSE = -inf.  wl / wr are the left /
 * right widths of a sliding (local) window around the diagonal key, the
 * sliding-window variant that forks from the same scheduling skeleton
 * ("FlashAttention-2" explainer, "The Downstream Story"); -1 means no bound.
 *
 * Inputs are bf16 bit patterns; they are widened to double exactly.
 * Layouts: q [B,Nq,Hq,d], k and v [B,Nk,Hkv,d] (d contiguous).
 * Outputs: o [B,R,Hq,d] and lse [B,Hq,R] in double, where R is the number of
 * computed rows (all Nq rows, or the caller's row list).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const uint16_t *q, *k, *v;
    int B, Hq, Hkv, Nq, Nk, d, causal;
    int window_left, window_right; /* < 0: unbounded on that side */
    double scale;
    const int *rows;
    int n_rows;
    int k_begin, k_end;
    double *o, *lse;
    long n_items;
    long next_item; /* shared work counter, advanced atomically */
} oracle_job;

static double bf16_to_double(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Causal visibility with bottom-right alignment: key j is visible to query
 * row i when j <= i + (Nk - Nq).  For Nq == Nk this is the usual j <= i. */
static int key_visible(const oracle_job *J, int i, int j)
{
    if (j < J->k_begin || j >= J->k_end)
        return 0;
    if (J->causal && (long)j > (long)i + (long)J->Nk - (long)J->Nq)
        return 0;
    /* local window around the diagonal key g = i + Nk - Nq: g - wl <= j <= g + wr */
    const long g = (long)J->Nk - (long)J->Nq + (long)i;
    if (J->window_left >= 0 && (long)j < g - (long)J->window_left)
        return 0;
    if (J->window_right >= 0 && (long)j > g + (long)J->window_right)
        return 0;
    return 1;
}

/* One query row of one head: scores, max, exponentials, sum, weighted V,
 * one division, log-sum-exp.  `s` is scratch of Nk doubles. */
static void attention_row(const oracle_job *J, int b, int hq, int ri, double *s)
{
    const int d = J->d;
    const int i = J->rows ? J->rows[ri] : ri;
    const int group = J->Hq / J->Hkv;
    const int hk = hq / group;
    const uint16_t *qrow = J->q + (((size_t)b * J->Nq + i) * J->Hq + hq) * d;
    double *orow = J->o + (((size_t)b * J->n_rows + ri) * J->Hq + hq) * d;
    double *lse_out = J->lse + ((size_t)b * J->Hq + hq) * J->n_rows + ri;

    double qd[512];
    for (int c = 0; c < d; ++c)
        qd[c] = bf16_to_double(qrow[c]);

    double m = -INFINITY;
    int n_visible = 0;
    for (int j = 0; j < J->Nk; ++j) {
        if (!key_visible(J, i, j))
            continue;
        const uint16_t *krow = J->k + (((size_t)b * J->Nk + j) * J->Hkv + hk) * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
            dot += qd[c] * bf16_to_double(krow[c]);
        s[j] = J->scale * dot;
        if (s[j] > m)
            m = s[j];
        ++n_visible;
    }

    for (int c = 0; c < d; ++c)
        orow[c] = 0.0;
    if (n_visible == 0) {
        *lse_out = -INFINITY;
        return;
    }

    double l = 0.0;
    for (int j = 0; j < J->Nk; ++j) {
        if (!key_visible(J, i, j))
            continue;
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int j = 0; j < J->Nk; ++j) {
        if (!key_visible(J, i, j))
            continue;
        const uint16_t *vrow = J->v + (((size_t)b * J->Nk + j) * J->Hkv + hk) * d;
        const double w = s[j];
        for (int c = 0; c < d; ++c)
            orow[c] += w * bf16_to_double(vrow[c]);
    }
    for (int c = 0; c < d; ++c)
        orow[c] /= l;
    *lse_out = m + log(l);
}

#define ORACLE_ROWS_PER_ITEM 8

static void *oracle_worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    double *s = (double *)malloc(sizeof(double) * (size_t)(J->Nk > 0 ? J->Nk : 1));
    if (!s)
        return (void *)1;
    const long row_items = (J->n_rows + ORACLE_ROWS_PER_ITEM - 1) / ORACLE_ROWS_PER_ITEM;
    for (;;) {
        long it = __atomic_fetch_add(&J->next_item, 1, __ATOMIC_RELAXED);
        if (it >= J->n_items)
            break;
        const long bh = it / row_items;
        const int r0 = (int)(it % row_items) * ORACLE_ROWS_PER_ITEM;
        const int b = (int)(bh / J->Hq), hq = (int)(bh % J->Hq);
        for (int ri = r0; ri < r0 + ORACLE_ROWS_PER_ITEM && ri < J->n_rows; ++ri)
            attention_row(J, b, hq, ri, s);
    }
    free(s);
    return NULL;
}

/*
 * oracle_attention -- compute O and LSE for the rows listed in `rows`
 * (n_rows entries, indices into [0, Nq)), or for every row when rows == NULL
 * (then n_rows must equal Nq).  Keys are restricted to [k_begin, k_end)
 * intersected with the causal set and the window [g - window_left,
 * g + window_right] around the diagonal key g = i + Nk - Nq (a negative width
 * leaves that side open); pass 0, Nk and -1, -1 for the full range.
 * nthreads <= 0 uses every online core.  Returns 0 on success, 1 on bad
 * arguments, 2 on allocation or thread failure.
 */
int oracle_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                     int window_left, int window_right,
                     double scale, const int *rows, int n_rows, int k_begin, int k_end,
                     double *o, double *lse, int nthreads)
{
    if (!q || !k || !v || !o || !lse)
        return 1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0 || d > 512)
        return 1;
    if (Hq % Hkv != 0 || n_rows <= 0 || (!rows && n_rows != Nq))
        return 1;
    if (k_begin < 0 || k_end > Nk || k_begin > k_end)
        return 1;
    if (rows)
        for (int r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= Nq)
                return 1;

    oracle_job J;
    J.q = q; J.k = k; J.v = v;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Nq = Nq; J.Nk = Nk; J.d = d; J.causal = causal;
    J.window_left = window_left < 0 ? -1 : window_left;
    J.window_right = window_right < 0 ? -1 : window_right;
    J.scale = scale;
    J.rows = rows; J.n_rows = n_rows;
    J.k_begin = k_begin; J.k_end = k_end;
    J.o = o; J.lse = lse;
    J.n_items = (long)B * Hq * ((n_rows + ORACLE_ROWS_PER_ITEM - 1) / ORACLE_ROWS_PER_ITEM);
    J.next_item = 0;

    if (nthreads <= 0)
        nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 256)
        nthreads = 256;
    if ((long)nthreads > J.n_items)
        nthreads = (int)J.n_items;

    pthread_t tid[256];
    int started = 0, rc = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&tid[started], NULL, oracle_worker, &J) != 0) {
            rc = 2;
            break;
        }
        ++started;
    }
    if (oracle_worker(&J) != NULL)
        rc = 2;
    for (int t = 0; t < started; ++t) {
        void *ret = NULL;
        pthread_join(tid[t], &ret);
        if (ret != NULL)
            rc = 2;
    }
    return rc;
}

/* Number of worker threads oracle_attention uses for nthreads <= 0. */
int oracle_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n < 1 ? 1 : (n > 256 ? 256 : (int)n);
}

/* ------------------------------------------------------------------------
 * Backward pass (gradients of the attention output), from the definition.
 *
 * With P_ij = exp(s_ij - m_i) / l_i the probabilities of row i over its
 * visible keys J_i, O_i = sum_j P_ij v_j and an upstream gradient dO:
 *
 *   dV_j  = sum_i P_ij dO_i                         (over the rows i that see j)
 *   dP_ij = dO_i . v_j
 *   dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik)         (the softmax Jacobian)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 *
 * summed over the query heads of a KV head's group for dK and dV.  The
 * pages' headline numbers are forward+backward training numbers and name the
 * backward pass as the forward's counterpart ("FlashAttention 2: Three Places
 * the Chip Was Still Waiting", section 2.5); its arithmetic here is the chain
 * rule applied to the plain definition above, with no tiling and no
 * recomputation tricks.  dq is [B,Nq,Hq,d], dk and dv are [B,Nk,Hkv,d], all
 * double.  Returns 0, 1 on bad arguments, 2 on allocation or thread failure.
 * ------------------------------------------------------------------------ */
typedef struct {
    const oracle_job *J;
    const uint16_t *dout;
    double *dq, *dk, *dv;
    long next_group;  /* (b, hk) work counter, advanced atomically */
} oracle_bwd_job;

/* All query heads of one (batch, KV head) group: every row's probabilities,
 * then its dQ row and its contributions to the group's dK and dV rows. */
static void backward_group(const oracle_bwd_job *W, int b, int hk, double *p, double *dp)
{
    const oracle_job *J = W->J;
    const int d = J->d, group = J->Hq / J->Hkv;
    for (int hq = hk * group; hq < (hk + 1) * group; ++hq) {
        for (int i = 0; i < J->Nq; ++i) {
            const size_t row_at = (((size_t)b * J->Nq + i) * J->Hq + hq) * (size_t)d;
            const uint16_t *qrow = J->q + row_at;
            const uint16_t *gorow = W->dout + row_at;
            double *dqrow = W->dq + row_at;
            for (int c = 0; c < d; ++c)
                dqrow[c] = 0.0;
            double m = -INFINITY;
            int n_visible = 0;
            for (int j = 0; j < J->Nk; ++j) {
                if (!key_visible(J, i, j))
                    continue;
                const uint16_t *krow = J->k + (((size_t)b * J->Nk + j) * J->Hkv + hk) * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c)
                    dot += bf16_to_double(qrow[c]) * bf16_to_double(krow[c]);
                p[j] = J->scale * dot;
                if (p[j] > m)
                    m = p[j];
                ++n_visible;
            }
            if (n_visible == 0)
                continue;
            double l = 0.0;
            for (int j = 0; j < J->Nk; ++j) {
                if (!key_visible(J, i, j))
                    continue;
                p[j] = exp(p[j] - m);
                l += p[j];
            }
            double pdp = 0.0; /* sum_k P_ik dP_ik */
            for (int j = 0; j < J->Nk; ++j) {
                if (!key_visible(J, i, j))
                    continue;
                p[j] /= l;
                const uint16_t *vj = J->v + (((size_t)b * J->Nk + j) * J->Hkv + hk) * d;
                double g = 0.0;
                for (int c = 0; c < d; ++c)
                    g += bf16_to_double(gorow[c]) * bf16_to_double(vj[c]);
                dp[j] = g;
                pdp += p[j] * g;
            }
            for (int j = 0; j < J->Nk; ++j) {
                if (!key_visible(J, i, j))
                    continue;
                const double ds = p[j] * (dp[j] - pdp);
                const uint16_t *krow = J->k + (((size_t)b * J->Nk + j) * J->Hkv + hk) * d;
                double *dkrow = W->dk + (((size_t)b * J->Nk + j) * J->Hkv + hk) * d;
                double *dvrow = W->dv + (((size_t)b * J->Nk + j) * J->Hkv + hk) * d;
                for (int c = 0; c < d; ++c) {
                    dqrow[c] += J->scale * ds * bf16_to_double(krow[c]);
                    dkrow[c] += J->scale * ds * bf16_to_double(qrow[c]);
                    dvrow[c] += p[j] * bf16_to_double(gorow[c]);
                }
            }
        }
    }
}

static void *oracle_bwd_worker(void *arg)
{
    oracle_bwd_job *W = (oracle_bwd_job *)arg;
    const oracle_job *J = W->J;
    double *p = (double *)malloc(sizeof(double) * (size_t)J->Nk);
    double *dp = (double *)malloc(sizeof(double) * (size_t)J->Nk);
    if (!p || !dp) {
        free(p);
        free(dp);
        return (void *)1;
    }
    const long n_groups = (long)J->B * J->Hkv;
    for (;;) {
        long it = __atomic_fetch_add(&W->next_group, 1, __ATOMIC_RELAXED);
        if (it >= n_groups)
            break;
        backward_group(W, (int)(it / J->Hkv), (int)(it % J->Hkv), p, dp);
    }
    free(p);
    free(dp);
    return NULL;
}

int oracle_attention_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              const uint16_t *dout, int B, int Hq, int Hkv, int Nq, int Nk,
                              int d, int causal, int window_left, int window_right, double scale,
                              double *dq, double *dk, double *dv, int nthreads)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv)
        return 1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0 || d > 512 || Hq % Hkv != 0)
        return 1;
    oracle_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Nq = Nq; J.Nk = Nk; J.d = d; J.causal = causal;
    J.window_left = window_left < 0 ? -1 : window_left;
    J.window_right = window_right < 0 ? -1 : window_right;
    J.scale = scale;
    J.k_begin = 0; J.k_end = Nk;
    memset(dk, 0, sizeof(double) * (size_t)B * Nk * Hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)B * Nk * Hkv * d);
    oracle_bwd_job W;
    W.J = &J; W.dout = dout; W.dq = dq; W.dk = dk; W.dv = dv; W.next_group = 0;
    int nt = nthreads > 0 ? nthreads : oracle_default_threads();
    const long n_groups = (long)B * Hkv;
    if (nt > n_groups)
        nt = (int)n_groups;
    pthread_t tid[256];
    int started = 0, rc = 0;
    for (int t = 1; t < nt && t < 256; ++t) {
        if (pthread_create(&tid[started], NULL, oracle_bwd_worker, &W) != 0) {
            rc = 2;
            break;
        }
        ++started;
    }
    if (oracle_bwd_worker(&W) != NULL)
        rc = 2;
    for (int t = 0; t < started; ++t) {
        void *ret = NULL;
        pthread_join(tid[t], &ret);
        if (ret != NULL)
            rc = 2;
    }
    return rc;
}
