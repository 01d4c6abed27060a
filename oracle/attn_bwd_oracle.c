/*
 * attn_bwd_oracle.c -- plain fp64 CPU oracle for the gradients of packed
 * variable-length bidirectional multi-head attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests may load this file's library.  It
 * shares no code, header, table or helper with the CUDA path (nor with
 * attn_oracle.c: the few lines of bf16 widening and segment lookup are
 * repeated here on purpose).
 *
 * What it differentiates: the forward definition of attn_oracle.c (per
 * segment i of cu_seqlens, per head h, per query row r of the segment; the
 * SparseAttn page, section 3.1, and the Mage-Flow page, "Packing + Flash
 * Attention varlen"):
 *     s_rj = scale * q_r . k_j,   P_rj = exp(s_rj) / sum_l exp(s_rl),
 *     out_r = sum_j P_rj v_j                    (j over the keys of the segment)
 * Given dout = dL/dout, the chain rule through the softmax gives (the
 * standard result for y = softmax(x): dx_j = y_j (dy_j - sum_l y_l dy_l)):
 *     dP_rj = dout_r . v_j
 *     D_r   = sum_j P_rj dP_rj                  (= dout_r . out_r)
 *     dS_rj = P_rj (dP_rj - D_r)
 *     dq_r  = scale * sum_j dS_rj k_j
 *     dk_j  = scale * sum_r dS_rj q_r           (r over the queries of the segment)
 *     dv_j  = sum_r P_rj dout_r
 * P is recomputed from q and k in fp64 (two passes per row: max, then sum); no
 * forward output or log-sum-exp is taken from anywhere else.
 *
 * Work is split by (segment, head) units; a unit owns the dq, dk, dv rows of
 * its segment and head, so threads never write the same element.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define BWD_IN_F64 0
#define BWD_IN_BF16 1

#define BWD_OK 0
#define BWD_ERR_ARGS -1
#define BWD_ERR_CU -2
#define BWD_ERR_ROWS -3
#define BWD_ERR_NOMEM -4

static double bwd_widen(const void *base, int kind, int64_t index) {
    if (kind == BWD_IN_F64) return ((const double *)base)[index];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[index] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    int kind;
    const void *q, *k, *v, *dout;
    const int32_t *cu;
    int32_t batch, heads, d, dv;
    int64_t total;
    double scale;
    /* full mode: every (segment, head) unit, outputs dq [T,H,d], dk [T,H,d], dv [T,H,dv] */
    double *dq, *dk, *dvo;
    /* row mode (dq only): n_rows listed (token, head) pairs, dq_rows [n, d] */
    int64_t n_rows;
    const int64_t *row_token;
    const int32_t *row_head;
    double *dq_rows;
    int64_t n_units, next;
    pthread_mutex_t lock;
    int64_t max_len;
} bwd_job_t;

static int32_t bwd_segment_of(const int32_t *cu, int32_t batch, int64_t token) {
    int32_t lo = 0, hi = batch;
    while (hi - lo > 1) {
        int32_t mid = lo + (hi - lo) / 2;
        if ((int64_t)cu[mid] <= token) lo = mid; else hi = mid;
    }
    return lo;
}

#define IDX(t, h, c, width) ((((int64_t)(t)) * J->heads + (h)) * (int64_t)(width) + (c))

/* Row r of segment [beg, end), head h: P_r into p[], dP_r into dp[], returns D_r. */
static double row_softmax_and_dp(const bwd_job_t *J, int64_t r, int32_t h, int64_t beg, int64_t end,
                                 double *p, double *dp) {
    int64_t n = end - beg;
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int32_t c = 0; c < J->d; ++c)
            dot += bwd_widen(J->q, J->kind, IDX(r, h, c, J->d)) * bwd_widen(J->k, J->kind, IDX(beg + j, h, c, J->d));
        p[j] = J->scale * dot;
        if (p[j] > m) m = p[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        p[j] = exp(p[j] - m);
        l += p[j];
    }
    double D = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        p[j] /= l;
        double dot = 0.0;
        for (int32_t c = 0; c < J->dv; ++c)
            dot += bwd_widen(J->dout, J->kind, IDX(r, h, c, J->dv)) * bwd_widen(J->v, J->kind, IDX(beg + j, h, c, J->dv));
        dp[j] = dot;
        D += p[j] * dot;
    }
    return D;
}

/* One (segment, head) unit: dq, dk, dv of all its rows. */
static void one_unit(const bwd_job_t *J, int32_t seg, int32_t h, double *p, double *dp) {
    int64_t beg = J->cu[seg], end = J->cu[seg + 1], n = end - beg;
    for (int64_t j = 0; j < n; ++j) {
        for (int32_t c = 0; c < J->d; ++c) J->dk[IDX(beg + j, h, c, J->d)] = 0.0;
        for (int32_t c = 0; c < J->dv; ++c) J->dvo[IDX(beg + j, h, c, J->dv)] = 0.0;
    }
    for (int64_t i = 0; i < n; ++i) {
        int64_t r = beg + i;
        double D = row_softmax_and_dp(J, r, h, beg, end, p, dp);
        for (int32_t c = 0; c < J->d; ++c) J->dq[IDX(r, h, c, J->d)] = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double ds = p[j] * (dp[j] - D);
            for (int32_t c = 0; c < J->d; ++c) {
                J->dq[IDX(r, h, c, J->d)] += J->scale * ds * bwd_widen(J->k, J->kind, IDX(beg + j, h, c, J->d));
                J->dk[IDX(beg + j, h, c, J->d)] += J->scale * ds * bwd_widen(J->q, J->kind, IDX(r, h, c, J->d));
            }
            for (int32_t c = 0; c < J->dv; ++c)
                J->dvo[IDX(beg + j, h, c, J->dv)] += p[j] * bwd_widen(J->dout, J->kind, IDX(r, h, c, J->dv));
        }
    }
}

/* One listed query row: dq only. */
static void one_dq_row(const bwd_job_t *J, int64_t i, double *p, double *dp) {
    int64_t r = J->row_token[i];
    int32_t h = J->row_head[i];
    int32_t seg = bwd_segment_of(J->cu, J->batch, r);
    int64_t beg = J->cu[seg], end = J->cu[seg + 1], n = end - beg;
    double D = row_softmax_and_dp(J, r, h, beg, end, p, dp);
    double *out = J->dq_rows + i * (int64_t)J->d;
    for (int32_t c = 0; c < J->d; ++c) out[c] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double ds = p[j] * (dp[j] - D);
        for (int32_t c = 0; c < J->d; ++c) out[c] += J->scale * ds * bwd_widen(J->k, J->kind, IDX(beg + j, h, c, J->d));
    }
}

static void *bwd_worker(void *arg) {
    bwd_job_t *J = (bwd_job_t *)arg;
    size_t len = (size_t)(J->max_len > 0 ? J->max_len : 1);
    double *p = (double *)malloc(sizeof(double) * len);
    double *dp = (double *)malloc(sizeof(double) * len);
    if (!p || !dp) { free(p); free(dp); return (void *)1; }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t u = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units) break;
        if (J->row_token) one_dq_row(J, u, p, dp);
        else one_unit(J, (int32_t)(u / J->heads), (int32_t)(u % J->heads), p, dp);
    }
    free(p); free(dp);
    return NULL;
}

static int bwd_check(int in_kind, const int32_t *cu, int32_t batch, int64_t total, int32_t heads, int32_t d,
                     int32_t dv, int64_t *max_len) {
    if ((in_kind != BWD_IN_F64 && in_kind != BWD_IN_BF16) || batch < 0 || total < 0 || heads <= 0 || d <= 0 ||
        dv <= 0 || !cu)
        return BWD_ERR_ARGS;
    if (cu[0] != 0 || (int64_t)cu[batch] != total) return BWD_ERR_CU;
    *max_len = 0;
    for (int32_t i = 0; i < batch; ++i) {
        if (cu[i + 1] < cu[i]) return BWD_ERR_CU;
        int64_t len = (int64_t)cu[i + 1] - cu[i];
        if (len > *max_len) *max_len = len;
    }
    return BWD_OK;
}

static int bwd_run(bwd_job_t *J, int n_threads) {
    if (J->n_units == 0) return BWD_OK;
    pthread_mutex_init(&J->lock, NULL);
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if ((int64_t)n_threads > J->n_units) n_threads = (int)J->n_units;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!tid) { pthread_mutex_destroy(&J->lock); return BWD_ERR_NOMEM; }
    int started = 0, failed = 0;
    for (int t = 0; t < n_threads; ++t) {
        if (pthread_create(&tid[t], NULL, bwd_worker, J) != 0) break;
        ++started;
    }
    if (started == 0 && bwd_worker(J) != NULL) failed = 1;
    for (int t = 0; t < started; ++t) {
        void *ret = NULL;
        pthread_join(tid[t], &ret);
        if (ret) failed = 1;
    }
    free(tid);
    pthread_mutex_destroy(&J->lock);
    return failed ? BWD_ERR_NOMEM : BWD_OK;
}

/*
 * oracle_varlen_attn_bwd: dq [T,H,d], dk [T,H,d], dv [T,H,dv] for every row.
 * q, k: [T,H,d]; v, dout: [T,H,dv]; all fp64 or all bf16 bit patterns.
 */
int oracle_varlen_attn_bwd(int in_kind, const void *q, const void *k, const void *v, const void *dout,
                           const int32_t *cu_seqlens, int32_t batch, int64_t total_tokens, int32_t heads,
                           int32_t head_dim, int32_t v_dim, double scale, double *dq, double *dk, double *dv,
                           int n_threads) {
    bwd_job_t J;
    memset(&J, 0, sizeof J);
    int rc = bwd_check(in_kind, cu_seqlens, batch, total_tokens, heads, head_dim, v_dim, &J.max_len);
    if (rc != BWD_OK) return rc;
    if (total_tokens == 0) return BWD_OK;
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return BWD_ERR_ARGS;
    J.kind = in_kind; J.q = q; J.k = k; J.v = v; J.dout = dout; J.cu = cu_seqlens; J.batch = batch;
    J.total = total_tokens; J.heads = heads; J.d = head_dim; J.dv = v_dim; J.scale = scale;
    J.dq = dq; J.dk = dk; J.dvo = dv;
    J.n_units = (int64_t)batch * heads;
    return bwd_run(&J, n_threads);
}

/* oracle_varlen_attn_bwd_dq_rows: dq [n_rows, d] of the listed (token, head) rows only. */
int oracle_varlen_attn_bwd_dq_rows(int in_kind, const void *q, const void *k, const void *v, const void *dout,
                                   const int32_t *cu_seqlens, int32_t batch, int64_t total_tokens, int32_t heads,
                                   int32_t head_dim, int32_t v_dim, double scale, int64_t n_rows,
                                   const int64_t *row_token, const int32_t *row_head, double *dq_rows,
                                   int n_threads) {
    bwd_job_t J;
    memset(&J, 0, sizeof J);
    int rc = bwd_check(in_kind, cu_seqlens, batch, total_tokens, heads, head_dim, v_dim, &J.max_len);
    if (rc != BWD_OK) return rc;
    if (n_rows == 0) return BWD_OK;
    if (!q || !k || !v || !dout || !row_token || !row_head || !dq_rows) return BWD_ERR_ARGS;
    for (int64_t i = 0; i < n_rows; ++i)
        if (row_token[i] < 0 || row_token[i] >= total_tokens || row_head[i] < 0 || row_head[i] >= heads)
            return BWD_ERR_ROWS;
    J.kind = in_kind; J.q = q; J.k = k; J.v = v; J.dout = dout; J.cu = cu_seqlens; J.batch = batch;
    J.total = total_tokens; J.heads = heads; J.d = head_dim; J.dv = v_dim; J.scale = scale;
    J.n_rows = n_rows; J.row_token = row_token; J.row_head = row_head; J.dq_rows = dq_rows;
    J.n_units = n_rows;
    return bwd_run(&J, n_threads);
}
