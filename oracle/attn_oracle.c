/*
 * attn_oracle.c -- plain fp64 CPU oracle for packed variable-length
 * bidirectional multi-head attention (the block-diagonal softmax(QK^T*scale)V).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this file's library.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * What it computes (definitions followed, by page and section):
 *   - "AIGC fundamentals: SparseAttn", section 3.1: scaled scores
 *     s_ij = scale * q_i . k_j, weights p_ij = exp(s_ij) / sum_l exp(s_il),
 *     output y_i = sum_j p_ij v_j; a restricted softmax over the kept keys S_i
 *     equals softmax over S_i alone, and an empty S_i is undefined.
 *   - Mage-Flow page, "Packing + Flash Attention varlen": tokens of all images
 *     are concatenated; cu_seqlens = [0, L0, L0+L1, ...] marks image i as
 *     tokens [cu_i, cu_{i+1}); attention is non-causal and a token attends only
 *     to the tokens of its own image (block-diagonal mask, no padding).
 *   - GigaPath-Flash page, section 2.2: standard attention softmax(QK^T/sqrt(d))V
 *     computed with the whole score row materialised.
 *
 * For every query row r of segment i and head h:
 *     s_j   = scale * sum_c q[r,h,c] * k[j,h,c]        j in [cu_i, cu_{i+1})
 *     m     = max_j s_j
 *     w_j   = exp(s_j - m),   l = sum_j w_j
 *     out[r,h,:] = (sum_j w_j v[j,h,:]) / l
 *     lse[r,h]   = m + log(l)          (natural log)
 * Two plain passes over the row (max, then sum); no blocking, no online
 * rescaling.  The max is subtracted only to keep exp() finite; it cancels.
 *
 * Inputs are either fp64 arrays or bf16 bit patterns (uint16), widened
 * exactly to fp64 (a bf16 value is the top 16 bits of an IEEE fp32).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_IN_F64 0
#define ORACLE_IN_BF16 1

#define ORACLE_OK 0
#define ORACLE_ERR_ARGS -1
#define ORACLE_ERR_CU -2
#define ORACLE_ERR_ROWS -3
#define ORACLE_ERR_NOMEM -4

static double widen(const void *base, int kind, int64_t index) {
    if (kind == ORACLE_IN_F64) {
        return ((const double *)base)[index];
    }
    uint32_t bits = (uint32_t)((const uint16_t *)base)[index] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    int kind;
    const void *q, *k, *v;
    const int32_t *cu;
    int32_t batch;
    int64_t total;
    int32_t heads, d, dv;
    double scale;
    int64_t n_rows;            /* number of (token, head) rows to compute */
    const int64_t *row_token;  /* NULL: every (token, head) in token-major order */
    const int32_t *row_head;
    double *out, *lse;
    int64_t next;              /* shared work counter, guarded by lock */
    pthread_mutex_t lock;
    int64_t max_len;
} job_t;

/* Segment index i with cu[i] <= token < cu[i+1] (cu is non-decreasing). */
static int32_t segment_of(const int32_t *cu, int32_t batch, int64_t token) {
    int32_t lo = 0, hi = batch; /* answer in [lo, hi) */
    while (hi - lo > 1) {
        int32_t mid = lo + (hi - lo) / 2;
        if ((int64_t)cu[mid] <= token) lo = mid; else hi = mid;
    }
    return lo;
}

/* One query row: the definition above, written out. */
static void one_row(const job_t *J, int64_t r, int32_t h, double *s, double *acc,
                    double *out_row, double *lse_out) {
    int32_t seg = segment_of(J->cu, J->batch, r);
    int64_t beg = J->cu[seg], end = J->cu[seg + 1];
    int64_t n = end - beg;
    int64_t qbase = (r * J->heads + h) * (int64_t)J->d;

    /* pass 1: scores and their maximum */
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        int64_t kbase = ((beg + j) * J->heads + h) * (int64_t)J->d;
        double dot = 0.0;
        for (int32_t c = 0; c < J->d; ++c)
            dot += widen(J->q, J->kind, qbase + c) * widen(J->k, J->kind, kbase + c);
        s[j] = J->scale * dot;
        if (s[j] > m) m = s[j];
    }
    /* pass 2: weights, normaliser and weighted sum of values */
    double l = 0.0;
    for (int32_t c = 0; c < J->dv; ++c) acc[c] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double w = exp(s[j] - m);
        l += w;
        int64_t vbase = ((beg + j) * J->heads + h) * (int64_t)J->dv;
        for (int32_t c = 0; c < J->dv; ++c) acc[c] += w * widen(J->v, J->kind, vbase + c);
    }
    for (int32_t c = 0; c < J->dv; ++c) out_row[c] = acc[c] / l;
    *lse_out = m + log(l);
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    double *s = (double *)malloc(sizeof(double) * (size_t)(J->max_len > 0 ? J->max_len : 1));
    double *acc = (double *)malloc(sizeof(double) * (size_t)J->dv);
    if (!s || !acc) { free(s); free(acc); return (void *)1; }
    const int64_t chunk = 64;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t start = J->next;
        J->next += chunk;
        pthread_mutex_unlock(&J->lock);
        if (start >= J->n_rows) break;
        int64_t stop = start + chunk < J->n_rows ? start + chunk : J->n_rows;
        for (int64_t i = start; i < stop; ++i) {
            int64_t r; int32_t h;
            if (J->row_token) { r = J->row_token[i]; h = J->row_head[i]; }
            else { r = i / J->heads; h = (int32_t)(i % J->heads); }
            one_row(J, r, h, s, acc, J->out + i * (int64_t)J->dv, J->lse + i);
        }
    }
    free(s); free(acc);
    return NULL;
}

/*
 * oracle_varlen_attn: block-diagonal attention for every row (row_token == NULL:
 * out [T, H, dv], lse [T, H]) or for a list of n_rows (token, head) pairs
 * (out [n_rows, dv], lse [n_rows]).  Returns 0 or a negative error code.
 * n_threads <= 0 uses every online core.
 */
int oracle_varlen_attn(int in_kind, const void *q, const void *k, const void *v,
                       const int32_t *cu_seqlens, int32_t batch, int64_t total_tokens,
                       int32_t heads, int32_t head_dim, int32_t v_dim, double scale,
                       int64_t n_rows, const int64_t *row_token, const int32_t *row_head,
                       double *out, double *lse, int n_threads) {
    if ((in_kind != ORACLE_IN_F64 && in_kind != ORACLE_IN_BF16) || batch < 0 || total_tokens < 0 ||
        heads <= 0 || head_dim <= 0 || v_dim <= 0 || !cu_seqlens)
        return ORACLE_ERR_ARGS;
    /* cu_seqlens: starts at 0, never decreases, ends at total_tokens */
    if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[batch] != total_tokens) return ORACLE_ERR_CU;
    int64_t max_len = 0;
    for (int32_t i = 0; i < batch; ++i) {
        if (cu_seqlens[i + 1] < cu_seqlens[i]) return ORACLE_ERR_CU;
        int64_t len = (int64_t)cu_seqlens[i + 1] - cu_seqlens[i];
        if (len > max_len) max_len = len;
    }
    if (!row_token) n_rows = total_tokens * heads;
    if (n_rows == 0) return ORACLE_OK;
    if (!q || !k || !v || !out || !lse) return ORACLE_ERR_ARGS;
    if (row_token) {
        if (!row_head) return ORACLE_ERR_ROWS;
        for (int64_t i = 0; i < n_rows; ++i)
            if (row_token[i] < 0 || row_token[i] >= total_tokens || row_head[i] < 0 || row_head[i] >= heads)
                return ORACLE_ERR_ROWS;
    }
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = in_kind; J.q = q; J.k = k; J.v = v; J.cu = cu_seqlens; J.batch = batch;
    J.total = total_tokens; J.heads = heads; J.d = head_dim; J.dv = v_dim; J.scale = scale;
    J.n_rows = n_rows; J.row_token = row_token; J.row_head = row_head; J.out = out; J.lse = lse;
    J.next = 0; J.max_len = max_len;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if ((int64_t)n_threads > n_rows) n_threads = (int)n_rows;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!tid) { pthread_mutex_destroy(&J.lock); return ORACLE_ERR_NOMEM; }
    int started = 0, failed = 0;
    for (int t = 0; t < n_threads; ++t) {
        if (pthread_create(&tid[t], NULL, worker, &J) != 0) break;
        ++started;
    }
    if (started == 0 && worker(&J) != NULL) failed = 1;
    for (int t = 0; t < started; ++t) {
        void *ret = NULL;
        pthread_join(tid[t], &ret);
        if (ret) failed = 1;
    }
    free(tid);
    pthread_mutex_destroy(&J.lock);
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* Number of worker threads a call with n_threads <= 0 uses. */
int oracle_default_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n < 1 ? 1 : (int)n;
}
