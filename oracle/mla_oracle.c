/*
 * Test infrastructure only -- NOT part of the product path.
 *
 * Plain, slow, fp64 CPU statement of variable-length, causally masked
 * Multi-head Latent Attention prefill, as the "MLA Prefill" page
 * (Ascend Transformer Boost C API, AtbMLAPreFillGetWorkspaceSize members
 * table) describes the operation.  Only the tests, the package's smoke check
 * and the CPU-baseline leg of the benchmark may load this file.  It shares no
 * code, header, table or helper with the CUDA path.
 *
 * What is computed (every step is written out, no blocking or fusion):
 *
 *   For sequence b with query length Lq_b (qSeqLen row) and key length Lk_b
 *   (kvSeqLen row), packed at token offsets cq_b = sum_{b'<b} Lq_b' and
 *   ck_b = sum_{b'<b} Lk_b' (the packed [batch*seq, head, dim] layouts of the
 *   Q / QRope / K / kRope / V rows), for every query head h with kv head
 *   kh = h / (headNum / kvHeadNum), every query row i < Lq_b and key j < Lk_b:
 *
 *     s_ij = qkScale * ( sum_d Q[cq_b+i,h,d]  * K[ck_b+j,kh,d]
 *                      + sum_r QR[cq_b+i,h,r] * KR[ck_b+j,kh,r] )
 *        -- "scaling coefficient post-multiplied by Q*K^T" (qkScale row); the
 *           rope halves (QRope / kRope rows) are part of the same product.
 *     visible(i,j) = (mask == causal) ? j <= i + (Lk_b - Lq_b) : true
 *        -- the causal mask (Mask row, MASK_TYPE_CAUSAL_MASK), aligned to the
 *           bottom-right corner when Lq_b < Lk_b; the all-zero mask of the
 *           maskType row (UNDEFINED) hides nothing.
 *     p_ij = exp(s_ij - m_i) / sum_{visible k} exp(s_ik - m_i),  m_i = max s_ij
 *            over the visible j; p_ij = 0 where not visible.
 *     O[cq_b+i,h,:] = sum_{visible j} p_ij * V[ck_b+j,kh,:]   (attenOut row)
 *
 *   A row with no visible key has O = 0.  qkScale is a float32 argument, and
 *   its float value is widened to double.  All inputs are given as doubles
 *   (the exact widening of the 16-bit values) and all arithmetic is fp64.
 *
 * Readings of points the page leaves open are stated where they are used.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARGS 1
#define ORACLE_ERR_SEQLEN 2
#define ORACLE_ERR_NOMEM 3

/* maskType values: 0 = no mask (UNDEFINED: all-zero mask), 1 = causal. */
#define ORACLE_MASK_NONE 0
#define ORACLE_MASK_CAUSAL 1

typedef struct {
    const double *q, *q_rope, *k, *k_rope, *v;
    const int32_t *q_seqlen, *kv_seqlen;
    int64_t batch, t_q, t_k, head_num, kv_head_num;
    int64_t d_nope, d_rope, d_v;
    int mask_type;
    double scale;
    /* derived */
    int64_t *cq, *ck; /* exclusive prefix sums, length batch + 1 */
} oracle_problem;

/* Which sequence owns packed query token t, or -1 if t lies past sum(Lq). */
static int64_t seq_of_token(const oracle_problem *pb, int64_t t) {
    for (int64_t b = 0; b < pb->batch; ++b)
        if (t >= pb->cq[b] && t < pb->cq[b + 1]) return b;
    return -1;
}

/*
 * The attention weights of one query row (token t, head h) over the keys of
 * its sequence: p[j] for j < Lk_b.  Returns the number of visible keys.
 */
static int64_t row_probs(const oracle_problem *pb, int64_t b, int64_t t, int64_t h, double *p) {
    const int64_t lq = pb->q_seqlen[b], lk = pb->kv_seqlen[b];
    const int64_t i = t - pb->cq[b];
    const int64_t group = pb->head_num / pb->kv_head_num;
    const int64_t kh = h / group; /* contiguous head groups */
    const int64_t off = lk - lq;  /* bottom-right alignment of the causal mask */
    int64_t n_vis = 0;
    double m = -INFINITY;
    for (int64_t j = 0; j < lk; ++j) {
        const int vis = (pb->mask_type == ORACLE_MASK_CAUSAL) ? (j <= i + off) : 1;
        if (!vis) {
            p[j] = 0.0;
            continue;
        }
        const double *qn = pb->q + (t * pb->head_num + h) * pb->d_nope;
        const double *kn = pb->k + ((pb->ck[b] + j) * pb->kv_head_num + kh) * pb->d_nope;
        double dot = 0.0;
        for (int64_t d = 0; d < pb->d_nope; ++d) dot += qn[d] * kn[d];
        if (pb->d_rope > 0) {
            const double *qr = pb->q_rope + (t * pb->head_num + h) * pb->d_rope;
            const double *kr = pb->k_rope + ((pb->ck[b] + j) * pb->kv_head_num + kh) * pb->d_rope;
            for (int64_t r = 0; r < pb->d_rope; ++r) dot += qr[r] * kr[r];
        }
        p[j] = pb->scale * dot; /* the raw score, turned into a weight below */
        if (p[j] > m) m = p[j];
        ++n_vis;
    }
    if (n_vis == 0) return 0;
    double denom = 0.0;
    for (int64_t j = 0; j < lk; ++j) {
        const int vis = (pb->mask_type == ORACLE_MASK_CAUSAL) ? (j <= i + off) : 1;
        if (vis) {
            p[j] = exp(p[j] - m);
            denom += p[j];
        }
    }
    for (int64_t j = 0; j < lk; ++j) {
        const int vis = (pb->mask_type == ORACLE_MASK_CAUSAL) ? (j <= i + off) : 1;
        if (vis) p[j] /= denom;
    }
    (void)lq;
    return n_vis;
}

/* One output row: O[t, h, :] = sum_j p_j V[ck_b + j, kh, :]. */
static void row_output(const oracle_problem *pb, int64_t b, int64_t t, int64_t h, double *p, double *out) {
    const int64_t lk = pb->kv_seqlen[b];
    const int64_t kh = h / (pb->head_num / pb->kv_head_num);
    double *o = out + (t * pb->head_num + h) * pb->d_v;
    for (int64_t d = 0; d < pb->d_v; ++d) o[d] = 0.0;
    if (row_probs(pb, b, t, h, p) == 0) return; /* no visible key: O = 0 */
    for (int64_t j = 0; j < lk; ++j) {
        if (p[j] == 0.0) continue;
        const double *vr = pb->v + ((pb->ck[b] + j) * pb->kv_head_num + kh) * pb->d_v;
        for (int64_t d = 0; d < pb->d_v; ++d) o[d] += p[j] * vr[d];
    }
}

static int prepare(oracle_problem *pb) {
    if (pb->batch < 0 || pb->head_num < 1 || pb->kv_head_num < 1 || pb->head_num % pb->kv_head_num != 0 ||
        pb->d_nope < 0 || pb->d_rope < 0 || pb->d_v < 1 || pb->t_q < 0 || pb->t_k < 0)
        return ORACLE_ERR_ARGS;
    if (pb->mask_type != ORACLE_MASK_NONE && pb->mask_type != ORACLE_MASK_CAUSAL) return ORACLE_ERR_ARGS;
    pb->cq = (int64_t *)calloc((size_t)pb->batch + 1, sizeof(int64_t));
    pb->ck = (int64_t *)calloc((size_t)pb->batch + 1, sizeof(int64_t));
    if (!pb->cq || !pb->ck) return ORACLE_ERR_NOMEM;
    for (int64_t b = 0; b < pb->batch; ++b) {
        if (pb->q_seqlen[b] < 0 || pb->kv_seqlen[b] < 0) return ORACLE_ERR_SEQLEN;
        pb->cq[b + 1] = pb->cq[b] + pb->q_seqlen[b];
        pb->ck[b + 1] = pb->ck[b] + pb->kv_seqlen[b];
    }
    if (pb->cq[pb->batch] > pb->t_q || pb->ck[pb->batch] > pb->t_k) return ORACLE_ERR_SEQLEN;
    return ORACLE_OK;
}

static void release(oracle_problem *pb) {
    free(pb->cq);
    free(pb->ck);
}

typedef struct {
    const oracle_problem *pb;
    const int64_t *rows; /* token indices to compute, or NULL = all tokens */
    int64_t n_rows;
    int64_t next; /* shared work counter, guarded by lock */
    pthread_mutex_t lock;
    double *out;
    int64_t max_lk;
} oracle_job;

static void *worker(void *arg) {
    oracle_job *job = (oracle_job *)arg;
    const oracle_problem *pb = job->pb;
    double *p = (double *)malloc(sizeof(double) * (size_t)(job->max_lk > 0 ? job->max_lk : 1));
    if (!p) return (void *)1;
    const int64_t n_items = job->n_rows * pb->head_num;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        const int64_t start = job->next;
        job->next += 16;
        pthread_mutex_unlock(&job->lock);
        if (start >= n_items) break;
        const int64_t stop = start + 16 < n_items ? start + 16 : n_items;
        for (int64_t it = start; it < stop; ++it) {
            const int64_t r = it / pb->head_num, h = it % pb->head_num;
            const int64_t t = job->rows ? job->rows[r] : r;
            const int64_t b = seq_of_token(pb, t);
            if (b < 0) continue; /* padding token: attenOut row left untouched */
            row_output(pb, b, t, h, p, job->out);
        }
    }
    free(p);
    return NULL;
}

/*
 * Full or row-sampled prefill.
 *   q      [t_q, head_num, d_nope]     q_rope [t_q, head_num, d_rope]
 *   k      [t_k, kv_head_num, d_nope]  k_rope [t_k, kv_head_num, d_rope]
 *   v      [t_k, kv_head_num, d_v]     out    [t_q, head_num, d_v]
 * all contiguous doubles; q_seqlen / kv_seqlen [batch] int32 on the host.
 * rows: NULL for every token, else n_rows packed token indices; only those
 * rows of out are written.  n_threads <= 0 uses every online core.
 * Returns 0, or a nonzero ORACLE_ERR_* code with out untouched.
 */
int mla_oracle_prefill(const double *q, const double *q_rope, const double *k, const double *k_rope,
                       const double *v, const int32_t *q_seqlen, const int32_t *kv_seqlen, int64_t batch,
                       int64_t t_q, int64_t t_k, int64_t head_num, int64_t kv_head_num, int64_t d_nope,
                       int64_t d_rope, int64_t d_v, int mask_type, float qk_scale, const int64_t *rows,
                       int64_t n_rows, double *out, int n_threads) {
    oracle_problem pb = {q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, batch, t_q, t_k, head_num, kv_head_num,
                         d_nope, d_rope, d_v, mask_type, (double)qk_scale, NULL, NULL};
    int rc = prepare(&pb);
    if (rc != ORACLE_OK) {
        release(&pb);
        return rc;
    }
    if (rows) {
        for (int64_t r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= t_q) {
                release(&pb);
                return ORACLE_ERR_ARGS;
            }
    } else {
        n_rows = t_q;
    }
    oracle_job job;
    job.pb = &pb;
    job.rows = rows;
    job.n_rows = n_rows;
    job.next = 0;
    job.out = out;
    job.max_lk = 0;
    for (int64_t b = 0; b < batch; ++b)
        if (kv_seqlen[b] > job.max_lk) job.max_lk = kv_seqlen[b];
    pthread_mutex_init(&job.lock, NULL);
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    int started = 0;
    if (tid)
        for (; started < n_threads; ++started)
            if (pthread_create(&tid[started], NULL, worker, &job) != 0) break;
    if (started == 0) worker(&job);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    pthread_mutex_destroy(&job.lock);
    release(&pb);
    return ORACLE_OK;
}

/*
 * The attention weights of one query row: p[j] for j < kvSeqLen[b] of the
 * sequence that owns packed token `token`, for query head `head`.
 * p must hold max(kvSeqLen) doubles.  Returns the number of visible keys,
 * or -1 (bad arguments / token past sum(Lq)).
 */
int64_t mla_oracle_row_probs(const double *q, const double *q_rope, const double *k, const double *k_rope,
                             const int32_t *q_seqlen, const int32_t *kv_seqlen, int64_t batch, int64_t t_q,
                             int64_t t_k, int64_t head_num, int64_t kv_head_num, int64_t d_nope, int64_t d_rope,
                             int mask_type, float qk_scale, int64_t token, int64_t head, double *p) {
    oracle_problem pb = {q, q_rope, k, k_rope, NULL, q_seqlen, kv_seqlen, batch, t_q, t_k, head_num, kv_head_num,
                         d_nope, d_rope, 1, mask_type, (double)qk_scale, NULL, NULL};
    if (prepare(&pb) != ORACLE_OK || token < 0 || token >= t_q || head < 0 || head >= head_num) {
        release(&pb);
        return -1;
    }
    const int64_t b = seq_of_token(&pb, token);
    int64_t n = -1;
    if (b >= 0) n = row_probs(&pb, b, token, head, p);
    release(&pb);
    return n;
}
