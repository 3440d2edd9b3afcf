/*
 * Plain FP64 CPU oracle for exact softmax attention (forward and backward).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it computes.  "FlashAttention: Fast and Memory-Efficient Exact
 * Attention with IO-Awareness" (opendecode.dev summary, section "The key
 * idea") and "FlashAttention, Decoded" (abstract gloss, sentence 4) both say
 * the tiled method gives an output identical to standard attention.  The
 * oracle is therefore the plain definition of standard attention, written
 * out one query row at a time:
 *
 *   M(r,c) = (!causal || c <= r) && (kv_len == NULL || c < L_b)
 *            && (block_mask == NULL || block_mask[(r/128)*nt + c/128] != 0)
 *            with L_b = kv_len[b] clamped into [0, N] and nt = ceil(N / 128)
 *            (a last, partial tile holds the rest)
 *   S_rc   = scale * sum_k Q_rk K_ck          if M(r,c), else -inf
 *   m_r    = max_c S_rc,  l_r = sum_c exp(S_rc - m_r)
 *   P_rc   = exp(S_rc - m_r) / l_r,  LSE_r = m_r + ln l_r  (natural log)
 *   O_r    = sum_c P_rc V_c
 *
 * The backward pass is the chain rule on L = sum(O * dO):
 *   dV_c = sum_r P_rc dO_r,  dP_rc = dO_r . V_c,  D_r = sum_c P_rc dP_rc,
 *   dS_rc = P_rc (dP_rc - D_r),  dQ_r = scale sum_c dS_rc K_c,
 *   dK_c = scale sum_r dS_rc Q_r.
 *
 * A row with no allowed key has O_r = 0, LSE_r = -inf and zero gradients.
 * There is no tiling, no online softmax and no reordering: one full score
 * row is formed, then normalised.  Work is split over (b, h) heads with
 * POSIX threads; each head is computed by exactly one thread, so the result
 * does not depend on the thread count.
 *
 * Layout: every tensor is contiguous [B][H][N][d] (row-major), LSE and D
 * are [B][H][N].
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_MASK_TILE 128

typedef struct {
    const double *q, *k, *v, *dout;
    double *o, *lse, *dq, *dk, *dv, *delta;
    int B, H, N, d;
    double scale;
    int causal;
    const uint8_t *block_mask;
    const int32_t *kv_len;
    int backward;
    int dropout;            /* keep mask Z and scale below apply (see dropout_keep) */
    uint32_t drop_t;        /* drop when the element's 16-bit draw is below drop_t */
    double drop_scale;      /* 65536 / (65536 - drop_t) */
    uint32_t seed_lo, seed_hi, offset;
    int r_begin, r_end;     /* query rows computed in every head */
    int next_head;          /* shared work counter, guarded by lock */
    pthread_mutex_t lock;
} oracle_job;

/*
 * Philox-4x32-10, the counter-based generator of Salmon, Moraes, Dror and
 * Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC 2011): ten rounds,
 * each multiplying counter words 0 and 2 by the two round constants into
 * 64-bit products and mixing their halves with words 1 and 3 and the key,
 * the key being advanced by the two Weyl constants between rounds.
 */
static void philox4x32_10(const uint32_t ctr_in[4], uint32_t k0, uint32_t k1, uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        const uint32_t n0 = hi1 ^ c1 ^ k0;
        const uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/*
 * Dropout draw for element (head bh, query r, key c): Philox-4x32-10 with
 * counter (c / 8, r, bh, offset) and key (seed_lo, seed_hi) gives eight
 * 16-bit values, for keys 8*(c/8) .. 8*(c/8)+7 in order (value k is the low
 * half of word k/2 for even k, the high half for odd k).  The element is kept
 * when its value is at least drop_t = floor(p * 65536).
 */
static uint32_t dropout_u16(int bh, int r, int c, uint32_t seed_lo, uint32_t seed_hi,
                            uint32_t offset)
{
    const uint32_t ctr[4] = {(uint32_t)c >> 3, (uint32_t)r, (uint32_t)bh, offset};
    uint32_t w[4];
    philox4x32_10(ctr, seed_lo, seed_hi, w);
    const int kk = c & 7;
    return (w[kk >> 1] >> (16 * (kk & 1))) & 0xFFFFu;
}

/* Z_rc * scale for the job's dropout (1 without dropout). */
static double dropout_weight(const oracle_job *job, int bh, int r, int c)
{
    if (!job->dropout) return 1.0;
    const uint32_t u = dropout_u16(bh, r, c, job->seed_lo, job->seed_hi, job->offset);
    return u >= job->drop_t ? job->drop_scale : 0.0;
}

/*
 * Key limit L_b of the mask: keys c >= L_b are padding.  Without key lengths
 * every key is allowed (L_b = N); a given length is taken clamped into
 * [0, N], so a negative one allows no key and one above N allows them all
 * (the contract of the library's kv_len argument).
 */
static int key_limit(int has_kv_len, int kv_len_b, int N)
{
    if (!has_kv_len) return N;
    return kv_len_b < 0 ? 0 : (kv_len_b > N ? N : kv_len_b);
}

/* The mask M(r,c) exactly as defined above, with L = key_limit(...). */
static int allowed(int r, int c, int N, int causal, const uint8_t *block_mask, int L)
{
    if (causal && c > r) return 0;
    if (c >= L) return 0;
    if (block_mask) {
        /* nt = ceil(N / 128): a last, partial tile holds the remaining positions */
        int nt = (N + ORACLE_MASK_TILE - 1) / ORACLE_MASK_TILE;
        if (!block_mask[(size_t)(r / ORACLE_MASK_TILE) * nt + (c / ORACLE_MASK_TILE)]) return 0;
    }
    return 1;
}

/*
 * One softmax row.  Fills p[0..N) with P_rc (0 where masked) and returns the
 * row's m and l through the pointers.  Returns the number of allowed keys.
 */
static int softmax_row(const double *qr, int r, const double *K, int N, int d, double scale,
                       int causal, const uint8_t *block_mask, int L, double *p,
                       double *m_out, double *l_out)
{
    int count = 0;
    double m = -INFINITY;
    for (int c = 0; c < N; ++c) {
        if (!allowed(r, c, N, causal, block_mask, L)) {
            p[c] = -INFINITY;
            continue;
        }
        const double *kc = K + (size_t)c * d;
        double s = 0.0;
        for (int x = 0; x < d; ++x) s += qr[x] * kc[x];
        s *= scale;
        p[c] = s;
        if (s > m) m = s;
        ++count;
    }
    double l = 0.0;
    for (int c = 0; c < N; ++c) {
        if (p[c] == -INFINITY) { p[c] = 0.0; continue; }
        p[c] = exp(p[c] - m);
        l += p[c];
    }
    if (count > 0)
        for (int c = 0; c < N; ++c) p[c] /= l;
    *m_out = m;
    *l_out = l;
    return count;
}

static void forward_head(const oracle_job *job, int bh, double *p)
{
    const int N = job->N, d = job->d;
    const int b = bh / job->H;
    const size_t off = (size_t)bh * N * d;
    const double *Q = job->q + off, *K = job->k + off, *V = job->v + off;
    double *O = job->o + off;
    double *lse = job->lse + (size_t)bh * N;
    const int L = key_limit(job->kv_len != NULL, job->kv_len ? job->kv_len[b] : 0, N);
    for (int r = job->r_begin; r < job->r_end; ++r) {
        double m, l;
        int count = softmax_row(Q + (size_t)r * d, r, K, N, d, job->scale, job->causal,
                                job->block_mask, L, p, &m, &l);
        double *orow = O + (size_t)r * d;
        for (int x = 0; x < d; ++x) orow[x] = 0.0;
        if (count == 0) {
            lse[r] = -INFINITY;
            continue;
        }
        for (int c = 0; c < N; ++c) {
            if (p[c] == 0.0) continue;
            const double *vc = V + (size_t)c * d;
            const double pw = p[c] * dropout_weight(job, bh, r, c);
            for (int x = 0; x < d; ++x) orow[x] += pw * vc[x];
        }
        lse[r] = m + log(l);
    }
}

static void backward_head(const oracle_job *job, int bh, double *p, double *dp)
{
    const int N = job->N, d = job->d;
    const int b = bh / job->H;
    const size_t off = (size_t)bh * N * d;
    const double *Q = job->q + off, *K = job->k + off, *V = job->v + off, *dO = job->dout + off;
    double *dQ = job->dq + off, *dK = job->dk + off, *dV = job->dv + off;
    const int L = key_limit(job->kv_len != NULL, job->kv_len ? job->kv_len[b] : 0, N);
    memset(dK, 0, sizeof(double) * (size_t)N * d);
    memset(dV, 0, sizeof(double) * (size_t)N * d);
    for (int r = job->r_begin; r < job->r_end; ++r) {
        const double *qr = Q + (size_t)r * d;
        const double *dor = dO + (size_t)r * d;
        double *dqr = dQ + (size_t)r * d;
        double m, l;
        int count = softmax_row(qr, r, K, N, d, job->scale, job->causal, job->block_mask, L, p,
                                &m, &l);
        for (int x = 0; x < d; ++x) dqr[x] = 0.0;
        if (count == 0) {
            if (job->delta) job->delta[(size_t)bh * N + r] = 0.0;
            continue;
        }
        /* With dropout O_r = sum_c P_rc W_rc V_c, W = Z * scale: by the chain rule
           the gradient reaching P_rc is W_rc dP_rc with dP_rc = dO_r . V_c, and
           D_r = sum_c P_rc W_rc dP_rc (= dO_r . O_r); without dropout W = 1. */
        double D = 0.0;
        for (int c = 0; c < N; ++c) {
            if (p[c] == 0.0) { dp[c] = 0.0; continue; }
            const double *vc = V + (size_t)c * d;
            double s = 0.0;
            for (int x = 0; x < d; ++x) s += dor[x] * vc[x];
            dp[c] = s * dropout_weight(job, bh, r, c);
            D += p[c] * dp[c];
        }
        if (job->delta) job->delta[(size_t)bh * N + r] = D;
        for (int c = 0; c < N; ++c) {
            if (p[c] == 0.0) continue;
            const double ds = p[c] * (dp[c] - D);
            const double pw = p[c] * dropout_weight(job, bh, r, c);
            const double *kc = K + (size_t)c * d;
            double *dkc = dK + (size_t)c * d;
            double *dvc = dV + (size_t)c * d;
            for (int x = 0; x < d; ++x) {
                dqr[x] += job->scale * ds * kc[x];
                dkc[x] += job->scale * ds * qr[x];
                dvc[x] += pw * dor[x];
            }
        }
    }
}

static void *worker(void *arg)
{
    oracle_job *job = (oracle_job *)arg;
    double *p = (double *)malloc(sizeof(double) * (size_t)job->N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)job->N);
    if (!p || !dp) {
        free(p);
        free(dp);
        return (void *)1;
    }
    for (;;) {
        pthread_mutex_lock(&job->lock);
        int bh = job->next_head++;
        pthread_mutex_unlock(&job->lock);
        if (bh >= job->B * job->H) break;
        if (job->backward)
            backward_head(job, bh, p, dp);
        else
            forward_head(job, bh, p);
    }
    free(p);
    free(dp);
    return NULL;
}

static int run_job(oracle_job *job, int nthreads)
{
    if (job->B <= 0 || job->H <= 0 || job->N <= 0 || job->d <= 0) return -3;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > job->B * job->H) nthreads = job->B * job->H;
    pthread_mutex_init(&job->lock, NULL);
    job->next_head = 0;
    pthread_t *tids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int rc = 0, started = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&tids[t], NULL, worker, job) != 0) { rc = -6; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) {
        void *ret = NULL;
        pthread_join(tids[t], &ret);
        if (ret) rc = -6;
    }
    free(tids);
    pthread_mutex_destroy(&job->lock);
    return rc;
}

/*
 * Forward (or backward) for query rows [r_begin, r_end) of every head.  The
 * backward's dK and dV then hold the contributions of those rows only, and
 * dQ, O and LSE rows outside the band are left untouched.  The *_band forms
 * exist to time bounded samples of a large workload; the plain forms are the
 * band [0, N).
 */
int oracle_attention_forward_band(const double *q, const double *k, const double *v, double *o,
                                  double *lse, int B, int H, int N, int d, double scale,
                                  int causal, const uint8_t *block_mask, const int32_t *kv_len,
                                  int r_begin, int r_end, int nthreads)
{
    if (r_begin < 0 || r_end > N || r_begin > r_end) return -3;
    oracle_job job;
    memset(&job, 0, sizeof(job));
    job.q = q; job.k = k; job.v = v; job.o = o; job.lse = lse;
    job.B = B; job.H = H; job.N = N; job.d = d; job.scale = scale; job.causal = causal;
    job.block_mask = block_mask; job.kv_len = kv_len; job.backward = 0;
    job.r_begin = r_begin; job.r_end = r_end;
    return run_job(&job, nthreads);
}

int oracle_attention_backward_band(const double *q, const double *k, const double *v,
                                   const double *dout, double *dq, double *dk, double *dv,
                                   double *delta, int B, int H, int N, int d, double scale,
                                   int causal, const uint8_t *block_mask, const int32_t *kv_len,
                                   int r_begin, int r_end, int nthreads)
{
    if (r_begin < 0 || r_end > N || r_begin > r_end) return -3;
    oracle_job job;
    memset(&job, 0, sizeof(job));
    job.q = q; job.k = k; job.v = v; job.dout = dout;
    job.dq = dq; job.dk = dk; job.dv = dv; job.delta = delta;
    job.B = B; job.H = H; job.N = N; job.d = d; job.scale = scale; job.causal = causal;
    job.block_mask = block_mask; job.kv_len = kv_len; job.backward = 1;
    job.r_begin = r_begin; job.r_end = r_end;
    return run_job(&job, nthreads);
}

int oracle_attention_forward(const double *q, const double *k, const double *v, double *o,
                             double *lse, int B, int H, int N, int d, double scale, int causal,
                             const uint8_t *block_mask, const int32_t *kv_len, int nthreads)
{
    return oracle_attention_forward_band(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask,
                                         kv_len, 0, N, nthreads);
}

int oracle_attention_backward(const double *q, const double *k, const double *v,
                              const double *dout, double *dq, double *dk, double *dv,
                              double *delta, int B, int H, int N, int d, double scale, int causal,
                              const uint8_t *block_mask, const int32_t *kv_len, int nthreads)
{
    return oracle_attention_backward_band(q, k, v, dout, dq, dk, dv, delta, B, H, N, d, scale,
                                          causal, block_mask, kv_len, 0, N, nthreads);
}

/*
 * Dropout (applied to P before P V, as the pages' fused operation lists
 * dropout among the steps standard attention runs separately: [HF] "Standard
 * Attention Algorithm"): the threshold is drop_t = floor(p_drop * 65536) taken
 * in single precision (p_drop * 65536 is exact there), an element is kept when
 * its 16-bit draw (dropout_u16) is >= drop_t, and kept entries are scaled by
 * 65536 / (65536 - drop_t), which makes the expectation of P Z exactly P.
 * LSE is the softmax's, unaffected by dropout.
 */
static int set_dropout(oracle_job *job, float p_drop, uint64_t seed, uint32_t offset)
{
    if (!(p_drop >= 0.0f && p_drop < 1.0f)) return -8;
    job->dropout = 1;
    job->drop_t = (uint32_t)(p_drop * 65536.0f);
    job->drop_scale = 65536.0 / (65536.0 - (double)job->drop_t);
    job->seed_lo = (uint32_t)seed;
    job->seed_hi = (uint32_t)(seed >> 32);
    job->offset = offset;
    return 0;
}

int oracle_attention_forward_dropout(const double *q, const double *k, const double *v,
                                     double *o, double *lse, int B, int H, int N, int d,
                                     double scale, int causal, const uint8_t *block_mask,
                                     const int32_t *kv_len, float p_drop, uint64_t seed,
                                     uint32_t offset, int nthreads)
{
    oracle_job job;
    memset(&job, 0, sizeof(job));
    job.q = q; job.k = k; job.v = v; job.o = o; job.lse = lse;
    job.B = B; job.H = H; job.N = N; job.d = d; job.scale = scale; job.causal = causal;
    job.block_mask = block_mask; job.kv_len = kv_len; job.backward = 0;
    job.r_begin = 0; job.r_end = N;
    int rc = set_dropout(&job, p_drop, seed, offset);
    return rc ? rc : run_job(&job, nthreads);
}

int oracle_attention_backward_dropout(const double *q, const double *k, const double *v,
                                      const double *dout, double *dq, double *dk, double *dv,
                                      double *delta, int B, int H, int N, int d, double scale,
                                      int causal, const uint8_t *block_mask,
                                      const int32_t *kv_len, float p_drop, uint64_t seed,
                                      uint32_t offset, int nthreads)
{
    oracle_job job;
    memset(&job, 0, sizeof(job));
    job.q = q; job.k = k; job.v = v; job.dout = dout;
    job.dq = dq; job.dk = dk; job.dv = dv; job.delta = delta;
    job.B = B; job.H = H; job.N = N; job.d = d; job.scale = scale; job.causal = causal;
    job.block_mask = block_mask; job.kv_len = kv_len; job.backward = 1;
    job.r_begin = 0; job.r_end = N;
    int rc = set_dropout(&job, p_drop, seed, offset);
    return rc ? rc : run_job(&job, nthreads);
}

/* The dropout keep mask Z as uint8 [BH][N][N] (1 = kept), and raw 16-bit draws
   as uint16 [BH][N][N] when draws is not NULL. */
int oracle_dropout_keep(uint8_t *keep, uint16_t *draws, int BH, int N, float p_drop,
                        uint64_t seed, uint32_t offset)
{
    oracle_job job;
    memset(&job, 0, sizeof(job));
    if (set_dropout(&job, p_drop, seed, offset)) return -8;
    for (int bh = 0; bh < BH; ++bh)
        for (int r = 0; r < N; ++r)
            for (int c = 0; c < N; ++c) {
                const uint32_t u = dropout_u16(bh, r, c, job.seed_lo, job.seed_hi, offset);
                const size_t i = ((size_t)bh * N + r) * N + c;
                keep[i] = (uint8_t)(u >= job.drop_t);
                if (draws) draws[i] = (uint16_t)u;
            }
    return 0;
}

/* Philox-4x32-10 itself, for the tests: out = philox(counter, key). */
void oracle_philox4x32_10(const uint32_t counter[4], uint32_t k0, uint32_t k1, uint32_t out[4])
{
    philox4x32_10(counter, k0, k1, out);
}

/*
 * Forward for a chosen subset of query rows of ONE head.  q_rows is
 * [R][d] (row i holds query number rows[i]); K and V are the head's full
 * [N][d]; has_kv_len = 0 means no key padding, else keys c >= kv_len_b
 * (clamped into [0, N], see key_limit) are padding.  Used to check sampled rows at
 * sizes where the whole head is too slow on the CPU; each row is the same
 * computation as in oracle_attention_forward.
 */
int oracle_attention_forward_rows(const double *q_rows, const int64_t *rows, int R,
                                  const double *k, const double *v, double *o_rows,
                                  double *lse_rows, int N, int d, double scale, int causal,
                                  const uint8_t *block_mask, int has_kv_len, int kv_len_b)
{
    if (R < 0 || N <= 0 || d <= 0) return -3;
    const int L = key_limit(has_kv_len, kv_len_b, N);
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    if (!p) return -6;
    for (int i = 0; i < R; ++i) {
        const int r = (int)rows[i];
        double m, l;
        int count = softmax_row(q_rows + (size_t)i * d, r, k, N, d, scale, causal, block_mask,
                                L, p, &m, &l);
        double *orow = o_rows + (size_t)i * d;
        for (int x = 0; x < d; ++x) orow[x] = 0.0;
        if (count == 0) { lse_rows[i] = -INFINITY; continue; }
        for (int c = 0; c < N; ++c) {
            if (p[c] == 0.0) continue;
            const double *vc = v + (size_t)c * d;
            for (int x = 0; x < d; ++x) orow[x] += p[c] * vc[x];
        }
        lse_rows[i] = m + log(l);
    }
    free(p);
    return 0;
}

/*
 * Backward quantities that depend on one query row only, for a chosen subset
 * of rows of ONE head: dQ_r = scale sum_c dS_rc K_c and D_r = sum_c P_rc dP_rc
 * (same computation as in oracle_attention_backward, row by row).  q_rows and
 * dout_rows are [R][d]; K and V are the head's [N][d].
 */
int oracle_attention_backward_dq_rows(const double *q_rows, const double *dout_rows,
                                      const int64_t *rows, int R, const double *k,
                                      const double *v, double *dq_rows, double *delta_rows,
                                      int N, int d, double scale, int causal,
                                      const uint8_t *block_mask, int has_kv_len, int kv_len_b)
{
    if (R < 0 || N <= 0 || d <= 0) return -3;
    const int L = key_limit(has_kv_len, kv_len_b, N);
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    if (!p || !dp) { free(p); free(dp); return -6; }
    for (int i = 0; i < R; ++i) {
        const int r = (int)rows[i];
        const double *qr = q_rows + (size_t)i * d;
        const double *dor = dout_rows + (size_t)i * d;
        double *dqr = dq_rows + (size_t)i * d;
        double m, l;
        int count = softmax_row(qr, r, k, N, d, scale, causal, block_mask, L, p, &m, &l);
        for (int x = 0; x < d; ++x) dqr[x] = 0.0;
        delta_rows[i] = 0.0;
        if (count == 0) continue;
        double D = 0.0;
        for (int c = 0; c < N; ++c) {
            if (p[c] == 0.0) { dp[c] = 0.0; continue; }
            const double *vc = v + (size_t)c * d;
            double s = 0.0;
            for (int x = 0; x < d; ++x) s += dor[x] * vc[x];
            dp[c] = s;
            D += p[c] * s;
        }
        delta_rows[i] = D;
        for (int c = 0; c < N; ++c) {
            if (p[c] == 0.0) continue;
            const double ds = p[c] * (dp[c] - D);
            const double *kc = k + (size_t)c * d;
            for (int x = 0; x < d; ++x) dqr[x] += scale * ds * kc[x];
        }
    }
    free(p);
    free(dp);
    return 0;
}

/*
 * dK and dV for a chosen subset of key columns of ONE head:
 *   dV_c = sum_r P_rc dO_r,  dK_c = scale sum_r P_rc (dP_rc - D_r) Q_r
 * for c in cols[0..C).  Every row r still needs its full softmax row and D_r,
 * so this costs a full pass over the head; rows are split into fixed chunks
 * of 256 handled by worker threads, and the per-chunk partial sums are added
 * in chunk order, so the result does not depend on the thread count.
 * q, k, v, dout are the head's [N][d]; dk_cols, dv_cols are [C][d].
 */
typedef struct {
    const double *q, *k, *v, *dout;
    const int64_t *cols;
    int C, N, d;
    double scale;
    int causal;
    const uint8_t *block_mask;
    int L;
    double *partial; /* [nchunks][2][C][d] */
    int nchunks;
    int next_chunk;
    pthread_mutex_t lock;
} kvcols_job;

#define KVCOLS_CHUNK 256

static void *kvcols_worker(void *arg)
{
    kvcols_job *job = (kvcols_job *)arg;
    const int N = job->N, d = job->d, C = job->C;
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    if (!p || !dp) { free(p); free(dp); return (void *)1; }
    for (;;) {
        pthread_mutex_lock(&job->lock);
        int ch = job->next_chunk++;
        pthread_mutex_unlock(&job->lock);
        if (ch >= job->nchunks) break;
        double *dk = job->partial + (size_t)ch * 2 * C * d;
        double *dv = dk + (size_t)C * d;
        memset(dk, 0, sizeof(double) * 2 * (size_t)C * d);
        const int r_end = (ch + 1) * KVCOLS_CHUNK < N ? (ch + 1) * KVCOLS_CHUNK : N;
        for (int r = ch * KVCOLS_CHUNK; r < r_end; ++r) {
            const double *qr = job->q + (size_t)r * d;
            const double *dor = job->dout + (size_t)r * d;
            double m, l;
            int count = softmax_row(qr, r, job->k, N, d, job->scale, job->causal,
                                    job->block_mask, job->L, p, &m, &l);
            if (count == 0) continue;
            double D = 0.0;
            for (int c = 0; c < N; ++c) {
                if (p[c] == 0.0) { dp[c] = 0.0; continue; }
                const double *vc = job->v + (size_t)c * d;
                double s = 0.0;
                for (int x = 0; x < d; ++x) s += dor[x] * vc[x];
                dp[c] = s;
                D += p[c] * s;
            }
            for (int i = 0; i < C; ++i) {
                const int c = (int)job->cols[i];
                if (p[c] == 0.0) continue;
                const double ds = p[c] * (dp[c] - D);
                for (int x = 0; x < d; ++x) {
                    dk[(size_t)i * d + x] += job->scale * ds * qr[x];
                    dv[(size_t)i * d + x] += p[c] * dor[x];
                }
            }
        }
    }
    free(p);
    free(dp);
    return NULL;
}

int oracle_attention_backward_kv_cols(const double *q, const double *k, const double *v,
                                      const double *dout, const int64_t *cols, int C,
                                      double *dk_cols, double *dv_cols, int N, int d,
                                      double scale, int causal, const uint8_t *block_mask,
                                      int has_kv_len, int kv_len_b, int nthreads)
{
    if (C < 0 || N <= 0 || d <= 0) return -3;
    for (int i = 0; i < C; ++i)
        if (cols[i] < 0 || cols[i] >= N) return -3;
    kvcols_job job;
    memset(&job, 0, sizeof(job));
    job.q = q; job.k = k; job.v = v; job.dout = dout; job.cols = cols; job.C = C;
    job.N = N; job.d = d; job.scale = scale; job.causal = causal;
    job.block_mask = block_mask; job.L = key_limit(has_kv_len, kv_len_b, N);
    job.nchunks = (N + KVCOLS_CHUNK - 1) / KVCOLS_CHUNK;
    job.partial = (double *)malloc(sizeof(double) * (size_t)job.nchunks * 2 * C * d + 1);
    if (!job.partial) return -6;
    pthread_mutex_init(&job.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > job.nchunks) nthreads = job.nchunks;
    pthread_t *tids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int rc = 0, started = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&tids[t], NULL, kvcols_worker, &job) != 0) { rc = -6; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) {
        void *ret = NULL;
        pthread_join(tids[t], &ret);
        if (ret) rc = -6;
    }
    free(tids);
    pthread_mutex_destroy(&job.lock);
    if (rc == 0) {
        memset(dk_cols, 0, sizeof(double) * (size_t)C * d);
        memset(dv_cols, 0, sizeof(double) * (size_t)C * d);
        for (int ch = 0; ch < job.nchunks; ++ch) {
            const double *pk = job.partial + (size_t)ch * 2 * C * d;
            const double *pv = pk + (size_t)C * d;
            for (size_t e = 0; e < (size_t)C * d; ++e) {
                dk_cols[e] += pk[e];
                dv_cols[e] += pv[e];
            }
        }
    }
    free(job.partial);
    return rc;
}

/*
 * Which (query tile, key tile) pairs hold at least one allowed (r, c).
 * visits is [B][i_end - i_begin][n_t] with n_t = ceil(N / T) (a last, partial
 * tile holds the remaining positions): the entry for query tile i
 * (i_begin <= i < i_end) and key tile j is 1 when some r < N in tile i and
 * some c < N in tile j have M(r,c), else 0.  Brute force over the entries of each
 * tile pair (stopping at the first allowed one), straight from the
 * definition of M; heads share the mask, so only b matters.
 */
int oracle_tile_visits(uint8_t *visits, int B, int N, int T, int causal,
                       const uint8_t *block_mask, const int32_t *kv_len, int i_begin, int i_end)
{
    if (T <= 0 || N <= 0) return -3;
    const int nt = (N + T - 1) / T;
    if (i_begin < 0 || i_end > nt || i_begin > i_end) return -3;
    const int ni = i_end - i_begin;
    for (int b = 0; b < B; ++b) {
        const int L = key_limit(kv_len != NULL, kv_len ? kv_len[b] : 0, N);
        for (int i = i_begin; i < i_end; ++i)
            for (int j = 0; j < nt; ++j) {
                int any = 0;
                for (int r = i * T; r < (i + 1) * T && r < N && !any; ++r)
                    for (int c = j * T; c < (j + 1) * T && c < N; ++c)
                        if (allowed(r, c, N, causal, block_mask, L)) { any = 1; break; }
                visits[((size_t)b * ni + (i - i_begin)) * nt + j] = (uint8_t)any;
            }
    }
    return 0;
}
