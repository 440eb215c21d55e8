/*
 * gdn_ref.c -- fp64 CPU oracle for the Gated DeltaNet layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (plain definition, token by token, no chunking):
 *   Gated DeltaNet is the linear-attention layer named in the Qwen3-Next-80B-A3B
 *   model card ("Highlights": Hybrid Attention; "Model Overview": Gated DeltaNet,
 *   32 linear-attention heads for V and 16 for QK, head dimension 128).  Its state
 *   update is the gated delta rule, per sequence and per V head, with the state S a
 *   d_v x d_k matrix:
 *       S_t = alpha_t * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *       o_t = S_t q_t                       (the output reads the updated state)
 *   with alpha_t = exp(g_t), k_t = k/sqrt(|k|^2 + eps), and
 *   q_t = q/sqrt(|q|^2 + eps) / sqrt(d_k).  V head h reads QK head
 *   h / (num_v_heads / num_qk_heads) (contiguous grouping: V heads 2j and 2j+1 share
 *   QK head j in the 16/32 layout).
 *
 *   The product S (I - beta k k^T) is evaluated literally as S - beta (S k) k^T, so
 *   one token costs two matrix-vector products and one rank-1 update.
 *
 * Layouts (all row-major, fp64):
 *   q, k           [total_tokens][num_qk_heads][d_k]
 *   v              [total_tokens][num_v_heads][d_v]
 *   g, beta        [total_tokens][num_v_heads]
 *   initial_state  [num_seqs][num_v_heads][d_v][d_k]   (NULL means zeros)
 *   final_state    [num_seqs][num_v_heads][d_v][d_k]   (NULL means not written)
 *   out            [total_tokens][num_v_heads][d_v]
 *   cu_seqlens     [num_seqs + 1], cu_seqlens[0] = 0, non-decreasing
 *
 * Work is split over (sequence, V head) pairs across num_threads POSIX threads;
 * each pair is an independent recurrence, so the result does not depend on the
 * thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *s0;
    const int32_t *cu;
    int32_t num_seqs, hk, hv, dk, dv;
    double eps;
    double *out, *sT;
    int next_job; /* shared job counter (atomic) */
    int error;
} ref_ctx;

/* One (sequence n, V head h) recurrence. Returns 0 on success, -1 on allocation failure. */
static int run_pair(ref_ctx *c, int n, int h)
{
    const int dk = c->dk, dv = c->dv, hk = c->hk, hv = c->hv;
    const int qk_head = h / (hv / hk);
    double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
    double *kn = (double *)malloc(sizeof(double) * dk);
    double *qn = (double *)malloc(sizeof(double) * dk);
    double *u = (double *)malloc(sizeof(double) * dv);
    if (!S || !kn || !qn || !u) {
        free(S); free(kn); free(qn); free(u);
        return -1;
    }
    if (c->s0) {
        const double *src = c->s0 + ((size_t)n * hv + h) * dv * dk;
        memcpy(S, src, sizeof(double) * dv * dk);
    }
    for (int32_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
        const double *qt = c->q + ((size_t)t * hk + qk_head) * dk;
        const double *kt = c->k + ((size_t)t * hk + qk_head) * dk;
        const double *vt = c->v + ((size_t)t * hv + h) * dv;
        const double alpha = exp(c->g[(size_t)t * hv + h]);
        const double b = c->beta[(size_t)t * hv + h];

        /* L2 normalisation of k and q; q additionally scaled by 1/sqrt(d_k). */
        double ssk = 0.0, ssq = 0.0;
        for (int j = 0; j < dk; ++j) { ssk += kt[j] * kt[j]; ssq += qt[j] * qt[j]; }
        const double rk = 1.0 / sqrt(ssk + c->eps);
        const double rq = 1.0 / sqrt(ssq + c->eps) / sqrt((double)dk);
        for (int j = 0; j < dk; ++j) { kn[j] = kt[j] * rk; qn[j] = qt[j] * rq; }

        /* u = S k */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kn[j];
            u[i] = acc;
        }
        /* S <- alpha * (S - beta u k^T) + beta v k^T */
        for (int i = 0; i < dv; ++i) {
            for (int j = 0; j < dk; ++j) {
                double s = S[(size_t)i * dk + j];
                s = alpha * (s - b * u[i] * kn[j]) + b * vt[i] * kn[j];
                S[(size_t)i * dk + j] = s;
            }
        }
        /* o = S q (post-update state) */
        double *ot = c->out + ((size_t)t * hv + h) * dv;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qn[j];
            ot[i] = acc;
        }
    }
    if (c->sT) {
        double *dst = c->sT + ((size_t)n * hv + h) * dv * dk;
        memcpy(dst, S, sizeof(double) * dv * dk);
    }
    free(S); free(kn); free(qn); free(u);
    return 0;
}

static void *worker(void *arg)
{
    ref_ctx *c = (ref_ctx *)arg;
    const int total = c->num_seqs * c->hv;
    for (;;) {
        int job = __atomic_fetch_add(&c->next_job, 1, __ATOMIC_RELAXED);
        if (job >= total) break;
        if (run_pair(c, job / c->hv, job % c->hv) != 0)
            __atomic_store_n(&c->error, 1, __ATOMIC_RELAXED);
    }
    return NULL;
}

/*
 * Runs the recurrence for every (sequence, V head) pair.
 * Returns 0 on success, 1 on bad arguments, 2 on allocation or thread failure.
 */
int gdn_ref_forward(const double *q, const double *k, const double *v,
                    const double *g, const double *beta,
                    const double *initial_state, const int32_t *cu_seqlens,
                    int32_t num_seqs, int32_t num_qk_heads, int32_t num_v_heads,
                    int32_t d_k, int32_t d_v, double eps,
                    double *out, double *final_state, int32_t num_threads)
{
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !out) return 1;
    if (num_seqs < 0 || num_qk_heads <= 0 || num_v_heads <= 0 || d_k <= 0 || d_v <= 0) return 1;
    if (num_v_heads % num_qk_heads != 0) return 1;
    if (cu_seqlens[0] != 0) return 1;
    for (int n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;

    ref_ctx c;
    c.q = q; c.k = k; c.v = v; c.g = g; c.beta = beta; c.s0 = initial_state;
    c.cu = cu_seqlens; c.num_seqs = num_seqs; c.hk = num_qk_heads; c.hv = num_v_heads;
    c.dk = d_k; c.dv = d_v; c.eps = eps; c.out = out; c.sT = final_state;
    c.next_job = 0; c.error = 0;

    if (num_threads < 1) num_threads = 1;
    if (num_threads > 256) num_threads = 256;
    pthread_t tid[256];
    int started = 0;
    for (int i = 1; i < num_threads; ++i) {
        if (pthread_create(&tid[started], NULL, worker, &c) != 0) break;
        ++started;
    }
    worker(&c);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    return c.error ? 2 : 0;
}
