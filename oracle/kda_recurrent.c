/*
 * KDA oracle, form R: the token-by-token recurrence, in fp64, on the CPU.
 *
 * TEST INFRASTRUCTURE. This file is the definition the CUDA path is checked
 * against. Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load it. It shares no code, header or constant with the CUDA
 * library, and it includes nothing from it.
 *
 * What it follows (page "atlas_core/kimi_k3/kda.rs", module doc and
 * `kda_recurrent_step`; page "K3/kda/ops/api.py", `chunk_kda`):
 *   per sequence n and head h, state S (d_k x d_v, rows = key channels),
 *   S starts at initial_state[n,h] or 0, and for every token t in order:
 *     q^ = q_t / sqrt(sum q_t^2 + 1e-6), k^ likewise      (if use_qk_l2norm)
 *     g  = max(g_t, lower_bound)                          (if a bound is given)
 *     S  = diag(exp(g)) S            decay on the key axis, per channel
 *     d  = sigmoid(beta_t) (v_t - S^T k^)                 read of the decayed S
 *          (beta_t as given when it holds probabilities: api.py's
 *          use_beta_sigmoid_in_kernel = False)
 *     S  = S + k^ d^T                                     rank-1 write
 *     o_t = scale S^T q^                                  read of the updated S
 *   final_state[n,h] = S.
 *
 * Layout: q,k,g are [T_total, H, d_k], v and o are [T_total, H, d_v], beta is
 * [T_total, H] (logits, or probabilities), states are [N, H, d_k, d_v] with element (c, j) of a
 * head at c*d_v + j. Sequence n covers tokens cu_seqlens[n] .. cu_seqlens[n+1].
 * Every pair (n, h) is independent; pairs are spread over POSIX threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int N, H, Dk, Dv;
    const int64_t *cu_seqlens;
    const double *q, *k, *v, *g, *beta;
    double scale;
    const double *S0;
    double *o, *S_out;
    int use_qk_l2norm, has_lb;
    int beta_logit; /* 1: beta holds logits (sigmoid applied); 0: probabilities */
    double lb;
    int next_pair, npairs;
    pthread_mutex_t lock;
    int failed;
} rec_job;

/* x / sqrt(sum x^2 + 1e-6): the eps sits inside the square root
 * ("atlas_core/kimi_k3/kda.rs", `l2norm_rows`, `KDA_L2_EPS`). */
static void rec_l2norm(const double *x, double *y, int d)
{
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss + 1e-6);
    for (int i = 0; i < d; ++i) y[i] = x[i] * inv;
}

static double rec_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static int rec_pair(rec_job *J, int n, int h)
{
    const int H = J->H, Dk = J->Dk, Dv = J->Dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)Dk * Dv);
    double *qh = (double *)malloc(sizeof(double) * Dk);
    double *kh = (double *)malloc(sizeof(double) * Dk);
    double *delta = (double *)malloc(sizeof(double) * Dv);
    if (!S || !qh || !kh || !delta) {
        free(S); free(qh); free(kh); free(delta);
        return -1;
    }
    if (J->S0)
        memcpy(S, J->S0 + ((size_t)n * H + h) * Dk * Dv, sizeof(double) * (size_t)Dk * Dv);
    else
        memset(S, 0, sizeof(double) * (size_t)Dk * Dv);

    for (int64_t t = J->cu_seqlens[n]; t < J->cu_seqlens[n + 1]; ++t) {
        const double *qt = J->q + ((size_t)t * H + h) * Dk;
        const double *kt = J->k + ((size_t)t * H + h) * Dk;
        const double *vt = J->v + ((size_t)t * H + h) * Dv;
        const double *gt = J->g + ((size_t)t * H + h) * Dk;
        double *ot = J->o + ((size_t)t * H + h) * Dv;
        if (J->use_qk_l2norm) {
            rec_l2norm(qt, qh, Dk);
            rec_l2norm(kt, kh, Dk);
        } else {
            memcpy(qh, qt, sizeof(double) * Dk);
            memcpy(kh, kt, sizeof(double) * Dk);
        }
        /* S <- diag(exp(g)) S : row c of S (key channel c) is scaled. */
        for (int c = 0; c < Dk; ++c) {
            double gc = gt[c];
            if (J->has_lb && gc < J->lb) gc = J->lb;
            double a = exp(gc);
            for (int j = 0; j < Dv; ++j) S[(size_t)c * Dv + j] *= a;
        }
        /* delta = sigmoid(beta) (v - S^T k^) */
        double b = J->beta[(size_t)t * H + h];
        if (J->beta_logit) b = rec_sigmoid(b);
        for (int j = 0; j < Dv; ++j) {
            double kv = 0.0;
            for (int c = 0; c < Dk; ++c) kv += S[(size_t)c * Dv + j] * kh[c];
            delta[j] = b * (vt[j] - kv);
        }
        /* S <- S + k^ delta^T */
        for (int c = 0; c < Dk; ++c)
            for (int j = 0; j < Dv; ++j) S[(size_t)c * Dv + j] += kh[c] * delta[j];
        /* o = scale S^T q^ */
        for (int j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < Dk; ++c) acc += S[(size_t)c * Dv + j] * qh[c];
            ot[j] = J->scale * acc;
        }
    }
    if (J->S_out)
        memcpy(J->S_out + ((size_t)n * H + h) * Dk * Dv, S, sizeof(double) * (size_t)Dk * Dv);
    free(S); free(qh); free(kh); free(delta);
    return 0;
}

static void *rec_worker(void *arg)
{
    rec_job *J = (rec_job *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int p = J->next_pair++;
        pthread_mutex_unlock(&J->lock);
        if (p >= J->npairs) break;
        if (rec_pair(J, p / J->H, p % J->H) != 0) {
            pthread_mutex_lock(&J->lock);
            J->failed = 1;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int kda_oracle_recurrent(int N, int H, int Dk, int Dv, const int64_t *cu_seqlens,
                         const double *q, const double *k, const double *v, const double *g,
                         const double *beta, double scale, const double *initial_state,
                         double *o, double *final_state, int use_qk_l2norm, int has_lower_bound,
                         double lower_bound, int beta_is_logit, int nthreads)
{
    if (N < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || !cu_seqlens) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    rec_job J;
    J.N = N; J.H = H; J.Dk = Dk; J.Dv = Dv; J.cu_seqlens = cu_seqlens;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.scale = scale;
    J.beta_logit = beta_is_logit;
    J.S0 = initial_state; J.o = o; J.S_out = final_state;
    J.use_qk_l2norm = use_qk_l2norm; J.has_lb = has_lower_bound; J.lb = lower_bound;
    J.next_pair = 0; J.npairs = N * H; J.failed = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J.npairs) nthreads = J.npairs > 0 ? J.npairs : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    int started = 0;
    if (th) {
        for (int i = 0; i < nthreads; ++i) {
            if (pthread_create(&th[i], NULL, rec_worker, &J) != 0) break;
            ++started;
        }
    }
    if (started == 0) rec_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return J.failed ? -2 : 0;
}
