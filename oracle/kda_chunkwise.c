/*
 * KDA oracle, form C: the chunkwise (WY / UT) form, in fp64, on the CPU.
 *
 * TEST INFRASTRUCTURE. It exists to cross-check form R (kda_recurrent.c) with
 * an independently written second route to the same numbers, and it shares no
 * code with form R or with the CUDA library. Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg may load it.
 *
 * What it computes: the same result as the recurrence of page
 * "atlas_core/kimi_k3/kda.rs" (module doc, `kda_recurrent_step`), reached one
 * chunk of L <= C tokens at a time, as the `chunk_kda` boundary of page
 * "K3/kda/ops/api.py" does with its chunk_size. The chunk algebra is derived
 * here from that recurrence (the pages print the boundary, not the body):
 *
 *   inside a chunk, with S the state entering it and rows r, s of the chunk,
 *   G_r = sum_{u<=r} g_u (per key channel, inclusive),
 *   A_kk[r,s] = sum_c k^_r[c] k^_s[c] exp(G_r[c]-G_s[c])   (s < r)
 *   A_qk[r,s] = sum_c q^_r[c] k^_s[c] exp(G_r[c]-G_s[c])   (s <= r)
 *   T = (I + diag(beta) A_kk)^-1   by forward substitution
 *   W = T diag(beta) (k^ . exp(G)),   U = T diag(beta) V
 *   Delta = U - W S
 *   O = scale ((q^ . exp(G)) S + A_qk Delta)
 *   S <- diag(exp(G_last)) S + (k^ . exp(G_last - G))^T Delta
 *
 * Only differences of G that are <= 0 are exponentiated, so no factor exceeds
 * 1 for g <= 0. Gates must be finite here (form R also handles g = -inf).
 * Layout and threading as in form R.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int N, H, Dk, Dv, C;
    const int64_t *cu;
    const double *q, *k, *v, *g, *beta;
    double scale;
    const double *S0;
    double *o, *S_out;
    int l2, has_lb;
    double lb;
    int beta_logit; /* 1: beta holds logits (sigmoid applied); 0: probabilities */
    int next, npairs, failed;
    pthread_mutex_t mu;
} chk_job;

typedef struct {
    double *S, *qh, *kh, *vv, *G, *b, *Akk, *Aqk, *T, *W, *U, *D, *tmp;
} chk_buf;

static void chk_free(chk_buf *B)
{
    free(B->S); free(B->qh); free(B->kh); free(B->vv); free(B->G); free(B->b);
    free(B->Akk); free(B->Aqk); free(B->T); free(B->W); free(B->U); free(B->D); free(B->tmp);
}

static int chk_alloc(chk_buf *B, int C, int Dk, int Dv)
{
    memset(B, 0, sizeof(*B));
    size_t cc = (size_t)C * C, ck = (size_t)C * Dk, cv = (size_t)C * Dv;
    B->S = malloc(sizeof(double) * (size_t)Dk * Dv);
    B->qh = malloc(sizeof(double) * ck);
    B->kh = malloc(sizeof(double) * ck);
    B->vv = malloc(sizeof(double) * cv);
    B->G = malloc(sizeof(double) * ck);
    B->b = malloc(sizeof(double) * C);
    B->Akk = malloc(sizeof(double) * cc);
    B->Aqk = malloc(sizeof(double) * cc);
    B->T = malloc(sizeof(double) * cc);
    B->W = malloc(sizeof(double) * ck);
    B->U = malloc(sizeof(double) * cv);
    B->D = malloc(sizeof(double) * cv);
    B->tmp = malloc(sizeof(double) * (size_t)(Dk > Dv ? Dk : Dv) * Dv);
    if (!B->S || !B->qh || !B->kh || !B->vv || !B->G || !B->b || !B->Akk || !B->Aqk ||
        !B->T || !B->W || !B->U || !B->D || !B->tmp) {
        chk_free(B);
        return -1;
    }
    return 0;
}

/* One chunk of L tokens starting at token t0; S (Dk x Dv) is updated. */
static void chk_chunk(chk_job *J, chk_buf *B, int h, int64_t t0, int L)
{
    const int H = J->H, Dk = J->Dk, Dv = J->Dv;
    /* gather the chunk: normalised q, k; v; sigmoid(beta); inclusive cumsum G */
    for (int r = 0; r < L; ++r) {
        size_t row = (size_t)(t0 + r) * H + h;
        const double *qs = J->q + row * Dk, *ks = J->k + row * Dk, *gs = J->g + row * Dk;
        double nq = 1.0, nk = 1.0;
        if (J->l2) {
            double sq = 0.0, sk = 0.0;
            for (int c = 0; c < Dk; ++c) { sq += qs[c] * qs[c]; sk += ks[c] * ks[c]; }
            nq = 1.0 / sqrt(sq + 1e-6);
            nk = 1.0 / sqrt(sk + 1e-6);
        }
        for (int c = 0; c < Dk; ++c) {
            B->qh[(size_t)r * Dk + c] = qs[c] * nq;
            B->kh[(size_t)r * Dk + c] = ks[c] * nk;
            double gc = gs[c];
            if (J->has_lb && gc < J->lb) gc = J->lb;
            B->G[(size_t)r * Dk + c] = (r ? B->G[(size_t)(r - 1) * Dk + c] : 0.0) + gc;
        }
        memcpy(B->vv + (size_t)r * Dv, J->v + row * Dv, sizeof(double) * Dv);
        B->b[r] = J->beta_logit ? 1.0 / (1.0 + exp(-J->beta[row])) : J->beta[row];
    }
    /* gated key-key and query-key blocks, lower triangle only */
    for (int r = 0; r < L; ++r)
        for (int s = 0; s < L; ++s) {
            double akk = 0.0, aqk = 0.0;
            if (s <= r) {
                for (int c = 0; c < Dk; ++c) {
                    double e = exp(B->G[(size_t)r * Dk + c] - B->G[(size_t)s * Dk + c]);
                    akk += B->kh[(size_t)r * Dk + c] * B->kh[(size_t)s * Dk + c] * e;
                    aqk += B->qh[(size_t)r * Dk + c] * B->kh[(size_t)s * Dk + c] * e;
                }
            }
            B->Akk[(size_t)r * L + s] = (s < r) ? akk : 0.0;
            B->Aqk[(size_t)r * L + s] = (s <= r) ? aqk : 0.0;
        }
    /* T = (I + diag(b) Akk)^-1, unit lower triangular, column by column:
     * T[j][j] = 1, T[r][j] = -sum_{j<=s<r} b_r Akk[r][s] T[s][j]. */
    for (int j = 0; j < L; ++j) {
        for (int r = 0; r < L; ++r) B->T[(size_t)r * L + j] = 0.0;
        B->T[(size_t)j * L + j] = 1.0;
        for (int r = j + 1; r < L; ++r) {
            double acc = 0.0;
            for (int s = j; s < r; ++s) acc += B->Akk[(size_t)r * L + s] * B->T[(size_t)s * L + j];
            B->T[(size_t)r * L + j] = -B->b[r] * acc;
        }
    }
    /* W = T diag(b) (k^ . exp(G)),  U = T diag(b) V */
    for (int r = 0; r < L; ++r) {
        for (int c = 0; c < Dk; ++c) {
            double acc = 0.0;
            for (int s = 0; s <= r; ++s)
                acc += B->T[(size_t)r * L + s] * B->b[s] * B->kh[(size_t)s * Dk + c] *
                       exp(B->G[(size_t)s * Dk + c]);
            B->W[(size_t)r * Dk + c] = acc;
        }
        for (int j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int s = 0; s <= r; ++s)
                acc += B->T[(size_t)r * L + s] * B->b[s] * B->vv[(size_t)s * Dv + j];
            B->U[(size_t)r * Dv + j] = acc;
        }
    }
    /* Delta = U - W S */
    for (int r = 0; r < L; ++r)
        for (int j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < Dk; ++c) acc += B->W[(size_t)r * Dk + c] * B->S[(size_t)c * Dv + j];
            B->D[(size_t)r * Dv + j] = B->U[(size_t)r * Dv + j] - acc;
        }
    /* O = scale ((q^ . exp(G)) S + Aqk Delta) */
    for (int r = 0; r < L; ++r) {
        double *orow = J->o + ((size_t)(t0 + r) * H + h) * Dv;
        for (int j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < Dk; ++c)
                acc += B->qh[(size_t)r * Dk + c] * exp(B->G[(size_t)r * Dk + c]) *
                       B->S[(size_t)c * Dv + j];
            for (int s = 0; s <= r; ++s) acc += B->Aqk[(size_t)r * L + s] * B->D[(size_t)s * Dv + j];
            orow[j] = J->scale * acc;
        }
    }
    /* S <- diag(exp(G_last)) S + (k^ . exp(G_last - G))^T Delta */
    const double *Gl = B->G + (size_t)(L - 1) * Dk;
    for (int c = 0; c < Dk; ++c)
        for (int j = 0; j < Dv; ++j) {
            double acc = exp(Gl[c]) * B->S[(size_t)c * Dv + j];
            for (int s = 0; s < L; ++s)
                acc += B->kh[(size_t)s * Dk + c] * exp(Gl[c] - B->G[(size_t)s * Dk + c]) *
                       B->D[(size_t)s * Dv + j];
            B->tmp[(size_t)c * Dv + j] = acc;
        }
    memcpy(B->S, B->tmp, sizeof(double) * (size_t)Dk * Dv);
}

static int chk_pair(chk_job *J, int n, int h)
{
    chk_buf B;
    if (chk_alloc(&B, J->C, J->Dk, J->Dv) != 0) return -1;
    size_t st = (size_t)J->Dk * J->Dv;
    if (J->S0) memcpy(B.S, J->S0 + ((size_t)n * J->H + h) * st, sizeof(double) * st);
    else memset(B.S, 0, sizeof(double) * st);
    for (int64_t t0 = J->cu[n]; t0 < J->cu[n + 1]; t0 += J->C) {
        int64_t rem = J->cu[n + 1] - t0;
        chk_chunk(J, &B, h, t0, rem < J->C ? (int)rem : J->C);
    }
    if (J->S_out) memcpy(J->S_out + ((size_t)n * J->H + h) * st, B.S, sizeof(double) * st);
    chk_free(&B);
    return 0;
}

static void *chk_worker(void *arg)
{
    chk_job *J = (chk_job *)arg;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int p = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (p >= J->npairs) break;
        if (chk_pair(J, p / J->H, p % J->H) != 0) {
            pthread_mutex_lock(&J->mu);
            J->failed = 1;
            pthread_mutex_unlock(&J->mu);
        }
    }
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int kda_oracle_chunkwise(int N, int H, int Dk, int Dv, const int64_t *cu_seqlens,
                         const double *q, const double *k, const double *v, const double *g,
                         const double *beta, double scale, const double *initial_state,
                         double *o, double *final_state, int use_qk_l2norm, int has_lower_bound,
                         double lower_bound, int beta_is_logit, int chunk_size, int nthreads)
{
    if (N < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || chunk_size <= 0 || !cu_seqlens) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    chk_job J;
    J.N = N; J.H = H; J.Dk = Dk; J.Dv = Dv; J.C = chunk_size; J.cu = cu_seqlens;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.scale = scale;
    J.beta_logit = beta_is_logit;
    J.S0 = initial_state; J.o = o; J.S_out = final_state;
    J.l2 = use_qk_l2norm; J.has_lb = has_lower_bound; J.lb = lower_bound;
    J.next = 0; J.npairs = N * H; J.failed = 0;
    pthread_mutex_init(&J.mu, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J.npairs) nthreads = J.npairs > 0 ? J.npairs : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * nthreads);
    int started = 0;
    if (th)
        for (int i = 0; i < nthreads; ++i) {
            if (pthread_create(&th[i], NULL, chk_worker, &J) != 0) break;
            ++started;
        }
    if (started == 0) chk_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return J.failed ? -2 : 0;
}
