/*
 * M²RNN recurrence: plain fp64 CPU oracle.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * this file's library.  It shares no code with the CUDA path and is
 * deliberately slow and literal: naive loops, libm tanh, no blocking, no
 * reordering beyond the definitions below.
 *
 * What it computes (per batch element b and head h, independently):
 *   Z_t = tanh(H_{t-1} W + k_t v_tᵀ)                     (1)
 *   H_t = f_t H_{t-1} + (1 - f_t) Z_t                     (2)
 *   y_t = H_tᵀ q_t                                        (3)
 * (1) and (2) are the state-update equations of "M²RNN: Non-Linear RNNs with
 * Matrix-Valued States for Scalable Language Modeling" (gist.science technical
 * summary, §2.1 core architecture design; the wispaper.ai post "M2 RNN:
 * Breaking the Expressivity Ceiling...", §1 The Core Recurrence, prints the
 * same pair with garbled LaTeX).  H_t is K×V (same §2.1: matrix-valued
 * state), W is V×V per head (it right-multiplies H_{t-1}; §2.2 gives the GEMM
 * dimensions (K, V, V)), f_t is a scalar in [0,1] that depends only on the
 * input (§2.1 forget gate).  The pages define no readout: (3) is the library's
 * stated reading, using the updated state H_t.
 *
 * Indexing: array step t (0-based) consumes k[t], v[t], q[t], f[t] and
 * produces H_{t+1} and y[t].  H0 NULL means a zero initial state.
 *
 * Backward (BPTT): the exact chain rule of (1)-(3).  With G_t = dL/dH_t:
 *   G_T   = dHT + q_T dy_Tᵀ
 *   dq_t  = H_t dy_t
 *   dA_t  = (1 - f_t) G_t ⊙ (1 - Z_t²)
 *   df_t  = <G_t, H_{t-1} - Z_t>_F
 *   dk_t  = dA_t v_t,  dv_t = dA_tᵀ k_t,  dW += H_{t-1}ᵀ dA_t
 *   G_{t-1} = f_t G_t + dA_t Wᵀ + q_{t-1} dy_{t-1}ᵀ,   dH0 = G_0.
 * Z_t is recomputed from the stored H_{t-1} by (1), which is the same
 * recomputation the pages describe for the backward pass (§2.2: states are
 * recomputed rather than stored).  dW sums over batch and time; the batch sum
 * is taken in ascending b after all pairs finish, so results do not depend on
 * the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, H, T, K, V;
    const double *k, *v, *q, *f, *W, *H0, *dy, *dHT;
    double *y, *HT;
    double *dk, *dv, *dq, *df, *dWpart, *dH0;
    int backward;
    int nthreads;
    int next;              /* next pair to take (guarded by mu) */
    int failed;            /* allocation failure */
    pthread_mutex_t mu;
} job_t;

/* Offsets into the head-first contiguous layouts. */
static size_t off_bht(const job_t* j, int b, int h, int t, int n) {
    return (((size_t)b * j->H + h) * j->T + t) * (size_t)n;
}
static size_t off_state(const job_t* j, int b, int h) {
    return ((size_t)b * j->H + h) * (size_t)j->K * j->V;
}

/* A = Hprev W + k vᵀ ; written out element by element. */
static void preact(int K, int V, const double* Hprev, const double* W,
                   const double* kt, const double* vt, double* A) {
    for (int i = 0; i < K; ++i)
        for (int c = 0; c < V; ++c) {
            double s = 0.0;
            for (int l = 0; l < V; ++l) s += Hprev[(size_t)i * V + l] * W[(size_t)l * V + c];
            A[(size_t)i * V + c] = s + kt[i] * vt[c];
        }
}

static int run_pair(job_t* j, int b, int h) {
    const int K = j->K, V = j->V, T = j->T;
    const size_t KV = (size_t)K * V;
    const double* W = j->W + (size_t)h * V * V;
    /* States H_0..H_T kept only when the backward needs them. */
    double* Hs = (double*)malloc(sizeof(double) * KV * (j->backward ? (size_t)T + 1 : 2));
    double* A = (double*)malloc(sizeof(double) * KV);
    double* G = (double*)malloc(sizeof(double) * KV);
    double* dA = (double*)malloc(sizeof(double) * KV);
    if (!Hs || !A || !G || !dA) { free(Hs); free(A); free(G); free(dA); return -1; }

    if (j->H0) memcpy(Hs, j->H0 + off_state(j, b, h), sizeof(double) * KV);
    else memset(Hs, 0, sizeof(double) * KV);

    for (int t = 0; t < T; ++t) {
        const double* Hp = j->backward ? Hs + (size_t)t * KV : Hs + (size_t)(t & 1) * KV;
        double* Hn = j->backward ? Hs + (size_t)(t + 1) * KV : Hs + (size_t)((t + 1) & 1) * KV;
        const double* kt = j->k + off_bht(j, b, h, t, K);
        const double* vt = j->v + off_bht(j, b, h, t, V);
        const double* qt = j->q + off_bht(j, b, h, t, K);
        const double ft = j->f[((size_t)b * j->H + h) * T + t];
        preact(K, V, Hp, W, kt, vt, A);                               /* (1) inside tanh */
        for (size_t e = 0; e < KV; ++e)
            Hn[e] = ft * Hp[e] + (1.0 - ft) * tanh(A[e]);             /* (1), (2) */
        if (j->y) {
            double* yt = j->y + off_bht(j, b, h, t, V);
            for (int c = 0; c < V; ++c) {                               /* (3) */
                double s = 0.0;
                for (int i = 0; i < K; ++i) s += Hn[(size_t)i * V + c] * qt[i];
                yt[c] = s;
            }
        }
    }
    const double* HTp = j->backward ? Hs + (size_t)T * KV : Hs + (size_t)(T & 1) * KV;
    if (j->HT) memcpy(j->HT + off_state(j, b, h), HTp, sizeof(double) * KV);

    if (j->backward) {
        double* dWp = j->dWpart + ((size_t)b * j->H + h) * (size_t)V * V;
        memset(dWp, 0, sizeof(double) * (size_t)V * V);
        if (j->dHT) memcpy(G, j->dHT + off_state(j, b, h), sizeof(double) * KV);
        else memset(G, 0, sizeof(double) * KV);
        for (int t = T - 1; t >= 0; --t) {
            const double* Hp = Hs + (size_t)t * KV;        /* H_{t-1} in the paper's numbering */
            const double* Hn = Hs + (size_t)(t + 1) * KV;  /* H_t */
            const double* kt = j->k + off_bht(j, b, h, t, K);
            const double* vt = j->v + off_bht(j, b, h, t, V);
            const double* qt = j->q + off_bht(j, b, h, t, K);
            const double* dyt = j->dy + off_bht(j, b, h, t, V);
            const double ft = j->f[((size_t)b * j->H + h) * T + t];
            /* readout: G += q dyᵀ, dq = H_t dy */
            for (int i = 0; i < K; ++i)
                for (int c = 0; c < V; ++c) G[(size_t)i * V + c] += qt[i] * dyt[c];
            double* dqt = j->dq + off_bht(j, b, h, t, K);
            for (int i = 0; i < K; ++i) {
                double s = 0.0;
                for (int c = 0; c < V; ++c) s += Hn[(size_t)i * V + c] * dyt[c];
                dqt[i] = s;
            }
            /* recompute Z_t = tanh(A) from H_{t-1} */
            preact(K, V, Hp, W, kt, vt, A);
            double dft = 0.0;
            for (size_t e = 0; e < KV; ++e) {
                const double z = tanh(A[e]);
                dft += G[e] * (Hp[e] - z);
                dA[e] = (1.0 - ft) * G[e] * (1.0 - z * z);
            }
            j->df[((size_t)b * j->H + h) * T + t] = dft;
            double* dkt = j->dk + off_bht(j, b, h, t, K);
            for (int i = 0; i < K; ++i) {
                double s = 0.0;
                for (int c = 0; c < V; ++c) s += dA[(size_t)i * V + c] * vt[c];
                dkt[i] = s;
            }
            double* dvt = j->dv + off_bht(j, b, h, t, V);
            for (int c = 0; c < V; ++c) {
                double s = 0.0;
                for (int i = 0; i < K; ++i) s += dA[(size_t)i * V + c] * kt[i];
                dvt[c] = s;
            }
            for (int l = 0; l < V; ++l)
                for (int c = 0; c < V; ++c) {
                    double s = 0.0;
                    for (int i = 0; i < K; ++i) s += Hp[(size_t)i * V + l] * dA[(size_t)i * V + c];
                    dWp[(size_t)l * V + c] += s;
                }
            /* G_{t-1} = f G + dA Wᵀ (A is free again: use it as the new G) */
            for (int i = 0; i < K; ++i)
                for (int l = 0; l < V; ++l) {
                    double s = 0.0;
                    for (int c = 0; c < V; ++c) s += dA[(size_t)i * V + c] * W[(size_t)l * V + c];
                    A[(size_t)i * V + l] = ft * G[(size_t)i * V + l] + s;
                }
            memcpy(G, A, sizeof(double) * KV);
        }
        if (j->dH0) memcpy(j->dH0 + off_state(j, b, h), G, sizeof(double) * KV);
    }
    free(Hs); free(A); free(G); free(dA);
    return 0;
}

static void* worker(void* arg) {
    job_t* j = (job_t*)arg;
    const int npairs = j->B * j->H;
    for (;;) {
        pthread_mutex_lock(&j->mu);
        const int p = j->next++;
        pthread_mutex_unlock(&j->mu);
        if (p >= npairs) break;
        if (run_pair(j, p / j->H, p % j->H) != 0) {
            pthread_mutex_lock(&j->mu);
            j->failed = 1;
            pthread_mutex_unlock(&j->mu);
        }
    }
    return NULL;
}

static int run_job(job_t* j) {
    int nth = j->nthreads > 0 ? j->nthreads : 1;
    if (nth > j->B * j->H) nth = j->B * j->H;
    pthread_mutex_init(&j->mu, NULL);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nth);
    if (!th) return -1;
    int started = 0;
    for (int r = 0; r < nth; ++r)
        if (pthread_create(&th[r], NULL, worker, j) == 0) ++started;
    if (started == 0) worker(j);
    for (int r = 0; r < started; ++r) pthread_join(th[r], NULL);
    free(th);
    pthread_mutex_destroy(&j->mu);
    return j->failed ? -1 : 0;
}

/* Forward.  y [B,H,T,V] and HT [B,H,K,V] may each be NULL.  Returns 0 on success. */
int m2rnn_oracle_forward(int B, int H, int T, int K, int V,
                         const double* k, const double* v, const double* q,
                         const double* f, const double* W, const double* H0,
                         double* y, double* HT, int nthreads) {
    if (B < 1 || H < 1 || T < 0 || K < 1 || V < 1) return -2;
    job_t j;
    memset(&j, 0, sizeof j);
    j.B = B; j.H = H; j.T = T; j.K = K; j.V = V;
    j.k = k; j.v = v; j.q = q; j.f = f; j.W = W; j.H0 = H0;
    j.y = y; j.HT = HT; j.nthreads = nthreads;
    return run_job(&j);
}

/* Forward + backward.  dHT may be NULL (zero).  dW [H,V,V] sums over batch. */
int m2rnn_oracle_backward(int B, int H, int T, int K, int V,
                          const double* k, const double* v, const double* q,
                          const double* f, const double* W, const double* H0,
                          const double* dy, const double* dHT,
                          double* dk, double* dv, double* dq, double* df,
                          double* dW, double* dH0, int nthreads) {
    if (B < 1 || H < 1 || T < 0 || K < 1 || V < 1) return -2;
    job_t j;
    memset(&j, 0, sizeof j);
    j.B = B; j.H = H; j.T = T; j.K = K; j.V = V;
    j.k = k; j.v = v; j.q = q; j.f = f; j.W = W; j.H0 = H0;
    j.dy = dy; j.dHT = dHT;
    j.dk = dk; j.dv = dv; j.dq = dq; j.df = df; j.dH0 = dH0;
    j.backward = 1; j.nthreads = nthreads;
    j.dWpart = (double*)malloc(sizeof(double) * (size_t)B * H * V * V);
    if (!j.dWpart) return -1;
    int rc = run_job(&j);
    if (rc == 0) {
        for (int h = 0; h < H; ++h)
            for (size_t e = 0; e < (size_t)V * V; ++e) {
                double s = 0.0;
                for (int b = 0; b < B; ++b) s += j.dWpart[((size_t)b * H + h) * V * V + e];
                dW[(size_t)h * V * V + e] = s;
            }
    }
    free(j.dWpart);
    return rc;
}
