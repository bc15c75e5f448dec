/*
 * ssd_oracle.c -- fp64 CPU oracle for the Mamba-2 selective state-space layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (plain definitions, token by token, in double precision):
 *
 *   Selective SSM recurrence -- "Hybrid Architectures for Language Models:
 *   Systematic Analysis and Design Insights" (summary page), section 2
 *   Background: the state is updated as h_t = Abar h_{t-1} + Bbar x_t and the
 *   output is y_t = C h_t + D x_t, with input-dependent parameters.
 *   The pages leave the discretisation open; the reading taken here (the one
 *   the Mamba-2 layer uses) is
 *       dt    = softplus(dt_raw + dt_bias)            one scalar per (token, head)
 *       Abar  = exp(dt * A)                           A is a per-head scalar
 *       Bbar  = dt * B
 *   so, per head with state h[p][n]:
 *       h[p][n] <- exp(dt*A) * h[p][n] + dt * x[p] * B[n]
 *       y[p]     = sum_n C[n] * h[p][n] + D * x[p]
 *   Heads map to B/C groups contiguously: g = h / (H / G).
 *
 *   Causal depthwise convolution + SiLU -- the Mamba cache size formula of
 *   the same page, appendix C (Details for Computational and Memory Costs
 *   Comparison), counts N_conv * (2*d_state + d_ssm) conv-cache entries per
 *   layer: the short convolution runs over the x, B and C channels together
 *   and its cache holds N_conv (= k) past inputs per channel.  Tap order is
 *   cross-correlation with causal left padding:
 *       u[t][c] = SiLU(bias[c] + sum_{j<k} w[c][j] * e[t-k+1+j][c])
 *   where e[tau] is the input for tau >= 0 and the cached input (or 0) for
 *   tau < 0.  The conv kernel width 4 and the SiLU activation are the
 *   Mamba-2 settings listed in the Nemotron feasibility report, section 1.4.
 *
 *   Decode step -- the same recurrence run for one token from a given state.
 *
 * Precision: all arithmetic in IEEE double; softplus is evaluated as
 * max(v,0) + log1p(exp(-|v|)) with no threshold, SiLU as v / (1 + exp(-v)).
 * Work is split over (batch, head) pairs on POSIX threads; each pair is an
 * independent sequential recurrence, so the result does not depend on the
 * thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double softplus(double v) { return fmax(v, 0.0) + log1p(exp(-fabs(v))); }
static double silu(double v) { return v / (1.0 + exp(-v)); }

/* ------------------------------------------------------------------------ */
/* Causal depthwise conv1d + SiLU                                            */
/* ------------------------------------------------------------------------ */

/*
 * xBC        [b][L][conv_dim]   input channels (x | B | C)
 * out        [b][L][conv_dim]   SiLU(conv) output
 * w          [conv_dim][k]      taps; tap k-1 multiplies the current token
 * bias       [conv_dim]         may be NULL (zero)
 * conv_state [b][conv_dim][k]   may be NULL (zero left context, nothing kept).
 *                               On entry column j holds the input at time
 *                               j - k (relative to the first token of this
 *                               call); on exit it holds the last k inputs of
 *                               the extended sequence, oldest first.
 */
void oracle_conv1d_silu(const double* xBC, double* out, const double* w,
                        const double* bias, double* conv_state, int64_t b,
                        int64_t L, int64_t conv_dim, int64_t k)
{
    double* hist = (double*)malloc(sizeof(double) * (size_t)(L + k));
    for (int64_t bi = 0; bi < b; ++bi) {
        for (int64_t c = 0; c < conv_dim; ++c) {
            /* extended input e[tau], tau = -k .. L-1, stored at hist[tau + k] */
            for (int64_t j = 0; j < k; ++j)
                hist[j] = conv_state ? conv_state[(bi * conv_dim + c) * k + j] : 0.0;
            for (int64_t t = 0; t < L; ++t)
                hist[t + k] = xBC[(bi * L + t) * conv_dim + c];
            for (int64_t t = 0; t < L; ++t) {
                double acc = bias ? bias[c] : 0.0;
                for (int64_t j = 0; j < k; ++j)
                    acc += w[c * k + j] * hist[(t - k + 1 + j) + k];
                out[(bi * L + t) * conv_dim + c] = silu(acc);
            }
            if (conv_state)
                for (int64_t j = 0; j < k; ++j)
                    conv_state[(bi * conv_dim + c) * k + j] = hist[L + j];
        }
    }
    free(hist);
}

/* ------------------------------------------------------------------------ */
/* Token-by-token selective scan                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *x, *B, *C, *dt_raw, *dt_bias, *A, *D, *init_state;
    double *y, *final_state;
    int64_t b, L, H, P, N, G;
    int64_t next;           /* next (batch, head) pair to process */
    pthread_mutex_t lock;
} scan_job;

/*
 * One (batch bi, head h) recurrence.
 * x  [b][L][H][P], B and C [b][L][G][N], dt_raw [b][L][H], y [b][L][H][P],
 * states [b][H][P][N].
 */
static void scan_one(const scan_job* J, int64_t bi, int64_t h, double* hs)
{
    const int64_t L = J->L, H = J->H, P = J->P, N = J->N, G = J->G;
    const int64_t g = h / (H / G);
    const double A = J->A[h];
    const double Dh = J->D ? J->D[h] : 0.0;
    const double bias = J->dt_bias ? J->dt_bias[h] : 0.0;
    const int64_t sbase = (bi * H + h) * P * N;

    if (J->init_state) memcpy(hs, J->init_state + sbase, sizeof(double) * (size_t)(P * N));
    else memset(hs, 0, sizeof(double) * (size_t)(P * N));

    for (int64_t t = 0; t < L; ++t) {
        const double dt = softplus(J->dt_raw[(bi * L + t) * H + h] + bias);
        const double a = exp(dt * A);
        const double* xt = J->x + ((bi * L + t) * H + h) * P;
        const double* Bt = J->B + ((bi * L + t) * G + g) * N;
        const double* Ct = J->C + ((bi * L + t) * G + g) * N;
        double* yt = J->y + ((bi * L + t) * H + h) * P;
        for (int64_t p = 0; p < P; ++p) {
            double* row = hs + p * N;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                row[n] = a * row[n] + dt * xt[p] * Bt[n];
                acc += Ct[n] * row[n];
            }
            yt[p] = acc + Dh * xt[p];
        }
    }
    if (J->final_state) memcpy(J->final_state + sbase, hs, sizeof(double) * (size_t)(P * N));
}

static void* scan_worker(void* arg)
{
    scan_job* J = (scan_job*)arg;
    double* hs = (double*)malloc(sizeof(double) * (size_t)(J->P * J->N));
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t item = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (item >= J->b * J->H) break;
        scan_one(J, item / J->H, item % J->H, hs);
    }
    free(hs);
    return NULL;
}

/*
 * Full-sequence selective scan.  dt_bias and D may be NULL (zero);
 * init_state may be NULL (zero state); final_state may be NULL.
 * nthreads <= 0 means one thread.  Returns 0, or -1 on bad sizes.
 */
int oracle_selective_scan(const double* x, const double* B, const double* C,
                          const double* dt_raw, const double* dt_bias,
                          const double* A, const double* D,
                          const double* init_state, double* y,
                          double* final_state, int64_t b, int64_t L, int64_t H,
                          int64_t P, int64_t N, int64_t G, int nthreads)
{
    if (b < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
    scan_job J = {x, B, C, dt_raw, dt_bias, A, D, init_state, y, final_state,
                  b, L, H, P, N, G, 0, PTHREAD_MUTEX_INITIALIZER};
    if (nthreads < 1) nthreads = 1;
    if (nthreads > b * H) nthreads = (int)(b * H > 0 ? b * H : 1);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, scan_worker, &J);
    scan_worker(&J);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/*
 * Single-token decode step: the recurrence body once, from `state`, which is
 * updated in place.  x [b][H][P], B and C [b][G][N], dt_raw [b][H],
 * y [b][H][P], state [b][H][P][N].
 */
int oracle_state_update(double* state, const double* x, const double* B,
                        const double* C, const double* dt_raw,
                        const double* dt_bias, const double* A, const double* D,
                        double* y, int64_t b, int64_t H, int64_t P, int64_t N,
                        int64_t G, int nthreads)
{
    /* One token is a length-1 sequence whose initial and final state are the
       same buffer; the per-pair copy in scan_one makes the aliasing safe. */
    return oracle_selective_scan(x, B, C, dt_raw, dt_bias, A, D, state, y, state,
                                 b, 1, H, P, N, G, nthreads);
}
