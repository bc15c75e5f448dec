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
 *   Backward pass -- the gradient of a loss through the scan, for training
 *   (the Nemotron feasibility report plans forward and backward tests of the
 *   Mamba-2 layer, sections 3.2 and 3.3).  It is the reverse-mode derivative
 *   of the token loop above, written out: with g = dLoss/dh_t carried
 *   backwards from dLoss/d(final state),
 *       g      += dy_t C_t^T                      (y_t reads h_t)
 *       dC_t   += h_t^T dy_t
 *       dx_t    = D dy_t + dt g B_t
 *       dB_t   += dt g^T x_t
 *       ddt     = x_t^T g B_t + A exp(dt A) <g, h_{t-1}>
 *       dA     += dt exp(dt A) <g, h_{t-1}>,   dD += dy_t . x_t
 *       ddt_raw = ddt * sigmoid(dt_raw + dt_bias)  (softplus' = sigmoid)
 *       g       = exp(dt A) g                     (h_t reads h_{t-1})
 *   and dLoss/d(initial state) = g after the first token.
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

/* ------------------------------------------------------------------------ */
/* Backward pass of the selective scan                                       */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *x, *B, *C, *dt_raw, *dt_bias, *A, *D, *init_state, *dy, *dfinal;
    double *dx, *dB, *dC, *ddt_raw, *dinit;
    double *dA_part, *dD_part, *dbias_part;   /* [b][H] per-pair partial sums */
    int64_t b, L, H, P, N, G;
    int64_t next;           /* next (batch, group) pair to process */
    pthread_mutex_t lock;
} bwd_job;

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/*
 * One (batch bi, head h) pair: the forward recurrence again, keeping every
 * state h_0 .. h_L (hs, (L + 1) * P * N doubles: h_0 is the initial state),
 * then the reverse loop.  dB and dC of the head's group are accumulated
 * (the caller runs a group's heads in order, on one thread).
 */
static void bwd_one(const bwd_job* J, int64_t bi, int64_t h, double* hs, double* g)
{
    const int64_t L = J->L, H = J->H, P = J->P, N = J->N, G = J->G, PN = P * N;
    const int64_t grp = h / (H / G);
    const double A = J->A[h];
    const double Dh = J->D ? J->D[h] : 0.0;
    const double bias = J->dt_bias ? J->dt_bias[h] : 0.0;
    const int64_t sbase = (bi * H + h) * PN;

    if (J->init_state != NULL) memcpy(hs, J->init_state + sbase, sizeof(double) * (size_t)PN);
    else memset(hs, 0, sizeof(double) * (size_t)PN);
    for (int64_t t = 0; t < L; ++t) {
        const double dt = softplus(bias + J->dt_raw[(bi * L + t) * H + h]);
        const double a = exp(A * dt);
        const double* xt = J->x + ((bi * L + t) * H + h) * P;
        const double* Bt = J->B + ((bi * L + t) * G + grp) * N;
        const double* prev = hs + t * PN;
        double* cur = hs + (t + 1) * PN;
        for (int64_t p = 0; p < P; ++p)
            for (int64_t n = 0; n < N; ++n) cur[p * N + n] = a * prev[p * N + n] + dt * xt[p] * Bt[n];
    }

    if (J->dfinal) memcpy(g, J->dfinal + sbase, sizeof(double) * (size_t)PN);
    else memset(g, 0, sizeof(double) * (size_t)PN);
    double dA = 0.0, dD = 0.0, dbias = 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
        const double v = bias + J->dt_raw[(bi * L + t) * H + h];
        const double dt = softplus(v);
        const double a = exp(A * dt);
        const double* xt = J->x + ((bi * L + t) * H + h) * P;
        const double* Bt = J->B + ((bi * L + t) * G + grp) * N;
        const double* Ct = J->C + ((bi * L + t) * G + grp) * N;
        const double* dyt = J->dy + ((bi * L + t) * H + h) * P;
        const double* ht = hs + (t + 1) * PN;
        const double* hprev = hs + t * PN;
        double* dxt = J->dx + ((bi * L + t) * H + h) * P;
        double* dBt = J->dB + ((bi * L + t) * G + grp) * N;
        double* dCt = J->dC + ((bi * L + t) * G + grp) * N;

        /* y_t = h_t C_t + D x_t */
        for (int64_t p = 0; p < P; ++p)
            for (int64_t n = 0; n < N; ++n) g[p * N + n] += dyt[p] * Ct[n];
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t p = 0; p < P; ++p) acc += dyt[p] * ht[p * N + n];
            dCt[n] += acc;
        }
        double xgb = 0.0, gh = 0.0;
        for (int64_t p = 0; p < P; ++p) {
            double gb = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                gb += g[p * N + n] * Bt[n];
                gh += g[p * N + n] * hprev[p * N + n];
            }
            dxt[p] = Dh * dyt[p] + dt * gb;
            xgb += xt[p] * gb;
            dD += dyt[p] * xt[p];
        }
        /* h_t = exp(dt A) h_{t-1} + dt x_t B_t^T */
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t p = 0; p < P; ++p) acc += g[p * N + n] * xt[p];
            dBt[n] += dt * acc;
        }
        const double ddt = xgb + A * a * gh;
        dA += dt * a * gh;
        const double dv = ddt * sigmoid(v);
        J->ddt_raw[(bi * L + t) * H + h] = dv;
        dbias += dv;
        for (int64_t i = 0; i < PN; ++i) g[i] *= a;
    }
    if (J->dinit) memcpy(J->dinit + sbase, g, sizeof(double) * (size_t)PN);
    J->dA_part[bi * H + h] = dA;
    J->dD_part[bi * H + h] = dD;
    J->dbias_part[bi * H + h] = dbias;
}

static void* bwd_worker(void* arg)
{
    bwd_job* J = (bwd_job*)arg;
    double* hs = (double*)malloc(sizeof(double) * (size_t)((J->L + 1) * J->P * J->N));
    double* g = (double*)malloc(sizeof(double) * (size_t)(J->P * J->N));
    const int64_t hpg = J->H / J->G;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t item = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (item >= J->b * J->G) break;
        const int64_t bi = item / J->G, grp = item % J->G;
        for (int64_t k = 0; k < hpg; ++k) bwd_one(J, bi, grp * hpg + k, hs, g);
    }
    free(g);
    free(hs);
    return NULL;
}

/*
 * Gradient of Loss = sum(dy * y) + sum(dfinal * final_state) with respect to
 * every input of oracle_selective_scan.  dfinal may be NULL (zero); dinit may
 * be NULL (not wanted).  Outputs: dx [b][L][H][P], dB and dC [b][L][G][N],
 * ddt_raw [b][L][H], dA, dD and ddt_bias [H] (summed over the batch),
 * dinit [b][H][P][N].  Each worker keeps (L + 1) * P * N doubles of states.
 * The result does not depend on the thread count (a group's heads run in
 * order on one thread; batch partial sums are added in batch order).
 * Returns 0, or -1 on bad sizes.
 */
int oracle_selective_scan_bwd(const double* x, const double* B, const double* C,
                              const double* dt_raw, const double* dt_bias,
                              const double* A, const double* D,
                              const double* init_state, const double* dy,
                              const double* dfinal, double* dx, double* dB,
                              double* dC, double* ddt_raw, double* dA, double* dD,
                              double* ddt_bias, double* dinit, int64_t b, int64_t L,
                              int64_t H, int64_t P, int64_t N, int64_t G, int nthreads)
{
    if (b < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
    memset(dB, 0, sizeof(double) * (size_t)(b * L * G * N));
    memset(dC, 0, sizeof(double) * (size_t)(b * L * G * N));
    double* parts = (double*)calloc((size_t)(3 * b * H + 1), sizeof(double));
    bwd_job J = {x, B, C, dt_raw, dt_bias, A, D, init_state, dy, dfinal,
                 dx, dB, dC, ddt_raw, dinit, parts, parts + b * H, parts + 2 * b * H,
                 b, L, H, P, N, G, 0, PTHREAD_MUTEX_INITIALIZER};
    if (nthreads < 1) nthreads = 1;
    if (nthreads > b * G) nthreads = (int)(b * G > 0 ? b * G : 1);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, bwd_worker, &J);
    bwd_worker(&J);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    for (int64_t h = 0; h < H; ++h) {
        double sa = 0.0, sd = 0.0, sb = 0.0;
        for (int64_t bi = 0; bi < b; ++bi) {
            sa += J.dA_part[bi * H + h];
            sd += J.dD_part[bi * H + h];
            sb += J.dbias_part[bi * H + h];
        }
        dA[h] = sa;
        dD[h] = sd;
        ddt_bias[h] = sb;
    }
    free(parts);
    return 0;
}
