/*
 * ss_oracle.c -- plain, slow, fp64 CPU oracle for the selective scan (S6) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file:
 * only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg use it.  It shares no
 * code, header, table or helper with the CUDA library; the two agree only on the argument
 * conventions (layouts and the four direction codes), which both restate on their own.
 *
 * What it computes, step by step, for every batch row b and channel d (all in double):
 *
 *   for each scan direction k (an ordering of the L positions):
 *     h[n] = initial_state[k,b,d,n], or 0 without one     (the state before step 0)
 *     for t = 0 .. L-1:
 *       p     = spatial position visited at step t         (the direction's index map)
 *       u_t   = u[b,p,d], or, with a convolution given,    ("Understanding Mamba from zero"
 *               silu(conv_bias[k,d] + sum_j                 sec. 6.2 Step 2: a small depthwise
 *                 conv_weight[k,d,j] * u[b, p(t-w+1+j), d]) causal 1D conv before the SSM;
 *               over the taps j = 0..w-1 whose step        width d_conv = 4 in sec. 8; "Vision
 *               t-w+1+j is >= 0 (zero padding before the    Mamba" sec. 2.2: each direction
 *               first step), p(s) = position of step s      convolves its own scanned sequence;
 *                                                          the activation after the conv as in
 *                                                          Figure 2's caption and the VMamba
 *                                                          block of "S4 -> Mamba" sec. 3)
 *       Delta = softplus(delta[k,b,t,d] + bias[d])         ("Understanding Mamba from zero",
 *               (or the raw sum when softplus is off)       sec. 4.1 Algorithm 2 / sec. 6.2
 *                                                          Step 3: tau_Delta(Parameter+s_Delta))
 *               with int8 codes (delta_scale given), the   ("S4 -> Mamba" sec. 2.3: Delta
 *               raw value is delta[k,b,t,d] * delta_scale[d] quantised to int8 at inference)
 *       for n: Abar = exp(Delta * A[d,n])                  (same page, sec. 6.2 Step 4, eq. 4)
 *              Bbar = Delta * B[k,b,t,n]                   (first-order reading of eq. 4, as on
 *                                                          "Mamba-UNet" sec. 4: Bbar ~ Delta*B)
 *                     or, with zoh_exact, (exp(Delta*A)-1)/A * B   (eq. 4 exactly, diagonal A)
 *              h[n]  = Abar * h[n] + Bbar * u_t            (eq. 2a; the per-state scalar
 *                                                          recurrence h_t = a_t h_{t-1} + b_t of
 *                                                          sec. 5)
 *       y_k[p] = sum_n C[k,b,t,n] * h[n] + Dskip[d]*u_t    (eq. 2b plus the D(t)x(t) skip
 *                                                          term of "Mamba-UNet" sec. 4)
 *     last_state[k,b,d,n] = h[n] after the last step
 *   out[b,p,d] = (sum_k y_k[p]) * silu(z[b,p,d])          (Step 6 gate phi = SiLU; the Vim block's
 *                                                          sigma(z)*(y_fwd+y_bwd), "Vision Mamba"
 *                                                          sec. 2.2; SS2D merge, "S4 -> Mamba" sec. 3)
 *
 * With params_per_direction, direction k reads its own A[k], Dskip[k] and delta_bias[k] (VMamba's
 * cross-scan and Vim's two scan directions are separate S6 modules, each with its own parameters).
 * With u_per_direction, direction k reads its own input u[k] wherever u appears above.  This is
 * the cross-modal scan of Sigma's CroMB ("S4 -> Mamba" sec. 4.1): two modalities, each scanned
 * over its own input with the C of the other modality, outputs summed -- the caller stacks the
 * inputs as directions and passes C in swapped order.
 *
 * Direction maps (which spatial position p a scan visits at step t), for a sequence that is an
 * H x W image flattened row by row (raster order, "Understanding Mamba from zero" sec. 7.2):
 *   0 forward:          p = t
 *   1 reverse:          p = L-1-t                         (Vim backward scan)
 *   2 column-major:     step t visits row t mod H of column t div H, i.e. p = (t mod H)*W + t div H
 *   3 column-reverse:   the column-major order walked backwards, p = colmajor(L-1-t)
 * Directions 2 and 3 are the two other cross-scan orders of VMamba's SS2D ("S4 -> Mamba" sec. 3).
 *
 * Layouts (row-major, all double):
 *   u, z                 [batch, L, D]   spatial order (u: [K, batch, L, D] with u_per_direction)
 *   delta                [K, batch, L, D] scan order of direction k
 *   B, C                 [K, batch, L, N] scan order of direction k
 *   A                    [D, N] ([K, D, N] with params_per_direction)
 *   Dskip, delta_bias    [D] ([K, D] with params_per_direction) or NULL (NULL means zero)
 *   z                    NULL means no gate
 *   out                  [batch, L, D]
 *   last_state           [K, batch, D, N] or NULL
 *   initial_state        [K, batch, D, N] or NULL (zero)
 *   conv_weight          [K, D, conv_width] or NULL (no convolution: u_t = u[b,p,d])
 *   conv_bias            [K, D] or NULL (zero)
 *   delta_scale          [D] or NULL: delta holds int8 codes q, the raw value is q * scale[d]
 *
 * Parity is pinned by tests/test_oracle_pins.py against the LTI convolution form (eq. 3),
 * Theorem 1, the unrolled double sum, the Delta -> 0 limit, reversal and explicitly permuted
 * scans; see the header of that file.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEM 2

enum { ORACLE_DIR_FORWARD = 0, ORACLE_DIR_REVERSE = 1, ORACLE_DIR_COLUMN = 2, ORACLE_DIR_COLUMN_REVERSE = 3 };

/* Spatial position visited at step t of direction dir. Returns -1 for an unknown direction. */
int64_t ss_oracle_position(int32_t dir, int64_t L, int64_t H, int64_t W, int64_t t)
{
    int64_t s;
    switch (dir) {
    case ORACLE_DIR_FORWARD:
        return t;
    case ORACLE_DIR_REVERSE:
        return L - 1 - t;
    case ORACLE_DIR_COLUMN:
        return (t % H) * W + (t / H);
    case ORACLE_DIR_COLUMN_REVERSE:
        s = L - 1 - t;
        return (s % H) * W + (s / H);
    default:
        return -1;
    }
}

static double oracle_softplus(double x)
{
    /* log(1 + e^x) written so that neither branch overflows */
    return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

static double oracle_silu(double v)
{
    return v / (1.0 + exp(-v));
}

/* The input of step t of direction dir after the causal depthwise convolution and SiLU: tap j
 * (0 .. width-1) multiplies the input at step t - (width-1) + j of the same scan order, so the
 * last tap takes the current step; steps before 0 contribute nothing. */
static double oracle_conv_silu_step(const double* u, int64_t b, int64_t d, int64_t L, int64_t D,
                                    int32_t dir, int64_t H, int64_t W, int64_t t,
                                    const double* w, double bias, int64_t width)
{
    double c = bias;
    for (int64_t j = 0; j < width; ++j) {
        const int64_t s = t - (width - 1) + j;
        if (s >= 0)
            c += w[j] * u[(b * L + ss_oracle_position(dir, L, H, W, s)) * D + d];
    }
    return oracle_silu(c);
}

/* The convolved inputs on their own, for checking: out[k,b,t,d] = u_t of direction k (scan
 * order).  conv_bias may be NULL. */
int ss_oracle_conv_silu(int64_t batch, int64_t L, int64_t D, int32_t K, const int32_t* dirs,
                        int64_t H, int64_t W, const double* u, const double* conv_weight,
                        const double* conv_bias, int64_t conv_width, double* out)
{
    if (batch < 0 || L < 0 || D < 0 || K < 1 || K > 4 || conv_width < 1 || conv_width > 64)
        return ORACLE_BAD_ARG;
    if (!u || !conv_weight || !out || !dirs)
        return ORACLE_BAD_ARG;
    for (int32_t k = 0; k < K; ++k) {
        if (dirs[k] < 0 || dirs[k] > 3)
            return ORACLE_BAD_ARG;
        if ((dirs[k] == ORACLE_DIR_COLUMN || dirs[k] == ORACLE_DIR_COLUMN_REVERSE) &&
            (H <= 0 || W <= 0 || H * W != L))
            return ORACLE_BAD_ARG;
    }
    for (int32_t k = 0; k < K; ++k)
        for (int64_t b = 0; b < batch; ++b)
            for (int64_t t = 0; t < L; ++t)
                for (int64_t d = 0; d < D; ++d)
                    out[(((int64_t)k * batch + b) * L + t) * D + d] = oracle_conv_silu_step(
                        u, b, d, L, D, dirs[k], H, W, t,
                        conv_weight + ((int64_t)k * D + d) * conv_width,
                        conv_bias ? conv_bias[(int64_t)k * D + d] : 0.0, conv_width);
    return ORACLE_OK;
}

int ss_oracle_scan(int64_t batch, int64_t L, int64_t D, int64_t N, int32_t K,
                   const int32_t* dirs, int64_t H, int64_t W,
                   const double* u, const double* delta, const double* A,
                   const double* B, const double* C, const double* Dskip,
                   const double* z, const double* delta_bias,
                   int32_t softplus, int32_t zoh_exact,
                   double* out, double* last_state, int32_t nthreads,
                   const double* initial_state, const double* conv_weight,
                   const double* conv_bias, int64_t conv_width, int32_t u_per_direction,
                   const double* delta_scale, int32_t params_per_direction)
{
    int bad = 0;
    if (batch < 0 || L < 0 || D < 0 || N < 1 || K < 1 || K > 4)
        return ORACLE_BAD_ARG;
    if (conv_weight && (conv_width < 1 || conv_width > 64))
        return ORACLE_BAD_ARG;
    if (!u || !delta || !A || !B || !C || !out || !dirs)
        return ORACLE_BAD_ARG;
    for (int32_t k = 0; k < K; ++k) {
        if (dirs[k] < 0 || dirs[k] > 3)
            return ORACLE_BAD_ARG;
        if ((dirs[k] == ORACLE_DIR_COLUMN || dirs[k] == ORACLE_DIR_COLUMN_REVERSE) &&
            (H <= 0 || W <= 0 || H * W != L))
            return ORACLE_BAD_ARG;
    }
    if (batch == 0 || L == 0 || D == 0) {
        /* no step is taken: the final state is the initial one */
        if (last_state) {
            if (initial_state)
                memcpy(last_state, initial_state, sizeof(double) * (size_t)(K * batch * D * N));
            else
                memset(last_state, 0, sizeof(double) * (size_t)(K * batch * D * N));
        }
        return ORACLE_OK;
    }
    if (nthreads <= 0)
        nthreads = 1;

#pragma omp parallel num_threads(nthreads) reduction(| : bad)
    {
        double* yacc = (double*)malloc(sizeof(double) * (size_t)L);
        double* h = (double*)malloc(sizeof(double) * (size_t)N);
        if (!yacc || !h) {
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bd = 0; bd < batch * D; ++bd) {
                const int64_t b = bd / D, d = bd % D;
                memset(yacc, 0, sizeof(double) * (size_t)L);
                for (int32_t k = 0; k < K; ++k) {
                    const double* uk = u_per_direction ? u + (int64_t)k * batch * L * D : u;
                    const int64_t pk = params_per_direction ? (int64_t)k : 0;
                    const double* Ak = A + pk * D * N;
                    const double* Dk = Dskip ? Dskip + pk * D : NULL;
                    const double* biask = delta_bias ? delta_bias + pk * D : NULL;
                    for (int64_t n = 0; n < N; ++n)
                        h[n] = initial_state
                                   ? initial_state[(((int64_t)k * batch + b) * D + d) * N + n]
                                   : 0.0;
                    for (int64_t t = 0; t < L; ++t) {
                        const int64_t p = ss_oracle_position(dirs[k], L, H, W, t);
                        const double ut =
                            conv_weight
                                ? oracle_conv_silu_step(
                                      uk, b, d, L, D, dirs[k], H, W, t,
                                      conv_weight + ((int64_t)k * D + d) * conv_width,
                                      conv_bias ? conv_bias[(int64_t)k * D + d] : 0.0, conv_width)
                                : uk[(b * L + p) * D + d];
                        const int64_t row = ((int64_t)k * batch + b) * L + t;
                        const double draw = delta_scale ? delta[row * D + d] * delta_scale[d]
                                                        : delta[row * D + d];
                        double dt = draw + (biask ? biask[d] : 0.0);
                        if (softplus)
                            dt = oracle_softplus(dt);
                        double yt = 0.0;
                        for (int64_t n = 0; n < N; ++n) {
                            const double a = Ak[d * N + n];
                            const double abar = exp(dt * a);
                            double bcoef;
                            if (zoh_exact)
                                bcoef = (a != 0.0) ? expm1(dt * a) / a : dt;
                            else
                                bcoef = dt;
                            h[n] = abar * h[n] + bcoef * B[row * N + n] * ut;
                            yt += C[row * N + n] * h[n];
                        }
                        yacc[p] += yt + (Dk ? Dk[d] : 0.0) * ut;
                    }
                    if (last_state)
                        for (int64_t n = 0; n < N; ++n)
                            last_state[(((int64_t)k * batch + b) * D + d) * N + n] = h[n];
                }
                for (int64_t p = 0; p < L; ++p) {
                    const int64_t i = (b * L + p) * D + d;
                    out[i] = z ? yacc[p] * oracle_silu(z[i]) : yacc[p];
                }
            }
        }
        free(yacc);
        free(h);
    }
    return bad ? ORACLE_NO_MEM : ORACLE_OK;
}

int ss_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
