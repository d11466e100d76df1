/*
 * oracle.c -- plain FP64 CPU oracle for the FP32 NCHW grouped/depthwise/dense
 * conv2d forward and the conv -> +bias -> *scale -> sigmoid -> GroupNorm chain.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may link,
 * load or call this file; only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA implementation.
 *
 * Every quantity is computed straight from its definition: a loop nest over
 * (n, k, p, q, c, r, s) in double precision, reading the FP32 inputs as their
 * exact values.  There is no blocking, fusion or reordering.  OpenMP only
 * splits independent outputs (or independent GroupNorm groups) over threads;
 * the summation order inside one output is fixed, so results do not depend on
 * the thread count.
 *
 * Sources (web pages on the subject):
 *  [Atlas]   "GroupConv Atlas" (xiangguozhang.com/projects/groupconv-atlas),
 *            section "Fix the experiment": FP32, contiguous NCHW, grouped conv.
 *  [FusedGN] POPCORNBENCH "Kimi-K2.6__l2_p21" transcript: the Model that applies
 *            Conv2d, + bias[K,1,1], * scale[K,1,1], sigmoid, GroupNorm(eps=1e-5)
 *            with affine weight/bias, population variance; the direct-conv
 *            index formula input[n, ic, h+kh, w+kw] * weight[c, ic, kh, kw]
 *            (no kernel flip) and zero padding of the halo tile.
 *  [Dense]   POPCORNBENCH "Kimi-K2.6__l1_p62" transcript: output size
 *            (H + 2p - d(R-1) - 1)/s + 1 and the general-geometry index map
 *            in_y = out_y*stride - pad + kh*dilation.
 *
 * Readings taken where the pages are silent (each listed in the design notes):
 *  - group g of output channel k is k / (K/groups); it reads input channels
 *    [g*C/groups, (g+1)*C/groups)  (the usual grouped-conv convention);
 *  - the Sigma|w*x| magnitude returned for the tolerance also counts |bias|;
 *  - GroupNorm variance is computed two-pass (mean first, then the mean of
 *    squared deviations), population form, eps inside the square root.
 *
 * Parity status: every function here is pinned by tests against closed forms,
 * invariants and brute force (see tests/test_oracle.py).
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

/* Output extent along one axis, floor form ([Dense] output-size paragraph).
 * Returns <= 0 when the kernel does not fit. */
long oracle_out_extent(long in, long k, long stride, long pad, long dil)
{
    long span = in + 2 * pad - dil * (k - 1) - 1;
    if (stride <= 0) return -1;
    if (span < 0) return 0;
    return span / stride + 1;
}

typedef struct {
    int N, C, H, W, K, R, S, sh, sw, ph, pw, dh, dw, groups;
    long P, Q;
} geom_t;

static int make_geom(geom_t *g, int N, int C, int H, int W, int K, int R, int S,
                     int sh, int sw, int ph, int pw, int dh, int dw, int groups)
{
    if (N < 0 || C <= 0 || H <= 0 || W <= 0 || K <= 0 || R <= 0 || S <= 0) return ORACLE_BAD_ARG;
    if (sh <= 0 || sw <= 0 || ph < 0 || pw < 0 || dh <= 0 || dw <= 0 || groups <= 0) return ORACLE_BAD_ARG;
    if (C % groups != 0 || K % groups != 0) return ORACLE_BAD_ARG;
    g->N = N; g->C = C; g->H = H; g->W = W; g->K = K; g->R = R; g->S = S;
    g->sh = sh; g->sw = sw; g->ph = ph; g->pw = pw; g->dh = dh; g->dw = dw; g->groups = groups;
    g->P = oracle_out_extent(H, R, sh, ph, dh);
    g->Q = oracle_out_extent(W, S, sw, pw, dw);
    if (g->P <= 0 || g->Q <= 0) return ORACLE_BAD_ARG;
    return ORACLE_OK;
}

/* One output element of the grouped cross-correlation, straight from the
 * definition ([FusedGN] direct-conv index formula; [Dense] index map):
 *   y[n,k,p,q] = sum_{c < C/g, r < R, s < S} w[k,c,r,s] * x[n, gi*C/g + c, ih, iw]
 *   ih = p*sh - ph + r*dh,  iw = q*sw - pw + s*dw,  terms outside the image are 0.
 * *mag receives sum |w*x| over the same terms. */
static double conv_point(const geom_t *g, const float *x, const float *w,
                         long n, long k, long p, long q, double *mag)
{
    long cpg = g->C / g->groups;
    long kpg = g->K / g->groups;
    long gi = k / kpg;
    double acc = 0.0, m = 0.0;
    for (long c = 0; c < cpg; ++c) {
        long ci = gi * cpg + c;
        for (long r = 0; r < g->R; ++r) {
            long ih = p * g->sh - g->ph + r * g->dh;
            if (ih < 0 || ih >= g->H) continue;
            for (long s = 0; s < g->S; ++s) {
                long iw = q * g->sw - g->pw + s * g->dw;
                if (iw < 0 || iw >= g->W) continue;
                double wv = (double)w[((k * cpg + c) * g->R + r) * g->S + s];
                double xv = (double)x[((n * g->C + ci) * (long)g->H + ih) * g->W + iw];
                acc += wv * xv;
                m += fabs(wv * xv);
            }
        }
    }
    *mag = m;
    return acc;
}

/* Full convolution output y[N,K,P,Q] (double), optional bias[K] (NULL = none),
 * optional absacc[N,K,P,Q] = sum|w*x| + |bias|. */
int oracle_conv2d(const float *x, const float *w, const float *bias,
                  int N, int C, int H, int W, int K, int R, int S,
                  int sh, int sw, int ph, int pw, int dh, int dw, int groups,
                  double *y, double *absacc)
{
    geom_t g;
    int st = make_geom(&g, N, C, H, W, K, R, S, sh, sw, ph, pw, dh, dw, groups);
    if (st != ORACLE_OK) return st;
    long NK = (long)N * K;
#pragma omp parallel for schedule(dynamic, 1)
    for (long nk = 0; nk < NK; ++nk) {
        long n = nk / K, k = nk % K;
        double b = bias ? (double)bias[k] : 0.0;
        for (long p = 0; p < g.P; ++p) {
            for (long q = 0; q < g.Q; ++q) {
                double mag;
                double v = conv_point(&g, x, w, n, k, p, q, &mag);
                long o = (nk * g.P + p) * g.Q + q;
                y[o] = v + b;
                if (absacc) absacc[o] = mag + fabs(b);
            }
        }
    }
    return ORACLE_OK;
}

/* The same definition evaluated at `count` flat output indices
 * idx[i] = ((n*K + k)*P + p)*Q + q.  Used to check full-size runs on samples. */
int oracle_conv2d_at(const float *x, const float *w, const float *bias,
                     int N, int C, int H, int W, int K, int R, int S,
                     int sh, int sw, int ph, int pw, int dh, int dw, int groups,
                     long count, const long long *idx, double *y, double *absacc)
{
    geom_t g;
    int st = make_geom(&g, N, C, H, W, K, R, S, sh, sw, ph, pw, dh, dw, groups);
    if (st != ORACLE_OK) return st;
    long total = (long)N * K * g.P * g.Q;
    for (long i = 0; i < count; ++i)
        if (idx[i] < 0 || idx[i] >= total) return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        long o = (long)idx[i];
        long q = o % g.Q, t = o / g.Q;
        long p = t % g.P; t /= g.P;
        long k = t % K, n = t / K;
        double b = bias ? (double)bias[k] : 0.0;
        double mag;
        double v = conv_point(&g, x, w, n, k, p, q, &mag);
        y[i] = v + b;
        if (absacc) absacc[i] = mag + fabs(b);
    }
    return ORACLE_OK;
}

/* Logistic function 1/(1+e^-v) ([FusedGN] Model: torch.sigmoid), written in
 * the form that does not overflow for large |v|. */
static double sigmoid_f64(double v)
{
    if (v >= 0.0) return 1.0 / (1.0 + exp(-v));
    double e = exp(v);
    return e / (1.0 + e);
}

/* The fused chain on selected GroupNorm groups ([FusedGN] Model forward):
 *   z = conv(x, w) + b_conv[k] + b_extra[k]       (either bias may be NULL)
 *   v = z * scale[k]
 *   a = sigmoid(v)
 *   per (n, G): mu = mean(a), var = mean((a - mu)^2)  over the K/gn_groups
 *               channels of group G and all P*Q positions (population form)
 *   y = (a - mu) / sqrt(var + eps) * gamma[k] + beta[k]
 * pairs[2*i], pairs[2*i+1] = (n, G) of the i-th requested group; pairs == NULL
 * means every (n, G) in order, which makes the compact outputs below exactly
 * the [N,K,P,Q] tensors.  Outputs (each may be NULL except y_out):
 *   a_out, y_out, absacc_out : [npairs][K/gn_groups][P][Q]
 *   mean_out, var_out        : [npairs]
 * absacc_out holds sum|w*x| + |b_conv| + |b_extra| of the conv stage. */
int oracle_chain(const float *x, const float *w, const float *b_conv, const float *b_extra,
                 const float *scale, int gn_groups, const float *gamma, const float *beta,
                 double eps,
                 int N, int C, int H, int W, int K, int R, int S,
                 int sh, int sw, int ph, int pw, int dh, int dw, int groups,
                 long npairs, const int *pairs,
                 double *a_out, double *y_out, double *absacc_out,
                 double *mean_out, double *var_out)
{
    geom_t g;
    int st = make_geom(&g, N, C, H, W, K, R, S, sh, sw, ph, pw, dh, dw, groups);
    if (st != ORACLE_OK) return st;
    if (gn_groups <= 0 || K % gn_groups != 0 || !scale || !gamma || !beta || !y_out) return ORACLE_BAD_ARG;
    if (!(eps >= 0.0)) return ORACLE_BAD_ARG;
    long kg = K / gn_groups;
    long PQ = g.P * g.Q;
    long M = kg * PQ;
    if (pairs == NULL) npairs = (long)N * gn_groups;
    for (long i = 0; pairs && i < npairs; ++i)
        if (pairs[2 * i] < 0 || pairs[2 * i] >= N || pairs[2 * i + 1] < 0 || pairs[2 * i + 1] >= gn_groups)
            return ORACLE_BAD_ARG;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long i = 0; i < npairs; ++i) {
        long n = pairs ? pairs[2 * i] : i / gn_groups;
        long G = pairs ? pairs[2 * i + 1] : i % gn_groups;
        double *a = a_out ? a_out + i * M : (double *)malloc(sizeof(double) * M);
        if (!a) { bad = 1; continue; }
        /* conv + bias + scale + sigmoid for every element of the group */
        for (long kk = 0; kk < kg; ++kk) {
            long k = G * kg + kk;
            double bc = b_conv ? (double)b_conv[k] : 0.0;
            double be = b_extra ? (double)b_extra[k] : 0.0;
            double sc = (double)scale[k];
            for (long p = 0; p < g.P; ++p) {
                for (long q = 0; q < g.Q; ++q) {
                    double mag;
                    double z = conv_point(&g, x, w, n, k, p, q, &mag) + bc + be;
                    long o = (kk * g.P + p) * g.Q + q;
                    a[o] = sigmoid_f64(z * sc);
                    if (absacc_out) absacc_out[i * M + o] = mag + fabs(bc) + fabs(be);
                }
            }
        }
        /* GroupNorm statistics, two-pass */
        double sum = 0.0;
        for (long o = 0; o < M; ++o) sum += a[o];
        double mu = sum / (double)M;
        double ss = 0.0;
        for (long o = 0; o < M; ++o) { double d = a[o] - mu; ss += d * d; }
        double var = ss / (double)M;
        double inv = 1.0 / sqrt(var + eps);
        for (long kk = 0; kk < kg; ++kk) {
            long k = G * kg + kk;
            double ga = (double)gamma[k], be = (double)beta[k];
            for (long o = kk * PQ; o < (kk + 1) * PQ; ++o)
                y_out[i * M + o] = (a[o] - mu) * inv * ga + be;
        }
        if (mean_out) mean_out[i] = mu;
        if (var_out) var_out[i] = var;
        if (!a_out) free(a);
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* Threads the OpenMP runtime will use (reported with CPU timings). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for later calls (the benchmark times the oracle on all host cores
 * and on one); n < 1 leaves the setting unchanged.  Results do not depend on
 * it: threads only split independent outputs. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
