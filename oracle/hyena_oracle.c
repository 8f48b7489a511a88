/*
 * hyena_oracle.c -- float64 CPU oracle for the Hyena gated long convolution.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file.  Only tests/, __graft_entry__.smoke() and the cpu_baseline
 * leg of bench.py use it.  It shares no code, header, table or constant with
 * the CUDA library: it is written from the definitions on the pages.
 *
 * Sources (page title, section):
 *  [P4] "HyenaDNA operator walk-through" (adg.csdn.net/695241245b9f5f31781b4602),
 *       section 二.1 (HyenaOperator.__init__ / forward): in_proj output is
 *       rearranged to [b, d, l]; short_filter is a depthwise Conv1d with kernel
 *       3, padding 2, groups = inner width, truncated to the first l samples;
 *       the result is split channel-wise into x0..x(order-1) and v; for each
 *       o, x_i in enumerate(reversed(x[1:])): v = v * x_i, then
 *       v = fftconv(v, k[o], bias[o]); finally y = v * x[0].
 *       Section 二.2 (HyenaFilter.forward): fftconv(x, k, bias) is the FFT
 *       evaluation of a long causal convolution ("equivalent to Conv1d(x, k)").
 *  [P5] "Native Multi-Dimensional Subquadratic Operators via Input Dependent
 *       Long Convolutions" (gist.science summary), 方法论 (原生 ND 卷积,
 *       边界处理): the N-D global convolution is evaluated with an N-D FFT;
 *       the non-circular form zero-pads every axis to twice its length.
 *
 * Readings of points the pages leave open:
 *  - fftconv(x, k, D) = (k * x)[0:L] + D * x  (causal linear convolution plus
 *    a per-channel skip); evaluated either by its direct sum or by a
 *    zero-padded FFT of size >= 2L.
 *  - Conv1d is a cross-correlation: with padding 2 and the first L outputs
 *    kept, tap w[2] multiplies the current sample, w[0] the sample two back.
 *  - 2-D form: v[p][q] = sum_{i<=p, j<=q} K[i][j] w[p-i][q-j] + D w[p][q]
 *    (kernel anchored at (0,0), output cropped to [0:H, 0:W]).
 *  - 3-D form ([P5] 原生 ND 卷积 on L1 x L2 x L3 grids, e.g. 3-D medical
 *    volumes): v[a][p][q] = sum_{h<=a, i<=p, j<=q} K[h][i][j]
 *    w[a-h][p-i][q-j] + D w[a][p][q], kernel anchored at the origin, output
 *    cropped to the input grid (zero padding every axis to twice its length).
 *  - 2-D circular form ([P5] 边界处理: circular convolution for periodic
 *    systems, no padding): v[p][q] = sum_{i<H, j<W} K[i][j]
 *    w[(p-i) mod H][(q-j) mod W] + D w[p][q], with K on the same H x W grid.
 *
 * Every function works in double precision on exactly the values it is
 * given.  Radix-2 FFT twiddles come from cos/sin of the C library in double,
 * computed per index (no recurrence).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_PI 3.14159265358979323846264338327950288

/* ---------------------------------------------------------------------- */
/* Short depthwise causal conv, width 3 ([P4] 二.1, short_filter).        */
/* One channel row of length L.  bias may be 0.                           */
/* ---------------------------------------------------------------------- */
void oracle_shortconv_row(const double *u, double *out, const double w[3],
                          double bias, int64_t L)
{
    for (int64_t t = 0; t < L; ++t) {
        double um2 = (t >= 2) ? u[t - 2] : 0.0;
        double um1 = (t >= 1) ? u[t - 1] : 0.0;
        out[t] = w[0] * um2 + w[1] * um1 + w[2] * u[t] + bias;
    }
}

/* u: [rows][L] where row r uses weights w[(r % Ctot)*3 ..] and bias[r % Ctot]. */
void oracle_shortconv(const double *u, double *out, const double *w,
                      const double *bias, int64_t B, int64_t Ctot, int64_t L)
{
    int64_t rows = B * Ctot;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t j = r % Ctot;
        oracle_shortconv_row(u + r * L, out + r * L, w + 3 * j,
                             bias ? bias[j] : 0.0, L);
    }
}

/* ---------------------------------------------------------------------- */
/* Direct causal convolution with skip: the plain definition of fftconv.  */
/* out[t] = sum_{tau=0..t} k[tau] x[t-tau] + D x[t],  t < L.              */
/* ---------------------------------------------------------------------- */
void oracle_causal_conv_direct(const double *k, double D, const double *x,
                               double *out, int64_t L)
{
    for (int64_t t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int64_t tau = 0; tau <= t; ++tau) acc += k[tau] * x[t - tau];
        out[t] = acc + D * x[t];
    }
}

/* ---------------------------------------------------------------------- */
/* Iterative radix-2 complex FFT (Cooley-Tukey, bit reversal first).      */
/* sign = -1: forward  X[f] = sum_n x[n] exp(-2 pi i f n / n_)             */
/* sign = +1: unnormalised inverse.  n must be a power of two.            */
/* ---------------------------------------------------------------------- */
void oracle_fft(double *re, double *im, int64_t n, int sign)
{
    if (n <= 1) return;
    /* bit reversal permutation */
    for (int64_t i = 1, j = 0; i < n; ++i) {
        int64_t bit = n >> 1;
        for (; j & bit; bit >>= 1) j ^= bit;
        j ^= bit;
        if (i < j) {
            double t = re[i]; re[i] = re[j]; re[j] = t;
            t = im[i]; im[i] = im[j]; im[j] = t;
        }
    }
    /* twiddle table cos/sin(2 pi j / n), j < n/2, each from the C library */
    double *cw = (double *)malloc(sizeof(double) * (size_t)(n / 2));
    double *sw = (double *)malloc(sizeof(double) * (size_t)(n / 2));
    for (int64_t j = 0; j < n / 2; ++j) {
        double a = 2.0 * ORACLE_PI * (double)j / (double)n;
        cw[j] = cos(a);
        sw[j] = sin(a) * (double)sign;
    }
    for (int64_t len = 2; len <= n; len <<= 1) {
        int64_t half = len >> 1, step = n / len;
        for (int64_t s = 0; s < n; s += len) {
            for (int64_t j = 0; j < half; ++j) {
                double wr = cw[j * step], wi = sw[j * step];
                int64_t a = s + j, b = s + j + half;
                double tr = re[b] * wr - im[b] * wi;
                double ti = re[b] * wi + im[b] * wr;
                re[b] = re[a] - tr; im[b] = im[a] - ti;
                re[a] += tr;        im[a] += ti;
            }
        }
    }
    free(cw);
    free(sw);
}

static int64_t next_pow2(int64_t x)
{
    int64_t n = 1;
    while (n < x) n <<= 1;
    return n;
}

/* Causal convolution with skip by a zero-padded FFT of size n >= 2L-1
 * (n = next power of two >= 2L).  Same result as the direct sum. */
void oracle_causal_conv_fft(const double *k, double D, const double *x,
                            double *out, int64_t L)
{
    int64_t n = next_pow2(2 * L);
    double *kr = (double *)calloc((size_t)n, sizeof(double));
    double *ki = (double *)calloc((size_t)n, sizeof(double));
    double *xr = (double *)calloc((size_t)n, sizeof(double));
    double *xi = (double *)calloc((size_t)n, sizeof(double));
    memcpy(kr, k, sizeof(double) * (size_t)L);
    memcpy(xr, x, sizeof(double) * (size_t)L);
    oracle_fft(kr, ki, n, -1);
    oracle_fft(xr, xi, n, -1);
    for (int64_t f = 0; f < n; ++f) {
        double a = xr[f] * kr[f] - xi[f] * ki[f];
        double b = xr[f] * ki[f] + xi[f] * kr[f];
        xr[f] = a; xi[f] = b;
    }
    oracle_fft(xr, xi, n, +1);
    for (int64_t t = 0; t < L; ++t) out[t] = xr[t] / (double)n + D * x[t];
    free(kr); free(ki); free(xr); free(xi);
}

/* ---------------------------------------------------------------------- */
/* 2-D non-circular convolution ([P5] 原生 ND 卷积, 边界处理).            */
/* out[p][q] = sum_{i<=p, j<=q} K[i][j] x[p-i][q-j] + D x[p][q]           */
/* ---------------------------------------------------------------------- */
void oracle_conv2d_direct(const double *K, double D, const double *x,
                          double *out, int64_t H, int64_t W)
{
    for (int64_t p = 0; p < H; ++p)
        for (int64_t q = 0; q < W; ++q) {
            double acc = 0.0;
            for (int64_t i = 0; i <= p; ++i)
                for (int64_t j = 0; j <= q; ++j)
                    acc += K[i * W + j] * x[(p - i) * W + (q - j)];
            out[p * W + q] = acc + D * x[p * W + q];
        }
}

/* 2-D FFT of an nh x nw complex array: rows then columns, radix-2 each. */
static void oracle_fft2(double *re, double *im, int64_t nh, int64_t nw, int sign)
{
    for (int64_t r = 0; r < nh; ++r) oracle_fft(re + r * nw, im + r * nw, nw, sign);
    double *cr = (double *)malloc(sizeof(double) * (size_t)nh);
    double *ci = (double *)malloc(sizeof(double) * (size_t)nh);
    for (int64_t c = 0; c < nw; ++c) {
        for (int64_t r = 0; r < nh; ++r) { cr[r] = re[r * nw + c]; ci[r] = im[r * nw + c]; }
        oracle_fft(cr, ci, nh, sign);
        for (int64_t r = 0; r < nh; ++r) { re[r * nw + c] = cr[r]; im[r * nw + c] = ci[r]; }
    }
    free(cr); free(ci);
}

/* Zero-padded (2H x 2W, rounded up to powers of two) 2-D FFT convolution. */
void oracle_conv2d_fft(const double *K, double D, const double *x,
                       double *out, int64_t H, int64_t W)
{
    int64_t nh = next_pow2(2 * H), nw = next_pow2(2 * W);
    size_t n = (size_t)(nh * nw);
    double *kr = (double *)calloc(n, sizeof(double));
    double *ki = (double *)calloc(n, sizeof(double));
    double *xr = (double *)calloc(n, sizeof(double));
    double *xi = (double *)calloc(n, sizeof(double));
    for (int64_t p = 0; p < H; ++p)
        for (int64_t q = 0; q < W; ++q) {
            kr[p * nw + q] = K[p * W + q];
            xr[p * nw + q] = x[p * W + q];
        }
    oracle_fft2(kr, ki, nh, nw, -1);
    oracle_fft2(xr, xi, nh, nw, -1);
    for (size_t f = 0; f < n; ++f) {
        double a = xr[f] * kr[f] - xi[f] * ki[f];
        double b = xr[f] * ki[f] + xi[f] * kr[f];
        xr[f] = a; xi[f] = b;
    }
    oracle_fft2(xr, xi, nh, nw, +1);
    double scale = 1.0 / (double)n;
    for (int64_t p = 0; p < H; ++p)
        for (int64_t q = 0; q < W; ++q)
            out[p * W + q] = xr[p * nw + q] * scale + D * x[p * W + q];
    free(kr); free(ki); free(xr); free(xi);
}

/* ---------------------------------------------------------------------- */
/* 2-D circular convolution ([P5] 边界处理, periodic systems).            */
/* out[p][q] = sum_{i<H, j<W} K[i][j] x[(p-i) mod H][(q-j) mod W]         */
/*             + D x[p][q]                                               */
/* ---------------------------------------------------------------------- */
void oracle_conv2d_circ_direct(const double *K, double D, const double *x,
                               double *out, int64_t H, int64_t W)
{
    for (int64_t p = 0; p < H; ++p)
        for (int64_t q = 0; q < W; ++q) {
            double acc = 0.0;
            for (int64_t i = 0; i < H; ++i)
                for (int64_t j = 0; j < W; ++j)
                    acc += K[i * W + j] * x[((p - i + H) % H) * W + ((q - j + W) % W)];
            out[p * W + q] = acc + D * x[p * W + q];
        }
}

/* The same through an H x W FFT (powers of two; no padding: the DFT's own
 * periodicity is the circular boundary). */
void oracle_conv2d_circ_fft(const double *K, double D, const double *x,
                            double *out, int64_t H, int64_t W)
{
    size_t n = (size_t)(H * W);
    double *kr = (double *)malloc(sizeof(double) * n);
    double *ki = (double *)calloc(n, sizeof(double));
    double *xr = (double *)malloc(sizeof(double) * n);
    double *xi = (double *)calloc(n, sizeof(double));
    memcpy(kr, K, sizeof(double) * n);
    memcpy(xr, x, sizeof(double) * n);
    oracle_fft2(kr, ki, H, W, -1);
    oracle_fft2(xr, xi, H, W, -1);
    for (size_t f = 0; f < n; ++f) {
        double a = xr[f] * kr[f] - xi[f] * ki[f];
        double b = xr[f] * ki[f] + xi[f] * kr[f];
        xr[f] = a; xi[f] = b;
    }
    oracle_fft2(xr, xi, H, W, +1);
    double scale = 1.0 / (double)n;
    for (size_t t = 0; t < n; ++t) out[t] = xr[t] * scale + D * x[t];
    free(kr); free(ki); free(xr); free(xi);
}

/* ---------------------------------------------------------------------- */
/* 3-D non-circular convolution ([P5] 原生 ND 卷积, 边界处理).            */
/* out[a][p][q] = sum_{h<=a, i<=p, j<=q} K[h][i][j] x[a-h][p-i][q-j]      */
/*                + D x[a][p][q]                                         */
/* ---------------------------------------------------------------------- */
void oracle_conv3d_direct(const double *K, double D, const double *x,
                          double *out, int64_t N1, int64_t N2, int64_t N3)
{
    for (int64_t a = 0; a < N1; ++a)
        for (int64_t p = 0; p < N2; ++p)
            for (int64_t q = 0; q < N3; ++q) {
                double acc = 0.0;
                for (int64_t h = 0; h <= a; ++h)
                    for (int64_t i = 0; i <= p; ++i)
                        for (int64_t j = 0; j <= q; ++j)
                            acc += K[(h * N2 + i) * N3 + j] * x[((a - h) * N2 + (p - i)) * N3 + (q - j)];
                out[(a * N2 + p) * N3 + q] = acc + D * x[(a * N2 + p) * N3 + q];
            }
}

/* 3-D FFT of an n1 x n2 x n3 complex array: each axis in turn, radix-2. */
static void oracle_fft3(double *re, double *im, int64_t n1, int64_t n2, int64_t n3, int sign)
{
    int64_t nmax = n1 > n2 ? (n1 > n3 ? n1 : n3) : (n2 > n3 ? n2 : n3);
    double *lr = (double *)malloc(sizeof(double) * (size_t)nmax);
    double *li = (double *)malloc(sizeof(double) * (size_t)nmax);
    for (int64_t a = 0; a < n1; ++a)            /* axis 3: contiguous lines */
        for (int64_t p = 0; p < n2; ++p)
            oracle_fft(re + (a * n2 + p) * n3, im + (a * n2 + p) * n3, n3, sign);
    for (int64_t a = 0; a < n1; ++a)            /* axis 2 */
        for (int64_t q = 0; q < n3; ++q) {
            for (int64_t p = 0; p < n2; ++p) { lr[p] = re[(a * n2 + p) * n3 + q]; li[p] = im[(a * n2 + p) * n3 + q]; }
            oracle_fft(lr, li, n2, sign);
            for (int64_t p = 0; p < n2; ++p) { re[(a * n2 + p) * n3 + q] = lr[p]; im[(a * n2 + p) * n3 + q] = li[p]; }
        }
    for (int64_t p = 0; p < n2; ++p)            /* axis 1 */
        for (int64_t q = 0; q < n3; ++q) {
            for (int64_t a = 0; a < n1; ++a) { lr[a] = re[(a * n2 + p) * n3 + q]; li[a] = im[(a * n2 + p) * n3 + q]; }
            oracle_fft(lr, li, n1, sign);
            for (int64_t a = 0; a < n1; ++a) { re[(a * n2 + p) * n3 + q] = lr[a]; im[(a * n2 + p) * n3 + q] = li[a]; }
        }
    free(lr); free(li);
}

/* Zero-padded (every axis to twice its length, powers of two) 3-D FFT convolution. */
void oracle_conv3d_fft(const double *K, double D, const double *x,
                       double *out, int64_t N1, int64_t N2, int64_t N3)
{
    int64_t n1 = next_pow2(2 * N1), n2 = next_pow2(2 * N2), n3 = next_pow2(2 * N3);
    size_t n = (size_t)(n1 * n2 * n3);
    double *kr = (double *)calloc(n, sizeof(double));
    double *ki = (double *)calloc(n, sizeof(double));
    double *xr = (double *)calloc(n, sizeof(double));
    double *xi = (double *)calloc(n, sizeof(double));
    for (int64_t a = 0; a < N1; ++a)
        for (int64_t p = 0; p < N2; ++p)
            for (int64_t q = 0; q < N3; ++q) {
                kr[(a * n2 + p) * n3 + q] = K[(a * N2 + p) * N3 + q];
                xr[(a * n2 + p) * n3 + q] = x[(a * N2 + p) * N3 + q];
            }
    oracle_fft3(kr, ki, n1, n2, n3, -1);
    oracle_fft3(xr, xi, n1, n2, n3, -1);
    for (size_t f = 0; f < n; ++f) {
        double a = xr[f] * kr[f] - xi[f] * ki[f];
        double b = xr[f] * ki[f] + xi[f] * kr[f];
        xr[f] = a; xi[f] = b;
    }
    oracle_fft3(xr, xi, n1, n2, n3, +1);
    double scale = 1.0 / (double)n;
    for (int64_t a = 0; a < N1; ++a)
        for (int64_t p = 0; p < N2; ++p)
            for (int64_t q = 0; q < N3; ++q)
                out[(a * N2 + p) * N3 + q] = xr[(a * n2 + p) * n3 + q] * scale + D * x[(a * N2 + p) * N3 + q];
    free(kr); free(ki); free(xr); free(xi);
}

/*
 * The operator on nrows self-contained 3-D rows (N1 x N2 x N3 each, no short
 * conv: the pages give none for N-D): u_rows [nrows][order+1][n], k_rows
 * [nrows][order-1][n], D_rows [nrows][order-1], y [nrows][n]; the same gating
 * as the 1-D and 2-D forms ([P4] 二.1).  method: 1 direct, 2 FFT.
 */
int oracle_hyena_rows3(const double *u_rows, const double *k_rows, const double *D_rows, int64_t nrows,
                       int64_t N1, int64_t N2, int64_t N3, int order, int method, int nthreads, double *y)
{
    if (!u_rows || !k_rows || !D_rows || !y || nrows < 0 || N1 < 1 || N2 < 1 || N3 < 1 || order < 2)
        return -1;
    int64_t n = N1 * N2 * N3;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        const double *x = u_rows + r * (order + 1) * n;
        double *v = (double *)malloc(sizeof(double) * (size_t)n);
        double *w = (double *)malloc(sizeof(double) * (size_t)n);
        memcpy(v, x + (int64_t)order * n, sizeof(double) * (size_t)n);
        for (int s = 1; s <= order - 1; ++s) {
            const double *g = x + (int64_t)(order - s) * n;   /* gate x_{order-s} */
            for (int64_t t = 0; t < n; ++t) w[t] = g[t] * v[t];
            const double *ks = k_rows + (r * (order - 1) + (s - 1)) * n;
            double Ds = D_rows[r * (order - 1) + (s - 1)];
            if (method == 1) oracle_conv3d_direct(ks, Ds, w, v, N1, N2, N3);
            else             oracle_conv3d_fft(ks, Ds, w, v, N1, N2, N3);
        }
        for (int64_t t = 0; t < n; ++t) y[r * n + t] = x[t] * v[t];
        free(v); free(w);
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* The Hyena operator on one (b, c) row ([P4] 二.1 forward loop).         */
/*                                                                        */
/* Each row is self-contained (n = L in 1-D, n = H*W in 2-D):             */
/*  u_row  : [order+1][n]  projected chunks x0..x(order-1), v of (b, c),  */
/*           before the short conv                                       */
/*  k_row  : [order-1][n]  long filter of channel c for each step         */
/*  D_row  : [order-1]     skip ("bias") of channel c for each step       */
/*  scw_row: [order+1][3]  short-conv taps of the chunk channels, or NULL */
/*  scb_row: [order+1]     short-conv bias, or NULL                       */
/*  method : 1 direct sums, 2 FFT, 0 direct when small else FFT           */
/*  ndim   : 1, 2 (non-circular) or 3 meaning the 2-D circular form       */
/* Step s = 1..order-1 uses gate x_{order-s}, filter k[s-1], skip D[s-1]. */
/* ---------------------------------------------------------------------- */
static void hyena_row(const double *u_row, const double *k_row, const double *D_row,
                      const double *scw_row, const double *scb_row,
                      int64_t H, int64_t W, int ndim, int order, int method,
                      double *y_row)
{
    int64_t n = H * W;
    double *x = (double *)malloc(sizeof(double) * (size_t)(n * (order + 1)));
    double *w = (double *)malloc(sizeof(double) * (size_t)n);
    double *vn = (double *)malloc(sizeof(double) * (size_t)n);
    for (int j = 0; j <= order; ++j) {
        const double *src = u_row + (int64_t)j * n;
        double *dst = x + (int64_t)j * n;
        if (scw_row) {
            /* [P4] 二.1: short_filter (depthwise, causal after truncation) */
            oracle_shortconv_row(src, dst, scw_row + 3 * j, scb_row ? scb_row[j] : 0.0, n);
        } else {
            memcpy(dst, src, sizeof(double) * (size_t)n);
        }
    }
    double *v = x + (int64_t)order * n;     /* value branch: last chunk */
    /* [P4] 二.1: for o, x_i in enumerate(reversed(x[1:])): gate, then conv */
    for (int s = 1; s <= order - 1; ++s) {
        const double *gate = x + (int64_t)(order - s) * n;
        const double *ks = k_row + (int64_t)(s - 1) * n;
        double Ds = D_row[s - 1];
        for (int64_t t = 0; t < n; ++t) w[t] = gate[t] * v[t];
        int direct = (method == 1) ||
                     (method == 0 && ((ndim == 1 && W <= 4096) ||
                                      (ndim != 1 && H <= 64 && W <= 64)));
        if (ndim == 1) {
            if (direct) oracle_causal_conv_direct(ks, Ds, w, vn, W);
            else        oracle_causal_conv_fft(ks, Ds, w, vn, W);
        } else if (ndim == 2) {
            if (direct) oracle_conv2d_direct(ks, Ds, w, vn, H, W);
            else        oracle_conv2d_fft(ks, Ds, w, vn, H, W);
        } else {
            if (direct) oracle_conv2d_circ_direct(ks, Ds, w, vn, H, W);
            else        oracle_conv2d_circ_fft(ks, Ds, w, vn, H, W);
        }
        memcpy(v, vn, sizeof(double) * (size_t)n);
    }
    /* [P4] 二.1: y = v * x[0] */
    for (int64_t t = 0; t < n; ++t) y_row[t] = x[t] * v[t];
    free(x); free(w); free(vn);
}

/*
 * The operator over nrows self-contained rows (layouts as for hyena_row,
 * stacked row-major).  y: [nrows][n].  nthreads <= 0: OpenMP default.
 * Returns 0 on success, -1 on bad arguments.
 */
int oracle_hyena_rows(const double *u_rows, const double *k_rows, const double *D_rows,
                      const double *scw_rows, const double *scb_rows, int64_t nrows,
                      int64_t H, int64_t W, int ndim, int order, int method,
                      int nthreads, double *y)
{
    if (!u_rows || !k_rows || !D_rows || !y || nrows < 0 || H < 1 || W < 1 || order < 2)
        return -1;
    if (ndim != 1 && ndim != 2 && ndim != 3) return -1;
    if (ndim == 1 && H != 1) return -1;
    if (ndim != 1 && scw_rows) return -1;
    int64_t n = H * W;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        hyena_row(u_rows + i * (order + 1) * n, k_rows + i * (order - 1) * n,
                  D_rows + i * (order - 1),
                  scw_rows ? scw_rows + i * (order + 1) * 3 : NULL,
                  scb_rows ? scb_rows + i * (order + 1) : NULL,
                  H, W, ndim, order, method, y + i * n);
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Split of the projected stream ([P4] 二.1: after in_proj and the short   */
/* filter the stream u[b][(order+1) d][l] is cut along the channel axis   */
/* into blocks of d, `*x, v = uc.split(d_model, dim=1)`, so x_0..x_(order-1) */
/* come first and v last).  Chunk j of row (b, c) is channel j*C + c of   */
/* batch b.  The short filter is depthwise over all (order+1) C channels, */
/* so its taps and bias split the same way.  The long filters            */
/* k[order-1][FC][n] and skips D[order-1][FC] of step s are taken at      */
/* index c (shared by the batch, [P4] 二.1 'l (o d) -> o d l'), or at     */
/* b*C + c when every sample brings its own filters ([P5] 方法论, input-   */
/* dependent kernels; FC = B*C).                                          */
/*                                                                        */
/* Stored values are read exactly: kind 0 = float64, 1 = float32,         */
/* 2 = bfloat16 bit patterns (the upper 16 bits of an IEEE binary32).     */
/* ---------------------------------------------------------------------- */
static double stored_value(const void *base, int kind, int64_t i)
{
    if (kind == 0) return ((const double *)base)[i];
    if (kind == 1) return (double)((const float *)base)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Gathers the self-contained rows (layouts of oracle_hyena_rows) of the
 * listed row ids r = b*C + c from the stacked tensors.
 *   u     [B][(order+1)*C][n] (u_kind)      k  [order-1][FC][n] (k_kind)
 *   D     [order-1][FC] or NULL (= 0)       sc_w [(order+1)*C][3] or NULL,
 *   sc_b  [(order+1)*C] or NULL (= 0)
 * Outputs: u_rows [R][order+1][n], k_rows [R][order-1][n], D_rows
 * [R][order-1], scw_rows [R][order+1][3] and scb_rows [R][order+1] (both
 * only when sc_w is given).  Returns 0, or -1 on bad arguments.
 */
int oracle_split_rows(const void *u, int u_kind, const void *k, int k_kind, const double *D,
                      const double *sc_w, const double *sc_b, int64_t B, int64_t C, int order,
                      int64_t n, int per_sample, const int64_t *rows, int64_t nrows,
                      double *u_rows, double *k_rows, double *D_rows, double *scw_rows,
                      double *scb_rows)
{
    if (!u || !k || !rows || !u_rows || !k_rows || !D_rows || B < 1 || C < 1 || order < 2 || n < 1)
        return -1;
    if (u_kind < 0 || u_kind > 2 || k_kind < 0 || k_kind > 2) return -1;
    if (sc_w && (!scw_rows || !scb_rows)) return -1;
    const int64_t Ctot = (int64_t)(order + 1) * C;
    const int64_t FC = per_sample ? B * C : C;
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t r = rows[i];
        if (r < 0 || r >= B * C) return -1;
        const int64_t b = r / C, c = r % C;
        for (int j = 0; j <= order; ++j) {
            const int64_t ch = (int64_t)j * C + c;             /* block j, channel c */
            const int64_t src = (b * Ctot + ch) * n;
            double *dst = u_rows + (i * (order + 1) + j) * n;
            for (int64_t t = 0; t < n; ++t) dst[t] = stored_value(u, u_kind, src + t);
            if (sc_w) {
                for (int m = 0; m < 3; ++m) scw_rows[(i * (order + 1) + j) * 3 + m] = sc_w[ch * 3 + m];
                scb_rows[i * (order + 1) + j] = sc_b ? sc_b[ch] : 0.0;
            }
        }
        const int64_t f = per_sample ? b * C + c : c;          /* filter index */
        for (int s = 0; s < order - 1; ++s) {
            const int64_t src = ((int64_t)s * FC + f) * n;
            double *dst = k_rows + (i * (order - 1) + s) * n;
            for (int64_t t = 0; t < n; ++t) dst[t] = stored_value(k, k_kind, src + t);
            D_rows[i * (order - 1) + s] = D ? D[(int64_t)s * FC + f] : 0.0;
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Projections around the operator ([P4] 二.1, HyenaOperator: in_proj =   */
/* nn.Linear(d_model, (order+1) d_model) on u[b][l][:], then              */
/* rearrange 'b l d -> b d l'; at the end y = rearrange(v * x[0],         */
/* 'b d l -> b l d') and out_proj = nn.Linear(d_model, d_model)).          */
/* nn.Linear(x) = x W^T + bias with the weight stored W[out][in].          */
/* ---------------------------------------------------------------------- */
/* x [B][L][D] -> u [B][J][L]:  u[b][j][l] = sum_i x[b][l][i] W[j][i] + bias[j] */
void oracle_in_proj(const double *x, const double *W, const double *bias, int64_t B, int64_t L,
                    int64_t D, int64_t J, double *u)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t j = 0; j < J; ++j) {
            for (int64_t l = 0; l < L; ++l) {
                double acc = bias ? bias[j] : 0.0;
                for (int64_t i = 0; i < D; ++i) acc += x[(b * L + l) * D + i] * W[j * D + i];
                u[(b * J + j) * L + l] = acc;
            }
        }
    }
}

/* y [B][D][L] -> out [B][L][J]:  out[b][l][j] = sum_i y[b][i][l] W[j][i] + bias[j] */
void oracle_out_proj(const double *y, const double *W, const double *bias, int64_t B, int64_t L,
                     int64_t D, int64_t J, double *out)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t l = 0; l < L; ++l) {
            for (int64_t j = 0; j < J; ++j) {
                double acc = bias ? bias[j] : 0.0;
                for (int64_t i = 0; i < D; ++i) acc += y[(b * D + i) * L + l] * W[j * D + i];
                out[(b * L + l) * J + j] = acc;
            }
        }
    }
}

/* Number of threads an OpenMP parallel region would use. */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
