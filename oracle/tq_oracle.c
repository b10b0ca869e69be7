/*
 * tq_oracle.c -- plain, slow, obviously correct CPU oracle for the
 * TurboQuant inner-product vector quantizer (encode + score + top-k).
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests/, by the smoke check and by the
 * CPU-baseline leg of bench.py.  It shares no code with the CUDA library.
 *
 * Page references (titles of the reference pages):
 *   [QPD] quant_prune_distill #674 "TurboQuant" summary
 *         - para "two problem statements": MSE-optimal and inner-product-
 *           optimal quantization, the latter unbiased;
 *         - para "for MSE-optimised TurboQuant": random orthogonal rotation
 *           (not Hadamard), then a Lloyd-Max grid for the target bit width;
 *         - para "for inner product": MSE quantizer at (bits - 1), residual
 *           quantized with 1-bit QJL: random matrix, then the sign;
 *           dequantization is the inverse rotation and renormalisation.
 *   [RSC] RecSysChannel #256 "TurboQuant: Redefining AI efficiency with
 *         extreme compression"
 *         - para "uniform on the unit sphere": coordinates nearly N(0,1/d),
 *           nearly independent;
 *         - item 1): thresholds computed in advance for that distribution;
 *         - item 2): a 1-bit per-coordinate correction making the inner
 *           product estimate unbiased;
 *         - caveat 1: vectors must be normalised and multiplied by a random
 *           matrix.
 *   [SEA] seeallochnaya #3476
 *         - step 1): random rotation spreads outliers; 1-D k-means
 *           boundaries denser in the centre; each coordinate rounded
 *           independently on the fixed grid;
 *         - step 2): residual multiplied by a random matrix, keep the sign.
 *
 * Readings where the pages are silent (the plainest reading each time):
 *   R1  random numbers: SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) in
 *       counter form, keyed by (seed, stream); Box-Muller for Gaussians.
 *   R2  Pi = Q * diag(sign R_jj) from the Householder QR of a Gaussian
 *       matrix (the Haar-distributed orthogonal matrix).
 *   R3  S has iid N(0,1) entries (the sqrt(pi/2)/d constant is exact only
 *       for Gaussian rows).
 *   R4  codebook: Lloyd-Max for N(0,1), scaled by 1/sqrt(d).
 *   R5  a value exactly on a boundary goes to the upper cell; sign(0) = +1.
 *   R6  the estimator s = |x| (<Pi q, yhat> + |r| sqrt(pi/2)/d <S Pi q, z>),
 *       z in {-1,+1}^d.
 *   R7  code layout (blocks of 32 coordinates, b words each), below.
 */
#include "tq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define TQO_GAMMA 0x9E3779B97F4A7C15ULL

/* ------------------------------------------------------------------------ */
/* R1: SplitMix64.  The generator advances its state by the golden-ratio     */
/* increment and returns a bijective 64-bit mix of the state.  The i-th      */
/* output (i = 0, 1, ...) of a stream started at state s0 is therefore       */
/* mix64(s0 + (i + 1) * gamma), which is what makes it counter-based.       */
/* ------------------------------------------------------------------------ */
uint64_t tqo_mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Starting state of stream `stream` under `seed`:
 * s0 = mix64(seed XOR stream * gamma).  Stream 0 = Pi, 1 = S. */
uint64_t tqo_stream_key(uint64_t seed, uint64_t stream)
{
    return tqo_mix64(seed ^ (stream * TQO_GAMMA));
}

uint64_t tqo_u64(uint64_t seed, uint64_t stream, uint64_t i)
{
    uint64_t s0 = tqo_stream_key(seed, stream);
    return tqo_mix64(s0 + (i + 1) * TQO_GAMMA);
}

/* Box-Muller (1958).  Pair m uses outputs 2m and 2m+1:
 *   u1 = ((a >> 11) + 1) * 2^-53  in (0, 1]
 *   u2 = (b >> 11) * 2^-53         in [0, 1)
 *   rho = sqrt(-2 ln u1);  g[2m] = rho cos(2 pi u2);  g[2m+1] = rho sin(2 pi u2)
 * A count that is odd drops the last sine. */
void tqo_gaussian(uint64_t seed, uint64_t stream, int64_t count, double *out)
{
    const double two_m53 = 1.0 / 9007199254740992.0; /* 2^-53 */
    const double two_pi = 6.283185307179586476925286766559;
    int64_t m;
    for (m = 0; 2 * m < count; m++) {
        uint64_t a = tqo_u64(seed, stream, (uint64_t)(2 * m));
        uint64_t b = tqo_u64(seed, stream, (uint64_t)(2 * m + 1));
        double u1 = (double)((a >> 11) + 1) * two_m53;
        double u2 = (double)(b >> 11) * two_m53;
        double rho = sqrt(-2.0 * log(u1));
        out[2 * m] = rho * cos(two_pi * u2);
        if (2 * m + 1 < count)
            out[2 * m + 1] = rho * sin(two_pi * u2);
    }
}

/* ------------------------------------------------------------------------ */
/* R4: Lloyd-Max quantizer for the standard normal ([QPD] "Lloyd-Max grid";  */
/* [SEA] "1-D k-means, boundaries denser in the centre"; [RSC] item 1       */
/* "thresholds computed in advance").  Alternate the two optimality          */
/* conditions: boundaries at midpoints of neighbouring centroids, centroids  */
/* at the conditional mean of their cell,                                    */
/*   c_j = (phi(b_{j-1}) - phi(b_j)) / (Phi(b_j) - Phi(b_{j-1})).           */
/* The density is log-concave, so the fixed point is unique and any start    */
/* converges.  The codebook is kept exactly symmetric (c_{L-1-j} = -c_j).   */
/* ------------------------------------------------------------------------ */
static double tqo_phi(double t)
{
    if (isinf(t)) return 0.0;
    return exp(-0.5 * t * t) / sqrt(2.0 * 3.14159265358979323846);
}

/* P(a < X <= b) for X ~ N(0,1), computed from the tail on the side where
 * both limits lie to avoid cancellation. */
static double tqo_mass(double a, double b)
{
    const double r2 = 1.4142135623730950488;
    if (a >= 0.0) return 0.5 * (erfc(a / r2) - erfc(b / r2));
    if (b <= 0.0) return 0.5 * (erfc(-b / r2) - erfc(-a / r2));
    return 1.0 - 0.5 * erfc(-a / r2) - 0.5 * erfc(b / r2);
}

int tqo_lloyd_max(int levels, double *c, double *beta, double *distortion, int *iters)
{
    int L = levels, j, it;
    double *lo, *hi;
    if (L < 1 || L > 256) return -1;
    if (L == 1) {
        c[0] = 0.0;
        if (distortion) *distortion = 1.0;
        if (iters) *iters = 0;
        return 0;
    }
    lo = (double *)malloc(sizeof(double) * (size_t)L);
    hi = (double *)malloc(sizeof(double) * (size_t)L);
    for (j = 0; j < L; j++) c[j] = -3.0 + 6.0 * (j + 0.5) / L;
    for (it = 0; it < 1000000; it++) {
        double maxdelta = 0.0;
        for (j = 0; j + 1 < L; j++) beta[j] = 0.5 * (c[j] + c[j + 1]);
        for (j = 0; j < L; j++) {
            double a = (j == 0) ? -INFINITY : beta[j - 1];
            double b = (j == L - 1) ? INFINITY : beta[j];
            double nc = (tqo_phi(a) - tqo_phi(b)) / tqo_mass(a, b);
            lo[j] = nc;
        }
        for (j = 0; j < L; j++) { /* enforce exact symmetry */
            double s = 0.5 * (lo[j] - lo[L - 1 - j]);
            hi[j] = s;
        }
        for (j = 0; j < L; j++) {
            double dlt = fabs(hi[j] - c[j]);
            if (dlt > maxdelta) maxdelta = dlt;
            c[j] = hi[j];
        }
        if (maxdelta < 1e-13) { it++; break; }
    }
    for (j = 0; j + 1 < L; j++) beta[j] = 0.5 * (c[j] + c[j + 1]);
    if (distortion) {
        /* D = E[(X - Q(X))^2] = sum over cells [a, b] of
         *   int (x - c_j)^2 phi = P + a phi(a) - b phi(b)
         *                         - 2 c_j (phi(a) - phi(b)) + c_j^2 P,
         * using int x phi = phi(a) - phi(b) and
         *       int x^2 phi = P + a phi(a) - b phi(b)  over [a, b]. */
        double acc = 0.0;
        for (j = 0; j < L; j++) {
            double a = (j == 0) ? -INFINITY : beta[j - 1];
            double b = (j == L - 1) ? INFINITY : beta[j];
            double P = tqo_mass(a, b);
            double aphi = isinf(a) ? 0.0 : a * tqo_phi(a);
            double bphi = isinf(b) ? 0.0 : b * tqo_phi(b);
            acc += P + aphi - bphi - 2.0 * c[j] * (tqo_phi(a) - tqo_phi(b))
                   + c[j] * c[j] * P;
        }
        *distortion = acc;
    }
    if (iters) *iters = it;
    free(lo);
    free(hi);
    return 0;
}

/* fp32 tables for dimension d: centroids and boundaries of the (b-1)-bit
 * Lloyd-Max quantizer of N(0,1), multiplied by sigma = 1/sqrt(d) (the
 * N(0, 1/d) marginal of a rotated unit vector, [RSC] "nearly normal"). */
int tqo_codebook(int d, int b, float *c, float *beta)
{
    int k = b - 1, L, j;
    double cd[256], bd[256], sigma;
    if (d <= 0 || b < 1 || b > 8) return -1;
    L = 1 << k;
    if (k == 0) return 0;
    if (tqo_lloyd_max(L, cd, bd, NULL, NULL)) return -1;
    sigma = 1.0 / sqrt((double)d);
    for (j = 0; j < L; j++) c[j] = (float)(cd[j] * sigma);
    for (j = 0; j + 1 < L; j++) beta[j] = (float)(bd[j] * sigma);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* R2: Pi from the Householder QR of a Gaussian matrix ([QPD] "random         */
/* orthogonal matrix (not Hadamard)").  G[i][j] = gaussian(seed, stream 0)   */
/* element i*d + j.  Textbook Householder (Golub & Van Loan, Alg. 5.2.1):    */
/* for column j, v = x + sign(x_0)|x| e_1, H_j = I - 2 v v^T / (v^T v),      */
/* R_jj = -sign(x_0)|x|.  Q = H_0 H_1 ... H_{d-1}.  Pi = Q diag(sign R_jj)  */
/* so that G = Pi * (upper triangular with positive diagonal).              */
/* pi_d (optional) receives Pi in double, row-major; pi_f the fp32 copy.    */
/* ------------------------------------------------------------------------ */
int tqo_rotation(int d, uint64_t seed, double *pi_d, float *pi_f, double *rdiag)
{
    size_t n = (size_t)d;
    double *A, *Q, *V, *vtv, *rd, *g;
    int64_t j;
    if (d <= 0) return -1;
    A = (double *)malloc(sizeof(double) * n * n);   /* column-major */
    Q = (double *)malloc(sizeof(double) * n * n);   /* column-major */
    V = (double *)calloc(n * n, sizeof(double));    /* v_j in column j */
    vtv = (double *)malloc(sizeof(double) * n);
    rd = (double *)malloc(sizeof(double) * n);
    g = (double *)malloc(sizeof(double) * n * n);
    tqo_gaussian(seed, 0, (int64_t)(n * n), g);
    for (size_t i = 0; i < n; i++)
        for (size_t jj = 0; jj < n; jj++)
            A[i + jj * n] = g[i * n + jj];
    free(g);

    for (j = 0; j < d; j++) {
        size_t m = n - (size_t)j;
        double *x = &A[(size_t)j + (size_t)j * n];
        double *v = &V[(size_t)j + (size_t)j * n];
        double nx = 0.0, s, vv = 0.0;
        int64_t col;
        for (size_t i = 0; i < m; i++) nx += x[i] * x[i];
        nx = sqrt(nx);
        s = (x[0] >= 0.0) ? 1.0 : -1.0;
        for (size_t i = 0; i < m; i++) v[i] = x[i];
        v[0] = x[0] + s * nx;
        for (size_t i = 0; i < m; i++) vv += v[i] * v[i];
        vtv[j] = vv;
        rd[j] = -s * nx;
        if (vv == 0.0) continue;
#pragma omp parallel for schedule(static)
        for (col = j; col < d; col++) {
            double *a = &A[(size_t)j + (size_t)col * n];
            double w = 0.0;
            for (size_t i = 0; i < m; i++) w += v[i] * a[i];
            w = 2.0 * w / vv;
            for (size_t i = 0; i < m; i++) a[i] -= w * v[i];
        }
    }
    /* Q = H_0 H_1 ... H_{d-1} I, applied from the last reflector. */
    for (size_t i = 0; i < n * n; i++) Q[i] = 0.0;
    for (size_t i = 0; i < n; i++) Q[i + i * n] = 1.0;
    for (j = d - 1; j >= 0; j--) {
        size_t m = n - (size_t)j;
        const double *v = &V[(size_t)j + (size_t)j * n];
        double vv = vtv[j];
        int64_t col;
        if (vv == 0.0) continue;
#pragma omp parallel for schedule(static)
        for (col = 0; col < d; col++) {
            double *q = &Q[(size_t)j + (size_t)col * n];
            double w = 0.0;
            for (size_t i = 0; i < m; i++) w += v[i] * q[i];
            w = 2.0 * w / vv;
            for (size_t i = 0; i < m; i++) q[i] -= w * v[i];
        }
    }
    for (size_t i = 0; i < n; i++) {
        for (size_t jj = 0; jj < n; jj++) {
            double sgn = (rd[jj] >= 0.0) ? 1.0 : -1.0;
            double val = Q[i + jj * n] * sgn;
            if (pi_d) pi_d[i * n + jj] = val;
            if (pi_f) pi_f[i * n + jj] = (float)val;
        }
    }
    if (rdiag)
        for (size_t i = 0; i < n; i++) rdiag[i] = fabs(rd[i]);
    free(A); free(Q); free(V); free(vtv); free(rd);
    return 0;
}

/* R3: S[i][j] = gaussian(seed, stream 1) element i*d + j, rounded to fp32
 * ([SEA] step 2 "multiplied by a random matrix"). */
int tqo_qjl_matrix(int d, uint64_t seed, float *S)
{
    size_t n = (size_t)d * (size_t)d;
    double *g;
    if (d <= 0) return -1;
    g = (double *)malloc(sizeof(double) * n);
    tqo_gaussian(seed, 1, (int64_t)n, g);
    for (size_t i = 0; i < n; i++) S[i] = (float)g[i];
    free(g);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* R7: code layout.  A vector's record is d/32 blocks; block w holds          */
/* coordinates 32w .. 32w+31 in b consecutive 32-bit words.  With k = b-1   */
/* index bits and one sign bit per coordinate:                               */
/*   b = 1: word 0 bit j = z_j                                               */
/*   b = 2: 2-bit fields, word (j / 16), bits 2(j%16)..: idx_j | z_j << 1    */
/*   b = 4: 4-bit fields, word (j / 8),  bits 4(j%8)..:  idx_j | z_j << 3    */
/*   b = 3: 2-bit index fields in words 0..1 (16 per word), word 2 bit j=z_j */
/* where z_j = 1 iff (S r)_j >= 0.                                           */
/* ------------------------------------------------------------------------ */
int64_t tqo_words_per_vector(int d, int b)
{
    return (int64_t)(d / 32) * b;
}

static void tqo_pack_block(int b, const int32_t *idx, const int32_t *z, uint32_t *w)
{
    int j;
    for (j = 0; j < b; j++) w[j] = 0u;
    for (j = 0; j < 32; j++) {
        uint32_t iv = (uint32_t)idx[j], zv = (uint32_t)z[j];
        if (b == 1) {
            w[0] |= zv << j;
        } else if (b == 2) {
            w[j / 16] |= (iv | (zv << 1)) << (2 * (j % 16));
        } else if (b == 4) {
            w[j / 8] |= (iv | (zv << 3)) << (4 * (j % 8));
        } else { /* b == 3 */
            w[j / 16] |= iv << (2 * (j % 16));
            w[2] |= zv << j;
        }
    }
}

static void tqo_unpack_block(int b, const uint32_t *w, int32_t *idx, int32_t *z)
{
    int j;
    for (j = 0; j < 32; j++) {
        uint32_t f;
        if (b == 1) {
            idx[j] = 0;
            z[j] = (int32_t)((w[0] >> j) & 1u);
        } else if (b == 2) {
            f = (w[j / 16] >> (2 * (j % 16))) & 3u;
            idx[j] = (int32_t)(f & 1u);
            z[j] = (int32_t)(f >> 1);
        } else if (b == 4) {
            f = (w[j / 8] >> (4 * (j % 8))) & 15u;
            idx[j] = (int32_t)(f & 7u);
            z[j] = (int32_t)(f >> 3);
        } else {
            idx[j] = (int32_t)((w[j / 16] >> (2 * (j % 16))) & 3u);
            z[j] = (int32_t)((w[2] >> j) & 1u);
        }
    }
}

static int tqo_check_db(int d, int b)
{
    if (d <= 0 || d % 32 != 0) return -1;
    if (b < 1 || b > 4) return -1;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Encode, one vector at a time, steps in the pages' order:                  */
/*  1. |x| and the unit vector x/|x|        ([RSC] caveat 1: normalised)     */
/*  2. y = Pi x / |x|                        ([QPD], [SEA] step 1: rotate)   */
/*  3. idx_i = #{j : beta_j <= y_i}          ([SEA] round each coordinate   */
/*     on the fixed grid; R5 for ties)                                       */
/*  4. yhat_i = c[idx_i], r = y - yhat, |r|  ([QPD] MSE quantizer at b-1     */
/*     bits, then the residual; [SEA] step 2 "the difference")               */
/*  5. p = S r, z_i = [p_i >= 0]             ([QPD] QJL: random matrix, sign)*/
/*  6. pack (R7); store |x| and |r| in fp32.                                  */
/* A zero vector gets y = 0 and is otherwise encoded by the same steps.      */
/* Optional diagnostics: y, p in double and the index of every coordinate.   */
/* ------------------------------------------------------------------------ */
int tqo_encode(int d, int b, const float *c, const float *beta,
               const float *Pi, const float *S, int64_t n, const double *x,
               uint32_t *codes, float *xnorm, float *rnorm,
               double *y_out, double *p_out, int32_t *idx_out)
{
    int k = b - 1, L = 1 << (b - 1);
    int64_t wpv, v;
    if (tqo_check_db(d, b)) return -1;
    wpv = tqo_words_per_vector(d, b);
#pragma omp parallel for schedule(dynamic, 16)
    for (v = 0; v < n; v++) {
        const double *xv = x + (size_t)v * d;
        double *y = (double *)malloc(sizeof(double) * (size_t)d);
        double *r = (double *)malloc(sizeof(double) * (size_t)d);
        double *p = (double *)malloc(sizeof(double) * (size_t)d);
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        int32_t *z = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        double nx = 0.0, nr = 0.0;
        int i, j, w;
        for (j = 0; j < d; j++) nx += xv[j] * xv[j];
        nx = sqrt(nx);
        for (i = 0; i < d; i++) {
            double acc = 0.0;
            for (j = 0; j < d; j++) acc += (double)Pi[(size_t)i * d + j] * xv[j];
            y[i] = (nx > 0.0) ? acc / nx : 0.0;
        }
        for (i = 0; i < d; i++) {
            int cnt = 0;
            for (j = 0; j + 1 < L; j++)
                if ((double)beta[j] <= y[i]) cnt++;
            idx[i] = cnt;
            r[i] = y[i] - ((k > 0) ? (double)c[cnt] : 0.0);
            nr += r[i] * r[i];
        }
        nr = sqrt(nr);
        for (i = 0; i < d; i++) {
            double acc = 0.0;
            for (j = 0; j < d; j++) acc += (double)S[(size_t)i * d + j] * r[j];
            p[i] = acc;
            z[i] = (acc >= 0.0) ? 1 : 0;
        }
        for (w = 0; w < d / 32; w++)
            tqo_pack_block(b, idx + 32 * w, z + 32 * w,
                           codes + (size_t)v * wpv + (size_t)w * b);
        xnorm[v] = (float)nx;
        rnorm[v] = (float)nr;
        if (y_out) memcpy(y_out + (size_t)v * d, y, sizeof(double) * (size_t)d);
        if (p_out) memcpy(p_out + (size_t)v * d, p, sizeof(double) * (size_t)d);
        if (idx_out) memcpy(idx_out + (size_t)v * d, idx, sizeof(int32_t) * (size_t)d);
        free(y); free(r); free(p); free(idx); free(z);
    }
    return 0;
}

int tqo_unpack(int d, int b, int64_t n, const uint32_t *codes, int32_t *idx, int32_t *z)
{
    int64_t wpv, v;
    if (tqo_check_db(d, b)) return -1;
    wpv = tqo_words_per_vector(d, b);
    for (v = 0; v < n; v++)
        for (int w = 0; w < d / 32; w++)
            tqo_unpack_block(b, codes + (size_t)v * wpv + (size_t)w * b,
                             idx + (size_t)v * d + 32 * w, z + (size_t)v * d + 32 * w);
    return 0;
}

/* Dequantization ([QPD] "inverse rotation and renormalisation"):
 *   xhat = |x| Pi^T (yhat + |r| sqrt(pi/2)/d S^T (2z - 1)). */
int tqo_decode(int d, int b, const float *c, const float *Pi, const float *S,
               int64_t n, const uint32_t *codes, const float *xnorm,
               const float *rnorm, double *xhat)
{
    int k = b - 1;
    int64_t wpv, v;
    const double kappa0 = sqrt(3.14159265358979323846 / 2.0) / (double)d;
    if (tqo_check_db(d, b)) return -1;
    wpv = tqo_words_per_vector(d, b);
#pragma omp parallel for schedule(dynamic, 16)
    for (v = 0; v < n; v++) {
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        int32_t *z = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        double *e = (double *)malloc(sizeof(double) * (size_t)d);
        double kap = kappa0 * (double)rnorm[v];
        int i, j, w;
        for (w = 0; w < d / 32; w++)
            tqo_unpack_block(b, codes + (size_t)v * wpv + (size_t)w * b,
                             idx + 32 * w, z + 32 * w);
        for (j = 0; j < d; j++) {
            double acc = 0.0;
            for (i = 0; i < d; i++)
                acc += (double)S[(size_t)i * d + j] * (z[i] ? 1.0 : -1.0);
            e[j] = ((k > 0) ? (double)c[idx[j]] : 0.0) + kap * acc;
        }
        for (j = 0; j < d; j++) {
            double acc = 0.0;
            for (i = 0; i < d; i++) acc += (double)Pi[(size_t)i * d + j] * e[i];
            xhat[(size_t)v * d + j] = (double)xnorm[v] * acc;
        }
        free(idx); free(z); free(e);
    }
    return 0;
}

/* Query transform: qr = Pi q, u = S qr (in double from the fp32 matrices). */
int tqo_query(int d, const float *Pi, const float *S, int64_t nq,
              const double *q, double *qr, double *u)
{
    int64_t t;
    if (d <= 0) return -1;
    for (t = 0; t < nq; t++) {
        const double *qv = q + (size_t)t * d;
        double *a = qr + (size_t)t * d, *bb = u + (size_t)t * d;
        for (int i = 0; i < d; i++) {
            double acc = 0.0;
            for (int j = 0; j < d; j++) acc += (double)Pi[(size_t)i * d + j] * qv[j];
            a[i] = acc;
        }
        for (int i = 0; i < d; i++) {
            double acc = 0.0;
            for (int j = 0; j < d; j++) acc += (double)S[(size_t)i * d + j] * a[j];
            bb[i] = acc;
        }
    }
    return 0;
}

/* R6: unbiased inner-product estimate from a packed record ([QPD] "unbiased"
 * requirement; [RSC] item 2):
 *   s = |x| ( sum_i qr_i c[idx_i] + |r| sqrt(pi/2)/d sum_i u_i (2 z_i - 1) ).
 * scores[t][v] for query t and vector v. */
int tqo_score(int d, int b, const float *c, int64_t n, const uint32_t *codes,
              const float *xnorm, const float *rnorm, int64_t nq,
              const double *qr, const double *u, double *scores)
{
    int k = b - 1;
    int64_t wpv, v;
    const double kappa0 = sqrt(3.14159265358979323846 / 2.0) / (double)d;
    if (tqo_check_db(d, b)) return -1;
    wpv = tqo_words_per_vector(d, b);
#pragma omp parallel for schedule(dynamic, 64)
    for (v = 0; v < n; v++) {
        int32_t idx[32], z[32];
        for (int64_t t = 0; t < nq; t++) {
            const double *a = qr + (size_t)t * d, *bb = u + (size_t)t * d;
            double mse = 0.0, qjl = 0.0;
            for (int w = 0; w < d / 32; w++) {
                tqo_unpack_block(b, codes + (size_t)v * wpv + (size_t)w * b, idx, z);
                for (int j = 0; j < 32; j++) {
                    int i = 32 * w + j;
                    if (k > 0) mse += a[i] * (double)c[idx[j]];
                    qjl += bb[i] * (z[j] ? 1.0 : -1.0);
                }
            }
            scores[(size_t)t * n + v] =
                (double)xnorm[v] * (mse + kappa0 * (double)rnorm[v] * qjl);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Fractional bit widths ([QPD] experiments: quality neutral at 3.5 bits per */
/* channel on LongBench, a mild loss at 2.5; comuna.ru, the KV-cache         */
/* paragraph).  The pages give only the average width.  Reading (R13): the   */
/* first d/2 rotated coordinates take b total bits (b-1 index bits and the   */
/* sign), the last d/2 take b-1 (b-2 index bits and the sign), each half     */
/* rounded on the Lloyd-Max grid of its own level count for the same         */
/* N(0, 1/d) marginal; the QJL sign covers every coordinate.  The record is  */
/* the first half's d/64 blocks in the R7 layout of width b, then the second */
/* half's d/64 blocks in the layout of width b-1: b - 1/2 bits a coordinate. */
/* ------------------------------------------------------------------------ */
int64_t tqo_split_words_per_vector(int d, int b)
{
    return (int64_t)(d / 64) * (2 * b - 1);
}

static int tqo_check_split(int d, int b)
{
    if (d <= 0 || d % 64 != 0) return -1;
    if (b < 2 || b > 4) return -1;
    return 0;
}

/* width and first word of 32-coordinate block w of a split record */
static int tqo_split_block_bits(int d, int b, int w)
{
    return (w < d / 64) ? b : b - 1;
}

static int64_t tqo_split_block_offset(int d, int b, int w)
{
    const int h = d / 64;
    return (w < h) ? (int64_t)w * b : (int64_t)h * b + (int64_t)(w - h) * (b - 1);
}

/* Encode with the steps of tqo_encode; coordinate i is rounded on the grid of
 * its half (c_hi, beta_hi: 2^(b-1) levels for i < d/2; c_lo, beta_lo:
 * 2^(b-2) levels after, none when b = 2). */
int tqo_split_encode(int d, int b, const float *c_hi, const float *beta_hi,
                     const float *c_lo, const float *beta_lo, const float *Pi,
                     const float *S, int64_t n, const double *x, uint32_t *codes,
                     float *xnorm, float *rnorm, double *y_out, double *p_out,
                     int32_t *idx_out)
{
    int64_t wpv, v;
    if (tqo_check_split(d, b)) return -1;
    wpv = tqo_split_words_per_vector(d, b);
#pragma omp parallel for schedule(dynamic, 16)
    for (v = 0; v < n; v++) {
        const double *xv = x + (size_t)v * d;
        double *y = (double *)malloc(sizeof(double) * (size_t)d);
        double *r = (double *)malloc(sizeof(double) * (size_t)d);
        double *p = (double *)malloc(sizeof(double) * (size_t)d);
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        int32_t *z = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        double nx = 0.0, nr = 0.0;
        int i, j, w;
        for (j = 0; j < d; j++) nx += xv[j] * xv[j];
        nx = sqrt(nx);
        for (i = 0; i < d; i++) {
            double acc = 0.0;
            for (j = 0; j < d; j++) acc += (double)Pi[(size_t)i * d + j] * xv[j];
            y[i] = (nx > 0.0) ? acc / nx : 0.0;
        }
        for (i = 0; i < d; i++) {
            const int hi = i < d / 2;
            const int k = hi ? b - 1 : b - 2;
            const float *c = hi ? c_hi : c_lo, *beta = hi ? beta_hi : beta_lo;
            int cnt = 0;
            for (j = 0; j + 1 < (1 << k); j++)
                if ((double)beta[j] <= y[i]) cnt++;
            idx[i] = cnt;
            r[i] = y[i] - ((k > 0) ? (double)c[cnt] : 0.0);
            nr += r[i] * r[i];
        }
        nr = sqrt(nr);
        for (i = 0; i < d; i++) {
            double acc = 0.0;
            for (j = 0; j < d; j++) acc += (double)S[(size_t)i * d + j] * r[j];
            p[i] = acc;
            z[i] = (acc >= 0.0) ? 1 : 0;
        }
        for (w = 0; w < d / 32; w++)
            tqo_pack_block(tqo_split_block_bits(d, b, w), idx + 32 * w, z + 32 * w,
                           codes + (size_t)v * wpv + tqo_split_block_offset(d, b, w));
        xnorm[v] = (float)nx;
        rnorm[v] = (float)nr;
        if (y_out) memcpy(y_out + (size_t)v * d, y, sizeof(double) * (size_t)d);
        if (p_out) memcpy(p_out + (size_t)v * d, p, sizeof(double) * (size_t)d);
        if (idx_out) memcpy(idx_out + (size_t)v * d, idx, sizeof(int32_t) * (size_t)d);
        free(y); free(r); free(p); free(idx); free(z);
    }
    return 0;
}

int tqo_split_unpack(int d, int b, int64_t n, const uint32_t *codes, int32_t *idx, int32_t *z)
{
    int64_t wpv, v;
    if (tqo_check_split(d, b)) return -1;
    wpv = tqo_split_words_per_vector(d, b);
    for (v = 0; v < n; v++)
        for (int w = 0; w < d / 32; w++)
            tqo_unpack_block(tqo_split_block_bits(d, b, w),
                             codes + (size_t)v * wpv + tqo_split_block_offset(d, b, w),
                             idx + (size_t)v * d + 32 * w, z + (size_t)v * d + 32 * w);
    return 0;
}

/* yhat_i of a split record: the centroid of coordinate i's half (0 where that
 * half has no index bits). */
static double tqo_split_yhat(int d, int b, const float *c_hi, const float *c_lo, int i,
                             int32_t idx)
{
    if (i < d / 2) return (double)c_hi[idx];
    return (b - 2 > 0) ? (double)c_lo[idx] : 0.0;
}

/* Dequantization of a split record, as tqo_decode. */
int tqo_split_decode(int d, int b, const float *c_hi, const float *c_lo, const float *Pi,
                     const float *S, int64_t n, const uint32_t *codes, const float *xnorm,
                     const float *rnorm, double *xhat)
{
    int64_t v;
    const double kappa0 = sqrt(3.14159265358979323846 / 2.0) / (double)d;
    if (tqo_check_split(d, b)) return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (v = 0; v < n; v++) {
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        int32_t *z = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        double *e = (double *)malloc(sizeof(double) * (size_t)d);
        double kap = kappa0 * (double)rnorm[v];
        int i, j;
        tqo_split_unpack(d, b, 1, codes + (size_t)v * tqo_split_words_per_vector(d, b), idx, z);
        for (j = 0; j < d; j++) {
            double acc = 0.0;
            for (i = 0; i < d; i++)
                acc += (double)S[(size_t)i * d + j] * (z[i] ? 1.0 : -1.0);
            e[j] = tqo_split_yhat(d, b, c_hi, c_lo, j, idx[j]) + kap * acc;
        }
        for (j = 0; j < d; j++) {
            double acc = 0.0;
            for (i = 0; i < d; i++) acc += (double)Pi[(size_t)i * d + j] * e[i];
            xhat[(size_t)v * d + j] = (double)xnorm[v] * acc;
        }
        free(idx); free(z); free(e);
    }
    return 0;
}

/* The estimator of tqo_score on split records. */
int tqo_split_score(int d, int b, const float *c_hi, const float *c_lo, int64_t n,
                    const uint32_t *codes, const float *xnorm, const float *rnorm, int64_t nq,
                    const double *qr, const double *u, double *scores)
{
    int64_t wpv, v;
    const double kappa0 = sqrt(3.14159265358979323846 / 2.0) / (double)d;
    if (tqo_check_split(d, b)) return -1;
    wpv = tqo_split_words_per_vector(d, b);
#pragma omp parallel for schedule(dynamic, 64)
    for (v = 0; v < n; v++) {
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        int32_t *z = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        tqo_split_unpack(d, b, 1, codes + (size_t)v * wpv, idx, z);
        for (int64_t t = 0; t < nq; t++) {
            const double *a = qr + (size_t)t * d, *bb = u + (size_t)t * d;
            double mse = 0.0, qjl = 0.0;
            for (int i = 0; i < d; i++) {
                mse += a[i] * tqo_split_yhat(d, b, c_hi, c_lo, i, idx[i]);
                qjl += bb[i] * (z[i] ? 1.0 : -1.0);
            }
            scores[(size_t)t * n + v] =
                (double)xnorm[v] * (mse + kappa0 * (double)rnorm[v] * qjl);
        }
        free(idx); free(z);
    }
    return 0;
}

/* Top-k per query: order by score descending, then id ascending; by plain
 * selection (k passes over the row). */
int tqo_topk(int64_t nq, int64_t n, const double *scores, int k,
             double *vals, int64_t *ids)
{
    int64_t t;
    if (k < 0 || (int64_t)k > n) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < nq; t++) {
        const double *s = scores + (size_t)t * n;
        char *taken = (char *)calloc((size_t)n, 1);
        for (int r = 0; r < k; r++) {
            int64_t best = -1;
            for (int64_t v = 0; v < n; v++) {
                if (taken[v]) continue;
                if (best < 0 || s[v] > s[best]) best = v;
            }
            taken[best] = 1;
            vals[(size_t)t * k + r] = s[best];
            ids[(size_t)t * k + r] = best;
        }
        free(taken);
    }
    return 0;
}

/* Exact inner products <q_t, x_v> in double. */
int tqo_exact_scores(int d, int64_t n, const double *x, int64_t nq,
                     const double *q, double *out)
{
    int64_t v;
#pragma omp parallel for schedule(static)
    for (v = 0; v < n; v++)
        for (int64_t t = 0; t < nq; t++) {
            double acc = 0.0;
            for (int j = 0; j < d; j++)
                acc += q[(size_t)t * d + j] * x[(size_t)v * d + j];
            out[(size_t)t * n + v] = acc;
        }
    return 0;
}

/* The MSE-only quantizer ([QPD] "for MSE-optimised TurboQuant"): all `bits`
 * go to the Lloyd-Max index, no QJL.  Its inner-product estimate
 * |x| <Pi q, yhat> is the biased one the pages contrast with. */
int tqo_mse_estimate(int d, int bits, const float *c, const float *beta,
                     const float *Pi, const double *x, const double *q,
                     double *estimate)
{
    int L = 1 << bits;
    double nx = 0.0, acc = 0.0;
    if (d <= 0 || bits < 1) return -1;
    for (int j = 0; j < d; j++) nx += x[j] * x[j];
    nx = sqrt(nx);
    for (int i = 0; i < d; i++) {
        double yi = 0.0, qi = 0.0;
        int cnt = 0;
        for (int j = 0; j < d; j++) {
            yi += (double)Pi[(size_t)i * d + j] * x[j];
            qi += (double)Pi[(size_t)i * d + j] * q[j];
        }
        yi = (nx > 0.0) ? yi / nx : 0.0;
        for (int j = 0; j + 1 < L; j++)
            if ((double)beta[j] <= yi) cnt++;
        acc += qi * (double)c[cnt];
    }
    *estimate = nx * acc;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The MSE-only quantizer as a stored code ([QPD] "for MSE-optimised          */
/* TurboQuant": all b bits go to the Lloyd-Max index, no QJL).  Steps 1-4 of  */
/* tqo_encode with 2^b levels (c, beta: the b-bit tables, i.e. tqo_codebook  */
/* at b + 1).  R11: the record keeps the layout of R7, the b-bit index split  */
/* into its low b-1 bits (the idx field) and its top bit (the z position);   */
/* |r| = |y - c[idx]| is stored as well.                                     */
/* ------------------------------------------------------------------------ */
static int32_t tqo_mse_index(int b, int32_t idx, int32_t z)
{
    return (b == 1) ? z : (idx | (z << (b - 1)));
}

int tqo_mse_encode(int d, int b, const float *c, const float *beta, const float *Pi,
                   int64_t n, const double *x, uint32_t *codes, float *xnorm, float *rnorm,
                   double *y_out, int32_t *idx_out)
{
    int L = 1 << b;
    int64_t wpv, v;
    if (tqo_check_db(d, b)) return -1;
    wpv = tqo_words_per_vector(d, b);
#pragma omp parallel for schedule(dynamic, 16)
    for (v = 0; v < n; v++) {
        const double *xv = x + (size_t)v * d;
        double *y = (double *)malloc(sizeof(double) * (size_t)d);
        int32_t *lo = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        int32_t *top = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        int32_t *full = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
        double nx = 0.0, nr = 0.0;
        int i, j, w;
        for (j = 0; j < d; j++) nx += xv[j] * xv[j];
        nx = sqrt(nx);
        for (i = 0; i < d; i++) {
            double acc = 0.0;
            for (j = 0; j < d; j++) acc += (double)Pi[(size_t)i * d + j] * xv[j];
            y[i] = (nx > 0.0) ? acc / nx : 0.0;
        }
        for (i = 0; i < d; i++) {
            int cnt = 0;
            double r;
            for (j = 0; j + 1 < L; j++)
                if ((double)beta[j] <= y[i]) cnt++;
            full[i] = cnt;
            lo[i] = (b == 1) ? 0 : (cnt & ((1 << (b - 1)) - 1));
            top[i] = (b == 1) ? cnt : (cnt >> (b - 1));
            r = y[i] - (double)c[cnt];
            nr += r * r;
        }
        for (w = 0; w < d / 32; w++)
            tqo_pack_block(b, lo + 32 * w, top + 32 * w, codes + (size_t)v * wpv + (size_t)w * b);
        xnorm[v] = (float)nx;
        rnorm[v] = (float)sqrt(nr);
        if (y_out) memcpy(y_out + (size_t)v * d, y, sizeof(double) * (size_t)d);
        if (idx_out) memcpy(idx_out + (size_t)v * d, full, sizeof(int32_t) * (size_t)d);
        free(y); free(lo); free(top); free(full);
    }
    return 0;
}

/* The MSE estimate from stored records: s = |x| sum_i qr_i c[idx_i]
 * (qr = Pi q from tqo_query; [QPD]: biased, the contrast to the QJL one). */
int tqo_mse_score(int d, int b, const float *c, int64_t n, const uint32_t *codes,
                  const float *xnorm, int64_t nq, const double *qr, double *scores)
{
    int64_t wpv, v;
    if (tqo_check_db(d, b)) return -1;
    wpv = tqo_words_per_vector(d, b);
#pragma omp parallel for schedule(dynamic, 64)
    for (v = 0; v < n; v++) {
        int32_t idx[32], z[32];
        for (int64_t t = 0; t < nq; t++) {
            const double *a = qr + (size_t)t * d;
            double acc = 0.0;
            for (int w = 0; w < d / 32; w++) {
                tqo_unpack_block(b, codes + (size_t)v * wpv + (size_t)w * b, idx, z);
                for (int j = 0; j < 32; j++)
                    acc += a[32 * w + j] * (double)c[tqo_mse_index(b, idx[j], z[j])];
            }
            scores[(size_t)t * n + v] = (double)xnorm[v] * acc;
        }
    }
    return 0;
}

/* MSE dequantization: xhat = |x| Pi^T c[idx]. */
int tqo_mse_decode(int d, int b, const float *c, const float *Pi, int64_t n,
                   const uint32_t *codes, const float *xnorm, double *out)
{
    int64_t wpv, v;
    if (tqo_check_db(d, b)) return -1;
    wpv = tqo_words_per_vector(d, b);
#pragma omp parallel for schedule(dynamic, 16)
    for (v = 0; v < n; v++) {
        int32_t idx[32], z[32];
        double *yh = (double *)malloc(sizeof(double) * (size_t)d);
        for (int w = 0; w < d / 32; w++) {
            tqo_unpack_block(b, codes + (size_t)v * wpv + (size_t)w * b, idx, z);
            for (int j = 0; j < 32; j++) yh[32 * w + j] = (double)c[tqo_mse_index(b, idx[j], z[j])];
        }
        for (int i = 0; i < d; i++) {
            double acc = 0.0;
            for (int j = 0; j < d; j++) acc += (double)Pi[(size_t)j * d + i] * yh[j];
            out[(size_t)v * d + i] = (double)xnorm[v] * acc;
        }
        free(yh);
    }
    return 0;
}


/* ---------------------------------------------------------------------------
 * Decode attention over quantized keys and values (a reading: the pages stop
 * at the attention logits of quant_prune_distill #674 and the comuna.ru
 * summary; softmax and the value sum are the standard attention that those
 * logits feed).  For every query row t:
 *   l_j = scale * s_tj            (s: the estimated inner products)
 *   p_j = exp(l_j - max_j l_j) / sum_j exp(l_j - max_j l_j)
 *   out_t = sum_j p_j v_j         (v: the dequantized value rows)
 * logits [nq][n], values [n][d], out [nq][d]; n >= 1.
 * ------------------------------------------------------------------------- */
int tqo_softmax_weighted_sum(int64_t nq, int64_t n, int d, const double *logits,
                             const double *values, double *out)
{
    if (nq < 0 || n < 1 || d < 1) return -1;
    for (int64_t t = 0; t < nq; t++) {
        const double *l = logits + (size_t)t * n;
        double mx = l[0], sum = 0.0;
        for (int64_t j = 1; j < n; j++)
            if (l[j] > mx) mx = l[j];
        double *o = out + (size_t)t * d;
        for (int i = 0; i < d; i++) o[i] = 0.0;
        for (int64_t j = 0; j < n; j++) {
            const double w = exp(l[j] - mx);
            sum += w;
            for (int i = 0; i < d; i++) o[i] += w * values[(size_t)j * d + i];
        }
        for (int i = 0; i < d; i++) o[i] /= sum;
    }
    return 0;
}

