// E0: the method's parameters -- the Lloyd-Max codebook (host, fp64), the
// random rotation Pi (device: Gaussian matrix + fp64 Householder QR) and the
// QJL matrix S (device: Gaussian matrix).
//
// Pages: quant_prune_distill #674 (rotation by a random orthogonal matrix,
// not Hadamard; Lloyd-Max grid for the target bit width; residual sketched by
// a random matrix and a sign), RecSysChannel #256 item 1 (thresholds
// precomputed for the near-Gaussian coordinate distribution), seeallochnaya
// #3476 step 1 (1-D k-means boundaries, denser in the centre).
#include <cmath>
#include <cstring>

#include "tq_internal.cuh"

namespace tq {
namespace {

// SplitMix64 output mixer (Steele, Lea & Flood, OOPSLA 2014).
__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}
static uint64_t mix64_host(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

// Gaussian d x d matrix of (seed, stream): element e = i*d + j is the e-th
// output of Box-Muller over the counter-form SplitMix64 stream whose state
// starts at key = mix64(seed ^ stream*gamma): pair m uses outputs 2m, 2m+1,
// u1 = ((a>>11)+1) 2^-53, u2 = (b>>11) 2^-53, rho = sqrt(-2 ln u1),
// element 2m = rho cos(2 pi u2), element 2m+1 = rho sin(2 pi u2).
// Written column-major in fp64 (QR input) and/or row-major in fp32.
__global__ void k_gaussian(uint64_t key, int d, double* __restrict__ colmajor,
                           float* __restrict__ rowmajor) {
    const int64_t count = (int64_t)d * d;
    const int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (2 * m >= count) return;
    const uint64_t a = mix64(key + (uint64_t)(2 * m + 1) * kGamma);
    const uint64_t b = mix64(key + (uint64_t)(2 * m + 2) * kGamma);
    const double u1 = (double)((a >> 11) + 1) * 0x1p-53;
    const double u2 = (double)(b >> 11) * 0x1p-53;
    const double two_pi = 6.283185307179586476925286766559;
    const double rho = sqrt(-2.0 * log(u1));
    double v[2];
    v[0] = rho * cos(two_pi * u2);
    v[1] = rho * sin(two_pi * u2);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t e = 2 * m + h;
        if (e >= count) break;
        const int64_t i = e / d, j = e % d;
        if (colmajor) colmajor[i + j * d] = v[h];
        if (rowmajor) rowmajor[e] = (float)v[h];
    }
}

template <int NT>
__device__ double block_sum(double v, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x / 32, l = threadIdx.x % 32;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    double t = 0.0;
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) t += red[i];
    return t;
}

// Householder reflector of column j of the column-major matrix A (lda = d):
// x = A[j:, j], v = x + sign(x_0)|x| e_1 written over x, vtv[j] = v^T v,
// rd[j] = -sign(x_0)|x| (the R diagonal before the sign fix).
__global__ void k_hh_reflector(double* __restrict__ A, int d, int j, double* __restrict__ vtv,
                               double* __restrict__ rd) {
    __shared__ double red[8];
    double* x = A + j + (int64_t)j * d;
    const int m = d - j;
    double ss = 0.0;
    for (int i = threadIdx.x; i < m; i += 256) ss += x[i] * x[i];
    ss = block_sum<256>(ss, red);
    const double nx = sqrt(ss);
    const double x0 = x[0];
    const double s = (x0 >= 0.0) ? 1.0 : -1.0;
    __syncthreads();
    if (threadIdx.x == 0) x[0] = x0 + s * nx;
    __syncthreads();
    double vv = 0.0;
    for (int i = threadIdx.x; i < m; i += 256) vv += x[i] * x[i];
    vv = block_sum<256>(vv, red);
    if (threadIdx.x == 0) {
        vtv[j] = vv;
        rd[j] = -s * nx;
    }
}

// Apply H_j = I - 2 v v^T / v^T v (v = V[j:, j]) to rows j.. of columns
// col0 + blockIdx.x of M (column-major, lda = d).
__global__ void k_hh_apply(const double* V, double* M, int d, int j,
                           int col0, const double* __restrict__ vtv) {
    __shared__ double red[4];
    const double vv = vtv[j];
    if (vv == 0.0) return;
    const int col = col0 + blockIdx.x;
    const double* v = V + j + (int64_t)j * d;
    double* a = M + j + (int64_t)col * d;
    const int m = d - j;
    double w = 0.0;
    for (int i = threadIdx.x; i < m; i += 128) w += v[i] * a[i];
    w = block_sum<128>(w, red);
    w = 2.0 * w / vv;
    for (int i = threadIdx.x; i < m; i += 128) a[i] -= w * v[i];
}

__global__ void k_identity(double* __restrict__ Q, int d) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)d * d) return;
    Q[e] = ((e % d) == (e / d)) ? 1.0 : 0.0;
}

// Pi[i][j] = Q[i][j] * sign(R_jj), rounded to fp32, row-major.
__global__ void k_finish_pi(const double* __restrict__ Q, const double* __restrict__ rd, int d,
                            float* __restrict__ Pi) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)d * d) return;
    const int64_t i = e / d, j = e % d;
    const double sgn = (rd[j] >= 0.0) ? 1.0 : -1.0;
    Pi[e] = (float)(Q[i + j * d] * sgn);
}

// Lloyd-Max for N(0,1) with L (even) levels, on the positive half-line:
// p_0 < ... < p_{H-1} (H = L/2), thresholds t_0 = 0, t_i = (p_{i-1}+p_i)/2,
// t_H = inf; centroid of [t_i, t_{i+1}) is (phi(t_i) - phi(t_{i+1})) /
// (Q(t_i) - Q(t_{i+1})) with Q the upper tail; the negative half mirrors it.
void lloyd_max_host(int L, double* c, double* beta, double* distortion) {
    const int H = L / 2;  // L <= 16
    double p[8], t[9];
    for (int i = 0; i < H; ++i) p[i] = (i + 0.5) * (3.0 / H);
    auto phi = [](double x) { return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI); };
    auto tail = [](double x) { return std::isinf(x) ? 0.0 : 0.5 * std::erfc(x / std::sqrt(2.0)); };
    for (int it = 0; it < 2000000; ++it) {
        t[0] = 0.0;
        for (int i = 1; i < H; ++i) t[i] = 0.5 * (p[i - 1] + p[i]);
        t[H] = INFINITY;
        double delta = 0.0;
        for (int i = 0; i < H; ++i) {
            const double np = (phi(t[i]) - phi(t[i + 1])) / (tail(t[i]) - tail(t[i + 1]));
            delta = std::fmax(delta, std::fabs(np - p[i]));
            p[i] = np;
        }
        if (delta < 1e-14) break;
    }
    t[0] = 0.0;
    for (int i = 1; i < H; ++i) t[i] = 0.5 * (p[i - 1] + p[i]);
    t[H] = INFINITY;
    for (int i = 0; i < H; ++i) {
        c[H + i] = p[i];
        c[H - 1 - i] = -p[i];
    }
    for (int i = 0; i < H; ++i) {
        beta[H - 1 + i] = t[i];
        if (i > 0) beta[H - 1 - i] = -t[i];
    }
    double acc = 0.0;  // centroid condition: D = 1 - sum_cells c^2 P(cell)
    for (int i = 0; i < H; ++i) acc += 2.0 * p[i] * p[i] * (tail(t[i]) - tail(t[i + 1]));
    if (distortion) *distortion = 1.0 - acc;
}

}  // namespace
}  // namespace tq

namespace tq {
namespace {

// Pi_g (and, with d_S, S_g) of every group: Gaussian draws, Householder QR in
// fp64 on the device, Pi = Q diag(sign R_jj).
int build_matrices(int d, uint64_t seed, int G, float* d_Pi, float* d_S, void* d_ws,
                   cudaStream_t s) {
    const size_t dd = (size_t)d * d;
    double* A = (double*)d_ws;
    double* Q = (double*)((char*)d_ws + align256(dd * sizeof(double)));
    double* vtv = (double*)((char*)Q + align256(dd * sizeof(double)));
    double* rd = (double*)((char*)vtv + align256(d * sizeof(double)));
    const int gthreads = 256;
    const unsigned gblocks = (unsigned)((dd / 2 + gthreads) / gthreads);
    for (int g = 0; g < G; ++g) {
        const uint64_t sg = seed + (uint64_t)g;
        const uint64_t key_pi = mix64_host(sg ^ (0ULL * kGamma));
        const uint64_t key_s = mix64_host(sg ^ (1ULL * kGamma));
        if (d_S) k_gaussian<<<gblocks, gthreads, 0, s>>>(key_s, d, nullptr, d_S + (size_t)g * dd);
        k_gaussian<<<gblocks, gthreads, 0, s>>>(key_pi, d, A, nullptr);
        TQ_CHECK_LAUNCH();
        for (int j = 0; j < d; ++j) {
            k_hh_reflector<<<1, 256, 0, s>>>(A, d, j, vtv, rd);
            if (j + 1 < d) k_hh_apply<<<d - j - 1, 128, 0, s>>>(A, A, d, j, j + 1, vtv);
        }
        TQ_CHECK_LAUNCH();
        k_identity<<<(unsigned)((dd + 255) / 256), 256, 0, s>>>(Q, d);
        for (int j = d - 1; j >= 0; --j) k_hh_apply<<<d - j, 128, 0, s>>>(A, Q, d, j, j, vtv);
        k_finish_pi<<<(unsigned)((dd + 255) / 256), 256, 0, s>>>(Q, rd, d, d_Pi + (size_t)g * dd);
        TQ_CHECK_LAUNCH();
    }
    return TQ_OK;
}

// Host codebook: `levels` Lloyd-Max levels of N(0,1) scaled by 1/sqrt(d).
tq_codebook_t make_codebook(int d, int b, uint64_t seed, int G, int levels, int variant) {
    tq_codebook_t out;
    std::memset(&out, 0, sizeof(out));
    out.d = d;
    out.b = b;
    out.groups = G;
    out.seed = seed;
    out.levels = levels;
    out.variant = variant;
    out.distortion = 1.0;
    if (levels > 0) {
        double c[16], beta[16];
        lloyd_max_host(levels, c, beta, &out.distortion);
        const double sigma = 1.0 / std::sqrt((double)d);
        for (int i = 0; i < levels; ++i) out.centroids[i] = (float)(c[i] * sigma);
        for (int i = 0; i + 1 < levels; ++i) out.boundaries[i] = (float)(beta[i] * sigma);
    }
    return out;
}

}  // namespace
}  // namespace tq

extern "C" int tq_build_codebook(int d, int b, uint64_t seed, int G, tq_codebook_t* cb,
                                 float* d_Pi, float* d_S, void* d_ws, size_t ws_bytes,
                                 void* stream) {
    using namespace tq;
    if (!cb || G < 1) return TQ_ERR_ARG;
    if (!valid_db(d, b)) return TQ_ERR_UNSUPPORTED;
    if (!d_Pi || !d_S || !d_ws) return TQ_ERR_ARG;
    if (ws_bytes < tq_workspace_bytes(TQ_OP_BUILD, d, b, G, 0, 0, 0)) return TQ_ERR_WORKSPACE;
    const int rc = build_matrices(d, seed, G, d_Pi, d_S, d_ws, (cudaStream_t)stream);
    if (rc) return rc;
    *cb = make_codebook(d, b, seed, G, (b == 1) ? 0 : (1 << (b - 1)), TQ_VARIANT_PROD);
    return TQ_OK;
}

extern "C" int tq_build_codebook_split(int d, int b, uint64_t seed, int G, tq_codebook_t* cb,
                                       float* d_Pi, float* d_S, void* d_ws, size_t ws_bytes,
                                       void* stream) {
    using namespace tq;
    if (!cb || G < 1) return TQ_ERR_ARG;
    if (!valid_db(d, b) || b < 2) return TQ_ERR_UNSUPPORTED;
    if (!d_Pi || !d_S || !d_ws) return TQ_ERR_ARG;
    if (ws_bytes < tq_workspace_bytes(TQ_OP_BUILD, d, b, G, 0, 0, 0)) return TQ_ERR_WORKSPACE;
    const int rc = build_matrices(d, seed, G, d_Pi, d_S, d_ws, (cudaStream_t)stream);
    if (rc) return rc;
    // the first half's grid (b bits: 2^(b-1) levels), the second half's (b - 1 bits)
    tq_codebook_t out = make_codebook(d, b, seed, G, 1 << (b - 1), TQ_VARIANT_PROD);
    const tq_codebook_t lo = make_codebook(d, b - 1, seed, G, (b == 2) ? 0 : (1 << (b - 2)),
                                           TQ_VARIANT_PROD);
    out.split = 1;
    out.levels_lo = lo.levels;
    for (int i = 0; i < 16; ++i) {
        out.centroids_lo[i] = lo.centroids[i];
        out.boundaries_lo[i] = lo.boundaries[i];
    }
    *cb = out;
    return TQ_OK;
}

extern "C" int tq_build_codebook_mse(int d, int b, uint64_t seed, int G, tq_codebook_t* cb,
                                     float* d_Pi, void* d_ws, size_t ws_bytes, void* stream) {
    using namespace tq;
    if (!cb || G < 1) return TQ_ERR_ARG;
    if (!valid_db(d, b)) return TQ_ERR_UNSUPPORTED;
    if (!d_Pi || !d_ws) return TQ_ERR_ARG;
    if (ws_bytes < tq_workspace_bytes(TQ_OP_BUILD, d, b, G, 0, 0, 0)) return TQ_ERR_WORKSPACE;
    const int rc = build_matrices(d, seed, G, d_Pi, nullptr, d_ws, (cudaStream_t)stream);
    if (rc) return rc;
    *cb = make_codebook(d, b, seed, G, 1 << b, TQ_VARIANT_MSE);
    return TQ_OK;
}
