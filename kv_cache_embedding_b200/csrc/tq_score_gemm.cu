// S1 scoring of many queries at d >= 256 as one GEMM per key chunk on the
// tensor cores (tq_gemm_tc.cu), the decoded-key form of the estimate
//   s = |x| ( <qr, c[idx]> + <u, kappa (2z - 1)> ),  kappa = |r| sqrt(pi/2)/d,
// i.e. s[t][v] = |x_v| sum_k A[v][k] B[t][k] over K = 2d with
//   A[v] = ( c[idx_v,0..d) | kappa_v (2 z_v - 1) ),   B[t] = ( Pi q_t | S Pi q_t ).
// (MSE-only variant: A[v] = (c[cell] | 0), B[t] = (Pi q_t | 0).)
//
// Pages: quant_prune_distill #674 (inner-product estimate from the codes; MSE
// part plus the 1-bit QJL correction); comuna.ru "Google speeds up LLMs 8x"
// (vector search over the quantized database).
//
// A and B are two bf16 pieces each (x = hi + lo to ~2^-16 of |x|) and the GEMM
// sums hi hi + hi lo + lo hi, an error well inside the score tolerance.  With
// one 128-query tile the keys' pieces are decoded from the records inside the
// GEMM (two warps write them into each shared-memory stage), so only the
// records cross HBM; with 256 or more queries they are decoded once per chunk
// of 37,888 keys into the workspace and the product runs on CTA pairs
// (256 x 256 tiles).  The queries' pieces come by TMA.  Scores go out
// transposed ([query][key], coalesced over keys) with the maximum of every
// 128-key tile per query for the top-k threshold.
#include <cuda_bf16.h>

#include "tq_internal.cuh"

namespace tq {
namespace {

constexpr float kSqrtHalfPi = 1.2533141373155002512f;
constexpr int64_t kMaxRows = (int64_t)1 << 30;  // a multiple of 128

__device__ __forceinline__ void split2(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
    hi = __float2bfloat16_rn(v);
    lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

// Cell and sign bit of coordinate j (0..31) of a block (layout of tq.h).
template <int B>
__device__ __forceinline__ void field_of(const uint32_t* w, int j, int& cell, int& z) {
    if (B == 1) {
        cell = 0;
        z = (int)((w[0] >> j) & 1u);
    } else if (B == 2) {
        const uint32_t f = (w[j >> 4] >> (2 * (j & 15))) & 3u;
        cell = (int)(f & 1u);
        z = (int)(f >> 1);
    } else if (B == 3) {
        cell = (int)((w[j >> 4] >> (2 * (j & 15))) & 3u);
        z = (int)((w[2] >> j) & 1u);
    } else {
        const uint32_t f = (w[j >> 3] >> (4 * (j & 7))) & 15u;
        cell = (int)(f & 7u);
        z = (int)(f >> 3);
    }
}

// A pieces [2][rows][2d] of the records of one key chunk; one thread per
// (key, 8 coordinates), so a warp's 16-byte stores to each of the four
// planes are contiguous (whole sectors: no read-for-ownership of partly
// written sectors).
template <int B>
__global__ void k_key_operand(const uint32_t* __restrict__ codes, const float* __restrict__ rnorm,
                              int64_t rows, int d, KCodebook cb, __nv_bfloat16* __restrict__ out) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int nc = d / 8;  // 8-coordinate chunks per key
    if (e >= rows * nc) return;
    const int64_t v = e / nc;
    const int ch = (int)(e % nc);
    const int blk = ch >> 2, j0 = 8 * (ch & 3);
    const uint32_t* w = codes + v * (int64_t)(d / 32 * B) + blk * B;
    uint32_t ww[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < B; ++i) ww[i] = __ldg(w + i);
    const float kap = kSqrtHalfPi / (float)d * __ldg(rnorm + v);
    const int64_t K = 2 * (int64_t)d, plane = rows * K;
    __nv_bfloat16* row = out + v * K + 8 * ch;
    uint32_t chi[4] = {0u, 0u, 0u, 0u}, clo[4] = {0u, 0u, 0u, 0u};
    uint32_t shi[4] = {0u, 0u, 0u, 0u}, slo[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        int cell, z;
        field_of<B>(ww, j0 + h, cell, z);
        float c, sgn;
        if (cb.mse) {
            c = cb.c[(B == 1) ? z : (cell | (z << (B - 1)))];
            sgn = 0.f;
        } else {
            c = (B == 1) ? 0.f : cb.c[cell];
            sgn = z ? kap : -kap;
        }
        __nv_bfloat16 c1, c2, s1, s2;
        split2(c, c1, c2);
        split2(sgn, s1, s2);
        const int sft = 16 * (h & 1);
        chi[h >> 1] |= (uint32_t)__bfloat16_as_ushort(c1) << sft;
        clo[h >> 1] |= (uint32_t)__bfloat16_as_ushort(c2) << sft;
        shi[h >> 1] |= (uint32_t)__bfloat16_as_ushort(s1) << sft;
        slo[h >> 1] |= (uint32_t)__bfloat16_as_ushort(s2) << sft;
    }
    *reinterpret_cast<uint4*>(row) = make_uint4(chi[0], chi[1], chi[2], chi[3]);
    *reinterpret_cast<uint4*>(row + plane) = make_uint4(clo[0], clo[1], clo[2], clo[3]);
    *reinterpret_cast<uint4*>(row + d) = make_uint4(shi[0], shi[1], shi[2], shi[3]);
    *reinterpret_cast<uint4*>(row + plane + d) = make_uint4(slo[0], slo[1], slo[2], slo[3]);
}

// B pieces [2][nq_pad][2d] of one group's queries (rows >= nq are zero).
__global__ void k_query_operand(const float* __restrict__ qr, const float* __restrict__ u, int nq,
                                int nq_pad, int d, __nv_bfloat16* __restrict__ out) {
    const int64_t K = 2 * (int64_t)d;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= nq_pad * K) return;
    const int t = (int)(e / K);
    const int i = (int)(e % K);
    float v = 0.f;
    if (t < nq) v = (i < d) ? qr[(int64_t)t * d + i] : u[(int64_t)t * d + (i - d)];
    __nv_bfloat16 hi, lo;
    split2(v, hi, lo);
    out[e] = hi;
    out[(int64_t)nq_pad * K + e] = lo;
}

}  // namespace

bool score_gemm_supported(int d, int nq) {
    return d >= 256 && nq >= kScoreGemmMinQueries && gemm_tc_supported(128, 2 * d);
}

bool topk_materialized(int d, int G, int64_t n, int nq) {
    return (int64_t)G * nq * n <= kTopkMaterialize || score_gemm_supported(d, nq);
}

// Query counts padded to a multiple of 256 take the decoded keys through HBM,
// once per chunk of keys, and the CTA-pair GEMM (256 x 256 tiles: each key
// tile is read once per 256 queries); a single 128-query tile decodes the keys
// inside the one-CTA GEMM, so only the records cross HBM.  Beyond 256 queries
// re-decoding every key tile for each query tile costs more than the round
// trip of the decoded keys.
constexpr int kDecodeInGemmMaxQueries = 256;
constexpr int64_t kScoreGemmChunk = 148 * 256;  // keys decoded per GEMM: 2 row tiles per pair

bool score_gemm_materialises(int64_t nq_pad) {
    return nq_pad > kDecodeInGemmMaxQueries || nq_pad % 256 == 0;
}

size_t score_gemm_workspace(int d, int64_t n, int nq) {
    const int64_t nq_pad = (nq + 127) / 128 * 128;
    size_t bytes = align256((size_t)2 * nq_pad * 2 * d * 2);
    if (score_gemm_materialises(nq_pad)) {
        const int64_t chunk = n < kScoreGemmChunk ? n : kScoreGemmChunk;
        bytes += align256((size_t)2 * chunk * 2 * d * 2);
    }
    return bytes;
}

int score_gemm(const tq_codebook_t* cb, int G, int64_t n, const uint32_t* d_codes,
               const float* d_xnorm, const float* d_rnorm, int nq, const float* qr,
               const float* u, float* scores, float* tmax, int64_t ntm, void* op_ws, int* d_err,
               cudaStream_t s) {
    const int d = cb->d, b = cb->b;
    const int W = words_per_vector(d, b);
    const int nq_pad = (nq + 127) / 128 * 128;
    __nv_bfloat16* Bq = (__nv_bfloat16*)op_ws;
    KeyDecode kd{};
    kd.d = d;
    kd.b = b;
    kd.mse = is_mse(cb) ? 1 : 0;
    kd.kscale = kSqrtHalfPi / (float)d;
    for (int c = 0; c < 16; ++c) {  // bf16 pieces of every centroid
        const float v = c < cb->levels ? cb->centroids[c] : 0.f;
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
        kd.tab[c] = (uint32_t)__bfloat16_as_ushort(h) | ((uint32_t)__bfloat16_as_ushort(l) << 16);
    }
    for (int g = 0; g < G; ++g) {
        const int64_t qn = (int64_t)nq_pad * 2 * d;
        k_query_operand<<<(unsigned)((qn + 255) / 256), 256, 0, s>>>(
            qr + (int64_t)g * nq * d, u + (int64_t)g * nq * d, nq, nq_pad, d, Bq);
        TQ_CHECK_LAUNCH();
        if (score_gemm_materialises(nq_pad)) {  // decoded keys through HBM, chunk by chunk
            __nv_bfloat16* Ak =
                (__nv_bfloat16*)((char*)op_ws + align256((size_t)2 * nq_pad * 2 * d * 2));
            const KCodebook kc = make_kcodebook(cb);
            const int64_t chunk = n < kScoreGemmChunk ? n : kScoreGemmChunk;
            for (int64_t r0 = 0; r0 < n; r0 += chunk) {
                const int64_t rows = (n - r0) < chunk ? (n - r0) : chunk;
                const int64_t off = (int64_t)g * n + r0;
                const unsigned blocks = (unsigned)((rows * (d / 8) + 255) / 256);
                switch (b) {
                    case 1: k_key_operand<1><<<blocks, 256, 0, s>>>(d_codes + off * W, d_rnorm + off, rows, d, kc, Ak); break;
                    case 2: k_key_operand<2><<<blocks, 256, 0, s>>>(d_codes + off * W, d_rnorm + off, rows, d, kc, Ak); break;
                    case 3: k_key_operand<3><<<blocks, 256, 0, s>>>(d_codes + off * W, d_rnorm + off, rows, d, kc, Ak); break;
                    default: k_key_operand<4><<<blocks, 256, 0, s>>>(d_codes + off * W, d_rnorm + off, rows, d, kc, Ak); break;
                }
                TQ_CHECK_LAUNCH();
                float* tm = tmax ? tmax + (int64_t)g * nq * ntm + r0 / 128 : nullptr;
                const int rc = launch_gemm_tc((int)rows, nq_pad, 2 * d, Ak, 2, Bq,
                                              scores + (int64_t)g * nq * n + r0, n, d_xnorm + off,
                                              2, d_err, s, 2, true, nq, tm, ntm);
                if (rc) return rc;
            }
            continue;
        }
        // key ranges of at most 2^30 (the GEMM's row count is an int); in
        // practice one launch per group
        for (int64_t r0 = 0; r0 < n; r0 += kMaxRows) {
            const int64_t rows = (n - r0) < kMaxRows ? (n - r0) : kMaxRows;
            const int64_t off = (int64_t)g * n + r0;
            kd.codes = d_codes + off * W;
            kd.rnorm = d_rnorm + off;
            float* tm = tmax ? tmax + (int64_t)g * nq * ntm + r0 / 128 : nullptr;
            const int rc = launch_gemm_tc_decoded((int)rows, nq_pad, kd, Bq,
                                                  scores + (int64_t)g * nq * n + r0, n,
                                                  d_xnorm + off, d_err, s, nq, tm, ntm);
            if (rc) return rc;
        }
    }
    return TQ_OK;
}

}  // namespace tq
