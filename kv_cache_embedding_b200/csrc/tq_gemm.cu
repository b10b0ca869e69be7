// FP32 SIMT GEMM with a per-row scale, used for the small dense products of
// the support paths (query transform, dequantization, exact search) and as
// the portable rotation of the encode path for dimensions the tensor-core
// kernel does not cover.
//
//   C[m][n] = scale(m) * sum_k A[m][k] * B(n, k)
//   B(n, k) = B[n*ldb + k]  (b_nk = true)   or   B[k*ldb + n]  (b_nk = false)
//   scale(m) = 1 (mode 0), 1/row_scale[m] or 0 if row_scale[m] == 0 (mode 1),
//              row_scale[m] (mode 2)
//
// Products are summed in fp32 over chunks of 128 of K, and the chunk sums are
// added into a separate running total: the rounding error of a rotated
// coordinate then stays near 2^-24 * 0.4 * sqrt(128) of its scale for any d,
// instead of growing with sqrt(d) as one long fp32 sum would.
//
// 128x128x8 tiles, 256 threads, an 8x8 register tile per thread, fp32
// accumulation in k order.  Requirements: K % 8 == 0, lda/ldb/ldc % 4 == 0,
// 16-byte aligned bases; M and N may be ragged (N % 4 == 0 when !b_nk).
#include "tq_internal.cuh"

namespace tq {
namespace {

constexpr int BM = 128, BN = 128, BK = 8;

template <typename TA>
struct ALoad;
template <>
struct ALoad<float> {
    __device__ static void load4(const float* p, float v[4]) {
        float4 t = *reinterpret_cast<const float4*>(p);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    }
};
template <>
struct ALoad<__nv_bfloat16> {
    __device__ static void load4(const __nv_bfloat16* p, float v[4]) {
        uint2 t = *reinterpret_cast<const uint2*>(p);
        v[0] = __uint_as_float(t.x << 16);
        v[1] = __uint_as_float(t.x & 0xffff0000u);
        v[2] = __uint_as_float(t.y << 16);
        v[3] = __uint_as_float(t.y & 0xffff0000u);
    }
};

template <typename TA, bool B_NK>
__global__ __launch_bounds__(256) void k_sgemm(int M, int N, int K, const TA* __restrict__ A,
                                               int lda, const float* __restrict__ B, int ldb,
                                               float* __restrict__ C, int ldc,
                                               const float* __restrict__ row_scale,
                                               int scale_mode) {
    __shared__ __align__(16) float As[2][BK][BM];
    __shared__ __align__(16) float Bs[2][BK][BN];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    const int64_t m0 = (int64_t)blockIdx.y * BM;
    const int64_t n0 = (int64_t)blockIdx.x * BN;

    // loader coordinates
    const int a_r = tid / 2, a_k = (tid % 2) * 4;          // A: 128 rows x 8 k
    const int bnk_r = tid / 2, bnk_k = (tid % 2) * 4;      // B [N][K]: 128 n x 8 k
    const int bkn_k = tid / 32, bkn_n = (tid % 32) * 4;    // B [K][N]: 8 k x 128 n

    float a_reg[4], b_reg[4];
    auto load_tiles = [&](int k0) {
        int64_t m = m0 + a_r;
        if (m < M) {
            ALoad<TA>::load4(A + m * lda + k0 + a_k, a_reg);
        } else {
            a_reg[0] = a_reg[1] = a_reg[2] = a_reg[3] = 0.f;
        }
        if (B_NK) {
            int64_t n = n0 + bnk_r;
            if (n < N) {
                ALoad<float>::load4(B + n * ldb + k0 + bnk_k, b_reg);
            } else {
                b_reg[0] = b_reg[1] = b_reg[2] = b_reg[3] = 0.f;
            }
        } else {
            int64_t n = n0 + bkn_n;
            if (n < N) {
                ALoad<float>::load4(B + (int64_t)(k0 + bkn_k) * ldb + n, b_reg);
            } else {
                b_reg[0] = b_reg[1] = b_reg[2] = b_reg[3] = 0.f;
            }
        }
    };
    auto store_tiles = [&](int buf) {
#pragma unroll
        for (int i = 0; i < 4; ++i) As[buf][a_k + i][a_r] = a_reg[i];
        if (B_NK) {
#pragma unroll
            for (int i = 0; i < 4; ++i) Bs[buf][bnk_k + i][bnk_r] = b_reg[i];
        } else {
            *reinterpret_cast<float4*>(&Bs[buf][bkn_k][bkn_n]) =
                make_float4(b_reg[0], b_reg[1], b_reg[2], b_reg[3]);
        }
    };

    float acc[8][8], tot[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = tot[i][j] = 0.f;

    load_tiles(0);
    store_tiles(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = 0; k0 < K; k0 += BK) {
        const bool more = k0 + BK < K;
        if (more) load_tiles(k0 + BK);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[8], b[8];
            float4 t;
            t = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
            a[0] = t.x; a[1] = t.y; a[2] = t.z; a[3] = t.w;
            t = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
            a[4] = t.x; a[5] = t.y; a[6] = t.z; a[7] = t.w;
            t = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
            b[0] = t.x; b[1] = t.y; b[2] = t.z; b[3] = t.w;
            t = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
            b[4] = t.x; b[5] = t.y; b[6] = t.z; b[7] = t.w;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (((k0 + BK) & 127) == 0 || !more) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    tot[i][j] += acc[i][j];
                    acc[i][j] = 0.f;
                }
        }
        if (more) {
            store_tiles(buf ^ 1);
            __syncthreads();
            buf ^= 1;
        }
    }

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
        if (m >= M) continue;
        float sc = 1.f;
        if (scale_mode == 1) {
            float s = row_scale[m];
            sc = (s > 0.f) ? 1.f / s : 0.f;
        } else if (scale_mode == 2) {
            sc = row_scale[m];
        }
#pragma unroll
        for (int jh = 0; jh < 2; ++jh) {
            const int64_t n = n0 + jh * 64 + tx * 4;
            float* dst = C + m * ldc + n;
            if (n + 3 < N) {
                *reinterpret_cast<float4*>(dst) =
                    make_float4(tot[i][jh * 4 + 0] * sc, tot[i][jh * 4 + 1] * sc,
                                tot[i][jh * 4 + 2] * sc, tot[i][jh * 4 + 3] * sc);
            } else {
                for (int j = 0; j < 4; ++j)
                    if (n + j < N) dst[j] = tot[i][jh * 4 + j] * sc;
            }
        }
    }
}

}  // namespace

int launch_sgemm(int M, int N, int K, const void* A, int a_dtype, int lda, const float* B,
                 bool b_nk, int ldb, float* C, int ldc, const float* row_scale, int scale_mode,
                 cudaStream_t s) {
    if (M <= 0 || N <= 0) return TQ_OK;
    if (K % BK != 0 || lda % 4 || ldb % 4 || ldc % 4) return TQ_ERR_ARG;
    if (!b_nk && N % 4) return TQ_ERR_ARG;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
    if (grid.y > 65535) return TQ_ERR_ARG;
    if (a_dtype == TQ_F32) {
        if (b_nk)
            k_sgemm<float, true><<<grid, 256, 0, s>>>(M, N, K, (const float*)A, lda, B, ldb, C,
                                                      ldc, row_scale, scale_mode);
        else
            k_sgemm<float, false><<<grid, 256, 0, s>>>(M, N, K, (const float*)A, lda, B, ldb, C,
                                                       ldc, row_scale, scale_mode);
    } else {
        if (b_nk)
            k_sgemm<__nv_bfloat16, true><<<grid, 256, 0, s>>>(
                M, N, K, (const __nv_bfloat16*)A, lda, B, ldb, C, ldc, row_scale, scale_mode);
        else
            k_sgemm<__nv_bfloat16, false><<<grid, 256, 0, s>>>(
                M, N, K, (const __nv_bfloat16*)A, lda, B, ldb, C, ldc, row_scale, scale_mode);
    }
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

}  // namespace tq
