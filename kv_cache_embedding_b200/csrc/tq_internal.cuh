// Internal helpers of libtq (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq.h"

namespace tq {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;
constexpr int kMinD = 128;
constexpr int kMaxD = 4096;
constexpr int kMaxK = 32;           // largest top-k
constexpr int kTopkTile = 256;      // keys per top-k tile (one partial list each)
constexpr int64_t kEncodeChunk = 65536;  // rows per encode/decode chunk

// Codebook passed to kernels by value (kernel parameter space).
struct KCodebook {
    float c[16];
    float beta[16];
    float c_lo[16];     // fractional widths: the last d/2 coordinates' grid
    float beta_lo[16];
    int levels;   // PROD: 2^(b-1), 0 for b = 1; MSE: 2^b
    int levels_lo;
    int mse;      // 1: MSE-only variant (b-bit index, no QJL)
    int split;    // 1: fractional width (b - 1/2 bits a coordinate)
};

inline KCodebook make_kcodebook(const tq_codebook_t* cb) {
    KCodebook k;
    for (int i = 0; i < 16; ++i) {
        k.c[i] = cb->centroids[i];
        k.beta[i] = cb->boundaries[i];
        k.c_lo[i] = cb->split ? cb->centroids_lo[i] : 0.f;
        k.beta_lo[i] = cb->split ? cb->boundaries_lo[i] : 0.f;
    }
    k.levels = cb->levels;
    k.levels_lo = cb->split ? cb->levels_lo : 0;
    k.mse = cb->variant == TQ_VARIANT_MSE ? 1 : 0;
    k.split = cb->split ? 1 : 0;
    return k;
}

inline bool is_mse(const tq_codebook_t* cb) { return cb->variant == TQ_VARIANT_MSE; }
inline bool is_split(const tq_codebook_t* cb) { return cb->split != 0; }

__host__ __device__ inline int words_per_vector(int d, int b) { return d / 32 * b; }
// Record words of a codebook: d/32 b, or d/64 (2b - 1) for a fractional width.
inline int record_words(const tq_codebook_t* cb) {
    return is_split(cb) ? cb->d / 64 * (2 * cb->b - 1) : words_per_vector(cb->d, cb->b);
}

__device__ __forceinline__ float load_f32(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_f32(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}

// Strictly better in top-k order: larger value, then smaller id.
__device__ __forceinline__ bool better(float va, int64_t ia, float vb, int64_t ib) {
    return va > vb || (va == vb && ia < ib);
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// tq_topk writes the whole score matrix (and per-chunk maxima) to its
// workspace when it has at most this many scores, then selects per row; larger
// searches run the fused score + running-list kernel instead.
constexpr int64_t kTopkMaterialize = (int64_t)1 << 24;
constexpr int kTopkCandidates = 4096;  // gathered candidates per row on that path
// (also when the scores come from the decoded-key GEMM, whatever their number)
bool topk_materialized(int d, int G, int64_t n, int nq);

inline bool valid_db(int d, int b) {
    return d >= kMinD && d <= kMaxD && d % 128 == 0 && b >= 1 && b <= 4;
}

}  // namespace tq

#define TQ_TRY_CUDA(expr)                               \
    do {                                                \
        cudaError_t tq_e_ = (expr);                     \
        if (tq_e_ != cudaSuccess) return TQ_ERR_CUDA;   \
    } while (0)

#define TQ_CHECK_LAUNCH() TQ_TRY_CUDA(cudaPeekAtLastError())

// Entry points of the individual translation units (C++ linkage, internal).
namespace tq {
int launch_sgemm(int M, int N, int K, const void* A, int a_dtype, int lda, const float* B,
                 bool b_nk, int ldb, float* C, int ldc, const float* row_scale, int scale_mode,
                 cudaStream_t s);
// qr = Q Pi^T and u = qr S^T (S may be null: u = 0) for every group's nq
// query rows (fp32 or bf16); clears the device status word *err.
int query_prep(const float* d_Pi, const float* d_S, int G, int d, int nq, const void* d_q,
               int q_dtype, float* qr, float* u, int* err, cudaStream_t s);
// Argument checks shared by the scoring entry points.
int check_common(const tq_codebook_t* cb, int G, int64_t n, int nq, int q_dtype);
// Decode attention (tq_attention.cu): workspace of tq_attention_decode.
size_t attn_workspace_bytes(int b, int G, int64_t n, int nq);
bool encode_tc_supported(const tq_codebook_t* cb, int x_dtype, int G, int64_t n);
// Split-precision tcgen05 GEMM (tq_gemm_tc.cu): C = scale(m) * A B^T from
// Encode epilogues of the CTA-pair GEMM over one chunk of M rows (N = K = d,
// d % 256 == 0, inner-product records).  Mode 1, on the rotation product:
// bucketize y = C, write the cells, the fp16 pieces of rscale * r and |r|^2 of
// every 128 coordinates.  Mode 2, on the QJL product: the signs of C with the
// cells -> code records, and |r| from the partial sums.  Mode 4 (one-CTA GEMM,
// d = 128, the MSE-only variant): bucketize, |r| and the MSE-only records of
// whole rows.  Mode 0 stores C.
struct EncodeEpi {
    int mode;
    int b;
    float rscale;      // power of two
    uint8_t* idx;      // [M][d] cells (mode 1 writes, mode 2 reads)
    __half* rp;        // [2][M][d] fp16 pieces hi, lo of rscale * r (mode 1)
    float* rn2;        // [d/128][M] |r|^2 per 128 coordinates (mode 1 writes, mode 2 sums)
    float* rnorm;      // [M] |r| (mode 2)
    uint32_t* codes;   // [M][record words] (mode 2)
    KCodebook cb;
};
// 16-bit pieces of A ([pa][M][K]) and B ([pb][N][K]) -- bf16, or fp16 with
// `fp16` (the pointers then address __half data); d_err as the encode
// kernels' status word.  Row-major products with N % 256 == 0 run on CTA
// pairs (256 x 256 tiles) unless pair_form is false.
bool gemm_tc_supported(int N, int K);
int split_bf16x3(const float* x, int64_t count, __nv_bfloat16* out, cudaStream_t s);
// fp16 pieces [2][count] of scale * x (scale a power of two).
int split_f16x2(const float* x, int64_t count, float scale, __half* out, cudaStream_t s);
int launch_gemm_tc(int M, int N, int K, const __nv_bfloat16* A, int pa, const __nv_bfloat16* B,
                   float* C, int64_t ldc, const float* row_scale, int scale_mode, int* d_err,
                   cudaStream_t s, int pb = 3, bool transposed = false, int n_store = 0,
                   float* tmax = nullptr, int64_t ldt = 0, bool fp16 = false,
                   bool pair_form = true, const EncodeEpi* epi = nullptr);
// A operand decoded from code records inside the GEMM (scoring of many
// queries): row m of A = (c[idx] | kappa_m (2z - 1)) over K = 2d as bf16
// pieces hi, lo (kappa_m = kscale |r_m|; the MSE-only variant has c[cell] and
// zeros); tab[cell] = bf16 hi | bf16 lo << 16 of the centroid.
struct KeyDecode {
    const uint32_t* codes;  // [M][d/32 * b] records
    const float* rnorm;     // [M]
    int d, b, mse;
    float kscale;           // sqrt(pi/2) / d
    uint32_t tab[16];
};
// C^T tile store with per-128-row maxima, A decoded from records (pa = pb = 2).
int launch_gemm_tc_decoded(int M, int N, const KeyDecode& kd, const __nv_bfloat16* B, float* C,
                           int64_t ldc, const float* row_scale, int* d_err, cudaStream_t s,
                           int n_store, float* tmax, int64_t ldt);
// The general encode path's dense products run on the tensor-core GEMM (fp16
// pieces) at every d; its workspace holds their operands.
inline bool encode_gemm_tc(int d) { return d >= kMinD; }
// Scoring of many queries at d >= 256 as a GEMM over decoded keys
// (tq_score_gemm.cu): scores [G][nq][n] (and per-128-key maxima [G][nq][ntm]).
constexpr int kScoreGemmMinQueries = 64;
bool score_gemm_supported(int d, int nq);
size_t score_gemm_workspace(int d, int64_t n, int nq);
int score_gemm(const tq_codebook_t* cb, int G, int64_t n, const uint32_t* d_codes,
               const float* d_xnorm, const float* d_rnorm, int nq, const float* qr,
               const float* u, float* scores, float* tmax, int64_t ntm, void* op_ws, int* d_err,
               cudaStream_t s);
// Scoring of up to 16 queries per pass at d = 128 as exact int8 tensor-core
// products (tq_score_i8.cu); inner-product records with b = 2..4 whose code
// array is 16-byte aligned.  Same outputs as launch_score_tc.  With k0 and
// n_stride (>= 0) it scores keys k0 .. k0 + n of arrays holding n_stride keys
// per group, into scores [G][nq][n] (and maxima [G][nq][ceil(n / 128)]).
bool score_i8_supported(const tq_codebook_t* cb, int G, int64_t n, int nq, const void* d_codes);
int launch_score_i8(const tq_codebook_t* cb, int G, int64_t n, const uint32_t* d_codes,
                    const float* d_xnorm, const float* d_rnorm, int nq, const float* qr,
                    const float* u, float* d_scores, float* tmax, int* zero_cnt, int* d_err,
                    cudaStream_t s, int64_t n_stride = -1, int64_t k0 = 0);
bool score_tc_supported(int d, int b, int G, int64_t n, int nq);
int launch_score_tc(const tq_codebook_t* cb, int G, int64_t n, const uint32_t* d_codes,
                    const float* d_xnorm, const float* d_rnorm, int nq, const float* qr,
                    const float* u, float* d_scores, float* tmax, int* zero_cnt, int* d_err,
                    cudaStream_t s);
// Top-k with the path chosen by the caller: materialised scores (`materialize`)
// or the fused running-list kernel.
int topk_run(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G, int64_t n,
             const uint32_t* d_codes, const float* d_xnorm, const float* d_rnorm, int nq,
             const void* d_q, int q_dtype, int k, float* d_vals, int64_t* d_ids, void* d_ws,
             size_t ws_bytes, bool materialize, cudaStream_t s, float* scores_out = nullptr);
// scores_in_ws: the materialised path keeps the score matrix in the workspace
// (false when the caller's score output holds it, as in tq_score_topk)
size_t topk_workspace_bytes(int d, int b, int G, int64_t n, int nq, int k, bool materialize,
                            bool scores_in_ws = true);
// tq_topk's argument checks: TQ_OK to run, kTopkNothing when there is nothing
// to compute (a successful no-op), else the error status.
constexpr int kTopkNothing = 1;
int topk_validate(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G, int64_t n,
                  const uint32_t* d_codes, const float* d_xnorm, const float* d_rnorm, int nq,
                  const void* d_q, int q_dtype, int k, const float* d_vals, const int64_t* d_ids);
int launch_encode_tc(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G,
                     int64_t n, const void* d_x, uint32_t* d_codes, float* d_xnorm,
                     float* d_rnorm, int* d_err, cudaStream_t s);
}
