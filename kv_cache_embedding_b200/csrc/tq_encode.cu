// E1-E6, encode: norm, rotation, Lloyd-Max bucketize, residual, QJL sign.
//
// Pages: quant_prune_distill #674 (the inner-product quantizer: MSE quantizer
// at b-1 bits, then 1-bit QJL of the residual -- random matrix, sign);
// RecSysChannel #256 caveat 1 (vectors normalised and multiplied by a random
// matrix); seeallochnaya #3476 steps 1-2 (rotate; round every coordinate on
// the precomputed grid; residual -> random matrix -> sign).
//
// Portable path (any supported d; the only path of the MSE-only variant): per
// group and row chunk
//   k_rownorm      |x| in fp64 accumulation                       (E1)
//   GEMM           Y = X Pi^T / |x|                                (E2)
//   k_quantize     idx = #{beta_j <= y}, r = y - c[idx], |r|       (E3, E4)
//   GEMM           P = R S^T                                       (E5)
//   k_pack         fields idx | z -> code words                    (E3, E6)
// The GEMMs run on the tensor cores (split bf16 pieces, tq_gemm_tc.cu) for
// d >= 256, else as fp32 SIMT GEMMs (tq_gemm.cu).
#include "tq_internal.cuh"

namespace tq {
namespace {

template <typename T>
__global__ void k_rownorm(const T* __restrict__ x, int64_t rows, int d,
                          float* __restrict__ xnorm) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const T* xr = x + row * d;
    double acc = 0.0;
    for (int i = lane; i < d; i += 32) {
        const double v = (double)load_f32(xr, i);
        acc = fma(v, v, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) xnorm[row] = (float)sqrt(acc);
}

// One warp per row: bucketize each rotated coordinate, write the residual over
// it, the cell index to a byte array, and |r|.
__global__ void k_quantize(float* __restrict__ yr, uint8_t* __restrict__ idx, int64_t rows, int d,
                           KCodebook cb, float* __restrict__ rnorm) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    float* y = yr + row * d;
    uint8_t* ix = idx + row * d;
    float rr = 0.f;
    for (int i = lane; i < d; i += 32) {
        const float v = y[i];
        int cell = 0;
        float r = v;
        if (cb.levels > 0) {
#pragma unroll
            for (int j = 0; j < 15; ++j)
                if (j + 1 < cb.levels && cb.beta[j] <= v) ++cell;
            r = v - cb.c[cell];
        }
        y[i] = r;
        ix[i] = (uint8_t)cell;
        rr = fmaf(r, r, rr);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rr += __shfl_xor_sync(0xffffffffu, rr, o);
    if (lane == 0) rnorm[row] = sqrtf(rr);
}

// One warp per row; lane j handles coordinate 32w + j of block w.  Fields of
// neighbouring lanes are OR-combined with a butterfly inside each word's lanes.
// MSE: no projection; the b-bit cell is split into its low b-1 bits (idx
// field) and its top bit (the z position).
template <int B, bool MSE>
__global__ void k_pack(const float* __restrict__ p, const uint8_t* __restrict__ idx, int64_t rows,
                       int d, uint32_t* __restrict__ codes) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const int W = words_per_vector(d, B);
    for (int w = 0; w < d / 32; ++w) {
        const int i = 32 * w + lane;
        const uint32_t cell = idx[row * d + i];
        const uint32_t z = MSE ? (cell >> (B - 1)) : ((p[row * d + i] >= 0.f) ? 1u : 0u);
        const uint32_t iv = MSE ? (cell & ((1u << (B - 1)) - 1u)) : cell;
        uint32_t* out = codes + row * W + w * B;
        if (B == 1) {
            const uint32_t word = __ballot_sync(0xffffffffu, z != 0u);
            if (lane == 0) out[0] = word;
        } else if (B == 2 || B == 4) {
            constexpr int per = 32 / B;  // coordinates per word
            uint32_t f = (iv | (z << (B - 1))) << (B * (lane % per));
#pragma unroll
            for (int o = 1; o < per; o <<= 1) f |= __shfl_xor_sync(0xffffffffu, f, o);
            if (lane % per == 0) out[lane / per] = f;
        } else {  // B == 3: 2-bit index fields (16 per word), then the sign word
            uint32_t f = iv << (2 * (lane % 16));
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) f |= __shfl_xor_sync(0xffffffffu, f, o);
            const uint32_t zw = __ballot_sync(0xffffffffu, z != 0u);
            if (lane % 16 == 0) out[lane / 16] = f;
            if (lane == 0) out[2] = zw;
        }
    }
}

}  // namespace
}  // namespace tq

extern "C" int tq_encode(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G,
                         int64_t n, const void* d_x, int x_dtype, uint32_t* d_codes,
                         float* d_xnorm, float* d_rnorm, void* d_ws, size_t ws_bytes,
                         void* stream) {
    using namespace tq;
    if (!cb || G < 1 || n < 0) return TQ_ERR_ARG;
    if (x_dtype != TQ_F32 && x_dtype != TQ_BF16) return TQ_ERR_ARG;
    const int d = cb->d, b = cb->b;
    if (!valid_db(d, b)) return TQ_ERR_UNSUPPORTED;
    if (cb->groups < G) return TQ_ERR_MISMATCH;
    if (n == 0) return TQ_OK;
    const bool mse = is_mse(cb);
    if (!d_Pi || (!mse && !d_S) || !d_x || !d_codes || !d_xnorm || !d_rnorm) return TQ_ERR_ARG;
    const size_t need = tq_workspace_bytes(TQ_OP_ENCODE, d, b, G, n, 0, 0);
    if (need > 0 && (!d_ws || ws_bytes < need)) return TQ_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    // the first 256 bytes of the workspace hold the device status word
    // d = 128 bf16 keys: fused tensor-core kernel (TMA source and 16-byte code
    // stores need 16-byte aligned buffers)
    if (!mse && encode_tc_supported(cb, x_dtype, G, n) && (uintptr_t)d_x % 16 == 0 &&
        (uintptr_t)d_codes % 16 == 0)
        return launch_encode_tc(cb, d_Pi, d_S, G, n, d_x, d_codes, d_xnorm, d_rnorm,
                                (int*)d_ws, s);
    TQ_TRY_CUDA(cudaMemsetAsync(d_ws, 0, sizeof(int), s));
    int* err = (int*)d_ws;
    const KCodebook kc = make_kcodebook(cb);
    const int64_t chunk = n < kEncodeChunk ? n : kEncodeChunk;
    float* Y = (float*)((char*)d_ws + 256);
    float* P = (float*)((char*)Y + align256((size_t)chunk * d * 4));
    uint8_t* IX = (uint8_t*)((char*)P + align256((size_t)chunk * d * 4));
    const int W = words_per_vector(d, b);
    const size_t esz = (x_dtype == TQ_F32) ? 4 : 2;
    const size_t dd = (size_t)d * d;
    // tensor-core GEMMs: bf16 pieces of Pi_g, S_g and of the chunk's operand
    const bool tcg = encode_gemm_tc(d) && gemm_tc_supported(d, d);
    __nv_bfloat16* PiP = (__nv_bfloat16*)(IX + align256((size_t)chunk * d));
    __nv_bfloat16* SP = (__nv_bfloat16*)((char*)PiP + align256(3 * dd * 2));
    __nv_bfloat16* AP = (__nv_bfloat16*)((char*)SP + align256(3 * dd * 2));
    for (int g = 0; g < G; ++g) {
        if (tcg) {
            int rc = split_bf16x3(d_Pi + g * dd, (int64_t)dd, PiP, s);
            if (rc) return rc;
            if (!mse) {
                rc = split_bf16x3(d_S + g * dd, (int64_t)dd, SP, s);
                if (rc) return rc;
            }
        }
        for (int64_t r0 = 0; r0 < n; r0 += chunk) {
            const int64_t rows = (n - r0) < chunk ? (n - r0) : chunk;
            const int64_t off = (int64_t)g * n + r0;
            const void* xg = (const char*)d_x + (size_t)off * d * esz;
            float* xn = d_xnorm + off;
            float* rn = d_rnorm + off;
            const unsigned wblocks = (unsigned)((rows + 7) / 8);
            if (x_dtype == TQ_F32)
                k_rownorm<float><<<wblocks, 256, 0, s>>>((const float*)xg, rows, d, xn);
            else
                k_rownorm<__nv_bfloat16><<<wblocks, 256, 0, s>>>((const __nv_bfloat16*)xg, rows,
                                                                 d, xn);
            TQ_CHECK_LAUNCH();
            int rc;
            if (tcg) {  // Y = X Pi^T / |x| on the tensor cores
                const __nv_bfloat16* A = (const __nv_bfloat16*)xg;  // bf16 keys: one exact piece
                int pa = 1;
                if (x_dtype == TQ_F32) {
                    rc = split_bf16x3((const float*)xg, rows * d, AP, s);
                    if (rc) return rc;
                    A = AP;
                    pa = 3;
                }
                rc = launch_gemm_tc((int)rows, d, d, A, pa, PiP, Y, d, xn, 1, err, s);
            } else {
                rc = launch_sgemm((int)rows, d, d, xg, x_dtype, d, d_Pi + g * dd, true, d, Y, d,
                                  xn, 1, s);
            }
            if (rc) return rc;
            k_quantize<<<wblocks, 256, 0, s>>>(Y, IX, rows, d, kc, rn);
            TQ_CHECK_LAUNCH();
            uint32_t* cg = d_codes + (size_t)off * W;
            if (mse) {  // no QJL projection
                switch (b) {
                    case 1: k_pack<1, true><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    case 2: k_pack<2, true><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    case 3: k_pack<3, true><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    default: k_pack<4, true><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                }
                TQ_CHECK_LAUNCH();
                continue;
            }
            if (tcg) {  // P = R S^T on the tensor cores
                rc = split_bf16x3(Y, rows * d, AP, s);
                if (rc) return rc;
                rc = launch_gemm_tc((int)rows, d, d, AP, 3, SP, P, d, nullptr, 0, err, s);
            } else {
                rc = launch_sgemm((int)rows, d, d, Y, TQ_F32, d, d_S + g * dd, true, d, P, d,
                                  nullptr, 0, s);
            }
            if (rc) return rc;
            switch (b) {
                case 1: k_pack<1, false><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                case 2: k_pack<2, false><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                case 3: k_pack<3, false><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                default: k_pack<4, false><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
            }
            TQ_CHECK_LAUNCH();
        }
    }
    return TQ_OK;
}
