// E1-E6, encode: norm, rotation, Lloyd-Max bucketize, residual, QJL sign.
//
// Pages: quant_prune_distill #674 (the inner-product quantizer: MSE quantizer
// at b-1 bits, then 1-bit QJL of the residual -- random matrix, sign);
// RecSysChannel #256 caveat 1 (vectors normalised and multiplied by a random
// matrix); seeallochnaya #3476 steps 1-2 (rotate; round every coordinate on
// the precomputed grid; residual -> random matrix -> sign).
//
// General path (every d, fp32 rows, the MSE-only variant; bf16 keys at d = 128
// take the fused kernel of tq_encode_tc.cu): per group and row chunk
//   k_rownorm_split16   |x| in fp64 accumulation; fp16 pieces of 2^e x    (E1)
//   GEMM                Y = X Pi^T / |x| on the tensor cores              (E2)
//   k_quantize16        idx = #{beta_j <= y}, r = y - c[idx], |r|,
//                       fp16 pieces of 2^s r                              (E3, E4)
//   GEMM                P = R S^T on the tensor cores                     (E5)
//   k_pack              fields idx | z -> code words                      (E3, E6)
// The GEMMs (tq_gemm_tc.cu) take two fp16 pieces of each fp32 operand, every
// operand scaled by a power of two into fp16's range: rows of x so that
// |x| 2^e is in [2^10, 2^11) (then |2^e x_i| <= 2^11), Pi by 2^8 (its
// entries are ~ 1/sqrt(d); the scale keeps the low pieces normal), S by 2^4,
// r by 2^s with 2^s ~ 64 sqrt(d) (|r_i| <= 1.2 for |y| = 1).  The three
// products hi*hi + hi*lo + lo*hi leave ~2^-22 of each term: ~5e-7 sigma on a
// rotated coordinate and ~5e-7 |r| on a projection, far inside the 1e-5
// bands of the code parity.  The scales are exact and cancel: Y is divided by
// |x| 2^(e + 8); P only gives its signs.  Without the tensor-map encoder the
// products run as fp32 SIMT GEMMs (tq_gemm.cu) on the unsplit rows.
#include <cuda_fp16.h>

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

// One warp per row: |x| (fp64 accumulation), the row scale |x| 2^(e + 8) of the
// rotation's output (2^8: the scale of Pi's pieces), and the fp16 pieces of
// 2^e x with |x| 2^e in [2^10, 2^11) -- hi to out[0], lo to out[1] (fp32 rows
// only: a bf16 row scaled by 2^e is one exact fp16 piece).  x = 0 gives zero
// pieces and scale 0 (the GEMM then writes y = 0).
template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&v)[4]) {
    if constexpr (sizeof(T) == 4) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    } else {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xFFFF0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    }
}

// Rows whose start is 16-byte (fp32) or 8-byte (bf16) aligned are read 4
// values a lane; d is a multiple of 128.
template <typename T>
__global__ void k_rownorm_split16(const T* __restrict__ x, int64_t rows, int d,
                                  float* __restrict__ xnorm, float* __restrict__ rs,
                                  __half* __restrict__ out) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const T* xr = x + row * d;
    const bool vec = ((uintptr_t)xr % (4 * sizeof(T))) == 0;  // the same for every row
    double acc = 0.0;
    if (vec) {
        for (int i = 4 * lane; i < d; i += 128) {
            float v[4];
            load4(xr + i, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc = fma((double)v[e], (double)v[e], acc);
        }
    } else {
        for (int i = lane; i < d; i += 32) {
            const double v = (double)load_f32(xr, i);
            acc = fma(v, v, acc);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const double nrm = sqrt(acc);
    const float nf = (float)nrm;
    int E = 0;
    if (nf > 0.f) frexp((double)nf, &E);  // nf = m 2^E, m in [0.5, 1)
    const int e = nf > 0.f ? 11 - E : 0;
    const double sc = ldexp(1.0, e);      // exact; 2^e may exceed fp32's range
    if (lane == 0) {
        xnorm[row] = nf;
        rs[row] = (float)ldexp((double)nf, e + 8);  // in [2^18, 2^19), or 0
    }
    __half* hi = out + row * d;
    __half* lo = out + rows * d + row * d;
    if (vec) {
        for (int i = 4 * lane; i < d; i += 128) {
            float v[4];
            load4(xr + i, v);
            uint32_t hw[2], lw[2];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const float a = (float)((double)v[2 * p] * sc);  // exact, |a| <= 2^11
                const float b = (float)((double)v[2 * p + 1] * sc);
                const __half2 h = __floats2half2_rn(a, b);
                const float2 hf = __half22float2(h);
                const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
                hw[p] = *reinterpret_cast<const uint32_t*>(&h);
                lw[p] = *reinterpret_cast<const uint32_t*>(&l);
            }
            *reinterpret_cast<uint2*>(hi + i) = make_uint2(hw[0], hw[1]);
            if (sizeof(T) == 4) *reinterpret_cast<uint2*>(lo + i) = make_uint2(lw[0], lw[1]);
        }
    } else {
        for (int i = lane; i < d; i += 32) {
            const float v = (float)((double)load_f32(xr, i) * sc);  // exact, |v| <= 2^11
            const __half h = __float2half_rn(v);
            hi[i] = h;
            if (sizeof(T) == 4) lo[i] = __float2half_rn(v - __half2float(h));
        }
    }
}

// One warp per row: bucketize each rotated coordinate, the cell index to a byte
// array, |r|, and the fp16 pieces of rscale * r (r = y - c[idx]) -- hi to
// rp[0], lo to rp[1] -- as the operand of the QJL product.  Coordinates from
// `half` on take the second grid of a fractional width (c_lo, beta_lo).  A
// lane takes 4 consecutive coordinates per step (16-byte loads, 4-byte cell
// and 8-byte piece stores; d and `half` are multiples of 4); the grids sit in
// shared memory, read as broadcasts.
__global__ void __launch_bounds__(256)
k_quantize16(const float* __restrict__ yr, uint8_t* __restrict__ idx, int64_t rows, int d,
             KCodebook cb, float rscale, float* __restrict__ rnorm, __half* __restrict__ rp,
             int half) {
    __shared__ float s_c[2][16], s_b[2][16];
    if (threadIdx.x < 16) {
        s_c[0][threadIdx.x] = cb.c[threadIdx.x];
        s_b[0][threadIdx.x] = cb.beta[threadIdx.x];
    } else if (threadIdx.x < 32) {
        s_c[1][threadIdx.x - 16] = cb.c_lo[threadIdx.x - 16];
        s_b[1][threadIdx.x - 16] = cb.beta_lo[threadIdx.x - 16];
    }
    __syncthreads();
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const float4* y = reinterpret_cast<const float4*>(yr + row * d);
    uint32_t* ix = reinterpret_cast<uint32_t*>(idx + row * d);
    uint2* hi = reinterpret_cast<uint2*>(rp + row * d);
    uint2* lo = reinterpret_cast<uint2*>(rp + rows * d + row * d);
    float rr = 0.f;
    for (int i4 = lane; i4 < d / 4; i4 += 32) {
        const float4 v4 = y[i4];
        const int g = (4 * i4 >= half) ? 1 : 0;  // the second grid of a fractional width
        const int levels = g ? cb.levels_lo : cb.levels;
        const float v[4] = {v4.x, v4.y, v4.z, v4.w};
        uint32_t cells = 0u;
        __half h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int cell = 0;
            float r = v[e];
            if (levels > 0) {
#pragma unroll
                for (int j = 0; j < 15; ++j)
                    if (j + 1 < levels && s_b[g][j] <= v[e]) ++cell;
                r = v[e] - s_c[g][cell];
            }
            cells |= (uint32_t)cell << (8 * e);
            rr = fmaf(r, r, rr);
            const float t = r * rscale;  // exact: a power of two
            h[e] = __float2half_rn(t);
            l[e] = __float2half_rn(t - __half2float(h[e]));
        }
        ix[i4] = cells;
        hi[i4] = make_uint2((uint32_t)__half_as_ushort(h[0]) | ((uint32_t)__half_as_ushort(h[1]) << 16),
                            (uint32_t)__half_as_ushort(h[2]) | ((uint32_t)__half_as_ushort(h[3]) << 16));
        lo[i4] = make_uint2((uint32_t)__half_as_ushort(l[0]) | ((uint32_t)__half_as_ushort(l[1]) << 16),
                            (uint32_t)__half_as_ushort(l[2]) | ((uint32_t)__half_as_ushort(l[3]) << 16));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rr += __shfl_xor_sync(0xffffffffu, rr, o);
    if (lane == 0) rnorm[row] = sqrtf(rr);
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

// One 32-coordinate block of a record: lane j holds coordinate j's cell index
// field `iv` and sign z; the warp ORs neighbouring lanes' fields together with
// a butterfly inside each word's lanes and writes the block's B words.
template <int B>
__device__ __forceinline__ void pack_block(int lane, uint32_t iv, uint32_t z, uint32_t* out) {
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

// One warp per row; lane j handles coordinate 32w + j of block w.
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
        pack_block<B>(lane, iv, z, codes + row * W + w * B);
    }
}

// Fractional width b - 1/2: the first d/64 blocks in the layout of width B,
// the last d/64 in the layout of width B - 1, d/64 (2B - 1) words a record.
template <int B>
__global__ void k_pack_split(const float* __restrict__ p, const uint8_t* __restrict__ idx,
                             int64_t rows, int d, uint32_t* __restrict__ codes) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const int h = d / 64;  // blocks per half
    uint32_t* rec = codes + row * (int64_t)(h * (2 * B - 1));
    for (int w = 0; w < d / 32; ++w) {
        const int i = 32 * w + lane;
        const uint32_t cell = idx[row * d + i];
        const uint32_t z = (p[row * d + i] >= 0.f) ? 1u : 0u;
        if (w < h) pack_block<B>(lane, cell, z, rec + w * B);
        else pack_block<B - 1>(lane, cell, z, rec + h * B + (w - h) * (B - 1));
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
    const bool split = is_split(cb);
    if (split && (mse || b < 2 || d % 64)) return TQ_ERR_UNSUPPORTED;
    if (!mse && !split && encode_tc_supported(cb, x_dtype, G, n) && (uintptr_t)d_x % 16 == 0 &&
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
    const int W = record_words(cb);
    const size_t esz = (x_dtype == TQ_F32) ? 4 : 2;
    const size_t dd = (size_t)d * d;
    // the rotation and QJL products on the tensor cores, else fp32 SIMT GEMMs
    const bool tcg = gemm_tc_supported(d, d);
    if (split && !tcg) return TQ_ERR_UNSUPPORTED;  // the SIMT fallback has one grid
    // inner-product records at d % 256 == 0: the CTA-pair GEMMs with the
    // bucketize and packing in their epilogues
    int nsm_dev = 0, dev_id = 0;
    TQ_TRY_CUDA(cudaGetDevice(&dev_id));
    TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm_dev, cudaDevAttrMultiProcessorCount, dev_id));
    const bool fused = tcg && !mse && d % 256 == 0 && nsm_dev >= 2;
    // tensor-core GEMMs: fp16 pieces [2][d][d] of 2^8 Pi_g and of 2^4 S_g, the
    // chunk's operand pieces [2][chunk][d] (x, then r) and its row scales
    __half* PiP = (__half*)(IX + align256((size_t)chunk * d));
    __half* SP = (__half*)((char*)PiP + align256(3 * dd * 2));
    __half* AP = (__half*)((char*)SP + align256(3 * dd * 2));
    float* RS = (float*)((char*)AP + align256((size_t)2 * chunk * d * 2));
    int sr = 6;  // 2^sr ~ 64 sqrt(d)
    while ((1 << (2 * (sr - 6))) < d) ++sr;
    const float rscale = ldexpf(1.f, sr);
    for (int g = 0; g < G; ++g) {
        if (tcg) {
            int rc = split_f16x2(d_Pi + g * dd, (int64_t)dd, 256.f, PiP, s);
            if (rc) return rc;
            if (!mse) {
                rc = split_f16x2(d_S + g * dd, (int64_t)dd, 16.f, SP, s);
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
            int rc;
            if (tcg) {  // Y = X Pi^T / |x| on the tensor cores (fp16 pieces)
                if (x_dtype == TQ_F32)
                    k_rownorm_split16<float><<<wblocks, 256, 0, s>>>((const float*)xg, rows, d, xn,
                                                                     RS, AP);
                else
                    k_rownorm_split16<__nv_bfloat16><<<wblocks, 256, 0, s>>>(
                        (const __nv_bfloat16*)xg, rows, d, xn, RS, AP);
                TQ_CHECK_LAUNCH();
                if (fused) {
                    // the bucketize in the rotation's epilogue (cells, pieces of
                    // r in Y's space, |r|^2 partials in P's), the packing in the
                    // QJL product's: Y and P never reach HBM
                    uint32_t* cgf = d_codes + (size_t)off * W;
                    EncodeEpi e1 = {};
                    e1.mode = 1;
                    e1.b = b;
                    e1.rscale = rscale;
                    e1.idx = IX;
                    e1.rp = (__half*)Y;
                    e1.rn2 = P;
                    e1.cb = kc;
                    rc = launch_gemm_tc((int)rows, d, d, (const __nv_bfloat16*)AP,
                                        x_dtype == TQ_F32 ? 2 : 1, (const __nv_bfloat16*)PiP,
                                        nullptr, d, RS, 1, err, s, 2, false, 0, nullptr, 0, true,
                                        true, &e1);
                    if (rc) return rc;
                    EncodeEpi e2 = e1;
                    e2.mode = 2;
                    e2.codes = cgf;
                    e2.rnorm = rn;
                    rc = launch_gemm_tc((int)rows, d, d, (const __nv_bfloat16*)Y, 2,
                                        (const __nv_bfloat16*)SP, nullptr, d, nullptr, 0, err, s,
                                        2, false, 0, nullptr, 0, true, true, &e2);
                    if (rc) return rc;
                    continue;
                }
                if (mse && d == 128) {
                    // the rotation with the bucketize and packing of whole rows in
                    // its epilogue (the MSE-only records have no QJL product)
                    EncodeEpi e4 = {};
                    e4.mode = 4;
                    e4.b = b;
                    e4.codes = d_codes + (size_t)off * W;
                    e4.rnorm = rn;
                    e4.cb = kc;
                    rc = launch_gemm_tc((int)rows, d, d, (const __nv_bfloat16*)AP,
                                        x_dtype == TQ_F32 ? 2 : 1, (const __nv_bfloat16*)PiP,
                                        nullptr, d, RS, 1, err, s, 2, false, 0, nullptr, 0, true,
                                        false, &e4);
                    if (rc) return rc;
                    continue;
                }
                rc = launch_gemm_tc((int)rows, d, d, (const __nv_bfloat16*)AP,
                                    x_dtype == TQ_F32 ? 2 : 1, (const __nv_bfloat16*)PiP, Y, d, RS,
                                    1, err, s, 2, false, 0, nullptr, 0, true);
            } else {
                if (x_dtype == TQ_F32)
                    k_rownorm<float><<<wblocks, 256, 0, s>>>((const float*)xg, rows, d, xn);
                else
                    k_rownorm<__nv_bfloat16><<<wblocks, 256, 0, s>>>((const __nv_bfloat16*)xg,
                                                                     rows, d, xn);
                TQ_CHECK_LAUNCH();
                rc = launch_sgemm((int)rows, d, d, xg, x_dtype, d, d_Pi + g * dd, true, d, Y, d,
                                  xn, 1, s);
            }
            if (rc) return rc;
            uint32_t* cg = d_codes + (size_t)off * W;
            if (mse) {  // no QJL projection
                k_quantize<<<wblocks, 256, 0, s>>>(Y, IX, rows, d, kc, rn);
                TQ_CHECK_LAUNCH();
                switch (b) {
                    case 1: k_pack<1, true><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    case 2: k_pack<2, true><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    case 3: k_pack<3, true><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    default: k_pack<4, true><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                }
                TQ_CHECK_LAUNCH();
                continue;
            }
            if (tcg) {  // P = (2^sr R)(2^4 S)^T on the tensor cores: only its signs are kept
                k_quantize16<<<wblocks, 256, 0, s>>>(Y, IX, rows, d, kc, rscale, rn, AP,
                                                      split ? d / 2 : d);
                TQ_CHECK_LAUNCH();
                rc = launch_gemm_tc((int)rows, d, d, (const __nv_bfloat16*)AP, 2,
                                    (const __nv_bfloat16*)SP, P, d, nullptr, 0, err, s, 2, false,
                                    0, nullptr, 0, true);
            } else {
                k_quantize<<<wblocks, 256, 0, s>>>(Y, IX, rows, d, kc, rn);
                TQ_CHECK_LAUNCH();
                rc = launch_sgemm((int)rows, d, d, Y, TQ_F32, d, d_S + g * dd, true, d, P, d,
                                  nullptr, 0, s);
            }
            if (rc) return rc;
            if (split) {
                switch (b) {
                    case 2: k_pack_split<2><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    case 3: k_pack_split<3><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    default: k_pack_split<4><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                }
            } else {
                switch (b) {
                    case 1: k_pack<1, false><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    case 2: k_pack<2, false><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    case 3: k_pack<3, false><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                    default: k_pack<4, false><<<wblocks, 256, 0, s>>>(P, IX, rows, d, cg); break;
                }
            }
            TQ_CHECK_LAUNCH();
        }
    }
    return TQ_OK;
}
