// E1-E6 fused on the sm_100a tensor cores, for d = 128 and bf16 inputs
// (KV-cache keys): norm, rotation, Lloyd-Max bucketize, residual, QJL
// projection, sign and packing in one persistent kernel.
//
// Pages: quant_prune_distill #674 (rotate by a random orthogonal matrix;
// Lloyd-Max grid at b-1 bits; 1-bit QJL of the residual: random matrix,
// sign); RecSysChannel #256 caveat 1 (normalise and multiply by a random
// matrix); seeallochnaya #3476 (round every coordinate on the fixed grid;
// residual -> random matrix -> sign; "parallelises well on a GPU").
//
// Design (vector-major: a tile is 128 vectors = the MMA's M rows, the 128
// output coordinates its N columns, so a TMEM lane holds one vector):
//  * Keys are converted in shared memory from bf16 to fp16 after a power of
//    two per vector, 2^e, brings |x| into [128, 256): every bf16 value is
//    then an exact fp16 (8 significant bits of 11), so the rotation needs
//    only the pieces of Pi: 2^8 Pi = p1 + p2 (fp16, to ~2^-22), 2 passes.
//    The epilogue warps do this for tile k + 1 (4 threads per key, norm
//    combined by shuffles) before they process tile k.
//  * The weights are the MMA's B operand in shared memory (K-major, 128-byte
//    swizzle): 2^8 Pi as p1, p2 and S as s1, s2 (fp16), 128 KB per group.
//  * Epilogue thread = (vector, 32-coordinate block): y' = 2^10 y from D1,
//    bucketize (a table over y'/32 gives the cell below and the one boundary
//    that can fall inside each 32-wide interval), r' = y' - c'[idx], the block's part of |r'|^2, and r' as two
//    fp16 pieces written to TMEM as the A operand of D2 = R S^T (3 passes:
//    h1 s1 + h2 s1 + h1 s2).  Sign bits come back from D2 in the same
//    thread, so the block's code words are packed in registers and stored
//    whole: no cross-lane packing or reduction.  The second half of a tile
//    (signs, packing, stores) runs after the first half of the next tile so
//    the QJL MMA overlaps epilogue work.
//  * TMEM columns: [0,256) D1 x2 | [256,384) R pieces | [384,512) D2.
//  * Warp roles: 0 TMA producer, 1 TMEM owner + MMA issuer, 2-17 norms,
//    fp16 conversion and epilogue (4 lane quarters x 4 blocks).
//  * Every wait is bounded (1 s); a warp that gives up sets the abort flag and
//    the device status word, all roles leave their loops, in-flight TMA loads
//    and MMAs are drained (again bounded) and TMEM is released.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTN = 128;                     // vectors per tile (MMA M)
constexpr int kXS = 2;                       // key-tile stages
constexpr int kInv = 4;                      // slots of the per-vector scale ring
constexpr int kEpi = 16;                     // epilogue warps: 4 lane quarters x 4 blocks
constexpr int kThreads = 32 * (2 + kEpi);
constexpr int kLut = 128;                    // bucketize table: y'/32 rounded, mod 128
constexpr float kLutStep = 32.f;
constexpr uint32_t kColD1 = 0, kColR = 256, kColD2 = 384, kTmemCols = 512;
constexpr uint32_t kRegion = kTN * 128;      // 128 rows x 128 bytes: k < 64 or k >= 64
constexpr uint32_t kTileBytes = 2 * kRegion; // one 128 x 128 16-bit operand
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s per wait
constexpr float kRScale = 1024.f;            // r * 2^10 keeps fp16 pieces normal
constexpr float kPiScale = 256.f;            // 2^8 Pi keeps the second piece normal
constexpr uint32_t kIdescF16 = idesc_f16(0, 128, 128);  // fp16 x fp16 -> f32, K-major

struct Smem {
    uint8_t x[kXS][kTileBytes];    // keys: bf16 from TMA, then fp16 in place (1024-aligned)
    uint8_t wpi[2][kTileBytes];    // 2^8 Pi pieces p1, p2
    uint8_t ws[2][kTileBytes];     // S pieces s1, s2
    float4 lut[kLut][8];           // (boundary, c'[cell], c'[cell + 1], cell), 8 copies
    float inv[kInv][kTN];          // 2^10 / (|x| 2^e 2^8) per vector
    float rr[2][4][kTN];           // [tile parity][block] |r'|^2 partial sums
    float c[8];                    // 2^10 c
    float beta[8];                 // 2^10 beta
    uint64_t full_x[kXS], xready[kXS], empty_x[kXS];
    uint64_t d1_full[2], d1_empty[2], r_full, d2_full, d2_empty, w_ready, mma_done;
    uint32_t tmem_base;
    int abort;
    int zero;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

// Byte offset of 16-bit element (row, k) in a K-major 128 x 128 operand with
// the 128-byte swizzle (the layout TMA writes for a {64, 128} box).
__device__ __forceinline__ uint32_t sw128_offset(int row, int k) {
    return (uint32_t)(k >> 6) * kRegion + (uint32_t)row * 128u +
           ((((uint32_t)(k >> 3) & 7u) ^ ((uint32_t)row & 7u)) << 4) + (uint32_t)(k & 7) * 2u;
}

// Tiles of this CTA: groups are spread over CTAs (cpg CTAs per group when
// G <= #CTAs, else whole groups round-robin).  f(g, t, first, last) -> bool.
template <class F>
__device__ __forceinline__ void for_each_tile(int G, int tpg, F&& f) {
    const int cta = blockIdx.x, nctas = gridDim.x;
    if (G <= nctas) {
        const int cpg = nctas / G;
        if (cta >= cpg * G) return;
        const int g = cta / cpg, slot = cta % cpg;
        for (int t = slot; t < tpg; t += cpg)
            if (!f(g, t, t == slot, t + cpg >= tpg)) return;
    } else {
        for (int g = cta; g < G; g += nctas)
            for (int t = 0; t < tpg; ++t)
                if (!f(g, t, t == 0, t == tpg - 1)) return;
    }
}

// mbar_wait agreed by the whole warp (all lanes continue, or all give up), so
// that no partial warp reaches a .sync.aligned tcgen05 instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort, kWaitNs);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool give_up(volatile int* abort, int* err, int site) {
    *abort = 1;
    atomicCAS(err, 0, TQ_ERR_DEVICE_TIMEOUT * 1000 - site);
    return false;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Weights of one group into shared memory as fp16 pieces, by the 512
// epilogue threads (te): M (d x d fp32, row-major: B operand row n = output
// coordinate, k = input coordinate) times `scale` = hi + lo.  A thread
// converts 16-byte chunks (8 k of one row) and keeps its loads in flight.
__device__ __forceinline__ void weights_to_smem(const float* __restrict__ M, float scale,
                                                uint8_t* hi, uint8_t* lo, int te) {
    constexpr int kChunks = kD * kD / 8 / (32 * kEpi);  // 4
    float4 v[kChunks][2];
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
        const int c = te + 32 * kEpi * u;  // row c >> 4, k = 8 (c & 15) ..
        const float4* src = reinterpret_cast<const float4*>(M + (size_t)(c >> 4) * kD) + 2 * (c & 15);
        v[u][0] = __ldg(src);
        v[u][1] = __ldg(src + 1);
    }
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
        const int c = te + 32 * kEpi * u;
        const float e[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w,
                            v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float a = e[2 * p] * scale, b = e[2 * p + 1] * scale;
            const __half2 h = __floats2half2_rn(a, b);
            const float2 hf = __half22float2(h);
            wh[p] = h2_bits(h);
            wl[p] = h2_bits(__floats2half2_rn(a - hf.x, b - hf.y));
        }
        const uint32_t off = sw128_offset(c >> 4, 8 * (c & 15));
        *reinterpret_cast<uint4*>(hi + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        *reinterpret_cast<uint4*>(lo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    }
}

// Code words of one 32-coordinate block (layout of tq.h): the cell fields
// packed during bucketize and z = [p >= 0] for the QJL projections p.  Every
// z starts set and a negative p clears its bit (p + 0 turns -0 into +0, so the
// sign of the sum is exactly p < 0); the words are stored whole at dst.
template <int B>
__device__ __forceinline__ void store_block(const uint32_t (&cellw)[4], const uint32_t (&p)[32],
                                            uint32_t* __restrict__ dst) {
    constexpr uint32_t kZ = (B == 4) ? 0x88888888u : ((B == 2) ? 0xAAAAAAAAu : 0u);
    uint32_t w[4] = {cellw[0] | kZ, cellw[1] | kZ, cellw[2] | kZ, cellw[3] | kZ};
    uint32_t sw = 0xFFFFFFFFu;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint32_t neg = __float_as_uint(__uint_as_float(p[j]) + 0.f) >> 31;
        if (B == 4) w[j >> 3] -= neg << (4 * (j & 7) + 3);
        if (B == 2) w[j >> 4] -= neg << (2 * (j & 15) + 1);
        if (B == 1 || B == 3) sw -= neg << j;
    }
    if (B == 4) *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    if (B == 3) {
        dst[0] = w[0];
        dst[1] = w[1];
        dst[2] = sw;
    }
    if (B == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    if (B == 1) dst[0] = sw;
}

// Number of tiles of this CTA, and its k-th tile, in the order of for_each_tile.
__device__ __forceinline__ int tile_count(int G, int tpg) {
    const int cta = blockIdx.x, nctas = gridDim.x;
    if (G <= nctas) {
        const int cpg = nctas / G;
        if (cta >= cpg * G) return 0;
        const int slot = cta % cpg;
        return slot < tpg ? (tpg - slot + cpg - 1) / cpg : 0;
    }
    return cta < G ? ((G - cta + nctas - 1) / nctas) * tpg : 0;
}

__device__ __forceinline__ void tile_at(int k, int G, int tpg, int& g, int& t, bool& first) {
    const int cta = blockIdx.x, nctas = gridDim.x;
    if (G <= nctas) {
        const int cpg = nctas / G;
        g = cta / cpg;
        t = cta % cpg + k * cpg;
        first = k == 0;
    } else {
        g = cta + (k / tpg) * nctas;
        t = k % tpg;
        first = t == 0;
    }
}

template <int B>
__global__ void __launch_bounds__(kThreads, 1)
k_encode_tc(const __grid_constant__ CUtensorMap tmap_x, const float* __restrict__ Pi,
            const float* __restrict__ S, KCodebook cb, int G, int64_t n, int tpg,
            uint32_t* __restrict__ codes, float* __restrict__ xnorm, float* __restrict__ rnorm,
            int* __restrict__ err) {
    constexpr int L = (B == 1) ? 1 : (1 << (B - 1));
    constexpr int W = B * kD / 32;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment by pointer arithmetic on the shared array itself, so
    // every access below stays a shared-memory (not generic) access
    const uint32_t sbase = smem_u32(smem_raw);
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kXS; ++s) {
            mbar_init(&sm.full_x[s], 1);
            mbar_init(&sm.xready[s], kEpi);  // converted by every epilogue warp
            mbar_init(&sm.empty_x[s], 1);    // MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.d1_full[b], 1);
            mbar_init(&sm.d1_empty[b], kEpi);
        }
        mbar_init(&sm.r_full, kEpi);
        mbar_init(&sm.d2_full, 1);
        mbar_init(&sm.d2_empty, kEpi);
        mbar_init(&sm.w_ready, kEpi);
        mbar_init(&sm.mma_done, 1);
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // static indices: the codebook stays out of local memory
            sm.c[k] = cb.c[k] * kRScale;      // exact (power of two)
            sm.beta[k] = cb.beta[k] * kRScale;
        }
        sm.abort = 0;
        sm.zero = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tmap_x);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    if (B >= 3) {
        // Bucketize table over i = round(y'/32) + 64 (mod 128): y' in
        // [(i - 64.5) 32, (i - 63.5) 32] has `below` boundaries under the
        // interval and at most one inside it (the host checks that the
        // boundaries are more than 32 apart).  Entry: (that boundary or
        // +huge, c'[below], c'[below + 1], below).
        for (int e = threadIdx.x; e < kLut * 8; e += blockDim.x) {
            const int li = e >> 3;
            const float lo = ((float)li - 64.5f) * kLutStep, hi = ((float)li - 63.5f) * kLutStep;
            int below = 0;
            float bstar = 3.0e38f;
            for (int k = 0; k + 1 < L; ++k) {
                const float bk = sm.beta[k];
                if (bk < lo) ++below;
                else if (bk <= hi && bstar == 3.0e38f) bstar = bk;
            }
            const int above = below + 1 < L ? below + 1 : below;
            sm.lut[li][e & 7] = make_float4(bstar, sm.c[below], sm.c[above],
                                            __uint_as_float((uint32_t)below));
        }
        __syncthreads();
    }

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        uint32_t i = 0;
        for_each_tile(G, tpg, [&](int g, int t, bool, bool) {
            const int s = i % kXS;
            if (i >= (uint32_t)kXS &&
                !mbar_wait(&sm.empty_x[s], ((i / kXS) - 1) & 1, abort, kWaitNs))
                return give_up(abort, err, 1);
            mbar_arrive_expect_tx(&sm.full_x[s], kTileBytes);
            const int32_t row = (int32_t)((int64_t)g * n + (int64_t)t * kTN);
            tma_load_2d(sm.x[s], &tmap_x, 0, row, &sm.full_x[s]);
            tma_load_2d(sm.x[s] + kRegion, &tmap_x, 64, row, &sm.full_x[s]);
            ++i;
            return true;
        });
        // no TMA write may still be in flight when the CTA exits
        for (uint32_t j = (i > (uint32_t)kXS ? i - kXS : 0); j < i; ++j)
            mbar_wait(&sm.full_x[j % kXS], (j / kXS) & 1, &sm.zero, kWaitNs);
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        uint32_t i = 0, gi = 0;
        auto qjl = [&](uint32_t j) -> bool {
            if (!mbar_wait(&sm.r_full, j & 1, abort, kWaitNs)) return give_up(abort, err, 2);
            if (j >= 1 && !mbar_wait(&sm.d2_empty, (j - 1) & 1, abort, kWaitNs))
                return give_up(abort, err, 12);
            tc_fence_after();
#pragma unroll
            for (int combo = 0; combo < 3; ++combo) {  // h1 s1, h2 s1, h1 s2
                const uint32_t a = tbase + kColR + (combo == 1 ? 64u : 0u);
                const uint32_t wb = smem_u32(sm.ws[combo == 2 ? 1 : 0]);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)  // 16 coordinates per step
                    mma_f16_ts(tbase + kColD2, a + ks * 8,
                               smem_desc_kmajor_sw128(wb + (ks >> 2) * kRegion + (ks & 3) * 32),
                               kIdescF16, (combo | ks) != 0);
            }
            tc_commit(&sm.d2_full);
            return true;
        };
        for_each_tile(G, tpg, [&](int, int, bool first, bool last) {
            if (first) {
                if (!mbar_wait(&sm.w_ready, gi & 1, abort, kWaitNs)) return give_up(abort, err, 3);
                ++gi;
                tc_fence_after();
            }
            const int s = i % kXS, b = i & 1;
            if (!mbar_wait(&sm.xready[s], (i / kXS) & 1, abort, kWaitNs))
                return give_up(abort, err, 4);
            if (i >= 2 && !mbar_wait(&sm.d1_empty[b], ((i >> 1) - 1) & 1, abort, kWaitNs))
                return give_up(abort, err, 5);
            tc_fence_after();
            const uint32_t xs = smem_u32(sm.x[s]);
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint32_t wb = smem_u32(sm.wpi[p]);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t ko = (ks >> 2) * kRegion + (ks & 3) * 32;
                    mma_f16_ss(tbase + kColD1 + 128u * b, smem_desc_kmajor_sw128(xs + ko),
                               smem_desc_kmajor_sw128(wb + ko), kIdescF16, (p | ks) != 0);
                }
            }
            tc_commit(&sm.empty_x[s]);
            tc_commit(&sm.d1_full[b]);
            if (!first && !qjl(i - 1)) return false;
            if (last && !qjl(i)) return false;
            ++i;
            return true;
        });
        // every issued MMA completes before TMEM is released
        tc_commit(&sm.mma_done);
        mbar_wait(&sm.mma_done, 0, &sm.zero, kWaitNs);
    } else if (warp >= 2) {
        // ---------------- norms, fp16 conversion and epilogue ----------------
        const int ew = warp - 2;                       // 0 .. kEpi - 1
        const int q = warp & 3, h = ew >> 2;           // lane quarter, 32-coordinate block
        const int m = q * 32 + lane;                   // vector within the tile
        const uint32_t lane_addr = tbase + ((uint32_t)(q * 32) << 16);
        const int te = threadIdx.x - 64;               // 0 .. 32*kEpi - 1
        const int cr = 8 * ew + (lane & 7), cj = lane >> 3;  // conversion: key row, quarter
        const float4* lut = &sm.lut[0][lane & 7];
        const float bt0 = sm.beta[0], c0 = sm.c[0], c1 = sm.c[1];
        const int ntile = tile_count(G, tpg);

        // Norm of key row cr of tile k (4 threads, 32 bf16 each), its power of
        // two 2^e, and the row converted in place to fp16 x 2^e.
        auto convert = [&](int k) -> bool {
            int g, t;
            bool first;
            tile_at(k, G, tpg, g, t, first);
            const int s = k % kXS;
            if (!warp_wait(&sm.full_x[s], (k / kXS) & 1, abort)) return give_up(abort, err, 6);
            uint8_t* rowp = sm.x[s] + cr * 128;
            uint32_t off[4];
            uint4 u[4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const int c = cj + 4 * kk;  // 16-byte chunk: k = 8c .. 8c + 7
                off[kk] = (uint32_t)(c >> 3) * kRegion + ((((uint32_t)c & 7u) ^ ((uint32_t)cr & 7u)) << 4);
                u[kk] = *reinterpret_cast<const uint4*>(rowp + off[kk]);
            }
            float a2[2] = {0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t w4[4] = {u[kk].x, u[kk].y, u[kk].z, u[kk].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = __uint_as_float(w4[e] << 16);
                    const float hi = __uint_as_float(w4[e] & 0xffff0000u);
                    a2[e & 1] = fmaf(lo, lo, a2[e & 1]);
                    a2[e & 1] = fmaf(hi, hi, a2[e & 1]);
                }
            }
            float sum = a2[0] + a2[1];
            sum += __shfl_xor_sync(0xffffffffu, sum, 8);
            sum += __shfl_xor_sync(0xffffffffu, sum, 16);
            float nx = sqrtf(sum);
            const bool odd = !(sum >= 0x1p-96f && sum <= 0x1p+126f);
            if (__any_sync(0xffffffffu, odd)) {
                // squares under- or overflow fp32 (or a zero row): fp64 sums
                double acc = 0.0;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t w4[4] = {u[kk].x, u[kk].y, u[kk].z, u[kk].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const double lo = (double)__uint_as_float(w4[e] << 16);
                        const double hi = (double)__uint_as_float(w4[e] & 0xffff0000u);
                        acc = fma(lo, lo, acc);
                        acc = fma(hi, hi, acc);
                    }
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 8);
                acc += __shfl_xor_sync(0xffffffffu, acc, 16);
                if (odd) nx = (float)sqrt(acc);
            }
            // 2^e with |x| 2^e in [128, 256) (clamped for extreme norms)
            const int eb = (int)((__float_as_uint(nx) >> 23) & 0xffu);
            int ex = (eb == 0) ? 126 : 134 - eb;
            ex = ex < -120 ? -120 : (ex > 126 ? 126 : ex);
            const float sc = __uint_as_float((uint32_t)(ex + 127) << 23);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t w4[4] = {u[kk].x, u[kk].y, u[kk].z, u[kk].w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o[e] = h2_bits(__floats2half2_rn(__uint_as_float(w4[e] << 16) * sc,
                                                     __uint_as_float(w4[e] & 0xffff0000u) * sc));
                *reinterpret_cast<uint4*>(rowp + off[kk]) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            if (cj == 0) {
                sm.inv[k % kInv][cr] = (nx > 0.f) ? (kRScale / kPiScale) / (nx * sc) : 0.f;
                const int64_t v = (int64_t)t * kTN + cr;
                if (v < n) xnorm[(int64_t)g * n + v] = nx;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.xready[s]);
            return true;
        };

        // The second half of a tile (sign bits, packing, stores) runs after the
        // first half of the next tile.  State of the pending tile:
        bool pend = false;
        int pg = 0, pt = 0;
        uint32_t pidx = 0;
        uint32_t pcell[4] = {0u, 0u, 0u, 0u};
        auto wait_d2 = [&]() -> bool {  // the QJL MMA of the pending tile is done
            if (!warp_wait(&sm.d2_full, pidx & 1, abort)) return give_up(abort, err, 9);
            tc_fence_after();
            return true;
        };
        auto finish = [&]() {
            uint32_t p[32];
            tmem_ld32(lane_addr + kColD2 + 32u * h, p);
            tmem_wait_ld();
            // |r'|^2 of the tile is complete: every epilogue warp stored its part
            // before arriving on r_full, which the QJL MMA behind d2_full waited for
            float rn = 0.f;
            if (h == 0) {
                const float (*rrb)[kTN] = sm.rr[pidx & 1];
                rn = sqrtf((rrb[0][m] + rrb[1][m]) + (rrb[2][m] + rrb[3][m])) * (1.f / kRScale);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.d2_empty);
            const int64_t v = (int64_t)pt * kTN + m;
            if (v < n) {
                const int64_t rec = (int64_t)pg * n + v;
                if (h == 0) rnorm[rec] = rn;
                store_block<B>(pcell, p, codes + rec * W + B * h);
            }
            pend = false;
        };
        bool running = ntile == 0 || convert(0);
        for (int k = 0; running && k < ntile; ++k) {
            int g, t;
            bool first;
            tile_at(k, G, tpg, g, t, first);
            if (k + 1 < ntile && !convert(k + 1)) {
                running = false;
                break;
            }
            if (first) {
                // every MMA of the previous group is done once its last QJL MMA is
                if (pend) {
                    if (!wait_d2()) {
                        running = false;
                        break;
                    }
                    finish();
                }
                weights_to_smem(Pi + (size_t)g * kD * kD, kPiScale, sm.wpi[0], sm.wpi[1], te);
                weights_to_smem(S + (size_t)g * kD * kD, 1.f, sm.ws[0], sm.ws[1], te);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.w_ready);
            }
            const int b = k & 1, s = k % kXS;
            if (!warp_wait(&sm.d1_full[b], (k >> 1) & 1, abort)) {
                running = give_up(abort, err, 7);
                break;
            }
            tc_fence_after();
            uint32_t acc[32];
            tmem_ld32(lane_addr + kColD1 + 128u * b + 32u * h, acc);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.d1_empty[b]);
            // the scale of tile k was written before every warp arrived on xready
            if (!warp_wait(&sm.xready[s], (k / kXS) & 1, abort)) {
                running = give_up(abort, err, 8);
                break;
            }
            const float inv = sm.inv[k % kInv][m];

            uint32_t cellw[4] = {0u, 0u, 0u, 0u};
            float rr = 0.f;
            uint32_t hp1[16], hp2[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                float sr[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float y = __uint_as_float(acc[j + e]) * inv;  // 2^10 y
                    float r = y;
                    if (B >= 3) {
                        const float tf = fmaf(y, 1.f / kLutStep, 12582912.f + 64.f);
                        const float4 en = lut[(__float_as_uint(tf) & (kLut - 1)) * 8];
                        const bool up = y >= en.x;
                        r = y - (up ? en.z : en.y);
                        const uint32_t cc = __float_as_uint(en.w) + (up ? 1u : 0u);
                        if (B == 4) cellw[(j + e) >> 3] += cc << (4 * ((j + e) & 7));
                        else cellw[(j + e) >> 4] += cc << (2 * ((j + e) & 15));
                    } else if (B == 2) {
                        const bool up = y >= bt0;
                        r = y - (up ? c1 : c0);
                        if (up) cellw[(j + e) >> 4] += 1u << (2 * ((j + e) & 15));
                    }
                    rr = fmaf(r, r, rr);
                    sr[e] = r;
                }
                const __half2 h1 = __floats2half2_rn(sr[0], sr[1]);
                const float2 f1 = __half22float2(h1);
                hp1[j >> 1] = h2_bits(h1);
                hp2[j >> 1] = h2_bits(__floats2half2_rn(sr[0] - f1.x, sr[1] - f1.y));
            }
            // the QJL MMA of the pending tile still reads the R columns
            if (pend && !wait_d2()) {
                running = false;
                break;
            }
            tmem_st16(lane_addr + kColR + 16u * h, hp1);
            tmem_st16(lane_addr + kColR + 64u + 16u * h, hp2);
            sm.rr[b][h][m] = rr;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.r_full);

            if (pend) finish();
            pend = true;
            pg = g;
            pt = t;
            pidx = (uint32_t)k;
#pragma unroll
            for (int u = 0; u < 4; ++u) pcell[u] = cellw[u];
        }
        if (running && pend && wait_d2()) finish();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

template <int B>
int launch_b(const CUtensorMap& map, const float* Pi, const float* S, const KCodebook& kc, int G,
             int64_t n, int tpg, int nctas, uint32_t* codes, float* xn, float* rn, int* err,
             cudaStream_t s) {
    TQ_TRY_CUDA(cudaFuncSetAttribute(k_encode_tc<B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kSmemBytes));
    k_encode_tc<B><<<nctas, kThreads, kSmemBytes, s>>>(map, Pi, S, kc, G, n, tpg, codes, xn, rn,
                                                       err);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

}  // namespace

bool encode_tc_supported(const tq_codebook_t* cb, int x_dtype, int G, int64_t n) {
    if (cb->d != kD || x_dtype != TQ_BF16 || (int64_t)G * n >= ((int64_t)1 << 31)) return false;
    // the bucketize table holds at most one boundary per 32 / 2^10 of y
    for (int k = 0; k + 2 < cb->levels; ++k)
        if (!(cb->boundaries[k + 1] - cb->boundaries[k] > kLutStep / kRScale)) return false;
    return encode_tiled_fn() != nullptr;
}

int launch_encode_tc(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G,
                     int64_t n, const void* d_x, uint32_t* d_codes, float* d_xnorm,
                     float* d_rnorm, int* d_err, cudaStream_t s) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return TQ_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)kD, (cuuint64_t)((int64_t)G * n)};
    const cuuint64_t gstride[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kTN};
    const cuuint32_t estride[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(d_x), gdim, gstride, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return TQ_ERR_CUDA;
    int dev = 0, nsm = 0;
    TQ_TRY_CUDA(cudaGetDevice(&dev));
    TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    const int tpg = (int)((n + kTN - 1) / kTN);
    const int64_t units = (int64_t)G * tpg;
    const int nctas = (int)(units < nsm ? units : nsm);
    TQ_TRY_CUDA(cudaMemsetAsync(d_err, 0, sizeof(int), s));
    const KCodebook kc = make_kcodebook(cb);
    switch (cb->b) {
        case 1: return launch_b<1>(map, d_Pi, d_S, kc, G, n, tpg, nctas, d_codes, d_xnorm, d_rnorm, d_err, s);
        case 2: return launch_b<2>(map, d_Pi, d_S, kc, G, n, tpg, nctas, d_codes, d_xnorm, d_rnorm, d_err, s);
        case 3: return launch_b<3>(map, d_Pi, d_S, kc, G, n, tpg, nctas, d_codes, d_xnorm, d_rnorm, d_err, s);
        default: return launch_b<4>(map, d_Pi, d_S, kc, G, n, tpg, nctas, d_codes, d_xnorm, d_rnorm, d_err, s);
    }
}

}  // namespace tq
