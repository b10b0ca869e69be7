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
// Design (transposed orientation: output coordinates are the MMA's M = 128
// rows, vectors its N = 64 columns):
//  * The weights live in tensor memory as the MMA's A operand for the whole
//    kernel: Pi as three bf16 pieces (Pi = p1 + p2 + p3 to ~2^-24) and S as
//    two fp16 pieces (S = s1 + s2 to ~2^-22).  TMEM columns:
//      [0,192) Pi pieces | [192,320) S pieces | [320,448) D1 x2 | [448,512) D2
//  * A tile of 64 bf16 key vectors arrives by TMA (128-byte swizzle) and is
//    the B operand as is: bf16 x bf16 products are exact, so the rotation
//    D1 = Pi X^T is fp32-accurate after 3 passes.
//  * Epilogue warps (thread = output coordinate) work in units scaled by 2^10
//    (exact: 1/|x|, boundaries and centroids are pre-multiplied): y' = 2^10 y,
//    bucketize, r' = y' - c'[idx], |r|^2, and r' as two fp16 pieces written
//    coordinate-major (one 128-byte row per coordinate, vectors contiguous):
//    the MN-major B operand of D2 = S R^T (3 passes: s1 h1 + s1 h2 + s2 h1).
//    Only the sign of D2 is kept.
//  * Warp roles: 0 TMA producer, 1 TMEM owner + MMA issuer, 2-3 norms,
//    4..11 epilogue (two warps per TMEM lane quarter, 32 vectors each).
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
constexpr int kTN = 64;                      // vectors per tile (MMA N)
constexpr int kXS = 4;                       // key-tile stages
constexpr int kThreads = 384;
constexpr uint32_t kColPi = 0, kColS = 192, kColD1 = 320, kColD2 = 448, kTmemCols = 512;
constexpr uint32_t kStageBytes = kTN * kD * 2;   // two 8 KB swizzled regions (k < 64, k >= 64)
constexpr uint64_t kWaitNs = 1000000000ull;      // 1 s per wait
constexpr float kRScale = 1024.f;                // r * 2^10 keeps fp16 pieces normal
constexpr uint32_t kIdescRot = idesc_f16(1, 128, kTN);  // bf16 x bf16 -> f32
constexpr uint32_t kIdescQjl = idesc_f16(0, 128, kTN) | (1u << 16);  // fp16 x fp16, B MN-major

struct Smem {
    uint8_t x[kXS][kStageBytes];   // 1024-aligned (first member)
    uint8_t r[2][2][kStageBytes];  // [tile parity][piece h1, h2]: B operand of the QJL MMA
    uint32_t codes[kTN][16];       // packed records of the tile (W <= 16 words)
    float inv[kXS][kTN];           // 1/|x| per stage
    float rr[2][4][kTN];           // [tile parity][lane quarter] |r|^2 partial sums
    float c[8];
    float beta[8];
    uint64_t full_x[kXS], empty_x[kXS], norm_full[kXS];
    uint64_t d1_full[2], d1_empty[2], r_full, d2_full, d2_empty, w_ready, epi_bar, mma_done;
    uint32_t tmem_base;
    int abort;
    int zero;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

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

__device__ __forceinline__ uint32_t pack_bf16(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}
__device__ __forceinline__ uint32_t pack_f16(__half lo, __half hi) {
    return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// Row `row` of Pi (3 bf16 pieces) or S (2 fp16 pieces) into TMEM lane `row`:
// column c of a piece holds k = 2c (low half) and k = 2c + 1 (high half).
__device__ void load_weights(const float* __restrict__ Pi, const float* __restrict__ S, int g,
                             int row, int h, uint32_t taddr_lane) {
    if (h == 0) {
        const float* src = Pi + ((size_t)g * kD + row) * kD;
        for (int half = 0; half < 2; ++half) {
            uint32_t p1[32], p2[32], p3[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float2 v = __ldg(reinterpret_cast<const float2*>(src + 64 * half + 2 * c));
                __nv_bfloat16 a1 = __float2bfloat16_rn(v.x);
                float ra = v.x - __bfloat162float(a1);
                __nv_bfloat16 a2 = __float2bfloat16_rn(ra);
                __nv_bfloat16 a3 = __float2bfloat16_rn(ra - __bfloat162float(a2));
                __nv_bfloat16 b1 = __float2bfloat16_rn(v.y);
                float rb = v.y - __bfloat162float(b1);
                __nv_bfloat16 b2 = __float2bfloat16_rn(rb);
                __nv_bfloat16 b3 = __float2bfloat16_rn(rb - __bfloat162float(b2));
                p1[c] = pack_bf16(a1, b1);
                p2[c] = pack_bf16(a2, b2);
                p3[c] = pack_bf16(a3, b3);
            }
            tmem_st32(taddr_lane + kColPi + 0 + 32 * half, p1);
            tmem_st32(taddr_lane + kColPi + 64 + 32 * half, p2);
            tmem_st32(taddr_lane + kColPi + 128 + 32 * half, p3);
        }
    } else {
        const float* src = S + ((size_t)g * kD + row) * kD;
        for (int half = 0; half < 2; ++half) {
            uint32_t s1[32], s2[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float2 v = __ldg(reinterpret_cast<const float2*>(src + 64 * half + 2 * c));
                __half a1 = __float2half_rn(v.x);
                __half a2 = __float2half_rn(v.x - __half2float(a1));
                __half b1 = __float2half_rn(v.y);
                __half b2 = __float2half_rn(v.y - __half2float(b1));
                s1[c] = pack_f16(a1, b1);
                s2[c] = pack_f16(a2, b2);
            }
            tmem_st32(taddr_lane + kColS + 0 + 32 * half, s1);
            tmem_st32(taddr_lane + kColS + 64 + 32 * half, s2);
        }
    }
}

// Sum of v[j] over the 32 lanes for every j; lane l returns the sum for j = l.
__device__ __forceinline__ float transpose_reduce32(const float (&v)[32], int lane) {
    float a[16], b[8], c[4], d[2];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const bool up = lane & 16;
        const float keep = up ? v[i + 16] : v[i], send = up ? v[i] : v[i + 16];
        a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 8;
        const float keep = up ? a[i + 8] : a[i], send = up ? a[i] : a[i + 8];
        b[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 4;
        const float keep = up ? b[i + 4] : b[i], send = up ? b[i] : b[i + 4];
        c[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 2;
        const float keep = up ? c[i + 2] : c[i], send = up ? c[i] : c[i + 2];
        d[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    const bool up = lane & 1;
    const float keep = up ? d[1] : d[0], send = up ? d[0] : d[1];
    return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

// OR-combine fields of F lanes (F = 8 or 16, fields already shifted into
// place) for 32 vectors: afterwards lane e (= lane % F) holds the finished
// words of vectors j = e + F*i, i < 32/F.
template <int F>
__device__ __forceinline__ void transpose_or(const uint32_t (&v)[32], int lane,
                                             uint32_t (&out)[32 / F]) {
    uint32_t a[16], b[8], c[4], d[2];
    const int e = lane % F;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const bool up = e & 1;
        const uint32_t lo = v[2 * i], hi = v[2 * i + 1];
        a[i] = (up ? hi : lo) | __shfl_xor_sync(0xffffffffu, up ? lo : hi, 1);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = e & 2;
        const uint32_t lo = a[2 * i], hi = a[2 * i + 1];
        b[i] = (up ? hi : lo) | __shfl_xor_sync(0xffffffffu, up ? lo : hi, 2);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = e & 4;
        const uint32_t lo = b[2 * i], hi = b[2 * i + 1];
        c[i] = (up ? hi : lo) | __shfl_xor_sync(0xffffffffu, up ? lo : hi, 4);
    }
    if (F == 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) out[i] = c[i];
    } else {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const bool up = e & 8;
            const uint32_t lo = c[2 * i], hi = c[2 * i + 1];
            d[i] = (up ? hi : lo) | __shfl_xor_sync(0xffffffffu, up ? lo : hi, 8);
        }
#pragma unroll
        for (int i = 0; i < 32 / F; ++i) out[i] = d[i];
    }
}

// Pack the fields of this lane's coordinate (block q, position `lane`) for the
// warp's 32 vectors into sm.codes rows [32h, 32h + 32).
template <int B>
__device__ __forceinline__ void pack_tile(const int (&cell)[32], const uint32_t (&pbits)[32],
                                          int lane, int q, int h, uint32_t (*codes)[16]) {
    uint32_t z[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) z[j] = (__uint_as_float(pbits[j]) >= 0.f) ? 1u : 0u;
    if (B == 1 || B == 3) {
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const uint32_t w = __ballot_sync(0xffffffffu, z[j] != 0u);
            if (lane == j) mine = w;
        }
        codes[32 * h + lane][B * q + (B == 1 ? 0 : 2)] = mine;
    }
    if (B == 4) {
        uint32_t v[32], out[4];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = ((uint32_t)cell[j] | (z[j] << 3)) << (4 * (lane & 7));
        transpose_or<8>(v, lane, out);
#pragma unroll
        for (int i = 0; i < 4; ++i) codes[32 * h + (lane & 7) + 8 * i][4 * q + (lane >> 3)] = out[i];
    }
    if (B == 2 || B == 3) {
        uint32_t v[32], out[2];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const uint32_t f = (B == 2) ? ((uint32_t)cell[j] | (z[j] << 1)) : (uint32_t)cell[j];
            v[j] = f << (2 * (lane & 15));
        }
        transpose_or<16>(v, lane, out);
#pragma unroll
        for (int i = 0; i < 2; ++i) codes[32 * h + (lane & 15) + 16 * i][B * q + (lane >> 4)] = out[i];
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
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kXS; ++s) {
            mbar_init(&sm.full_x[s], 1);
            mbar_init(&sm.empty_x[s], 11);  // MMA commit + 2 norm warps + 8 epilogue warps
            mbar_init(&sm.norm_full[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.d1_full[b], 1);
            mbar_init(&sm.d1_empty[b], 8);
        }
        mbar_init(&sm.r_full, 8);
        mbar_init(&sm.d2_full, 1);
        mbar_init(&sm.d2_empty, 8);
        mbar_init(&sm.w_ready, 8);
        mbar_init(&sm.epi_bar, 8);
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

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        uint32_t i = 0;
        for_each_tile(G, tpg, [&](int g, int t, bool, bool) {
            const int s = i % kXS;
            if (i >= (uint32_t)kXS &&
                !mbar_wait(&sm.empty_x[s], ((i / kXS) - 1) & 1, abort, kWaitNs))
                return give_up(abort, err, 1);
            mbar_arrive_expect_tx(&sm.full_x[s], kStageBytes);
            const int32_t row = (int32_t)((int64_t)g * n + (int64_t)t * kTN);
            tma_load_2d(sm.x[s], &tmap_x, 0, row, &sm.full_x[s]);
            tma_load_2d(sm.x[s] + kStageBytes / 2, &tmap_x, 64, row, &sm.full_x[s]);
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
            const uint32_t d = tbase + kColD2;
            const uint32_t rb0 = smem_u32(sm.r[j & 1][0]), rb1 = smem_u32(sm.r[j & 1][1]);
#pragma unroll
            for (int combo = 0; combo < 3; ++combo) {  // s1 h1, s1 h2, s2 h1
                const uint32_t a = tbase + kColS + (combo == 2 ? 64u : 0u);
                const uint32_t rb = (combo == 1) ? rb1 : rb0;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)  // 16 coordinates = 16 rows of 128 B per step
                    mma_f16_ts(d, a + ks * 8, smem_desc_mnmajor_sw128(rb + ks * 2048),
                               kIdescQjl, (combo | ks) != 0);
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
            if (!mbar_wait(&sm.full_x[s], (i / kXS) & 1, abort, kWaitNs))
                return give_up(abort, err, 4);
            if (i >= 2 && !mbar_wait(&sm.d1_empty[b], ((i >> 1) - 1) & 1, abort, kWaitNs))
                return give_up(abort, err, 5);
            tc_fence_after();
            const uint32_t d = tbase + kColD1 + 64u * b;
            const uint32_t xs = smem_u32(sm.x[s]);
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16_ts(d, tbase + kColPi + 64u * p + ks * 8,
                               smem_desc_kmajor_sw128(xs + (ks >> 2) * (kStageBytes / 2) +
                                                      (ks & 3) * 32),
                               kIdescRot, (p | ks) != 0);
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
    } else if (warp == 2 || warp == 3) {
        // ---------------- norms (two warps, 32 vectors each) ----------------
        uint32_t i = 0;
        const int nr = lane + 32 * (warp - 2);
        for_each_tile(G, tpg, [&](int g, int t, bool, bool) {
            const int s = i % kXS;
            if (!warp_wait(&sm.full_x[s], (i / kXS) & 1, abort)) return give_up(abort, err, 6);
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int reg = 0; reg < 2; ++reg) {
                const uint4* rowp =
                    reinterpret_cast<const uint4*>(sm.x[s] + reg * (kStageBytes / 2) + nr * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = rowp[c];
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(w4[e] << 16);
                        const float hi = __uint_as_float(w4[e] & 0xffff0000u);
                        a4[e] = fmaf(lo, lo, a4[e]);
                        a4[e] = fmaf(hi, hi, a4[e]);
                    }
                }
            }
            const float nx = sqrtf((a4[0] + a4[1]) + (a4[2] + a4[3]));
            sm.inv[s][nr] = (nx > 0.f) ? kRScale / nx : 0.f;
            const int64_t v = (int64_t)t * kTN + nr;
            if (v < n) xnorm[(int64_t)g * n + v] = nx;
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.norm_full[s]);
                mbar_arrive(&sm.empty_x[s]);
            }
            ++i;
            return true;
        });
    } else if (warp >= 4) {
        // ---------------- epilogue ----------------
        const int q = warp & 3, h = (warp - 4) >> 2;
        const int coord = q * 32 + lane;
        const uint32_t lane_addr = tbase + ((uint32_t)(q * 32) << 16);
        // residual row of this coordinate: 128 bytes, 16-byte chunk c (vectors
        // 8c..8c+7) at position c ^ (coord % 8); this warp writes chunks 4h..4h+3
        uint32_t roff[4];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
            roff[ii] = (uint32_t)coord * 128u + ((((uint32_t)(4 * h + ii)) ^ (uint32_t)(coord & 7)) << 4);
        float bt[7];
#pragma unroll
        for (int k = 0; k < 7; ++k) bt[k] = sm.beta[k];
        uint32_t i = 0, eb = 0;
        const int te = threadIdx.x - 128;  // 0..255 over the epilogue warps
        auto epi_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.epi_bar);
            const bool ok = warp_wait(&sm.epi_bar, eb & 1, abort);
            ++eb;
            return ok;
        };
        // The second half of a tile (sign bits, packing, stores) runs after the
        // first half of the next tile, so the QJL MMA of a tile overlaps the
        // epilogue work of its successor.  State of the pending tile:
        bool pend = false;
        int pg = 0, pt = 0;
        uint32_t pidx = 0;
        uint32_t pcell[4] = {0u, 0u, 0u, 0u};
        auto finish = [&]() -> bool {
            if (!warp_wait(&sm.d2_full, pidx & 1, abort)) return give_up(abort, err, 9);
            tc_fence_after();
            uint32_t pb[32];
            tmem_ld32(lane_addr + kColD2 + 32u * h, pb);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.d2_empty);
            int cell[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) cell[j] = (int)((pcell[j >> 3] >> (4 * (j & 7))) & 15u);
            pack_tile<B>(cell, pb, lane, q, h, sm.codes);
            if (!epi_sync()) return give_up(abort, err, 10);
            const int64_t v0 = (int64_t)pt * kTN;
            const int valid = (int)((n - v0) < kTN ? (n - v0) : kTN);
            uint32_t* dst = codes + ((int64_t)pg * n + v0) * W;
            for (int e = te; e < valid * W; e += 256) dst[e] = sm.codes[e / W][e % W];
            const float (*rrb)[kTN] = sm.rr[pidx & 1];
            if (te < valid)
                rnorm[(int64_t)pg * n + v0 + te] =
                    sqrtf(rrb[0][te] + rrb[1][te] + rrb[2][te] + rrb[3][te]) * (1.f / kRScale);
            if (!epi_sync()) return give_up(abort, err, 11);
            pend = false;
            return true;
        };
        bool running = true;
        for_each_tile(G, tpg, [&](int g, int t, bool first, bool) {
            if (first) {
                // every MMA of the previous group must be done before its weights go
                if (pend && !finish()) return running = false;
                load_weights(Pi, S, g, coord, h, lane_addr);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.w_ready);
            }
            const int s = i % kXS, b = i & 1;
            if (!warp_wait(&sm.d1_full[b], (i >> 1) & 1, abort))
                return running = give_up(abort, err, 7);
            tc_fence_after();
            uint32_t acc[32];
            tmem_ld32(lane_addr + kColD1 + 64u * b + 32u * h, acc);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.d1_empty[b]);
            if (!warp_wait(&sm.norm_full[s], (i / kXS) & 1, abort))
                return running = give_up(abort, err, 8);
            float inv[32];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 t4 = *reinterpret_cast<const float4*>(&sm.inv[s][32 * h + j]);
                inv[j] = t4.x;
                inv[j + 1] = t4.y;
                inv[j + 2] = t4.z;
                inv[j + 3] = t4.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty_x[s]);

            uint32_t ccur[4] = {0u, 0u, 0u, 0u};
            float rr[32];
            uint32_t hp1[16], hp2[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                float sr[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float y = __uint_as_float(acc[j + e]) * inv[j + e];  // 2^10 y
                    uint32_t cc = 0;
                    float r = y;
                    if (B == 4) {  // three compares down the boundary tree
                        const bool p2 = y >= bt[3];
                        const bool p1 = y >= (p2 ? bt[5] : bt[1]);
                        const bool p0 = y >= (p2 ? (p1 ? bt[6] : bt[4]) : (p1 ? bt[2] : bt[0]));
                        cc = (p2 ? 4u : 0u) + (p1 ? 2u : 0u) + (p0 ? 1u : 0u);
                    } else if (B > 1) {
#pragma unroll
                        for (int k = 0; k + 1 < L; ++k) cc += (y >= bt[k]) ? 1u : 0u;
                    }
                    if (B > 1) r = y - sm.c[cc];
                    ccur[(j + e) >> 3] += cc << (4 * ((j + e) & 7));
                    rr[j + e] = r * r;
                    sr[e] = r;
                }
                const __half2 h1 = __floats2half2_rn(sr[0], sr[1]);
                const float2 f1 = __half22float2(h1);
                const __half2 h2 = __floats2half2_rn(sr[0] - f1.x, sr[1] - f1.y);
                hp1[j >> 1] = *reinterpret_cast<const uint32_t*>(&h1);
                hp2[j >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            uint8_t* r0 = sm.r[b][0];
            uint8_t* r1 = sm.r[b][1];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                *reinterpret_cast<uint4*>(r0 + roff[ii]) =
                    make_uint4(hp1[4 * ii], hp1[4 * ii + 1], hp1[4 * ii + 2], hp1[4 * ii + 3]);
                *reinterpret_cast<uint4*>(r1 + roff[ii]) =
                    make_uint4(hp2[4 * ii], hp2[4 * ii + 1], hp2[4 * ii + 2], hp2[4 * ii + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.r_full);
            sm.rr[b][q][32 * h + lane] = transpose_reduce32(rr, lane);

            if (pend && !finish()) return running = false;
            pend = true;
            pg = g;
            pt = t;
            pidx = i;
#pragma unroll
            for (int u = 0; u < 4; ++u) pcell[u] = ccur[u];
            ++i;
            return true;
        });
        if (running && pend) finish();
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

bool encode_tc_supported(int d, int x_dtype, int G, int64_t n) {
    return d == kD && x_dtype == TQ_BF16 && (int64_t)G * n < ((int64_t)1 << 31) &&
           encode_tiled_fn() != nullptr;
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
