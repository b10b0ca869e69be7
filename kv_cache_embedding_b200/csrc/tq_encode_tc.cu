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
//  * Epilogue warps (thread = output coordinate, kVpw vectors per warp) work
//    in units scaled by 2^10 (exact: 1/|x|, boundaries and centroids are
//    pre-multiplied): y' = 2^10 y, bucketize, r' = y' - c'[idx], |r|^2, and r'
//    as two fp16 pieces written coordinate-major (one 128-byte row per
//    coordinate, vectors contiguous): the MN-major B operand of D2 = S R^T
//    (3 passes: s1 h1 + s1 h2 + s2 h1).  Only the sign of D2 is kept.  The
//    second half of a tile (signs, packing, stores) runs after the first half
//    of the next tile so the QJL MMA overlaps epilogue work.
//  * Warp roles: 0 TMA producer, 1 TMEM owner + MMA issuer, 2-3 norms,
//    4.. epilogue (kEpi warps; kEpi / 4 per TMEM lane quarter).
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
constexpr int kVpw = 16;                     // vectors per epilogue warp
constexpr int kNH = kTN / kVpw;              // epilogue warps per TMEM lane quarter
constexpr int kEpi = 4 * kNH;                // epilogue warps
constexpr int kThreads = 32 * (4 + kEpi);
constexpr uint32_t kColPi = 0, kColS = 192, kColD1 = 320, kColD2 = 448, kTmemCols = 512;
constexpr uint32_t kStageBytes = kTN * kD * 2;   // two 8 KB swizzled regions (k < 64, k >= 64)
constexpr uint64_t kWaitNs = 1000000000ull;      // 1 s per wait
constexpr float kRScale = 1024.f;                // r * 2^10 keeps fp16 pieces normal
constexpr uint32_t kIdescRot = idesc_f16(1, 128, kTN);                // bf16 x bf16 -> f32
constexpr uint32_t kIdescQjl = idesc_f16(0, 128, kTN) | (1u << 16);   // fp16 x fp16, B MN-major

struct Smem {
    uint8_t x[kXS][kStageBytes];   // 1024-aligned (first member)
    uint8_t r[2][2][kStageBytes];  // [tile parity][piece h1, h2]: B operand of the QJL MMA
    float inv[kXS][kTN];           // 2^10 / |x| per stage
    float rr[2][4][kTN];           // [tile parity][lane quarter] |r'|^2 partial sums
    float c[8];                    // 2^10 c
    float beta[8];                 // 2^10 beta
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

// 32 lanes x 32 bits, 16 consecutive columns: thread t of the warp gets lane
// (warp's quarter base + t), columns [taddr.col, +16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

template <int V>
__device__ __forceinline__ void tmem_ldv(uint32_t taddr, uint32_t (&r)[V]) {
    if constexpr (V == 16) tmem_ld16(taddr, r);
    else tmem_ld32(taddr, r);
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}

// Copy the d x d fp32 matrix M (row-major) transposed into shared memory,
// stage[k][m] = M[m][k], by the epilogue warps (te = 0 .. 32 kEpi - 1): lane
// = row m within a quarter, so the shared stores of a warp are contiguous;
// each thread keeps its 8 row loads in flight together.
__device__ __forceinline__ void stage_transposed(const float* __restrict__ M, float* stage, int te) {
    const int m = 32 * ((te >> 5) & 3) + (te & 31);
    const int kg = te >> 7;  // 0..3: which quarter of the 32 float4 of the row
    float4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        v[j] = __ldg(reinterpret_cast<const float4*>(M + (size_t)m * kD) + 8 * kg + j);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int k = 4 * (8 * kg + j);
        stage[(k + 0) * kD + m] = v[j].x;
        stage[(k + 1) * kD + m] = v[j].y;
        stage[(k + 2) * kD + m] = v[j].z;
        stage[(k + 3) * kD + m] = v[j].w;
    }
}

// Pieces of row `row` of the staged matrix (stage[k][row]) into TMEM lane
// `row`: Pi as bf16 pieces 0-2 (bits 0-2 of `mask`), S as fp16 pieces 0-1
// (bit 3).  Column c of a piece holds k = 2c (low half) and k = 2c + 1 (high
// half); written 8 columns at a time.
__device__ void pieces_to_tmem(const float* stage, bool is_pi, int row, int mask,
                               uint32_t taddr_lane) {
#pragma unroll 1
    for (int piece = 0; piece < 3; ++piece) {
        if (is_pi ? !(mask & (1 << piece)) : (piece == 2 || !(mask & 8))) continue;
        const uint32_t col0 = is_pi ? kColPi + 64u * piece : kColS + 64u * piece;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 8) {
            uint32_t w[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float vx = stage[(2 * (c0 + c)) * kD + row];
                const float vy = stage[(2 * (c0 + c) + 1) * kD + row];
                if (is_pi) {  // Pi = p1 + p2 + p3 (bf16)
                    __nv_bfloat16 a = __float2bfloat16_rn(vx), bb = __float2bfloat16_rn(vy);
                    float ra = vx - __bfloat162float(a), rb = vy - __bfloat162float(bb);
                    if (piece >= 1) {
                        a = __float2bfloat16_rn(ra);
                        bb = __float2bfloat16_rn(rb);
                        ra -= __bfloat162float(a);
                        rb -= __bfloat162float(bb);
                    }
                    if (piece == 2) {
                        a = __float2bfloat16_rn(ra);
                        bb = __float2bfloat16_rn(rb);
                    }
                    w[c] = pack_bf16(a, bb);
                } else {  // S = s1 + s2 (fp16)
                    __half a = __float2half_rn(vx), bb = __float2half_rn(vy);
                    if (piece == 1) {
                        a = __float2half_rn(vx - __half2float(a));
                        bb = __float2half_rn(vy - __half2float(bb));
                    }
                    w[c] = pack_f16(a, bb);
                }
            }
            tmem_st8(taddr_lane + col0 + (uint32_t)c0, w);
        }
    }
}

// One halving round of a transposed butterfly: lane keeps half of its n
// values (selected by `up`), sends the other half to lane ^ m and combines.
template <int N, class Op, class T>
__device__ __forceinline__ void halve(T (&v)[N], bool up, int m, Op op) {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        const T lo = v[2 * i], hi = v[2 * i + 1];
        v[i] = op(up ? hi : lo, __shfl_xor_sync(0xffffffffu, up ? lo : hi, m));
    }
}

// Sum over the 32 lanes of v[j], for every j < V (V = 16 or 32).  Rounds pair
// lanes by bits 0.. of the lane index against bits 0.. of j; lane l ends with
// the sum for j = l % V (lanes l and l + 16 agree when V = 16).
template <int V>
__device__ __forceinline__ float transpose_reduce(const float (&v)[V], int lane) {
    float cur[V];
#pragma unroll
    for (int i = 0; i < V; ++i) cur[i] = v[i];
    auto add = [](float a, float b) { return a + b; };
    halve<V>(cur, lane & 1, 1, add);
    halve<V / 2>(reinterpret_cast<float(&)[V / 2]>(cur), lane & 2, 2, add);
    halve<V / 4>(reinterpret_cast<float(&)[V / 4]>(cur), lane & 4, 4, add);
    halve<V / 8>(reinterpret_cast<float(&)[V / 8]>(cur), lane & 8, 8, add);
    float t;
    if constexpr (V == 32) {
        halve<2>(reinterpret_cast<float(&)[2]>(cur), lane & 16, 16, add);
        t = cur[0];
    } else {
        t = cur[0] + __shfl_xor_sync(0xffffffffu, cur[0], 16);
    }
    return t;
}

// OR-combine fields of F lanes (F = 8 or 16, already shifted into place) for
// V vectors: afterwards lane e (= lane % F) holds the finished words of
// vectors j = e + F*i, i < V/F.
template <int F, int V>
__device__ __forceinline__ void transpose_or(const uint32_t (&v)[V], int lane,
                                             uint32_t (&out)[V / F]) {
    uint32_t cur[V];
#pragma unroll
    for (int i = 0; i < V; ++i) cur[i] = v[i];
    auto orr = [](uint32_t a, uint32_t b) { return a | b; };
    halve<V>(cur, lane & 1, 1, orr);
    halve<V / 2>(reinterpret_cast<uint32_t(&)[V / 2]>(cur), lane & 2, 2, orr);
    halve<V / 4>(reinterpret_cast<uint32_t(&)[V / 4]>(cur), lane & 4, 4, orr);
    if constexpr (F == 16) halve<V / 8>(reinterpret_cast<uint32_t(&)[V / 8]>(cur), lane & 8, 8, orr);
#pragma unroll
    for (int i = 0; i < V / F; ++i) out[i] = cur[i];
}

// Pack the fields of this lane's coordinate (block q, position `lane`) for
// the warp's V vectors (rows V*h .. V*h + V - 1 of the tile) and store the
// finished words of block q straight to the tile's records `dst` (W words per
// record); rows at or beyond `valid` are not written.
template <int B, int V>
__device__ __forceinline__ void pack_store(const uint32_t (&cellw)[V / 8],
                                           const uint32_t (&pbits)[V], int lane, int q, int h,
                                           uint32_t* __restrict__ dst, int valid) {
    constexpr int W = B * kD / 32;
    uint32_t z[V];
#pragma unroll
    for (int j = 0; j < V; ++j) z[j] = (__uint_as_float(pbits[j]) >= 0.f) ? 1u : 0u;
    if (B == 1 || B == 3) {
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t w = __ballot_sync(0xffffffffu, z[j] != 0u);
            if (lane == j) mine = w;
        }
        if (lane < V && V * h + lane < valid)
            dst[(V * h + lane) * W + B * q + (B == 1 ? 0 : 2)] = mine;
    }
    if (B == 4) {
        uint32_t v[V], out[V / 8];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t cell = (cellw[j >> 3] >> (4 * (j & 7))) & 15u;
            v[j] = (cell | (z[j] << 3)) << (4 * (lane & 7));
        }
        transpose_or<8, V>(v, lane, out);
#pragma unroll
        for (int i = 0; i < V / 8; ++i) {
            const int row = V * h + (lane & 7) + 8 * i;
            if (row < valid) dst[row * W + 4 * q + (lane >> 3)] = out[i];
        }
    }
    if (B == 2 || B == 3) {
        uint32_t v[V], out[V / 16];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t cell = (cellw[j >> 3] >> (4 * (j & 7))) & 15u;
            const uint32_t f = (B == 2) ? (cell | (z[j] << 1)) : cell;
            v[j] = f << (2 * (lane & 15));
        }
        transpose_or<16, V>(v, lane, out);
#pragma unroll
        for (int i = 0; i < V / 16; ++i) {
            const int row = V * h + (lane & 15) + 16 * i;
            if (row < valid) dst[row * W + B * q + (lane >> 4)] = out[i];
        }
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
    constexpr int V = kVpw;
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
            mbar_init(&sm.empty_x[s], 1 + 2 + kEpi);  // MMA commit + norm warps + epilogue
            mbar_init(&sm.norm_full[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.d1_full[b], 1);
            mbar_init(&sm.d1_empty[b], kEpi);
        }
        mbar_init(&sm.r_full, kEpi);
        mbar_init(&sm.d2_full, 1);
        mbar_init(&sm.d2_empty, kEpi);
        mbar_init(&sm.w_ready, kEpi);
        mbar_init(&sm.epi_bar, kEpi);
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
        const int q = warp & 3, h = (warp - 4) >> 2;  // lane quarter, vector slice
        const int coord = q * 32 + lane;
        const uint32_t lane_addr = tbase + ((uint32_t)(q * 32) << 16);
        // residual row of this coordinate: 128 bytes, 16-byte chunk c (vectors
        // 8c..8c+7) at position c ^ (coord % 8); this warp writes chunks
        // (V/8) h .. (V/8) h + V/8 - 1
        uint32_t roff[V / 8];
#pragma unroll
        for (int ii = 0; ii < V / 8; ++ii)
            roff[ii] = (uint32_t)coord * 128u +
                       ((((uint32_t)(V / 8 * h + ii)) ^ (uint32_t)(coord & 7)) << 4);
        float bt[7];
#pragma unroll
        for (int k = 0; k < 7; ++k) bt[k] = sm.beta[k];
        // weight pieces this warp loads into TMEM at each group start
        const int wmask = (kNH == 4) ? (1 << h) : (h == 0 ? 7 : 8);
        uint32_t i = 0, eb = 0;
        const int te = threadIdx.x - 128;  // 0 .. 32*kEpi - 1 over the epilogue warps
        auto epi_sync = [&]() -> bool {  // all epilogue warps
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.epi_bar);
            const bool ok = warp_wait(&sm.epi_bar, eb & 1, abort);
            ++eb;
            return ok;
        };
        float* stage = reinterpret_cast<float*>(&sm.r[0][0][0]);  // 64 KB, free at group start
        // The second half of a tile (sign bits, packing, stores) runs after the
        // first half of the next tile.  State of the pending tile:
        bool pend = false;
        int pg = 0, pt = 0;
        uint32_t pidx = 0;
        uint32_t pcell[V / 8];
#pragma unroll
        for (int u = 0; u < V / 8; ++u) pcell[u] = 0u;
        auto finish = [&]() -> bool {
            if (!warp_wait(&sm.d2_full, pidx & 1, abort)) return give_up(abort, err, 9);
            tc_fence_after();
            uint32_t pb[V];
            tmem_ldv<V>(lane_addr + kColD2 + (uint32_t)(V * h), pb);
            tmem_wait_ld();
            const int64_t v0 = (int64_t)pt * kTN;
            const int valid = (int)((n - v0) < kTN ? (n - v0) : kTN);
            // |r|^2 of the tile is complete: every epilogue warp stored its part
            // before arriving on r_full, which the QJL MMA behind d2_full waited for
            if (q == 0 && lane < V && V * h + lane < valid) {
                const float (*rrb)[kTN] = sm.rr[pidx & 1];
                const int vv = V * h + lane;
                rnorm[(int64_t)pg * n + v0 + vv] =
                    sqrtf(rrb[0][vv] + rrb[1][vv] + rrb[2][vv] + rrb[3][vv]) * (1.f / kRScale);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.d2_empty);
            pack_store<B, V>(pcell, pb, lane, q, h, codes + ((int64_t)pg * n + v0) * W, valid);
            pend = false;
            return true;
        };
        bool running = true;
        for_each_tile(G, tpg, [&](int g, int t, bool first, bool) {
            if (first) {
                // every MMA of the previous group must be done before its weights go
                if (pend && !finish()) return running = false;
                // Pi, then S, staged transposed through shared memory
                for (int mat = 0; mat < 2; ++mat) {
                    if (!epi_sync()) return running = give_up(abort, err, 13);
                    stage_transposed((mat == 0 ? Pi : S) + (size_t)g * kD * kD, stage, te);
                    if (!epi_sync()) return running = give_up(abort, err, 14);
                    pieces_to_tmem(stage, mat == 0, coord, wmask, lane_addr);
                }
                if (!epi_sync()) return running = give_up(abort, err, 15);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.w_ready);
            }
            const int s = i % kXS, b = i & 1;
            if (!warp_wait(&sm.d1_full[b], (i >> 1) & 1, abort))
                return running = give_up(abort, err, 7);
            tc_fence_after();
            uint32_t acc[V];
            tmem_ldv<V>(lane_addr + kColD1 + 64u * b + (uint32_t)(V * h), acc);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.d1_empty[b]);
            if (!warp_wait(&sm.norm_full[s], (i / kXS) & 1, abort))
                return running = give_up(abort, err, 8);
            float inv[V];
#pragma unroll
            for (int j = 0; j < V; j += 4) {
                const float4 t4 = *reinterpret_cast<const float4*>(&sm.inv[s][V * h + j]);
                inv[j] = t4.x;
                inv[j + 1] = t4.y;
                inv[j + 2] = t4.z;
                inv[j + 3] = t4.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty_x[s]);

            uint32_t ccur[V / 8];
#pragma unroll
            for (int u = 0; u < V / 8; ++u) ccur[u] = 0u;
            float rr[V];
            uint32_t hp1[V / 2], hp2[V / 2];
#pragma unroll
            for (int j = 0; j < V; j += 2) {
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
            for (int ii = 0; ii < V / 8; ++ii) {
                *reinterpret_cast<uint4*>(r0 + roff[ii]) =
                    make_uint4(hp1[4 * ii], hp1[4 * ii + 1], hp1[4 * ii + 2], hp1[4 * ii + 3]);
                *reinterpret_cast<uint4*>(r1 + roff[ii]) =
                    make_uint4(hp2[4 * ii], hp2[4 * ii + 1], hp2[4 * ii + 2], hp2[4 * ii + 3]);
            }
            const float tot = transpose_reduce<V>(rr, lane);
            if (lane < V) sm.rr[b][q][V * h + lane] = tot;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.r_full);

            if (pend && !finish()) return running = false;
            pend = true;
            pg = g;
            pt = t;
            pidx = i;
#pragma unroll
            for (int u = 0; u < V / 8; ++u) pcell[u] = ccur[u];
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
