// FP32-accurate dense products of the encode path on the sm_100a tensor
// cores, for the dimensions the fused d = 128 kernel does not cover (E2 the
// rotation, E5 the QJL projection):
//
//   C[m][n] = scale(m) * sum_k A[m][k] * B[n][k]     (A [M][K], B [N][K], K-contiguous)
//   scale(m) = 1 (mode 0), 1/row_scale[m] or 0 if row_scale[m] == 0 (mode 1),
//              row_scale[m] (mode 2)
// stored row-major (C[m * ldc + n]) or transposed (C[n * ldc + m], columns
// n < n_store only), optionally with the maximum of every 128-row tile per
// column (tmax[n * ldt + m / 128]).  The transposed form with tile maxima is
// the decoded-key scoring of many queries: rows = keys, columns = queries.
//
// Pages: quant_prune_distill #674 (rotate by a random orthogonal matrix; QJL:
// multiply the residual by a random matrix, keep the sign); RecSysChannel #256
// caveat 1 (normalise, multiply by a random matrix).
//
// Precision: both operands are split into 16-bit pieces and the MMAs sum the
// products a_i b_j with i + j < max(pa, pb) (pa, pb pieces of A and B); 16-bit
// x 16-bit products are exact in fp32.
//  * fp16 pieces (the encode path): each operand scaled by a power of two into
//    fp16's range, A = a1 + a2 and B = b1 + b2 (~2^-22 of the value; a bf16
//    input scaled this way is one exact fp16 piece): 2 x 2 -> a1 b1 + a1 b2 +
//    a2 b1 (3 passes), 1 x 2 -> a1 b1 + a1 b2 (2 passes).
//  * bf16 pieces (the decoded-key scoring): 2 x 2 -> a1 b1 + a1 b2 + a2 b1
//    (~2^-16); 3 x 3 pieces (~2^-24) -> 6 products.  The accumulator in tensor memory is
// restarted every 128 of K and the chunk sums are added in fp32 registers,
// so the rounding of an output stays near that of a 128-term fp32 sum for
// any K, as in the SIMT path.
//
// Tiles: 128 rows (MMA M) x 128 columns (MMA N), K in blocks of 64 staged by
// TMA with the 128-byte swizzle, in as many stages as 12 pieces of 16 KB hold
// (2 for 3 + 3 pieces, 3 for 2 + 2, 4 for 1 + 2 ...).  Warp 0 issues the TMA loads,
// warp 1 owns tensor memory and issues the MMAs, warps 2-5 (one per TMEM lane
// quarter) add up the chunk sums and store the tile.  Every wait is bounded
// (1 s); a warp that gives up sets the abort flag and the status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {
namespace {

using namespace sm100;

constexpr int kTM = 128, kTN = 128, kKB = 64;        // tile rows, columns, K block
constexpr int kPieceBytes = kTM * kKB * 2;            // one bf16 piece of a tile (16 KB)
constexpr int kPool = 12;                             // 16 KB operand pieces in shared memory
constexpr int kMaxStages = 6;
constexpr int kThreads = 32 * 6;
constexpr int kThreadsDecode = 32 * 8;                // + 2 warps decoding A from records
constexpr uint32_t kTmemCols = 2 * kTN;               // two chunk accumulators
constexpr uint64_t kWaitNs = 1000000000ull;

struct SmemG {
    // stage s holds pieces [s (pa + pb), (s + 1)(pa + pb)): A's pa, then B's pb
    // (1024-aligned, first); as many stages as the pool holds, up to 6
    uint8_t pool[kPool][kPieceBytes];
    float tkey[4][kTN];                  // per epilogue warp: its 32 rows' maximum per column
    uint32_t dtab[16];                   // decoded-A mode: packed bf16 pieces of c[cell]
    uint2 dpair[256][8];                 // b = 4: code byte -> (hi pair, lo pair) words, 8 copies
    uint32_t dsign[256];                 // b = 4: code byte -> sign flips of the pair (z = 0)
    float g_c[16], g_b[16];              // MSE-only encode epilogue: the grid
    uint64_t full[kMaxStages], empty[kMaxStages], acc_full[2], acc_empty[2], mma_done, tmax_bar, tmax_bar2;
    uint32_t tmem_base;
    int abort;
    int zero;
};
constexpr size_t kSmemBytes = sizeof(SmemG) + 1024;

__device__ __forceinline__ bool give_up(volatile int* abort, int* err, int site) {
    *abort = 1;
    atomicCAS(err, 0, TQ_ERR_DEVICE_TIMEOUT * 1000 - site);
    return false;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort, kWaitNs);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, int32_t z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// Decoded-A mode: rows rl and rl + 32 of tile m0, K block kb (64 of the
// K = 2d columns: the centroid half, then the sign half), written as the
// bf16 pieces hi / lo in the 128-byte-swizzled K-major layout of a TMA box.
// The code words of rows rl and rl + 32 of tile m0 for K block kb (2 blocks
// of 32 coordinates = 2B words each) and those rows' |r|.
template <int B>
__device__ __forceinline__ void load_rows(const KeyDecode& kd, int64_t M, int m0, int kb, int rl,
                                          uint32_t (&w)[2][2 * B], float (&rn)[2]) {
    const int W = kd.d / 32 * B;
    const int c0 = kb * kKB >= kd.d ? kb * kKB - kd.d : kb * kKB;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int64_t row = (int64_t)m0 + rl + 32 * half;
        const int64_t src = row < M ? row : 0;  // rows past M decode row 0 (not stored)
        const uint32_t* rec = kd.codes + src * W + (c0 / 32) * B;
#pragma unroll
        for (int i = 0; i < 2 * B; ++i) w[half][i] = __ldg(rec + i);
        rn[half] = __ldg(kd.rnorm + src);
    }
}

template <int B>
__device__ __forceinline__ void decode_rows(const KeyDecode& kd, const uint32_t* dtab,
                                            const uint2* dpair, const uint32_t* dsign, int kb,
                                            int rl, const uint32_t (&wr)[2][2 * B],
                                            const float (&rn)[2], uint8_t* hi, uint8_t* lo) {
    const bool sgn = kb * kKB >= kd.d;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int r = rl + 32 * half;
        const uint32_t* w = wr[half];
        uint32_t kp = 0u;  // bf16 hi | lo << 16 of kappa
        if (sgn && !kd.mse) {
            const float kap = kd.kscale * rn[half];
            const __nv_bfloat16 h = __float2bfloat16_rn(kap);
            const __nv_bfloat16 l = __float2bfloat16_rn(kap - __bfloat162float(h));
            kp = (uint32_t)__bfloat16_as_ushort(h) | ((uint32_t)__bfloat16_as_ushort(l) << 16);
        }
        if (B == 4) {  // one code byte = one coordinate pair: table lookups
            const uint32_t khi = (kp & 0xffffu) * 0x10001u, klo = (kp >> 16) * 0x10001u;
#pragma unroll
            for (int u = 0; u < 8; ++u) {  // chunk u: word u of the two blocks
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t f = __byte_perm(w[u], 0u, 0x4440u | e);
                    if (!sgn) {
                        const uint2 pr = dpair[f * 8 + (rl & 7)];
                        hw[e] = pr.x;
                        lw[e] = pr.y;
                    } else if (kd.mse) {
                        hw[e] = 0u;
                        lw[e] = 0u;
                    } else {
                        const uint32_t fl = dsign[f];
                        hw[e] = khi ^ fl;
                        lw[e] = klo ^ fl;
                    }
                }
                const uint32_t off = (uint32_t)r * 128u + ((((uint32_t)u) ^ ((uint32_t)r & 7u)) << 4);
                *reinterpret_cast<uint4*>(hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            continue;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // 16-byte chunks of 8 coordinates
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint32_t v[2];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int j = 8 * u + 2 * e + h2, blk = j >> 5, jj = j & 31;
                    uint32_t idx, z;
                    if (B == 4) {
                        const uint32_t f = (w[blk * 4 + (jj >> 3)] >> (4 * (jj & 7))) & 15u;
                        idx = f & 7u;
                        z = f >> 3;
                    } else if (B == 3) {
                        idx = (w[blk * 3 + (jj >> 4)] >> (2 * (jj & 15))) & 3u;
                        z = (w[blk * 3 + 2] >> jj) & 1u;
                    } else if (B == 2) {
                        const uint32_t f = (w[blk * 2 + (jj >> 4)] >> (2 * (jj & 15))) & 3u;
                        idx = f & 1u;
                        z = f >> 1;
                    } else {
                        idx = 0u;
                        z = (w[blk] >> jj) & 1u;
                    }
                    if (!sgn) {
                        v[h2] = dtab[kd.mse ? (idx | (z << (B - 1))) : idx];
                    } else {
                        v[h2] = kd.mse ? 0u : (z ? kp : (kp ^ 0x80008000u));
                    }
                }
                hw[e] = __byte_perm(v[0], v[1], 0x5410);  // the two hi halves
                lw[e] = __byte_perm(v[0], v[1], 0x7632);  // the two lo halves
            }
            const uint32_t off = (uint32_t)r * 128u + ((((uint32_t)u) ^ ((uint32_t)r & 7u)) << 4);
            *reinterpret_cast<uint4*>(hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
    }
}

// Decoded-A producer (one of the two decode warps): every (tile, K block) in
// the order of the other roles, the next block's words loaded while the
// current one is decoded.  Returns false when a wait gave up.
template <int B>
__device__ bool decode_loop(const KeyDecode& kd, SmemG& sm, int64_t M, int tiles, int tn, int nkb,
                            int ns, int pa, int pb, int rl, volatile int* abort, int* err) {
    const int lane = threadIdx.x % 32;
    int t = blockIdx.x, kb = 0;
    if (t >= tiles) return true;
    uint32_t wc[2][2 * B], wn[2][2 * B];
    float rc[2], rnx[2];
    load_rows<B>(kd, M, (t / tn) * kTM, kb, rl, wc, rc);
    for (uint32_t it = 0;; ++it) {
        // the next (tile, K block)
        int t2 = t, kb2 = kb + 1;
        if (kb2 == nkb) {
            kb2 = 0;
            t2 += gridDim.x;
        }
        const bool more = t2 < tiles;
        if (more) load_rows<B>(kd, M, (t2 / tn) * kTM, kb2, rl, wn, rnx);
        const int s = (int)(it % (uint32_t)ns);
        if (it >= (uint32_t)ns && !warp_wait(&sm.empty[s], ((it / ns) - 1) & 1, abort))
            return give_up(abort, err, 47);
        decode_rows<B>(kd, sm.dtab, &sm.dpair[0][0], sm.dsign, kb, rl, wc, rc,
                       sm.pool[s * (pa + pb)], sm.pool[s * (pa + pb) + 1]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.full[s]);
        if (!more) return true;
        t = t2;
        kb = kb2;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rc[h] = rnx[h];
#pragma unroll
            for (int i = 0; i < 2 * B; ++i) wc[h][i] = wn[h][i];
        }
    }
}

// MSE-only encode epilogue (mode 4) of a whole row (N = K = d = 128: the
// tile holds every coordinate of its rows): y = sum * sc, the cell (the count
// of boundaries <= y, binary search over the 2^b-level grid), |r| = |y -
// c[cell]|, and the record of the MSE-only layout (the cell's low b - 1 bits
// in the index fields, its top bit in the sign positions) -- the arithmetic
// of k_quantize and k_pack, without the rotated rows crossing HBM.
template <int L, int B>
__device__ __forceinline__ void epi_mse_row(const float (&sum)[kTN], float sc, const float* bt,
                                            const float* ct, const EncodeEpi& ep, int64_t row) {
    constexpr int W = B * kTN / 32;
    uint32_t out[W];
#pragma unroll
    for (int i = 0; i < W; ++i) out[i] = 0u;
    float rr = 0.f;
#pragma unroll
    for (int j = 0; j < kTN; ++j) {
        const float y = sum[j] * sc;
        int cell = 0;
#pragma unroll
        for (int step = L >> 1; step > 0; step >>= 1)
            if (bt[cell + step - 1] <= y) cell += step;
        const float r = y - ct[cell];
        rr = fmaf(r, r, rr);
        const uint32_t iv = (uint32_t)cell & ((1u << (B - 1)) - 1u), z = (uint32_t)cell >> (B - 1);
        const int w = j >> 5, jj = j & 31;
        if (B == 1) {
            out[w] |= z << jj;
        } else if (B == 2) {
            out[2 * w + (jj >> 4)] |= (iv | (z << 1)) << (2 * (jj & 15));
        } else if (B == 3) {
            out[3 * w + (jj >> 4)] |= iv << (2 * (jj & 15));
            out[3 * w + 2] |= z << jj;
        } else {
            out[4 * w + (jj >> 3)] |= (iv | (z << 3)) << (4 * (jj & 7));
        }
    }
    uint4* dst = reinterpret_cast<uint4*>(ep.codes + row * W);
#pragma unroll
    for (int i = 0; i < W / 4; ++i)
        dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    ep.rnorm[row] = sqrtf(rr);
}

template <int B>
__device__ __forceinline__ void epi_mse_row_b(const float (&sum)[kTN], float sc, const float* bt,
                                              const float* ct, const EncodeEpi& ep, int64_t row) {
    switch (ep.cb.levels) {  // 2^b levels
        case 2: epi_mse_row<2, B>(sum, sc, bt, ct, ep, row); break;
        case 4: epi_mse_row<4, B>(sum, sc, bt, ct, ep, row); break;
        case 8: epi_mse_row<8, B>(sum, sc, bt, ct, ep, row); break;
        default: epi_mse_row<16, B>(sum, sc, bt, ct, ep, row); break;
    }
}

__global__ void __launch_bounds__(kThreadsDecode, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
          int M, int N, int K, int pa, int pb, float* __restrict__ C, int64_t ldc,
          const float* __restrict__ row_scale, int scale_mode, int transposed, int n_store,
          float* __restrict__ tmax, int64_t ldt, int* __restrict__ err, KeyDecode kd,
          int decode, uint32_t idesc, const __grid_constant__ EncodeEpi ep) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    SmemG& sm = *reinterpret_cast<SmemG*>(smem_raw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort = &sm.abort;
    const int tm = (M + kTM - 1) / kTM, tn = N / kTN;
    const int tiles = tm * tn;
    const int nkb = K / kKB;            // K blocks per tile
    const int nch = nkb / 2;            // 128-wide K chunks per tile
    const uint32_t stage_tx = (uint32_t)(decode ? pb : pa + pb) * kPieceBytes;
    const int ns = min(kMaxStages, kPool / (pa + pb));  // pipeline stages

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&sm.full[s], decode ? 3 : 1);  // TMA (+ the 2 decode warps)
            mbar_init(&sm.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.acc_full[i], 1);
            mbar_init(&sm.acc_empty[i], 4);
        }
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.tmax_bar, 4);
        mbar_init(&sm.tmax_bar2, 4);
        sm.abort = 0;
        sm.zero = 0;
        fence_mbar_init();
    }
    if (ep.mode == 4 && threadIdx.x >= 32 && threadIdx.x < 48) {
        sm.g_c[threadIdx.x - 32] = ep.cb.c[threadIdx.x - 32];
        sm.g_b[threadIdx.x - 32] = ep.cb.beta[threadIdx.x - 32];
    }
    if (decode && threadIdx.x < 16) {
        uint32_t v = 0u;
        switch (threadIdx.x) {  // static indices keep the table in parameter space
#define TQ_DT(F) case F: v = kd.tab[F]; break;
            TQ_DT(0) TQ_DT(1) TQ_DT(2) TQ_DT(3) TQ_DT(4) TQ_DT(5) TQ_DT(6) TQ_DT(7)
            TQ_DT(8) TQ_DT(9) TQ_DT(10) TQ_DT(11) TQ_DT(12) TQ_DT(13) TQ_DT(14) TQ_DT(15)
#undef TQ_DT
        }
        sm.dtab[threadIdx.x] = v;
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    if (decode && kd.b == 4) {  // pair tables from the centroid pieces
        for (int e = threadIdx.x; e < 256 * 8; e += blockDim.x) {
            const uint32_t f = (uint32_t)e >> 3;
            const uint32_t a = sm.dtab[kd.mse ? (f & 15u) : (f & 7u)];
            const uint32_t b = sm.dtab[kd.mse ? (f >> 4) : ((f >> 4) & 7u)];
            sm.dpair[f][e & 7] = make_uint2(__byte_perm(a, b, 0x5410), __byte_perm(a, b, 0x7632));
        }
        for (int f = threadIdx.x; f < 256; f += blockDim.x)
            sm.dsign[f] = ((f & 0x08) ? 0u : 0x8000u) | ((f & 0x80) ? 0u : 0x80000000u);
        __syncthreads();
    }

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const int m0 = (t / tn) * kTM, n0 = (t % tn) * kTN;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = (int)(it % (uint32_t)ns);
                if (it >= (uint32_t)ns &&
                    !mbar_wait(&sm.empty[s], ((it / ns) - 1) & 1, abort, kWaitNs)) {
                    ok = give_up(abort, err, 41);
                    break;
                }
                mbar_arrive_expect_tx(&sm.full[s], stage_tx);
                uint8_t* st = sm.pool[s * (pa + pb)];
                if (!decode)
                    for (int p = 0; p < pa; ++p)
                        tma_load_3d(st + p * kPieceBytes, &tmap_a, kb * kKB, m0, p, &sm.full[s]);
                for (int p = 0; p < pb; ++p)
                    tma_load_3d(st + (pa + p) * kPieceBytes, &tmap_b, kb * kKB, n0, p, &sm.full[s]);
            }
        }
        // no TMA write may still be in flight when the CTA exits
        for (uint32_t j = (it > (uint32_t)ns ? it - ns : 0); j < it; ++j)
            mbar_wait(&sm.full[j % ns], (j / ns) & 1, &sm.zero, kWaitNs);
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        // products a_i b_j with i + j < max(pa, pb), by increasing i + j
        int pi_[6], pj_[6], np = 0;
        const int pmax = pa > pb ? pa : pb;
        for (int sij = 0; sij < pmax; ++sij)
            for (int i = 0; i <= sij; ++i)
                if (i < pa && sij - i < pb) {
                    pi_[np] = i;
                    pj_[np] = sij - i;
                    ++np;
                }
        uint32_t it = 0, cc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            for (int c = 0; c < nch && ok; ++c, ++cc) {
                const uint32_t ab = cc & 1;
                if (cc >= 2 && !mbar_wait(&sm.acc_empty[ab], ((cc >> 1) - 1) & 1, abort, kWaitNs)) {
                    ok = give_up(abort, err, 42);
                    break;
                }
                tc_fence_after();
                const uint32_t d = tbase + ab * kTN;
                for (int h = 0; h < 2; ++h, ++it) {
                    const int s = (int)(it % (uint32_t)ns);
                    if (!mbar_wait(&sm.full[s], (it / ns) & 1, abort, kWaitNs)) {
                        ok = give_up(abort, err, 43);
                        break;
                    }
                    tc_fence_after();
                    for (int q = 0; q < np; ++q) {
                        const uint32_t as = smem_u32(sm.pool[s * (pa + pb) + pi_[q]]),
                                       bs = smem_u32(sm.pool[s * (pa + pb) + pa + pj_[q]]);
#pragma unroll
                        for (int ks = 0; ks < kKB / 16; ++ks)
                            mma_f16_ss(d, smem_desc_kmajor_sw128(as + ks * 32),
                                   smem_desc_kmajor_sw128(bs + ks * 32), idesc,
                                   (h | q | ks) != 0);
                    }
                    tc_commit(&sm.empty[s]);
                }
                if (ok) tc_commit(&sm.acc_full[ab]);
            }
        }
        // every issued MMA completes before tensor memory is released
        tc_commit(&sm.mma_done);
        mbar_wait(&sm.mma_done, 0, &sm.zero, kWaitNs);
    } else if (warp >= 6) {
        // ---------------- A from code records (decoded-A mode) ----------------
        const int rl = 64 * (warp - 6) + lane;  // rows rl, rl + 32 of every tile
        switch (kd.b) {
            case 1: decode_loop<1>(kd, sm, M, tiles, tn, nkb, ns, pa, pb, rl, abort, err); break;
            case 2: decode_loop<2>(kd, sm, M, tiles, tn, nkb, ns, pa, pb, rl, abort, err); break;
            case 3: decode_loop<3>(kd, sm, M, tiles, tn, nkb, ns, pa, pb, rl, abort, err); break;
            default: decode_loop<4>(kd, sm, M, tiles, tn, nkb, ns, pa, pb, rl, abort, err); break;
        }
    } else if (warp >= 2) {
        // ---------------- chunk sums and stores ----------------
        const int q = warp & 3;  // TMEM lane quarter: tile rows 32 q .. 32 q + 31
        const uint32_t lane_addr = tbase + ((uint32_t)(32 * q) << 16);
        uint32_t cc = 0, tb = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const int m0 = (t / tn) * kTM, n0 = (t % tn) * kTN;
            float sum[kTN];
#pragma unroll
            for (int j = 0; j < kTN; ++j) sum[j] = 0.f;
            for (int c = 0; c < nch; ++c, ++cc) {
                const uint32_t ab = cc & 1;
                if (!warp_wait(&sm.acc_full[ab], (cc >> 1) & 1, abort)) {
                    ok = give_up(abort, err, 44);
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int j0 = 0; j0 < kTN; j0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(lane_addr + ab * kTN + (uint32_t)j0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) sum[j0 + j] += __uint_as_float(v[j]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
            }
            if (!ok) break;
            const int64_t row = (int64_t)m0 + 32 * q + lane;
            const bool live = row < M;
            float sc = 1.f;
            if (live && scale_mode == 1) {
                const float r = row_scale[row];
                sc = (r != 0.f) ? 1.f / r : 0.f;
            } else if (live && scale_mode == 2) {
                sc = row_scale[row];
            }
            if (ep.mode == 4) {
                if (live) {
                    switch (ep.b) {
                        case 1: epi_mse_row_b<1>(sum, sc, sm.g_b, sm.g_c, ep, row); break;
                        case 2: epi_mse_row_b<2>(sum, sc, sm.g_b, sm.g_c, ep, row); break;
                        case 3: epi_mse_row_b<3>(sum, sc, sm.g_b, sm.g_c, ep, row); break;
                        default: epi_mse_row_b<4>(sum, sc, sm.g_b, sm.g_c, ep, row); break;
                    }
                }
            } else if (!transposed) {
                if (live) {
                    float4* dst = reinterpret_cast<float4*>(C + row * ldc + n0);
#pragma unroll
                    for (int j = 0; j < kTN; j += 4)
                        dst[j / 4] = make_float4(sum[j] * sc, sum[j + 1] * sc, sum[j + 2] * sc,
                                                 sum[j + 3] * sc);
                }
            } else {
                // column j of the tile -> C[(n0 + j) * ldc + row]: a warp writes 32
                // consecutive rows of each column
#pragma unroll
                for (int j = 0; j < kTN; ++j) {
                    const float v = sum[j] * sc;
                    if (live && n0 + j < n_store) C[(int64_t)(n0 + j) * ldc + row] = v;
                    if (tmax) {  // the tile's maximum per column, 4 warps merged in shared memory
                        float m = live ? v : -INFINITY;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1)
                            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        if (lane == 0) sm.tkey[q][j] = m;
                    }
                }
                if (tmax) {
                    // the 4 epilogue warps meet on a bounded barrier, then each
                    // writes the maxima of 32 columns
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.tmax_bar);
                    if (!warp_wait(&sm.tmax_bar, tb & 1, abort)) {
                        ok = give_up(abort, err, 45);
                        break;
                    }
                    ++tb;
                    const int j = 32 * q + lane;
                    if (n0 + j < n_store)
                        tmax[(int64_t)(n0 + j) * ldt + m0 / kTM] =
                            fmaxf(fmaxf(sm.tkey[0][j], sm.tkey[1][j]),
                                  fmaxf(sm.tkey[2][j], sm.tkey[3][j]));
                    // the slots are rewritten only after the next tile's barrier,
                    // which every warp reaches after this read
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.tmax_bar2);
                    if (!warp_wait(&sm.tmax_bar2, (tb - 1) & 1, abort)) {
                        ok = give_up(abort, err, 46);
                        break;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// ---- the CTA-pair form (row-major products with N % 256 == 0) --------------
// One 256 x 256 tile per cluster of two CTAs: CTA r stages rows m0 + 128 r of
// A and rows n0 + 128 r of B (its halves of the pair's operands), the
// leader's thread issues cta_group::2 MMAs of M = 256, N = 256, and each CTA's
// tensor memory holds its 128 rows x 256 columns.  Per SM that is twice the
// MMA work per staged byte of the 128 x 128 form above, whose MMA warp waits
// on its stages (ncu: tensor pipe ~46 %, TMA reads ~31 % of peak), and half
// the MMA instructions.  The accumulation and its 128-wide K chunks are the
// same.  Warps: 0 TMA (both CTAs), 1 tensor memory (both) and the MMA issue
// (leader), 4-11 chunk sums and stores (TMEM lane quarter warp % 4, column
// half (warp - 4) / 4); 2-3 idle.  The leader's full barrier counts the
// bytes of both CTAs; the leader's MMA commits release both CTAs' stages and
// accumulators; every epilogue warp of the pair arrives on the leader's
// accumulator-empty barrier.  Every wait is bounded.
constexpr int kPN = 256;                       // tile columns (MMA N); tile rows 2 x kTM
constexpr int kPairThreads = 32 * 12;
constexpr uint32_t kPairTmemCols = 2 * kPN;    // two chunk accumulators
constexpr uint32_t kPairEpiWarps = 8;

struct SmemP {
    uint8_t pool[kPool][kPieceBytes];  // stage s: A's pa pieces, then B's pb (1024-aligned)
    float g_c[2][16], g_b[2][16];      // encode epilogues: the grids (second: fractional width)
    int g_levels[2];
    float tkey[2][4][kTN];             // transposed store: per column half, warp, column maxima
    uint64_t full[kMaxStages], empty[kMaxStages], acc_full[2], acc_empty[2], mma_done;
    uint64_t tmax_bar[2], tmax_bar2[2];
    uint32_t tmem_base;
    int abort;
    int zero;
};
constexpr size_t kSmemPairBytes = sizeof(SmemP) + 1024;

template <int L>
__device__ __forceinline__ void epi_quantize_l(const float (&sum)[kTN], float sc, const float* bt,
                                               const float* ct, const EncodeEpi& ep, int M,
                                               int N, int64_t row, int n0) {
    uint8_t* ix = ep.idx + row * N + n0;
    __half* hi = ep.rp + row * N + n0;
    __half* lo = ep.rp + (int64_t)M * N + row * N + n0;
    float rr = 0.f;
#pragma unroll
    for (int j0 = 0; j0 < kTN; j0 += 8) {
        uint32_t cw[2] = {0u, 0u}, hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float t[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float y = sum[j0 + e + u] * sc;
                int cell = 0;
                float r = y;
                if constexpr (L > 0) {
#pragma unroll
                    for (int step = L >> 1; step > 0; step >>= 1)
                        if (bt[cell + step - 1] <= y) cell += step;
                    r = y - ct[cell];
                }
                cw[e >> 2] |= (uint32_t)cell << (8 * ((e + u) & 3));
                rr = fmaf(r, r, rr);
                t[u] = r * ep.rscale;  // exact: a power of two
            }
            // two coordinates' pieces at once (round to nearest, as __float2half_rn)
            const __half2 h = __floats2half2_rn(t[0], t[1]);
            const float2 hf = __half22float2(h);
            const __half2 l = __floats2half2_rn(t[0] - hf.x, t[1] - hf.y);
            hw[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            lw[e >> 1] = *reinterpret_cast<const uint32_t*>(&l);
        }
        *reinterpret_cast<uint2*>(ix + j0) = make_uint2(cw[0], cw[1]);
        *reinterpret_cast<uint4*>(hi + j0) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(lo + j0) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    ep.rn2[(int64_t)(n0 / kTN) * M + row] = rr;
}

// Rotation epilogue: coordinates n0 .. n0 + 127 of row `row`, y = sum * sc:
// the cell (the count of boundaries <= y, by binary search over the sorted
// grid of 2^k levels), r = y - c[cell], the fp16 pieces of rscale * r and the
// segment's |r|^2 -- the arithmetic of k_quantize16, per coordinate.
__device__ __forceinline__ void epi_quantize(const float (&sum)[kTN], float sc, const SmemP& sm,
                                             const EncodeEpi& ep, int M, int N, int64_t row,
                                             int n0) {
    const int g = (ep.cb.split && n0 >= N / 2) ? 1 : 0;
    const float* bt = sm.g_b[g];
    const float* ct = sm.g_c[g];
    switch (sm.g_levels[g]) {  // inner-product grids: 2^(b-1) levels (none at b = 1)
        case 0: epi_quantize_l<0>(sum, sc, bt, ct, ep, M, N, row, n0); break;
        case 2: epi_quantize_l<2>(sum, sc, bt, ct, ep, M, N, row, n0); break;
        case 4: epi_quantize_l<4>(sum, sc, bt, ct, ep, M, N, row, n0); break;
        default: epi_quantize_l<8>(sum, sc, bt, ct, ep, M, N, row, n0); break;
    }
}

// QJL epilogue: coordinates n0 .. n0 + 127 (4 blocks of 32) of row `row` --
// z = [P >= 0] with the cells into 4 blocks of BB words at `rec` (the record
// layout of width BB: a sign plane; 2-bit [idx | z] fields; 2-bit idx fields
// and a sign plane; 4-bit [idx | z] nibbles).
template <int BB>
__device__ __forceinline__ void epi_pack(const float (&sum)[kTN], const uint8_t* cells,
                                         uint32_t* rec) {
    uint32_t out[4 * BB];
#pragma unroll
    for (int i = 0; i < 4 * BB; ++i) out[i] = 0u;
    const uint4* cp = reinterpret_cast<const uint4*>(cells);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint4 c0 = cp[2 * w], c1 = cp[2 * w + 1];
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const uint32_t cell = (cw[j >> 2] >> (8 * (j & 3))) & 0xFFu;
            const uint32_t z = sum[32 * w + j] >= 0.f ? 1u : 0u;
            if (BB == 1) {
                out[w] |= z << j;
            } else if (BB == 2) {
                out[2 * w + (j >> 4)] |= ((cell & 1u) | (z << 1)) << (2 * (j & 15));
            } else if (BB == 3) {
                out[3 * w + (j >> 4)] |= (cell & 3u) << (2 * (j & 15));
                out[3 * w + 2] |= z << j;
            } else {
                out[4 * w + (j >> 3)] |= ((cell & 7u) | (z << 3)) << (4 * (j & 7));
            }
        }
    }
    uint4* dst = reinterpret_cast<uint4*>(rec);
#pragma unroll
    for (int i = 0; i < BB; ++i)
        dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
}

template <int EPI>
__global__ void __launch_bounds__(kPairThreads, 1)
k_gemm_pair(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
            int M, int N, int K, int pa, int pb, float* __restrict__ C, int64_t ldc,
            const float* __restrict__ row_scale, int scale_mode, int n_store,
            float* __restrict__ tmax, int64_t ldt, int* __restrict__ err, uint32_t idesc,
            const __grid_constant__ EncodeEpi ep) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    // the same offset in both CTAs: the MMA reads the peer's operands there
    SmemP& sm = *reinterpret_cast<SmemP*>(smem_raw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    volatile int* abort = &sm.abort;
    const int tm = (M + 2 * kTM - 1) / (2 * kTM), tn = N / kPN;
    const int tiles = tm * tn;
    const int pair = blockIdx.x / 2, npairs = gridDim.x / 2;
    const int nkb = K / kKB;   // K blocks per tile
    const int nch = nkb / 2;   // 128-wide K chunks per tile
    const uint32_t stage_tx = (uint32_t)(pa + pb) * kPieceBytes;  // one CTA's bytes per stage
    const int ns = min(kMaxStages, kPool / (pa + pb));

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&sm.full[s], 1);   // the leader's producer; the bytes of both CTAs
            mbar_init(&sm.empty[s], 1);  // the pair's MMA commit
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.acc_full[i], 1);
            mbar_init(&sm.acc_empty[i], 2 * kPairEpiWarps);  // used in the leader
        }
        mbar_init(&sm.mma_done, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.tmax_bar[i], 4);   // the 4 warps of a column half
            mbar_init(&sm.tmax_bar2[i], 4);
        }
        sm.abort = 0;
        sm.zero = 0;
        fence_mbar_init();
    }
    if ((EPI == 1 || EPI == 2) && threadIdx.x >= 32 && threadIdx.x < 64) {
        const int i = threadIdx.x - 32;
        if (i < 16) {
            sm.g_c[0][i] = ep.cb.c[i];
            sm.g_b[0][i] = ep.cb.beta[i];
        } else {
            sm.g_c[1][i - 16] = ep.cb.c_lo[i - 16];
            sm.g_b[1][i - 16] = ep.cb.beta_lo[i - 16];
        }
        if (i == 0) {
            sm.g_levels[0] = ep.cb.levels;
            sm.g_levels[1] = ep.cb.levels_lo;
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(&sm.tmem_base, kPairTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // barriers initialised and tensor memory allocated in both CTAs
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        uint32_t it = 0;
        bool ok = true;
        for (int t = pair; t < tiles && ok; t += npairs) {
            const int m0 = (t / tn) * 2 * kTM + (int)rank * kTM;
            const int n0 = (t % tn) * kPN + (int)rank * kTM;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = (int)(it % (uint32_t)ns);
                if (it >= (uint32_t)ns &&
                    !mbar_wait(&sm.empty[s], ((it / ns) - 1) & 1, abort, kWaitNs)) {
                    ok = give_up(abort, err, 51);
                    break;
                }
                if (leader) mbar_arrive_expect_tx(&sm.full[s], 2 * stage_tx);
                const uint32_t fb = mapa_shared(smem_u32(&sm.full[s]), 0);
                uint8_t* st = sm.pool[s * (pa + pb)];
                for (int p = 0; p < pa; ++p)
                    tma_load_3d_pair(st + p * kPieceBytes, &tmap_a, kb * kKB, m0, p, fb);
                for (int p = 0; p < pb; ++p)
                    tma_load_3d_pair(st + (pa + p) * kPieceBytes, &tmap_b, kb * kKB, n0, p, fb);
            }
        }
        // no TMA write may still be in flight when the pair exits: the leader's
        // barriers count both CTAs' bytes
        if (leader)
            for (uint32_t j = (it > (uint32_t)ns ? it - ns : 0); j < it; ++j)
                mbar_wait(&sm.full[j % ns], (j / ns) & 1, &sm.zero, kWaitNs);
    } else if (warp == 1 && lane == 0 && leader) {
        // ---------------- MMA issuer (leader) ----------------
        int pi_[6], pj_[6], np = 0;
        const int pmax = pa > pb ? pa : pb;
        for (int sij = 0; sij < pmax; ++sij)
            for (int i = 0; i <= sij; ++i)
                if (i < pa && sij - i < pb) {
                    pi_[np] = i;
                    pj_[np] = sij - i;
                    ++np;
                }
        uint32_t it = 0, cc = 0;
        bool ok = true;
        for (int t = pair; t < tiles && ok; t += npairs) {
            for (int c = 0; c < nch && ok; ++c, ++cc) {
                const uint32_t ab = cc & 1;
                if (cc >= 2 &&
                    !mbar_wait(&sm.acc_empty[ab], ((cc >> 1) - 1) & 1, abort, kWaitNs)) {
                    ok = give_up(abort, err, 52);
                    break;
                }
                tc_fence_after();
                const uint32_t d = tbase + ab * kPN;
                for (int h = 0; h < 2; ++h, ++it) {
                    const int s = (int)(it % (uint32_t)ns);
                    if (!mbar_wait(&sm.full[s], (it / ns) & 1, abort, kWaitNs)) {
                        ok = give_up(abort, err, 53);
                        break;
                    }
                    tc_fence_after();
                    for (int q = 0; q < np; ++q) {
                        const uint32_t as = smem_u32(sm.pool[s * (pa + pb) + pi_[q]]),
                                       bs = smem_u32(sm.pool[s * (pa + pb) + pa + pj_[q]]);
#pragma unroll
                        for (int ks = 0; ks < kKB / 16; ++ks)
                            mma_f16_ss_pair(d, smem_desc_kmajor_sw128(as + ks * 32),
                                            smem_desc_kmajor_sw128(bs + ks * 32), idesc,
                                            (h | q | ks) != 0);
                    }
                    tc_commit_pair(&sm.empty[s], 0x3);
                }
                if (ok) tc_commit_pair(&sm.acc_full[ab], 0x3);
            }
        }
        // every issued MMA completes before either CTA releases tensor memory
        tc_commit_pair(&sm.mma_done, 0x3);
        mbar_wait(&sm.mma_done, 0, &sm.zero, kWaitNs);
    } else if (warp == 1 && lane == 0) {
        // the leader's MMAs write this CTA's tensor memory and read its stages
        mbar_wait(&sm.mma_done, 0, &sm.zero, kWaitNs);
    } else if (warp >= 4) {
        // ---------------- chunk sums and stores (both CTAs) ----------------
        const int q = warp & 3;               // TMEM lane quarter: rows 32 q .. 32 q + 31
        const int hc = (warp - 4) >> 2;       // column half of the tile
        const uint32_t lane_addr = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(hc * kTN);
        const uint32_t empty_c[2] = {mapa_shared(smem_u32(&sm.acc_empty[0]), 0),
                                     mapa_shared(smem_u32(&sm.acc_empty[1]), 0)};
        uint32_t cc = 0, tb = 0;
        bool ok = true;
        for (int t = pair; t < tiles && ok; t += npairs) {
            const int m0 = (t / tn) * 2 * kTM + (int)rank * kTM;
            const int n0 = (t % tn) * kPN + hc * kTN;
            float sum[kTN];
#pragma unroll
            for (int j = 0; j < kTN; ++j) sum[j] = 0.f;
            for (int c = 0; c < nch; ++c, ++cc) {
                const uint32_t ab = cc & 1;
                if (!warp_wait(&sm.acc_full[ab], (cc >> 1) & 1, abort)) {
                    ok = give_up(abort, err, 54);
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int j0 = 0; j0 < kTN; j0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(lane_addr + ab * kPN + (uint32_t)j0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) sum[j0 + j] += __uint_as_float(v[j]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(empty_c[ab]);
            }
            if (!ok) break;
            const int64_t row = (int64_t)m0 + 32 * q + lane;
            if constexpr (EPI == 3) {
                // scores: column j of the tile -> C[(n0 + j) * ldc + row] (a warp writes 32
                // consecutive rows of each column), times row_scale; the maximum of the
                // CTA's 128 rows per column for the top-k threshold
                const bool live = row < M;
                const float sc = live ? row_scale[row] : 0.f;
#pragma unroll
                for (int j = 0; j < kTN; ++j) {
                    const float v = sum[j] * sc;
                    if (live && n0 + j < n_store) C[(int64_t)(n0 + j) * ldc + row] = v;
                    if (tmax) {
                        float m = live ? v : -INFINITY;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1)
                            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        if (lane == 0) sm.tkey[hc][q][j] = m;
                    }
                }
                if (tmax) {
                    // the 4 warps of this column half meet on a bounded barrier, then
                    // each writes the maxima of 32 columns
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.tmax_bar[hc]);
                    if (!warp_wait(&sm.tmax_bar[hc], tb & 1, abort)) {
                        ok = give_up(abort, err, 55);
                        break;
                    }
                    ++tb;
                    const int j = 32 * q + lane;
                    // a CTA whose 128 rows all lie past M (the second half of the
                    // last pair tile) has no tile maximum to write
                    if (n0 + j < n_store && m0 < M)
                        tmax[(int64_t)(n0 + j) * ldt + m0 / kTM] =
                            fmaxf(fmaxf(sm.tkey[hc][0][j], sm.tkey[hc][1][j]),
                                  fmaxf(sm.tkey[hc][2][j], sm.tkey[hc][3][j]));
                    // the slots are rewritten only after every warp has read them
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.tmax_bar2[hc]);
                    if (!warp_wait(&sm.tmax_bar2[hc], (tb - 1) & 1, abort)) {
                        ok = give_up(abort, err, 56);
                        break;
                    }
                }
            } else if (row < M) {
                float sc = 1.f;
                if (scale_mode == 1) {
                    const float r = row_scale[row];
                    sc = (r != 0.f) ? 1.f / r : 0.f;
                } else if (scale_mode == 2) {
                    sc = row_scale[row];
                }
                if constexpr (EPI == 0) {
                    float4* dst = reinterpret_cast<float4*>(C + row * ldc + n0);
#pragma unroll
                    for (int j = 0; j < kTN; j += 4)
                        dst[j / 4] = make_float4(sum[j] * sc, sum[j + 1] * sc, sum[j + 2] * sc,
                                                 sum[j + 3] * sc);
                } else if constexpr (EPI == 1) {
                    epi_quantize(sum, sc, sm, ep, M, N, row, n0);
                } else {
                    // the record words of these 4 blocks: width b, or for a
                    // fractional width b in the first half and b - 1 after
                    const int b = ep.b;
                    const bool second = ep.cb.split && n0 >= N / 2;
                    const int W = ep.cb.split ? N / 64 * (2 * b - 1) : b * N / 32;
                    const int wb = n0 / 32;
                    const int off = !second ? wb * b : (N / 64) * b + (wb - N / 64) * (b - 1);
                    uint32_t* rec = ep.codes + row * W + off;
                    const uint8_t* cells = ep.idx + row * N + n0;
                    switch (second ? b - 1 : b) {
                        case 1: epi_pack<1>(sum, cells, rec); break;
                        case 2: epi_pack<2>(sum, cells, rec); break;
                        case 3: epi_pack<3>(sum, cells, rec); break;
                        default: epi_pack<4>(sum, cells, rec); break;
                    }
                    if (n0 == 0) {  // |r| from the rotation epilogue's partial sums, in order
                        float rr = 0.f;
                        for (int t = 0; t < N / kTN; ++t) rr += ep.rn2[(int64_t)t * M + row];
                        ep.rnorm[row] = sqrtf(rr);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the pair's MMAs or arrivals may touch it
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tbase, kPairTmemCols);
}

// out[p][r][k]: the bf16 pieces of x (fp32), x = out[0] + out[1] + out[2] to
// ~2^-24 of |x| (each piece the bf16 rounding of what the previous ones left).
__global__ void k_split3(const float* __restrict__ x, int64_t count, __nv_bfloat16* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    const float v = x[i];
    const __nv_bfloat16 p1 = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(p1);
    const __nv_bfloat16 p2 = __float2bfloat16_rn(r1);
    const __nv_bfloat16 p3 = __float2bfloat16_rn(r1 - __bfloat162float(p2));
    out[i] = p1;
    out[count + i] = p2;
    out[2 * count + i] = p3;
}

// out[p][i]: the fp16 pieces of scale * x (scale a power of two, so the
// product is exact): out[0] + out[1] = scale * x to ~2^-22 of its magnitude.
__global__ void k_split2h(const float* __restrict__ x, int64_t count, float scale,
                          __half* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    const float v = x[i] * scale;
    const __half p1 = __float2half_rn(v);
    out[i] = p1;
    out[count + i] = __float2half_rn(v - __half2float(p1));
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tiled_encoder() {
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

// 3-D map over bf16 pieces [pieces][rows][K] (K contiguous), box 64 x 128 x 1,
// 128-byte swizzle; rows beyond `rows` read as zeros.
bool make_piece_map(CUtensorMap* map, const void* base, int pieces, int64_t rows, int K) {
    EncodeTiledFn enc = tiled_encoder();
    if (!enc) return false;
    const cuuint64_t gdim[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)pieces};
    const cuuint64_t gstride[2] = {(cuuint64_t)K * 2, (cuuint64_t)rows * K * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kKB, (cuuint32_t)kTM, 1};
    const cuuint32_t estride[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box,
               estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace

bool gemm_tc_supported(int N, int K) {
    return N > 0 && K > 0 && N % kTN == 0 && K % 128 == 0 && tiled_encoder() != nullptr;
}

int split_bf16x3(const float* x, int64_t count, __nv_bfloat16* out, cudaStream_t s) {
    if (count <= 0) return TQ_OK;
    k_split3<<<(unsigned)((count + 255) / 256), 256, 0, s>>>(x, count, out);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

int split_f16x2(const float* x, int64_t count, float scale, __half* out, cudaStream_t s) {
    if (count <= 0) return TQ_OK;
    k_split2h<<<(unsigned)((count + 255) / 256), 256, 0, s>>>(x, count, scale, out);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

int launch_gemm_tc(int M, int N, int K, const __nv_bfloat16* A, int pa, const __nv_bfloat16* B,
                   float* C, int64_t ldc, const float* row_scale, int scale_mode, int* d_err,
                   cudaStream_t s, int pb, bool transposed, int n_store, float* tmax,
                   int64_t ldt, bool fp16, bool pair_form, const EncodeEpi* epi) {
    if (M <= 0) return TQ_OK;
    if (!gemm_tc_supported(N, K) || pa < 1 || pa > 3 || pb < 1 || pb > 3) return TQ_ERR_ARG;
    if (!transposed && ldc % 4) return TQ_ERR_ARG;
    CUtensorMap ma, mb;
    if (!make_piece_map(&ma, A, pa, M, K) || !make_piece_map(&mb, B, pb, N, K)) return TQ_ERR_CUDA;
    int dev = 0, nsm = 0;
    TQ_TRY_CUDA(cudaGetDevice(&dev));
    TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    const int epi_mode = epi ? epi->mode : 0;
    if ((epi_mode == 1 || epi_mode == 2) &&
        (transposed || tmax || N % kPN != 0 || nsm < 2 || !pair_form))
        return TQ_ERR_ARG;
    if (epi_mode == 4 && (transposed || tmax || N != kTN || K != kTN)) return TQ_ERR_ARG;
    if (epi_mode != 4 && (transposed || !tmax) && N % kPN == 0 && nsm >= 2 && pair_form) {
        const int64_t ptiles = (int64_t)((M + 2 * kTM - 1) / (2 * kTM)) * (N / kPN);
        const int npairs = (int)(ptiles < nsm / 2 ? ptiles : nsm / 2);
        auto kern = transposed ? k_gemm_pair<3>
                    : epi_mode == 1 ? k_gemm_pair<1> : epi_mode == 2 ? k_gemm_pair<2> : k_gemm_pair<0>;
        TQ_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemPairBytes));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * npairs));
        cfg.blockDim = dim3(kPairThreads);
        cfg.dynamicSmemBytes = kSmemPairBytes;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        EncodeEpi e = {};
        if (epi) e = *epi;
        TQ_TRY_CUDA(cudaLaunchKernelEx(&cfg, kern, ma, mb, M, N, K, pa, pb, C, ldc, row_scale,
                                       scale_mode, n_store, tmax, ldt, d_err,
                                       idesc_f16(fp16 ? 0u : 1u, 2 * kTM, kPN), e));
        return TQ_OK;
    }
    const int64_t tiles = (int64_t)((M + kTM - 1) / kTM) * (N / kTN);
    const int nctas = (int)(tiles < nsm ? tiles : nsm);
    TQ_TRY_CUDA(cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kSmemBytes));
    EncodeEpi e1 = {};
    if (epi) e1 = *epi;
    k_gemm_tc<<<nctas, kThreads, kSmemBytes, s>>>(ma, mb, M, N, K, pa, pb, C, ldc, row_scale,
                                                  scale_mode, transposed ? 1 : 0, n_store, tmax,
                                                  ldt, d_err, KeyDecode{}, 0,
                                                  idesc_f16(fp16 ? 0u : 1u, kTM, kTN), e1);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

int launch_gemm_tc_decoded(int M, int N, const KeyDecode& kd, const __nv_bfloat16* B, float* C,
                           int64_t ldc, const float* row_scale, int* d_err, cudaStream_t s,
                           int n_store, float* tmax, int64_t ldt) {
    if (M <= 0) return TQ_OK;
    const int K = 2 * kd.d;
    if (!gemm_tc_supported(N, K) || kd.b < 1 || kd.b > 4) return TQ_ERR_ARG;
    CUtensorMap mb;
    if (!make_piece_map(&mb, B, 2, N, K)) return TQ_ERR_CUDA;
    int dev = 0, nsm = 0;
    TQ_TRY_CUDA(cudaGetDevice(&dev));
    TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    const int64_t tiles = (int64_t)((M + kTM - 1) / kTM) * (N / kTN);
    const int nctas = (int)(tiles < nsm ? tiles : nsm);
    TQ_TRY_CUDA(cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kSmemBytes));
    // the A map is unused in this mode: the B map stands in for the parameter
    k_gemm_tc<<<nctas, kThreadsDecode, kSmemBytes, s>>>(mb, mb, M, N, K, 2, 2, C, ldc, row_scale,
                                                        2, 1, n_store, tmax, ldt, d_err, kd, 1,
                                                        idesc_f16(1u, kTM, kTN), EncodeEpi{});
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

}  // namespace tq
