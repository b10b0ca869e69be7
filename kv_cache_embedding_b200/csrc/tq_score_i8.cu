// S1 scoring on the sm_100a tensor cores with exact integer products, d = 128,
// b = 2..4, inner-product records, up to 16 queries per pass:
//   s = |x| ( <qr, c[idx]> + |r| sqrt(pi/2)/d <u, 2z - 1> ),  qr = Pi q, u = S qr.
//
// Pages: quant_prune_distill #674 (inner-product quantization: the MSE part
// plus the 1-bit QJL correction, unbiased); RecSysChannel #256 item 2 (a
// 1-bit per-coordinate correction makes inner products unbiased); comuna.ru
// "Google speeds up LLMs 8x" (attention logits computed from 4-bit keys).
//
// Why integers.  fp32-accurate SIMT scoring of a key against its group's
// queries is bound by FMA issue (2 FMAs per coordinate and query) and by the
// shared-memory lookups that decode each coordinate; both exceed the time its
// 72-byte record takes to stream from HBM.  Here the product runs on the
// tensor core as kind::i8 MMAs with s32 accumulation, which is exact, so the
// only rounding is that of the operands:
//  * A (tensor memory, one key per TMEM lane, 128 keys per tile), K = 384 int8:
//      k in [0,128):   ch[idx_k]          C_t = round(c_t * scale_c) = 256 ch_t + cl_t,
//      k in [128,256): cl[idx_k]          |C_t| <= 127 * 256 (two signed bytes)
//      k in [256,384): 127 (1 - z_k)      (0 or 127)
//    decoded in registers: one byte permute (prmt) maps four 3-bit cells to
//    four table bytes, and the sign mode of the same instruction (selector
//    bit 3 = z) maps the sign bits to 127 or 0 -- no table in shared memory.
//  * B (shared memory, K-major, 128-byte swizzle), 6 columns per query j:
//      Q = round(qr * sq) = 2^16 q0 + 2^8 q1 + q2,  U = round(u * su) likewise,
//      |Q|, |U| <= 127 * 2^16 (three signed bytes each);
//      6j+0: q0 | 0  | 0      6j+3: 0 | 0 | u0
//      6j+1: q1 | q0 | 0      6j+4: 0 | 0 | u1
//      6j+2: q2 | q1 | 0      6j+5: 0 | 0 | u2
//    (blocks ch | cl | z of K), so that
//      2^8 (2^16 D0 + 2^8 D1 + D2) = sum_k C Q - sum_k cl q2
//      2^16 E0 + 2^8 E1 + E2 = sum_k 127 (1 - z_k) U_k,
//    sum_k (2z_k - 1) U_k = SU - (2/127) (2^16 E0 + 2^8 E1 + E2), SU = sum_k U_k.
//  * Error bound (|q| = |qr|, Pi orthogonal): the centroid rounding gives
//    |ds| <= |x| |qr|_1 max|c| / (2 * 32512) <= 3.4e-5 |q| |x| at b = 4 (the
//    scale is chosen among 1024 candidates to shrink it further); the query
//    pieces, the dropped cl * q2 term and the fp32 recombination add < 5e-6
//    |q| |x|.  The parity tolerance is 1e-4 |q| |x|.
//  * Warp groups of 4 warps (one per TMEM lane quarter, thread = key); group k
//    takes every kGroups-th tile of the CTA's segment: it decodes the tile into
//    its own A buffer, its first warp's lane 0 issues the 12 MMAs (K = 32 each)
//    into its D buffer, and the group writes the scores; the groups overlap
//    each other's MMAs.  Per-tile maxima (for the top-k threshold) go through
//    a double-buffered slot in shared memory, written out by the group's
//    issuing thread one tile later.
//  * Every wait is bounded (1 s); a warp that gives up sets the abort flag and
//    the device status word; in-flight MMAs are drained before TMEM is freed.
#include <cmath>

#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTM = 128;          // keys per tile (MMA M)
constexpr int kACols = 96;        // A: 384 int8 per key = 96 TMEM columns
constexpr int kKSteps = 12;       // MMAs of K = 32 per tile
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr float kPieceMax = 8323072.f;  // 127 * 2^16: three signed bytes per value
constexpr int kCMax = 32512;            // 127 * 256: two signed bytes per centroid
constexpr size_t kMinSmem = 120 * 1024;  // one CTA per SM (it takes all of TMEM)

template <int NQ>
struct CfgI8 {
    static constexpr int N = (6 * NQ + 15) / 16 * 16;             // MMA N, 6 columns per query
    static constexpr int kStride = (kACols + N + 31) / 32 * 32;   // TMEM columns per group
    static constexpr int kGroups = (512 / kStride) < 4 ? (512 / kStride) : 4;
    static constexpr int kWarps = 4 * kGroups;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kDCols = (6 * NQ + 7) / 8 * 8;           // D columns read back
};

template <int NQ>
struct SmemI8 {
    uint8_t b[3 * CfgI8<NQ>::N * 128];  // B: 3 K-atoms of N rows x 128 B (first, 1024-aligned)
    float mscale[NQ], qa[NQ], qb[NQ];   // per query of the current unit
    float wmax[4][2][4][NQ];            // [group][tile parity][lane quarter][query]
    uint64_t a_full[4], d_full[4], mma_done[4], cta_bar;
    uint32_t tmem_base;
    int abort;
    int zero;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort, kWaitNs);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool give_up(volatile int* abort, int* err, int site) {
    *abort = 1;
    atomicCAS(err, 0, TQ_ERR_DEVICE_TIMEOUT * 1000 - site);
    return false;
}

// Signed-byte pieces of an integer |v| <= 127 * 2^16: v = 2^16 p0 + 2^8 p1 + p2.
__device__ __forceinline__ void pieces3(int v, int& p0, int& p1, int& p2) {
    p2 = ((v + 128) & 255) - 128;
    const int v1 = (v - p2) >> 8;  // exact
    p1 = ((v1 + 128) & 255) - 128;
    p0 = (v1 - p1) >> 8;
}

__device__ __forceinline__ uint32_t pack_bytes(int a, int b, int c, int d) {
    return (uint32_t)(a & 255) | ((uint32_t)(b & 255) << 8) | ((uint32_t)(c & 255) << 16) |
           ((uint32_t)(d & 255) << 24);
}

// One record (b * 16 bytes) of a key.
template <int B>
__device__ __forceinline__ void load_record(const uint32_t* __restrict__ p, uint32_t (&w)[4 * B]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < B; ++i) {
        const uint4 t = __ldg(q + i);
        w[4 * i] = t.x;
        w[4 * i + 1] = t.y;
        w[4 * i + 2] = t.z;
        w[4 * i + 3] = t.w;
    }
}

// Coordinates 8m .. 8m+7 of a record as eight nibbles, nibble j = idx | z << 3
// (the b = 4 field; for b < 4 the cell index has fewer bits).
template <int B>
__device__ __forceinline__ uint32_t nibble_word(const uint32_t (&w)[4 * B], int m) {
    if constexpr (B == 4) {
        return w[m];
    } else {
        // 2-bit fields (b = 2: idx | z << 1; b = 3: the 2-bit cell) of the 8
        // coordinates, spread to bits 4k, 4k + 1
        uint32_t h = (w[B * (m >> 2) + ((m & 3) >> 1)] >> (16 * (m & 1))) & 0xFFFFu;
        h = (h | (h << 8)) & 0x00FF00FFu;
        h = (h | (h << 4)) & 0x0F0F0F0Fu;
        h = (h | (h << 2)) & 0x33333333u;
        if constexpr (B == 2) return (h & 0x11111111u) | ((h & 0x22222222u) << 2);
        // b = 3: the sign bits of the block's third word, spread to bits 4k + 3
        uint32_t z = (w[3 * (m >> 2) + 2] >> (8 * (m & 3))) & 0xFFu;
        z = (z | (z << 12)) & 0x000F000Fu;
        z = (z | (z << 6)) & 0x03030303u;
        z = (z | (z << 3)) & 0x11111111u;
        return h | (z << 3);
    }
}

template <int B, int NQ>
__global__ void __launch_bounds__(CfgI8<NQ>::kThreads, 1)
k_score_i8(const uint32_t* __restrict__ codes, const float* __restrict__ xnorm,
           const float* __restrict__ rnorm, int G, int64_t n, int64_t n_stride, int64_t k0, int nq,
           const float* __restrict__ qr, const float* __restrict__ u, uint4 ctab, float scale_c,
           float* __restrict__ scores, float* __restrict__ tmax, int ntm,
           int* __restrict__ zero_cnt, int* __restrict__ err) {
    using C = CfgI8<NQ>;
    constexpr int N = C::N;
    constexpr int NG = C::kGroups;
    constexpr int W = 4 * B;  // record words
    constexpr uint32_t kIdesc = idesc_i8(128, N);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    SmemI8<NQ>& sm = *reinterpret_cast<SmemI8<NQ>*>(smem_raw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int grp = warp >> 2, quarter = warp & 3;
    volatile int* abort = &sm.abort;
    const int npass = (nq + NQ - 1) / NQ;
    const int64_t tpu = (n + kTM - 1) / kTM;
    const int64_t total = (int64_t)G * npass * tpu;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) {
            mbar_init(&sm.a_full[i], 4);  // the group's 4 warps
            mbar_init(&sm.d_full[i], 1);  // MMA commit
            mbar_init(&sm.mma_done[i], 1);
        }
        mbar_init(&sm.cta_bar, C::kWarps);
        sm.abort = 0;
        sm.zero = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    const uint32_t bs = smem_u32(sm.b);
    const uint32_t a_col = (uint32_t)(grp * C::kStride);
    const uint32_t lane_addr = tbase + ((uint32_t)(32 * quarter) << 16);
    const bool leader = quarter == 0 && lane == 0;
    const float kqjl = 1.2533141373155002512f / (float)kD;  // sqrt(pi/2) / d

    uint32_t eb = 0;    // CTA barrier phases
    uint32_t mine = 0;  // tiles of this group so far (barrier parities, wmax slots)
    // the issuing thread's tile whose maxima are still to be written
    float* pend = nullptr;
    int pend_qn = 0;
    uint32_t pend_par = 0;
    auto flush = [&]() {
        if (pend) {
            for (int j = 0; j < pend_qn; ++j) {
                const float m = fmaxf(fmaxf(sm.wmax[grp][pend_par][0][j], sm.wmax[grp][pend_par][1][j]),
                                      fmaxf(sm.wmax[grp][pend_par][2][j], sm.wmax[grp][pend_par][3][j]));
                pend[(int64_t)j * ntm] = m;
            }
            pend = nullptr;
        }
    };
    auto cta_sync = [&]() -> bool {  // every warp; bounded
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.cta_bar);
        const bool ok = warp_wait(&sm.cta_bar, eb & 1, abort);
        ++eb;
        return ok;
    };

    bool running = true;
    int64_t pos = (int64_t)blockIdx.x * total / gridDim.x;
    const int64_t hi = ((int64_t)blockIdx.x + 1) * total / gridDim.x;
    while (pos < hi && running) {
        // ---- segment: tiles [t0, t0 + len) of one unit (group g, query pass)
        const int64_t unit = pos / tpu;
        const int64_t t0 = pos % tpu;
        const int64_t len = (tpu - t0) < (hi - pos) ? (tpu - t0) : (hi - pos);
        pos += len;
        const int g = (int)(unit / npass);
        const int q0 = (int)(unit % npass) * NQ;
        const int qn = min(NQ, nq - q0);
        const int64_t row0 = (int64_t)g * nq + q0;
        // every group has read back its MMAs of the previous segment
        if (!cta_sync()) {
            running = give_up(abort, err, 41);
            break;
        }
        if (leader) flush();
        // B: rows of the live queries (every byte of rows 6j .. 6j + 5), then
        // the padding rows; per-query scales
        for (int j = warp; j < NQ; j += C::kWarps) {
            float4 qv = make_float4(0.f, 0.f, 0.f, 0.f), uv = qv;
            if (j < qn) {
                qv = *reinterpret_cast<const float4*>(qr + (row0 + j) * kD + 4 * lane);
                uv = *reinterpret_cast<const float4*>(u + (row0 + j) * kD + 4 * lane);
            }
            float mq = fmaxf(fmaxf(fabsf(qv.x), fabsf(qv.y)), fmaxf(fabsf(qv.z), fabsf(qv.w)));
            float mu = fmaxf(fmaxf(fabsf(uv.x), fabsf(uv.y)), fmaxf(fabsf(uv.z), fabsf(uv.w)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
                mu = fmaxf(mu, __shfl_xor_sync(0xffffffffu, mu, o));
            }
            const float sq = mq > 0.f ? kPieceMax / mq : 0.f;
            const float su = mu > 0.f ? kPieceMax / mu : 0.f;
            const float qf[4] = {qv.x, qv.y, qv.z, qv.w};
            const float uf[4] = {uv.x, uv.y, uv.z, uv.w};
            int pq[3][4], pu[3][4];
            int sum_u = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int Q = (int)fminf(fmaxf(rintf(qf[c] * sq), -kPieceMax), kPieceMax);
                const int U = (int)fminf(fmaxf(rintf(uf[c] * su), -kPieceMax), kPieceMax);
                pieces3(Q, pq[0][c], pq[1][c], pq[2][c]);
                pieces3(U, pu[0][c], pu[1][c], pu[2][c]);
                sum_u += U;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum_u += __shfl_xor_sync(0xffffffffu, sum_u, o);
            uint32_t P[3], Uw[3];
#pragma unroll
            for (int p = 0; p < 3; ++p) {
                P[p] = pack_bytes(pq[p][0], pq[p][1], pq[p][2], pq[p][3]);
                Uw[p] = pack_bytes(pu[p][0], pu[p][1], pu[p][2], pu[p][3]);
            }
            // rows 6j + r, K-atoms a (ch | cl | z); this lane's 4 bytes at K 4 lane
            const uint32_t word[6][3] = {{P[0], 0u, 0u}, {P[1], P[0], 0u}, {P[2], P[1], 0u},
                                         {0u, 0u, Uw[0]}, {0u, 0u, Uw[1]}, {0u, 0u, Uw[2]}};
#pragma unroll
            for (int r = 0; r < 6; ++r) {
                const int row = 6 * j + r;
                const int phys = (((lane >> 2) ^ (row & 7)) << 4) | ((4 * lane) & 15);
#pragma unroll
                for (int a = 0; a < 3; ++a)
                    *reinterpret_cast<uint32_t*>(sm.b + a * (N * 128) + row * 128 + phys) = word[r][a];
            }
            if (lane == 0) {
                sm.mscale[j] = sq > 0.f ? 256.f / (scale_c * sq) : 0.f;
                sm.qa[j] = su > 0.f ? (float)sum_u / su : 0.f;
                sm.qb[j] = su > 0.f ? (-2.f / 127.f) / su : 0.f;
            }
        }
        if constexpr (N > 6 * NQ) {
            constexpr int kPad = (N - 6 * NQ) * 32;  // words of the padding rows per K-atom
            for (int e = threadIdx.x; e < 3 * kPad; e += C::kThreads)
                *reinterpret_cast<uint32_t*>(sm.b + (e / kPad) * (N * 128) + 6 * NQ * 128 +
                                             4 * (e % kPad)) = 0u;
        }
        if (zero_cnt && t0 == 0 && (int)threadIdx.x < 2 * qn)  // top-k counters of these rows
            zero_cnt[(threadIdx.x & 1) * (int64_t)G * nq + row0 + (threadIdx.x >> 1)] = 0;
        fence_proxy_async_smem();
        if (!cta_sync()) {  // B complete before any MMA of the segment
            running = give_up(abort, err, 42);
            break;
        }
        // keys k0 .. k0 + n of group g (records n_stride apart per group)
        const uint32_t* codes_g = codes + ((int64_t)g * n_stride + k0) * W;
        const float* xn_g = xnorm + (int64_t)g * n_stride + k0;
        const float* rn_g = rnorm + (int64_t)g * n_stride + k0;
        const int kq = 32 * quarter + lane;  // key offset within a tile
        auto fetch = [&](int64_t t, uint32_t (&w)[W], float& xn, float& rn, bool& ok) {
            const int64_t v = t * kTM + kq;
            ok = v < n;
            load_record<B>(codes_g + (ok ? v : 0) * W, w);
            xn = ok ? __ldg(xn_g + v) : 0.f;
            rn = ok ? __ldg(rn_g + v) : 0.f;
        };
        uint32_t wc[W];
        float xc = 0.f, rc = 0.f;
        bool okc = false;
        if (grp < len) fetch(t0 + grp, wc, xc, rc, okc);
        for (int64_t k = grp; k < len; k += NG) {
            const int64_t t = t0 + k;
            // prefetch this group's next tile
            uint32_t wn[W];
            float xnn = 0.f, rnn = 0.f;
            bool okn = false;
            if (k + NG < len) fetch(t + NG, wn, xnn, rnn, okn);
            // ---- decode into A (this group's buffer; its previous MMA has completed)
            const uint32_t a_addr = lane_addr + a_col;
            const uint32_t CH0 = ctab.x, CH1 = ctab.y, CL0 = ctab.z, CL1 = ctab.w;
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // nibble words 8h .. 8h + 7: columns 16h .. 16h + 15
                uint32_t nw[8], o[16];
#pragma unroll
                for (int m = 0; m < 8; ++m) nw[m] = nibble_word<B>(wc, 8 * h + m);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const uint32_t ms = nw[m] & 0x77777777u;
                    o[2 * m] = prmt(CH0, CH1, ms);
                    o[2 * m + 1] = prmt(CH0, CH1, ms >> 16);
                }
                tmem_st16(a_addr + (uint32_t)(16 * h), o);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const uint32_t ms = nw[m] & 0x77777777u;
                    o[2 * m] = prmt(CL0, CL1, ms);
                    o[2 * m + 1] = prmt(CL0, CL1, ms >> 16);
                }
                tmem_st16(a_addr + (uint32_t)(32 + 16 * h), o);
#pragma unroll
                for (int m = 0; m < 8; ++m) {  // sign mode: z = 1 -> 0x00, z = 0 -> 0x7F
                    o[2 * m] = prmt(0x7F7F7F7Fu, 0x7F7F7F7Fu, nw[m]);
                    o[2 * m + 1] = prmt(0x7F7F7F7Fu, 0x7F7F7F7Fu, nw[m] >> 16);
                }
                tmem_st16(a_addr + (uint32_t)(64 + 16 * h), o);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.a_full[grp]);
            if (quarter == 0) {  // the group's MMAs, issued by one thread
                bool ok = true;
                if (lane == 0) {
                    ok = mbar_wait(&sm.a_full[grp], mine & 1, abort, kWaitNs);
                    if (ok) {
                        tc_fence_after();
                        const uint32_t a = tbase + a_col;
                        const uint32_t d = tbase + a_col + kACols;
#pragma unroll
                        for (int ks = 0; ks < kKSteps; ++ks)
                            mma_i8_ts(d, a + (uint32_t)(8 * ks),
                                      smem_desc_kmajor_sw128(bs + (ks >> 2) * (N * 128) + (ks & 3) * 32),
                                      kIdesc, ks != 0);
                        tc_commit(&sm.d_full[grp]);
                        flush();  // the group's previous tile (the other wmax slot)
                    }
                }
                if (!__all_sync(0xffffffffu, ok)) {
                    running = give_up(abort, err, 43);
                    break;
                }
            }
            // ---- read back D and write the scores
            if (!warp_wait(&sm.d_full[grp], mine & 1, abort)) {
                running = give_up(abort, err, 44);
                break;
            }
            tc_fence_after();
            uint32_t dv[C::kDCols];
            const uint32_t d_addr = lane_addr + a_col + kACols;
#pragma unroll
            for (int c = 0; c < C::kDCols; c += 8) {
                uint32_t r8[8];
                tmem_ld8(d_addr + (uint32_t)c, r8);
#pragma unroll
                for (int i = 0; i < 8; ++i) dv[c + i] = r8[i];
            }
            tmem_wait_ld();
            const float kap = kqjl * rc;
            const int64_t v = t * kTM + kq;
            const uint32_t par = mine & 1;
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                const float m = fmaf((float)(int)dv[6 * j], 65536.f,
                                     fmaf((float)(int)dv[6 * j + 1], 256.f, (float)(int)dv[6 * j + 2]));
                const float z = fmaf((float)(int)dv[6 * j + 3], 65536.f,
                                     fmaf((float)(int)dv[6 * j + 4], 256.f, (float)(int)dv[6 * j + 5]));
                const float mse = m * sm.mscale[j];
                const float qjl = fmaf(sm.qb[j], z, sm.qa[j]);
                const float sc = xc * fmaf(kap, qjl, mse);
                const bool live = okc && j < qn;
                if (live) scores[(row0 + j) * n + v] = sc;
                if (tmax) {
                    float mx = live ? sc : -INFINITY;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    if (lane == 0) sm.wmax[grp][par][quarter][j] = mx;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (tmax && leader) {  // written out after the group's next MMA issue (or the segment's end)
                pend = tmax + row0 * ntm + t;
                pend_qn = qn;
                pend_par = par;
            }
#pragma unroll
            for (int c = 0; c < W; ++c) wc[c] = wn[c];
            xc = xnn;
            rc = rnn;
            okc = okn;
            ++mine;
        }
    }
    // the last tile maxima; every MMA a group issued completes before TMEM is
    // released (they have all been waited for unless a wait gave up)
    if (running && cta_sync() && leader) flush();
    if (leader) {
        tc_commit(&sm.mma_done[grp]);
        mbar_wait(&sm.mma_done[grp], 0, &sm.zero, kWaitNs);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

template <int B, int NQ>
int launch_bq(const uint32_t* codes, const float* xn, const float* rn, int G, int64_t n,
              int64_t n_stride, int64_t k0, int nq, const float* qr, const float* u, uint4 ctab,
              float scale_c, float* scores, float* tmax, int ntm, int* zero_cnt, int* err,
              cudaStream_t s) {
    using C = CfgI8<NQ>;
    auto kern = k_score_i8<B, NQ>;
    size_t smem = sizeof(SmemI8<NQ>) + 1024;
    if (smem < kMinSmem) smem = kMinSmem;
    TQ_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    int dev = 0, nsm = 0;
    TQ_TRY_CUDA(cudaGetDevice(&dev));
    TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    const int64_t tiles = (int64_t)G * ((nq + NQ - 1) / NQ) * ((n + kTM - 1) / kTM);
    const int nctas = (int)(tiles < nsm ? tiles : nsm);
    kern<<<nctas, C::kThreads, smem, s>>>(codes, xn, rn, G, n, n_stride, k0, nq, qr, u, ctab,
                                          scale_c, scores, tmax, ntm, zero_cnt, err);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

template <int B>
int launch_b(int nqp, const uint32_t* codes, const float* xn, const float* rn, int G, int64_t n,
             int64_t n_stride, int64_t k0, int nq, const float* qr, const float* u, uint4 ctab,
             float scale_c, float* scores, float* tmax, int ntm, int* zero_cnt, int* err,
             cudaStream_t s) {
#define TQ_I8(NQV)                                                                             \
    return launch_bq<B, NQV>(codes, xn, rn, G, n, n_stride, k0, nq, qr, u, ctab, scale_c, scores, \
                             tmax, ntm, zero_cnt, err, s)
    if (nqp <= 2) TQ_I8(2);
    if (nqp <= 4) TQ_I8(4);
    if (nqp <= 8) TQ_I8(8);
    TQ_I8(16);
#undef TQ_I8
}

}  // namespace

// Centroid scale and byte tables: C_t = round(c_t * scale_c) = 256 ch_t + cl_t
// with |C_t| <= 32512.  Among the scales that put max |C_t| in the top 1024
// integers of that range, the one with the smallest largest rounding error
// |c_t scale_c - C_t| is taken.
void score_i8_tables(const tq_codebook_t* cb, uint4* ctab, float* scale_c) {
    const int L = cb->levels < 8 ? cb->levels : 8;
    double cmax = 0.0;
    for (int t = 0; t < L; ++t) cmax = fmax(cmax, fabs((double)cb->centroids[t]));
    double best = cmax > 0.0 ? kCMax / cmax : 1.0, best_err = 2.0;
    for (int T = kCMax; cmax > 0.0 && T > kCMax - 1024; --T) {
        const double sc = T / cmax;
        double e = 0.0;
        for (int t = 0; t < L; ++t) {
            const double y = (double)cb->centroids[t] * sc;
            e = fmax(e, fabs(y - rint(y)));
        }
        if (e < best_err) {
            best_err = e;
            best = sc;
        }
    }
    uint32_t ch[2] = {0u, 0u}, cl[2] = {0u, 0u};
    for (int t = 0; t < L; ++t) {
        const int C = (int)rint((double)cb->centroids[t] * best);
        const int lo = ((C + 128) & 255) - 128;
        const int hi = (C - lo) / 256;
        ch[t >> 2] |= (uint32_t)(hi & 255) << (8 * (t & 3));
        cl[t >> 2] |= (uint32_t)(lo & 255) << (8 * (t & 3));
    }
    *ctab = make_uint4(ch[0], ch[1], cl[0], cl[1]);
    *scale_c = (float)best;
}

bool score_i8_supported(const tq_codebook_t* cb, int G, int64_t n, int nq, const void* d_codes) {
    return !is_mse(cb) && !is_split(cb) && cb->d == kD && cb->b >= 2 && cb->b <= 4 && nq > 0 &&
           n > 0 &&
           n < ((int64_t)1 << 31) / 128 * 128 && (int64_t)G * n < ((int64_t)1 << 40) &&
           ((uintptr_t)d_codes & 15u) == 0;
}

int launch_score_i8(const tq_codebook_t* cb, int G, int64_t n, const uint32_t* d_codes,
                    const float* d_xnorm, const float* d_rnorm, int nq, const float* qr,
                    const float* u, float* d_scores, float* tmax, int* zero_cnt, int* d_err,
                    cudaStream_t s, int64_t n_stride, int64_t k0) {
    if (n_stride < 0) n_stride = n;
    uint4 ctab;
    float scale_c;
    score_i8_tables(cb, &ctab, &scale_c);
    const int nqp = nq < 16 ? nq : 16;
    const int ntm = (int)((n + kTM - 1) / kTM);
    // d_err was cleared by the query transform that precedes this kernel
    switch (cb->b) {
        case 2: return launch_b<2>(nqp, d_codes, d_xnorm, d_rnorm, G, n, n_stride, k0, nq, qr, u, ctab, scale_c, d_scores, tmax, ntm, zero_cnt, d_err, s);
        case 3: return launch_b<3>(nqp, d_codes, d_xnorm, d_rnorm, G, n, n_stride, k0, nq, qr, u, ctab, scale_c, d_scores, tmax, ntm, zero_cnt, d_err, s);
        default: return launch_b<4>(nqp, d_codes, d_xnorm, d_rnorm, G, n, n_stride, k0, nq, qr, u, ctab, scale_c, d_scores, tmax, ntm, zero_cnt, d_err, s);
    }
}

}  // namespace tq
