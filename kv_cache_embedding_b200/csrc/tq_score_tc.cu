// S1 scoring on the sm_100a tensor cores, d = 128, b = 2..4: the estimate
//   s = |x| ( <qr, c[idx]> + |r| sqrt(pi/2)/d <u, 2z - 1> ),  qr = Pi q, u = S qr
// for every key of a group against up to 16 queries per pass, as one
// persistent kernel.
//
// Pages: quant_prune_distill #674 (inner-product quantization: MSE part plus
// the 1-bit QJL correction, unbiased); RecSysChannel #256 item 2 (1-bit
// per-coordinate correction -> unbiased inner products); comuna.ru "Google
// speeds up LLMs 8x" (attention logits computed from 4-bit keys).
//
// Design: scoring is a product [keys x K] . [K x columns]:
//  * A (tensor memory, one key per TMEM lane, 128 keys per tile), fp16, K = 384:
//      k in [0,128):   c_hi[idx_k]   (c scaled by 2^ec, split c = c_hi + c_lo)
//      k in [128,256): c_lo[idx_k]
//      k in [256,384): 2 z_k - 1
//    written by the decode warps from a byte-indexed table (two coordinates
//    per 16-byte entry, 8 interleaved copies so the loads of a quarter-warp
//    never conflict).
//  * B (shared memory, K-major, 128-byte swizzle), 4 columns per query j:
//      4j + 0: qr_hi against c_hi and c_lo       4j + 1: qr_lo against c_hi
//      4j + 2: u_hi against the signs            4j + 3: u_lo against the signs
//    (qr, u scaled by powers of two per query, split into fp16 hi + lo).
//    D[key][4j] + D[key][4j+1] = 2^(ec+eq) <qr, c[idx]> to ~2^-22, and
//    D[key][4j+2] + D[key][4j+3] = 2^eu <u, 2z - 1>; fp32 accumulation.
//  * Warp roles: two groups of 8 warps (4 TMEM lane quarters x 2 coordinate
//    halves); group k takes every other tile of the CTA: it decodes the tile
//    into A[k] (each thread half of one key), lane 0 of the group's first
//    warp issues the MMA into D[k] once all 8 have arrived, and the group
//    writes the tile's scores (each half-warp set half of the queries); the
//    two groups overlap each other's MMA.
//  * Optional per-tile maxima (for the top-k threshold) and zeroing of the
//    top-k counters of the rows it writes.
//  * Every wait is bounded (1 s); a warp that gives up sets the abort flag and
//    the device status word; in-flight MMAs are drained before TMEM is freed.
#include <cuda_fp16.h>

#include "tq_internal.cuh"
#include "tq_codes.cuh"
#include "tq_sm100.cuh"

namespace tq {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTM = 128;               // keys per tile (MMA M)
constexpr int kACols = 3 * kD / 2;     // 192 TMEM columns per A buffer (K = 384 fp16)
constexpr int kKSteps = 3 * kD / 16;   // 24 MMAs of K = 16 per tile
constexpr int kMaxNQ = 16;             // queries per pass
constexpr int kMaxN = 4 * kMaxNQ;      // MMA N
constexpr int kDec = 16;               // 2 groups x (4 lane quarters x 2 coordinate halves)
constexpr int kThreads = 32 * kDec;
constexpr uint32_t kColD = 2 * kACols;  // D double buffer after the two A buffers
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int kCopies = 8;

struct SmemS {
    uint8_t b[6 * kMaxN * 128];         // B: 6 K-regions of N rows x 128 B (first, 1024-aligned)
    float c[8];                         // 2^ec c
    float qscale[kMaxNQ], uscale[kMaxNQ];  // 2^-(ec+eq), 2^-eu
    int eq[kMaxNQ], eu[kMaxNQ];         // per-query exponents of the current unit
    uint32_t tkey[2][kMaxNQ];           // [tile parity][query] running max (ordered key)
    int tcnt[2][kMaxNQ];                // warps that have merged into tkey
    uint64_t a_full[2], d_full[2], mma_done[2], dec_bar;
    uint32_t tmem_base;
    int abort;
    int zero;
};
constexpr size_t kSmemBytes = sizeof(SmemS) + 1024;

// The tiles of this CTA: units (group, query pass) get nctas / units CTAs each
// when they fit (cpg > 0), else whole units go round-robin (cpg = 0).  The
// schedule (units, tiles per unit, cpg) is the same for every thread; a
// position is (unit, t), t >= tpu or unit >= units meaning "done".
struct Sched {
    int units, tpu, cpg;
    __device__ void init(int units_, int tpu_) {
        units = units_;
        tpu = tpu_;
        cpg = units <= (int)gridDim.x ? (int)gridDim.x / units : 0;
    }
    __device__ void start(int& unit, int& t) const {
        if (cpg) {
            unit = (int)blockIdx.x / cpg;
            t = (int)blockIdx.x % cpg;
            if ((int)blockIdx.x >= cpg * units) t = tpu;  // no tiles
        } else {
            unit = (int)blockIdx.x;
            t = 0;
        }
    }
    __device__ bool valid(int unit, int t) const { return unit < units && t < tpu; }
    __device__ bool first(int t) const { return cpg ? t == (int)blockIdx.x % cpg : t == 0; }
    __device__ void advance(int& unit, int& t) const {
        if (cpg) {
            t += cpg;
        } else if (++t >= tpu) {
            t = 0;
            unit += (int)gridDim.x;
        }
    }
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

__device__ __forceinline__ uint32_t pack_h2(__half lo, __half hi) {
    return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// 32 lanes x 32 bits, 8 consecutive columns (thread t: lane quarter base + t).
__device__ __forceinline__ void st_tmem8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}

// 16-byte shared-memory load by shared-window address.
__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(saddr));
    return v;
}

// Order-preserving map of floats to unsigned keys (0 is below every float).
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t x = __float_as_uint(f);
    return (x & 0x80000000u) ? ~x : (x | 0x80000000u);
}
__device__ __forceinline__ float order_val(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// 2^e for |e| < 127 (exact).
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Pair field of coordinates 2m, 2m + 1 (m < 16) of a 32-coordinate block.
template <int B>
__device__ __forceinline__ uint32_t pair_field(const uint32_t (&w)[4], int m) {
    if (B == 4) return (w[m >> 2] >> (8 * (m & 3))) & 0xFFu;            // two [idx|z] nibbles
    if (B == 2) return (w[m >> 3] >> (4 * (m & 7))) & 0xFu;             // two [idx|z] pairs
    return ((w[m >> 3] >> (4 * (m & 7))) & 0xFu) | (((w[2] >> (2 * m)) & 3u) << 4);  // B == 3
}

// (cell, sign bit) of the low (h = 0) / high (h = 1) coordinate of a pair field.
template <int B>
__device__ __forceinline__ void pair_cell(uint32_t f, int h, int& cell, int& z) {
    if (B == 4) {
        const uint32_t nib = (f >> (4 * h)) & 15u;
        cell = (int)(nib & 7u);
        z = (int)(nib >> 3);
    } else if (B == 2) {
        const uint32_t fl = (f >> (2 * h)) & 3u;
        cell = (int)(fl & 1u);
        z = (int)(fl >> 1);
    } else {
        cell = (int)((f >> (2 * h)) & 3u);
        z = (int)((f >> (4 + h)) & 1u);
    }
}

template <int B>
__device__ __forceinline__ void load_block(const uint32_t* __restrict__ p, uint32_t (&w)[4]) {
    if (B == 4) {
        const uint4 t = __ldg(reinterpret_cast<const uint4*>(p));
        w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
    } else if (B == 2) {
        const uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = t.x; w[1] = t.y; w[2] = 0u; w[3] = 0u;
    } else {
        w[0] = __ldg(p); w[1] = __ldg(p + 1); w[2] = __ldg(p + 2); w[3] = 0u;
    }
}

template <int B, int NQ>
__global__ void __launch_bounds__(kThreads, 1)
k_score_tc(const uint32_t* __restrict__ codes, const float* __restrict__ xnorm,
           const float* __restrict__ rnorm, int G, int64_t n, int nq, const float* __restrict__ qr,
           const float* __restrict__ u, KCodebook cb, float cscale, float* __restrict__ scores,
           float* __restrict__ tmax, int ntm, int* __restrict__ zero_cnt, int* __restrict__ err) {
    constexpr int N = 4 * NQ;
    constexpr int W = B * kD / 32;
    constexpr int E = 1 << (2 * B);  // pair fields
    constexpr uint32_t kIdesc = idesc_f16(0, 128, N);  // fp16 x fp16 -> f32, K-major A and B
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // decode table: [pair field][copy] -> (c_hi pair, c_lo pair, sign pair, 0)
    __shared__ __align__(128) uint4 s_lut[256 * kCopies];
    const uint32_t sbase = smem_u32(smem_raw);
    SmemS& sm = *reinterpret_cast<SmemS*>(smem_raw + (((sbase + 1023u) & ~1023u) - sbase));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort = &sm.abort;
    const int npass = (nq + NQ - 1) / NQ;
    const int tpu = (int)((n + kTM - 1) / kTM);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.a_full[i], 8);  // the group's 8 warps
            mbar_init(&sm.d_full[i], 1);  // MMA commit
        }
        mbar_init(&sm.mma_done[0], 1);
        mbar_init(&sm.mma_done[1], 1);
        mbar_init(&sm.dec_bar, kDec);
        for (int i = 0; i < 2 * kMaxNQ; ++i) {
            (&sm.tkey[0][0])[i] = 0u;
            (&sm.tcnt[0][0])[i] = 0;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) sm.c[k] = cb.c[k] * cscale;  // static indices
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

    {
        // ---------------- decode + epilogue warps ----------------
        constexpr int WH = W / 2;     // record words of one coordinate half
        constexpr int NQH = NQ / 2;   // queries of one half-warp set
        const int q = warp & 3;       // TMEM lane quarter: keys 32 q .. 32 q + 31 of a tile
        const int hf = (warp >> 2) & 1;  // coordinates 64 hf .. 64 hf + 63; queries NQH hf ..
        const int grp = warp >> 3;    // group: tiles i with i % 2 == grp, buffers A[grp], D[grp]
        const bool issuer = (warp & 7) == 0 && lane == 0;
        const int td = threadIdx.x;  // 0 .. 32 kDec - 1
        const uint32_t bs = smem_u32(sm.b);
        const uint32_t lane_addr = tbase + ((uint32_t)(32 * q) << 16);
        // decode table: entry f, copy c at byte f * 128 + c * 16
        for (int e = td; e < E * kCopies; e += 32 * kDec) {
            const uint32_t f = (uint32_t)(e / kCopies);
            __half ch[2], cl[2], sg[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                int cell, z;
                pair_cell<B>(f, h, cell, z);
                const float c = sm.c[cell];
                ch[h] = __float2half_rn(c);
                cl[h] = __float2half_rn(c - __half2float(ch[h]));
                sg[h] = __float2half_rn(z ? 1.f : -1.f);
            }
            s_lut[e] = make_uint4(pack_h2(ch[0], ch[1]), pack_h2(cl[0], cl[1]),
                                  pack_h2(sg[0], sg[1]), 0u);
        }
        const uint32_t lane16 = (uint32_t)(lane & (kCopies - 1)) << 4;
        const uint32_t lut_s = smem_u32(s_lut);  // shared-window address of the table
        const float k0 = 1.2533141373155002512f / (float)kD;  // sqrt(pi/2) / d
        const uint32_t a_addr = lane_addr + (uint32_t)(grp * kACols + 32 * hf);
        const uint32_t d_addr = lane_addr + kColD + (uint32_t)(grp * N + 4 * NQH * hf);

        Sched sch;
        sch.init(G * npass, tpu);
        int cu, ct;  // current position
        sch.start(cu, ct);
        // per-unit bases: this thread's key in tile 0 / the group's key 0
        const uint32_t *rec0 = codes, *recg = codes;
        const float *xn0 = xnorm, *rn0 = rnorm;
        float* sc0 = scores;  // row of the unit's first query, this thread's key in tile 0
        float* tm0 = tmax;    // row of the unit's first query
        int qn = 0;           // live queries of the unit
        const int64_t kq = 32 * q + lane;  // key offset within a tile
        auto set_unit = [&](int unit) {
            const int g = unit / npass, z = unit % npass;
            const int q0 = z * NQ;
            recg = codes + (int64_t)g * n * W + WH * hf;
            rec0 = recg + kq * W;
            xn0 = xnorm + (int64_t)g * n + kq;
            rn0 = rnorm + (int64_t)g * n + kq;
            qn = min(NQ, nq - q0);
            sc0 = scores + ((int64_t)g * nq + q0) * n + kq;
            tm0 = tmax ? tmax + ((int64_t)g * nq + q0) * ntm : nullptr;
        };
        // this thread's half record (WH words) and norms of its key in tile t
        auto fetch = [&](int t, uint32_t (&w)[WH], float& xn, float& rn, bool& ok) {
            const int64_t v = (int64_t)t * kTM;
            ok = v + kq < n;
            const uint32_t* rp = ok ? rec0 + v * W : recg;  // a dead lane reads key 0
            if constexpr (WH % 4 == 0) {
#pragma unroll
                for (int c = 0; c < WH / 4; ++c) {
                    const uint4 t4 = __ldg(reinterpret_cast<const uint4*>(rp) + c);
                    w[4 * c] = t4.x; w[4 * c + 1] = t4.y; w[4 * c + 2] = t4.z; w[4 * c + 3] = t4.w;
                }
            } else if constexpr (WH % 2 == 0) {
#pragma unroll
                for (int c = 0; c < WH / 2; ++c) {
                    const uint2 t2 = __ldg(reinterpret_cast<const uint2*>(rp) + c);
                    w[2 * c] = t2.x; w[2 * c + 1] = t2.y;
                }
            } else {
#pragma unroll
                for (int c = 0; c < WH; ++c) w[c] = __ldg(rp + c);
            }
            xn = ok ? __ldg(xn0 + v) : 0.f;
            rn = ok ? __ldg(rn0 + v) : 0.f;
        };
        uint32_t wc[WH];
#pragma unroll
        for (int c = 0; c < WH; ++c) wc[c] = 0u;
        float xc = 0.f, rc = 0.f;
        bool okc = false;
        uint32_t i = 0, mine = 0, eb = 0;  // CTA tile counter, this group's tile counter
        bool running = true;
        auto dec_sync = [&]() -> bool {  // all decode warps; bounded
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.dec_bar);
            const bool ok = warp_wait(&sm.dec_bar, eb & 1, abort);
            ++eb;
            return ok;
        };
        while (sch.valid(cu, ct) && running) {
            int nu = cu, nt = ct;  // next position
            sch.advance(nu, nt);
            const bool nvalid = sch.valid(nu, nt);
            const bool own = (int)(i & 1) == grp;
            if (sch.first(ct)) {
                // every MMA of the previous unit has been read back by its group
                if (!dec_sync()) {
                    running = give_up(abort, err, 26);
                    break;
                }
                set_unit(cu);
                const int g = cu / npass, z = cu % npass;
                const int q0 = z * NQ;
                if (warp < NQ && warp < kDec) {  // per-query power-of-two scales
                    for (int j = warp; j < NQ; j += kDec) {
                        float mq = 0.f, mu = 0.f;
                        if (j < qn) {
                            const float* qrow = qr + ((int64_t)g * nq + q0 + j) * kD;
                            const float* urow = u + ((int64_t)g * nq + q0 + j) * kD;
                            for (int i2 = lane; i2 < kD; i2 += 32) {
                                mq = fmaxf(mq, fabsf(qrow[i2]));
                                mu = fmaxf(mu, fabsf(urow[i2]));
                            }
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
                            mu = fmaxf(mu, __shfl_xor_sync(0xffffffffu, mu, o));
                        }
                        int eq = 0, eu = 0;
                        if (mq > 0.f) {
                            frexpf(mq, &eq);
                            eq = 14 - eq;  // max |qr| 2^eq in [2^13, 2^14)
                        }
                        if (mu > 0.f) {
                            frexpf(mu, &eu);
                            eu = 14 - eu;
                        }
                        if (lane == 0) {
                            sm.qscale[j] = pow2f(-eq) / cscale;
                            sm.uscale[j] = pow2f(-eu);
                            sm.eq[j] = eq;
                            sm.eu[j] = eu;
                        }
                    }
                }
                if (!dec_sync()) {
                    running = give_up(abort, err, 27);
                    break;
                }
                // B: rows nrow = 4 j + part, K pairs kp (k = 2 kp, 2 kp + 1)
                for (int e = td; e < N * (3 * kD / 2); e += 32 * kDec) {
                    const int nrow = e / (3 * kD / 2), kp = e % (3 * kD / 2);
                    const int k = 2 * kp, part = nrow & 3, j = nrow >> 2;
                    const int seg = k / kD, i2 = k % kD;
                    const float* src = nullptr;
                    float scale = 0.f;
                    if (j < qn) {
                        const int64_t row = (int64_t)g * nq + q0 + j;
                        if ((part == 0 && seg < 2) || (part == 1 && seg == 0)) {
                            src = qr + row * kD + i2;
                            scale = pow2f(sm.eq[j]);
                        } else if (part >= 2 && seg == 2) {
                            src = u + row * kD + i2;
                            scale = pow2f(sm.eu[j]);
                        }
                    }
                    uint32_t word = 0u;
                    if (src) {
                        const float2 x = *reinterpret_cast<const float2*>(src);
                        const float y0 = x.x * scale, y1 = x.y * scale;  // exact: powers of two
                        const __half h0 = __float2half_rn(y0), h1 = __float2half_rn(y1);
                        word = (part & 1) ? pack_h2(__float2half_rn(y0 - __half2float(h0)),
                                                    __float2half_rn(y1 - __half2float(h1)))
                                          : pack_h2(h0, h1);
                    }
                    const int r = k / 64;                 // K region of 64 elements (128 B)
                    const int ob = (k % 64) * 2;          // byte within the 128-byte row
                    const int phys = (((ob >> 4) ^ (nrow & 7)) << 4) | (ob & 15);
                    *reinterpret_cast<uint32_t*>(sm.b + r * (N * 128) + nrow * 128 + phys) = word;
                }
                if (zero_cnt && ct == 0 && td < 2 * qn)  // top-k counters of these rows
                    zero_cnt[(td & 1) * (int64_t)G * nq + (int64_t)g * nq + q0 + (td >> 1)] = 0;
                fence_proxy_async_smem();
                if (!dec_sync()) {  // B complete before any MMA of the unit
                    running = give_up(abort, err, 28);
                    break;
                }
                // this group's first tile of the unit: its own tile or the next one
                if (own) fetch(ct, wc, xc, rc, okc);
                else if (nvalid && nu == cu) fetch(nt, wc, xc, rc, okc);
            }
            if (!own) {  // the other group's tile
                cu = nu;
                ct = nt;
                ++i;
                continue;
            }
            // prefetch this group's next tile (two tiles on) of the same unit
            int u2 = nu, t2 = nt;
            if (nvalid) sch.advance(u2, t2);
            uint32_t wn[WH];
#pragma unroll
            for (int c = 0; c < WH; ++c) wn[c] = 0u;
            float xnn = 0.f, rnn = 0.f;
            bool okn = false;
            const bool pre = nvalid && nu == cu && sch.valid(u2, t2) && u2 == cu;
            if (pre) fetch(t2, wn, xnn, rnn, okn);
            // decode: A[grp] is free (the group read back its previous MMA)
#pragma unroll
            for (int blk = 0; blk < kD / 64; ++blk) {  // this half's two blocks
                uint32_t wb[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int c = 0; c < B; ++c) wb[c] = wc[blk * B + c];
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // 8 coordinate pairs at a time
                    uint32_t chi[8], clo[8], sgn[8];
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const uint4 e = lds128(lut_s + (pair_offset<B>(wb, 8 * h + m) | lane16));
                        chi[m] = e.x;
                        clo[m] = e.y;
                        sgn[m] = e.z;
                    }
                    const uint32_t col = (uint32_t)(16 * blk + 8 * h);
                    st_tmem8(a_addr + col, chi);
                    st_tmem8(a_addr + kD / 2 + col, clo);
                    st_tmem8(a_addr + kD + col, sgn);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.a_full[grp]);
            if ((warp & 7) == 0) {  // the group's MMA, issued by one thread
                bool ok = true;
                if (issuer) {
                    ok = mbar_wait(&sm.a_full[grp], mine & 1, abort, kWaitNs);
                    if (ok) {
                        tc_fence_after();
                        const uint32_t a = tbase + (uint32_t)(grp * kACols);
                        const uint32_t d = tbase + kColD + (uint32_t)(grp * N);
#pragma unroll
                        for (int ks = 0; ks < kKSteps; ++ks)
                            mma_f16_ts(d, a + ks * 8,
                                       smem_desc_kmajor_sw128(bs + (ks >> 2) * (N * 128) + (ks & 3) * 32),
                                       kIdesc, ks != 0);
                        tc_commit(&sm.d_full[grp]);
                    }
                }
                if (!__all_sync(0xffffffffu, ok)) {
                    running = give_up(abort, err, 22);
                    break;
                }
            }
            // read back D[grp] and write the scores
            if (!warp_wait(&sm.d_full[grp], mine & 1, abort)) {
                running = give_up(abort, err, 24);
                break;
            }
            tc_fence_after();
            const float kap = k0 * rc;
            const int64_t v = (int64_t)ct * kTM;
            constexpr int CH = (4 * NQH) < 16 ? (4 * NQH) : 16;  // columns per read
#pragma unroll
            for (int c0 = 0; c0 < 4 * NQH; c0 += CH) {
                uint32_t dv[16];
                if constexpr (CH == 16) {
                    tmem_ld16(d_addr + (uint32_t)c0, dv);
                } else {
                    uint32_t d8[8];
                    tmem_ld8(d_addr + (uint32_t)c0, d8);
#pragma unroll
                    for (int c = 0; c < 8; ++c) dv[c] = d8[c];
                }
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < CH / 4; ++jj) {
                    const int j = NQH * hf + c0 / 4 + jj;
                    const float mse = (__uint_as_float(dv[4 * jj]) + __uint_as_float(dv[4 * jj + 1])) * sm.qscale[j];
                    const float qjl = (__uint_as_float(dv[4 * jj + 2]) + __uint_as_float(dv[4 * jj + 3])) * sm.uscale[j];
                    const float sc = xc * (mse + kap * qjl);
                    const bool live = okc && j < qn;
                    if (live) sc0[(int64_t)j * n + v] = sc;
                    if (tmax) {
                        // tile maximum: the group's 4 lane-quarter warps merge into
                        // tkey; the last to merge writes it and resets the slot (next
                        // used by this group's next tile, after all 4 have arrived)
                        float m = live ? sc : -INFINITY;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        if (lane == 0) {
                            atomicMax(&sm.tkey[grp][j], order_key(m));
                            __threadfence_block();
                            if (atomicAdd(&sm.tcnt[grp][j], 1) == 3) {
                                const uint32_t key = atomicExch(&sm.tkey[grp][j], 0u);
                                sm.tcnt[grp][j] = 0;
                                if (j < qn) tm0[(int64_t)j * ntm + ct] = order_val(key);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < WH; ++c) wc[c] = wn[c];
            xc = xnn;
            rc = rnn;
            okc = okn;
            ++mine;
            cu = nu;
            ct = nt;
            ++i;
        }
    }

    // every MMA a group issued completes before TMEM is released (they have all
    // been waited for unless a wait gave up)
    if ((warp & 7) == 0 && lane == 0) {
        tc_commit(&sm.mma_done[warp >> 3]);
        mbar_wait(&sm.mma_done[warp >> 3], 0, &sm.zero, kWaitNs);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

template <int B, int NQ>
int launch_bq(const uint32_t* codes, const float* xn, const float* rn, int G, int64_t n, int nq,
              const float* qr, const float* u, const KCodebook& kc, float cscale, float* scores,
              float* tmax, int ntm, int* zero_cnt, int* err, cudaStream_t s) {
    auto kern = k_score_tc<B, NQ>;
    TQ_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kSmemBytes));
    int dev = 0, nsm = 0;
    TQ_TRY_CUDA(cudaGetDevice(&dev));
    TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    const int64_t tiles = (int64_t)G * ((nq + NQ - 1) / NQ) * ((n + kTM - 1) / kTM);
    const int nctas = (int)(tiles < nsm ? tiles : nsm);
    kern<<<nctas, kThreads, kSmemBytes, s>>>(codes, xn, rn, G, n, nq, qr, u, kc, cscale, scores,
                                             tmax, ntm, zero_cnt, err);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

template <int B>
int launch_b(int nqp, const uint32_t* codes, const float* xn, const float* rn, int G, int64_t n,
             int nq, const float* qr, const float* u, const KCodebook& kc, float cscale,
             float* scores, float* tmax, int ntm, int* zero_cnt, int* err, cudaStream_t s) {
    if (nqp <= 4)
        return launch_bq<B, 4>(codes, xn, rn, G, n, nq, qr, u, kc, cscale, scores, tmax, ntm,
                               zero_cnt, err, s);
    if (nqp <= 8)
        return launch_bq<B, 8>(codes, xn, rn, G, n, nq, qr, u, kc, cscale, scores, tmax, ntm,
                               zero_cnt, err, s);
    return launch_bq<B, 16>(codes, xn, rn, G, n, nq, qr, u, kc, cscale, scores, tmax, ntm,
                            zero_cnt, err, s);
}

}  // namespace

// The tensor-core path pays a fixed ~23 ns per MMA instruction for N <= 64
// (24 per 128-key tile, whatever the number of queries), while the SIMT kernel's
// cost grows with the queries: it is taken from 16 queries per group on.
bool score_tc_supported(int d, int b, int G, int64_t n, int nq) {
    return d == kD && b >= 2 && b <= 4 && nq >= kMaxNQ && n > 0 &&
           n < ((int64_t)1 << 31) / 128 * 128 && (int64_t)G * n < ((int64_t)1 << 40);
}

size_t score_tc_tiles(int64_t n) { return (size_t)((n + kTM - 1) / kTM); }

int launch_score_tc(const tq_codebook_t* cb, int G, int64_t n, const uint32_t* d_codes,
                    const float* d_xnorm, const float* d_rnorm, int nq, const float* qr,
                    const float* u, float* d_scores, float* tmax, int* zero_cnt, int* d_err,
                    cudaStream_t s) {
    // 2^ec: the largest |centroid| scaled into [2^13, 2^14)
    float cmax = 0.f;
    for (int k = 0; k < cb->levels && k < 8; ++k) cmax = fmaxf(cmax, fabsf(cb->centroids[k]));
    int ec = 0;
    if (cmax > 0.f) {
        frexpf(cmax, &ec);
        ec = 14 - ec;
    }
    const float cscale = ldexpf(1.f, ec);
    // d_err was cleared by the query transform that precedes this kernel
    const KCodebook kc = make_kcodebook(cb);
    const int nqp = nq < kMaxNQ ? nq : kMaxNQ;
    const int ntm = (int)score_tc_tiles(n);
    switch (cb->b) {
        case 2: return launch_b<2>(nqp, d_codes, d_xnorm, d_rnorm, G, n, nq, qr, u, kc, cscale, d_scores, tmax, ntm, zero_cnt, d_err, s);
        case 3: return launch_b<3>(nqp, d_codes, d_xnorm, d_rnorm, G, n, nq, qr, u, kc, cscale, d_scores, tmax, ntm, zero_cnt, d_err, s);
        default: return launch_b<4>(nqp, d_codes, d_xnorm, d_rnorm, G, n, nq, qr, u, kc, cscale, d_scores, tmax, ntm, zero_cnt, d_err, s);
    }
}

}  // namespace tq
