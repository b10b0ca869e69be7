// Device helpers shared by the SIMT scoring kernels (tq_score.cu) and the
// decode-attention kernel (tq_attention.cu): the code-record field decode of
// the layout in tq.h, the 16-entry decode table, the queries' (Pi q, S Pi q)
// pairs in shared memory and the (mse, qjl) accumulation of the estimator
//   s = |x| ( <qr, c[idx]> + |r| sqrt(pi/2)/d <u, 2z - 1> )
// (quant_prune_distill #674: inner-product estimate from the codes).
#pragma once

#include "tq_internal.cuh"

namespace tq {
namespace sc {

constexpr float kSqrtHalfPi = 1.2533141373155002512f;  // sqrt(pi/2)

// Decode coordinate j (0..31) of a block: cell index and sign bit.
template <int B>
__device__ __forceinline__ void field(const uint32_t* w, int j, int& cell, uint32_t& z) {
    if (B == 1) {
        cell = 0;
        z = (w[0] >> j) & 1u;
    } else if (B == 2) {
        const uint32_t f = (w[j >> 4] >> (2 * (j & 15))) & 3u;
        cell = (int)(f & 1u);
        z = f >> 1;
    } else if (B == 3) {
        cell = (int)((w[j >> 4] >> (2 * (j & 15))) & 3u);
        z = (w[2] >> j) & 1u;
    } else {
        const uint32_t f = (w[j >> 3] >> (4 * (j & 7))) & 15u;
        cell = (int)(f & 7u);
        z = f >> 3;
    }
}

// Block blk's B words; A16: the record is 16-byte aligned (false for the
// records of a fractional width, d/64 (2b - 1) words long: 8-byte loads).
template <int B, bool A16 = true>
__device__ __forceinline__ void load_block(const uint32_t* __restrict__ rec, int blk,
                                           uint32_t w[4]) {
    const uint32_t* p = rec + blk * B;
    if (B == 4 && A16) {
        const uint4 t = __ldg(reinterpret_cast<const uint4*>(p));
        w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
    } else if (B == 4) {
        const uint2 t0 = __ldg(reinterpret_cast<const uint2*>(p));
        const uint2 t1 = __ldg(reinterpret_cast<const uint2*>(p) + 1);
        w[0] = t0.x; w[1] = t0.y; w[2] = t1.x; w[3] = t1.y;
    } else if (B == 2) {
        const uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = t.x; w[1] = t.y;
    } else {
#pragma unroll
        for (int i = 0; i < B; ++i) w[i] = __ldg(p + i);
    }
}

// ---- scoring, v2 ---------------------------------------------------------
// Thread = KP keys; block = 128 threads; queries in passes of NQ.  Shared
// memory holds, per query, the pairs (qr_i, u_i) interleaved, and a 16-entry
// table mapping a coordinate's field f to (c[idx], 2z - 1), so decoding a
// coordinate is one bit-field extract and one conflict-free 8-byte load
// (every entry owns its own bank pair).  Each query pair is loaded once per
// two coordinates and reused by the thread's KP keys.  Accumulators are
// (mse, qjl) pairs; with F2 they are updated by the packed fma.rn.f32x2.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    return __ffma2_rn(a, b, c);  // fma.rn.f32x2: the register pairs stay packed
}

template <bool F2>
__device__ __forceinline__ float2 pair_fma(float2 a, float2 b, float2 c) {
    if (F2) return ffma2(a, b, c);
    return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
}

// Field of coordinate j (0..31) of a block as the decode-table index.
template <int B>
__device__ __forceinline__ uint32_t field_index(const uint32_t (&w)[4], int j) {
    if (B == 1) return (w[0] >> j) & 1u;
    if (B == 2) return (w[j >> 4] >> (2 * (j & 15))) & 3u;
    if (B == 3) return ((w[j >> 4] >> (2 * (j & 15))) & 3u) | (((w[2] >> j) & 1u) << 2);
    return (w[j >> 3] >> (4 * (j & 7))) & 15u;
}

// Decode table entry f -> (c[idx], 2z - 1) for the field layouts above; for
// the MSE-only variant the field is the whole b-bit cell: (c[f], 0).  LO: the
// second grid of a fractional width (c_lo).
template <int B, bool LO = false>
__device__ __forceinline__ float2 table_entry(const KCodebook& cb, int f) {
    if (cb.mse) return make_float2(cb.c[f & ((1 << B) - 1)], 0.f);
    if (B == 1) return make_float2(0.f, (f & 1) ? 1.f : -1.f);
    if (B == 2) return make_float2(LO ? cb.c_lo[f & 1] : cb.c[f & 1], (f & 2) ? 1.f : -1.f);
    if (B == 3) return make_float2(LO ? cb.c_lo[f & 3] : cb.c[f & 3], (f & 4) ? 1.f : -1.f);
    return make_float2(LO ? cb.c_lo[f & 7] : cb.c[f & 7], (f & 8) ? 1.f : -1.f);
}

// Shared-memory setup common to the scoring kernels: the 16-entry decode
// table (and, for a fractional width, the second half's table of width B - 1
// in s_tab[16 .. 32)) and the NQ queries' (qr_i, u_i) pairs starting at query q0.
template <int B, int NQ, bool SPLIT = false>
__device__ __forceinline__ void load_score_smem(const KCodebook& cb, const float* __restrict__ qr,
                                                const float* __restrict__ u, int64_t row0, int qn,
                                                int d, float2* s_qu, float2* s_tab) {
    if (threadIdx.x < 16) {
        float2 e = make_float2(0.f, 0.f);
        switch (threadIdx.x) {  // static indices keep the codebook in parameter space
#define TQ_TAB(F) case F: e = table_entry<B>(cb, F); break;
            TQ_TAB(0) TQ_TAB(1) TQ_TAB(2) TQ_TAB(3) TQ_TAB(4) TQ_TAB(5) TQ_TAB(6) TQ_TAB(7)
            TQ_TAB(8) TQ_TAB(9) TQ_TAB(10) TQ_TAB(11) TQ_TAB(12) TQ_TAB(13) TQ_TAB(14) TQ_TAB(15)
#undef TQ_TAB
        }
        s_tab[threadIdx.x] = e;
    } else if (SPLIT && threadIdx.x < 32) {
        constexpr int BL = B > 1 ? B - 1 : 1;
        float2 e = make_float2(0.f, 0.f);
        switch (threadIdx.x - 16) {
#define TQ_TAB(F) case F: e = table_entry<BL, true>(cb, F); break;
            TQ_TAB(0) TQ_TAB(1) TQ_TAB(2) TQ_TAB(3) TQ_TAB(4) TQ_TAB(5) TQ_TAB(6) TQ_TAB(7)
            TQ_TAB(8) TQ_TAB(9) TQ_TAB(10) TQ_TAB(11) TQ_TAB(12) TQ_TAB(13) TQ_TAB(14) TQ_TAB(15)
#undef TQ_TAB
        }
        s_tab[threadIdx.x] = e;
    }
    for (int e = threadIdx.x; e < NQ * d; e += blockDim.x) {
        const int qq = e / d, i = e % d;
        const int64_t row = row0 + qq;
        s_qu[e] = (qq < qn) ? make_float2(qr[row * d + i], u[row * d + i]) : make_float2(0.f, 0.f);
    }
}

// Accumulate (mse, qjl) pairs of KP records against NQ queries, over the
// records' first nblk blocks (all d/32 when nblk < 0); s_qu rows are d apart.
template <int B, int NQ, int KP, bool F2, bool A16 = true>
__device__ __forceinline__ void score_keys(const uint32_t* const (&rec)[KP], int d,
                                           const float2* s_qu, const float2* s_tab,
                                           float2 (&acc)[KP][NQ], int nblk = -1) {
    if (nblk < 0) nblk = d / 32;
    uint32_t wcur[KP][4], wnext[KP][4];
#pragma unroll
    for (int k = 0; k < KP; ++k) load_block<B, A16>(rec[k], 0, wcur[k]);
    for (int blk = 0; blk < nblk; ++blk) {
        if (blk + 1 < nblk) {
#pragma unroll
            for (int k = 0; k < KP; ++k) load_block<B, A16>(rec[k], blk + 1, wnext[k]);
        }
        const float2* qb = s_qu + blk * 32;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            float2 e0[KP], e1[KP];
#pragma unroll
            for (int k = 0; k < KP; ++k) {
                e0[k] = s_tab[field_index<B>(wcur[k], j)];
                e1[k] = s_tab[field_index<B>(wcur[k], j + 1)];
            }
#pragma unroll
            for (int qq = 0; qq < NQ; ++qq) {
                const float4 p = *reinterpret_cast<const float4*>(qb + qq * d + j);
                const float2 p0 = make_float2(p.x, p.y), p1 = make_float2(p.z, p.w);
#pragma unroll
                for (int k = 0; k < KP; ++k) {
                    acc[k][qq] = pair_fma<F2>(p0, e0[k], acc[k][qq]);
                    acc[k][qq] = pair_fma<F2>(p1, e1[k], acc[k][qq]);
                }
            }
        }
        if (blk + 1 < nblk) {
#pragma unroll
            for (int k = 0; k < KP; ++k)
#pragma unroll
                for (int w = 0; w < 4; ++w) wcur[k][w] = wnext[k][w];
        }
    }
}

// score_keys over a record of width B, or over a fractional-width record
// (SPLIT): its first d/64 blocks of width B against the first d/2 query
// coordinates and table s_tab, then its last d/64 blocks of width B - 1
// against the rest and table s_tab + 16.
template <int B, int NQ, int KP, bool F2, bool SPLIT>
__device__ __forceinline__ void score_record(const uint32_t* const (&rec)[KP], int d,
                                             const float2* s_qu, const float2* s_tab,
                                             float2 (&acc)[KP][NQ]) {
    if constexpr (!SPLIT) {
        score_keys<B, NQ, KP, F2>(rec, d, s_qu, s_tab, acc);
    } else {
        constexpr int BL = B > 1 ? B - 1 : 1;
        score_keys<B, NQ, KP, F2, false>(rec, d, s_qu, s_tab, acc, d / 64);
        const uint32_t* lo[KP];
#pragma unroll
        for (int k = 0; k < KP; ++k) lo[k] = rec[k] + (d / 64) * B;
        score_keys<BL, NQ, KP, F2, false>(lo, d, s_qu + d / 2, s_tab + 16, acc, d / 64);
    }
}

}  // namespace sc
}  // namespace tq
