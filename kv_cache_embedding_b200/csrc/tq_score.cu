// S0-S2: query transform, scoring over packed codes, top-k; dequantization;
// the unquantized fp32 logit baseline and the exact fp32 top-k.
//
// Pages: quant_prune_distill #674 (inner-product quantization, unbiased
// estimate; dequantization = inverse rotation and renormalisation);
// RecSysChannel #256 item 2 (1-bit per-coordinate correction -> unbiased
// inner products); comuna.ru "Google speeds up LLMs 8x" (attention logits
// from 4-bit keys vs 32-bit keys; vector-search recall).
//
// Estimator (for a record with norms |x|, |r|, cells idx, signs z):
//   s = |x| ( <qr, c[idx]> + |r| sqrt(pi/2)/d <u, 2z - 1> ),  qr = Pi q, u = S qr.
#include <algorithm>
#include <cmath>
#include <cstdlib>

#include "tq_internal.cuh"
#include "tq_score_common.cuh"

namespace tq {
namespace {

using namespace sc;

template <int B, int NQ, int KP, bool F2, bool SPLIT>
__global__ __launch_bounds__(128) void k_score2(const uint32_t* __restrict__ codes,
                                                const float* __restrict__ xnorm,
                                                const float* __restrict__ rnorm, int64_t n, int d,
                                                int nq, const float* __restrict__ qr,
                                                const float* __restrict__ u, KCodebook cb,
                                                float* __restrict__ scores,
                                                float* __restrict__ cmax, int nchunks,
                                                int* __restrict__ zero_cnt) {
    extern __shared__ __align__(16) float2 s_qu[];  // [NQ][d] pairs (qr_i, u_i)
    __shared__ float2 s_tab[SPLIT ? 32 : 16];
    __shared__ float s_max[4][NQ];
    const int g = blockIdx.y;
    const int q0 = blockIdx.z * NQ;
    const int qn = min(NQ, nq - q0);
    load_score_smem<B, NQ, SPLIT>(cb, qr, u, (int64_t)g * nq + q0, qn, d, s_qu, s_tab);
    __syncthreads();
    const int W = SPLIT ? d / 64 * (2 * B - 1) : words_per_vector(d, B);
    int64_t v[KP];
    bool ok[KP];
#pragma unroll
    for (int k = 0; k < KP; ++k) {
        v[k] = ((int64_t)blockIdx.x * KP + k) * blockDim.x + threadIdx.x;
        ok[k] = v[k] < n;
    }
    float2 acc[KP][NQ];
#pragma unroll
    for (int k = 0; k < KP; ++k)
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq) acc[k][qq] = make_float2(0.f, 0.f);
    const uint32_t* rec[KP];
#pragma unroll
    for (int k = 0; k < KP; ++k) rec[k] = codes + ((int64_t)g * n + (ok[k] ? v[k] : 0)) * W;

    score_record<B, NQ, KP, F2, SPLIT>(rec, d, s_qu, s_tab, acc);
    const float k0 = kSqrtHalfPi / (float)d;
    float mx[NQ];
#pragma unroll
    for (int qq = 0; qq < NQ; ++qq) mx[qq] = -INFINITY;
#pragma unroll
    for (int k = 0; k < KP; ++k) {
        if (!ok[k]) continue;
        const int64_t gv = (int64_t)g * n + v[k];
        const float xn = xnorm[gv];
        const float kap = k0 * rnorm[gv];
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq)
            if (qq < qn) {
                const float sc = xn * (acc[k][qq].x + kap * acc[k][qq].y);
                scores[((int64_t)g * nq + q0 + qq) * n + v[k]] = sc;
                mx[qq] = fmaxf(mx[qq], sc);
            }
    }
    if (zero_cnt && blockIdx.x == 0 && threadIdx.x < 2 * qn)  // top-k counters of these rows
        zero_cnt[(threadIdx.x & 1) * (int64_t)gridDim.y * nq + (int64_t)g * nq + q0 +
                 (threadIdx.x >> 1)] = 0;
    if (cmax) {  // the block's 128 KP keys form one chunk: its maximum per query
        const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                mx[qq] = fmaxf(mx[qq], __shfl_xor_sync(0xffffffffu, mx[qq], o));
            if (lane == 0) s_max[warp][qq] = mx[qq];
        }
        __syncthreads();
        if (threadIdx.x < qn) {
            const int qq = threadIdx.x;
            const float m = fmaxf(fmaxf(s_max[0][qq], s_max[1][qq]), fmaxf(s_max[2][qq], s_max[3][qq]));
            cmax[((int64_t)g * nq + q0 + qq) * nchunks + blockIdx.x] = m;
        }
    }
}

// ---- top-k -------------------------------------------------------------
// Warp-wide selection of the best K of `count` scores in shared memory
// (element e has id id0 + e); removed/invalid entries hold -inf.
// Results go to vals/ids[0..K).  Lane 0 writes.
__device__ void warp_select(float* s, int count, int64_t id0, int K, float* vals, int64_t* ids) {
    const int lane = threadIdx.x % 32;
    for (int r = 0; r < K; ++r) {
        float bv = -INFINITY;
        int be = -1;
        for (int e = lane; e < count; e += 32) {
            const float v = s[e];
            if (v != -INFINITY && (be < 0 || v > bv)) {  // ascending e: first max wins ties
                bv = v;
                be = e;
            }
        }
        int64_t bid = (be < 0) ? INT64_MAX : id0 + be;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int64_t oid = __shfl_xor_sync(0xffffffffu, bid, o);
            if (better(ov, oid, bv, bid)) {
                bv = ov;
                bid = oid;
            }
        }
        if (lane == 0) {
            vals[r] = bv;
            ids[r] = bid;
        }
        if (bid != INT64_MAX && (bid - id0) % 32 == lane) s[bid - id0] = -INFINITY;
        __syncwarp();
    }
}

// ---- running top-k lists ---------------------------------------------------
// A warp keeps a sorted list of the best K (K <= 32) (value, id) pairs seen so
// far in registers: lane r holds the r-th best by (value desc, id asc); empty
// slots hold (-inf, none).  New entries are screened against the K-th best with
// one ballot; the rare ones that beat it are inserted one at a time.
constexpr int kCandTile = 256;  // keys scored per pass of a block (thread = key)
static_assert(kCandTile == kTopkTile, "key ranges are bounded by the top-k workspace tiles");

template <typename Id>
__device__ __forceinline__ bool better_t(float va, Id ia, float vb, Id ib) {
    return va > vb || (va == vb && ia < ib);
}
template <typename Id>
__device__ __forceinline__ Id id_none() {
    // INT64_MAX, INT32_MAX, UINT32_MAX
    return (Id)(~(uint64_t)0 >> (sizeof(Id) == 8 ? 1 : ((Id)-1 < (Id)0 ? 33 : 32)));
}

template <typename Id>
struct WarpList {
    float v;     // this lane's slot
    Id id;
    float kv;    // the K-th best (same on every lane)
    Id kid;

    __device__ __forceinline__ void init() {
        v = -INFINITY;
        id = id_none<Id>();
        kv = -INFINITY;
        kid = id_none<Id>();
    }
    // Offer every lane's (cv, cid) where `want`; warp-uniform call.
    __device__ __forceinline__ void offer(bool want, float cv, Id cid, int K, int lane) {
        uint32_t m = __ballot_sync(0xffffffffu, want && better_t(cv, cid, kv, kid));
        while (m) {
            const int src = __ffs(m) - 1;
            m &= m - 1;
            const float nv = __shfl_sync(0xffffffffu, cv, src);
            const Id nid = __shfl_sync(0xffffffffu, cid, src);
            if (!better_t(nv, nid, kv, kid)) continue;  // the list moved on meanwhile
            // position = number of kept entries better than the new one
            const int p = __popc(__ballot_sync(0xffffffffu, lane < K && better_t(v, id, nv, nid)));
            const float uv = __shfl_up_sync(0xffffffffu, v, 1);
            const Id uid = __shfl_up_sync(0xffffffffu, id, 1);
            if (lane == p) {
                v = nv;
                id = nid;
            } else if (lane > p && lane < K) {
                v = uv;
                id = uid;
            }
            kv = __shfl_sync(0xffffffffu, v, K - 1);
            kid = __shfl_sync(0xffffffffu, id, K - 1);
        }
    }
};

// grid: (nblk key ranges of `span` keys, G, query passes of NQ <= 8); 256
// threads, thread = key.  Each warp keeps a running best-K list per query
// over the keys it scores; at the end the block's 8 lists per query are
// combined in shared memory.  Output: the range's best K per query (value,
// global key id; -inf / INT64_MAX where the range has fewer) in
// part_vals/part_ids [G][nq][nblk][K].
template <int B, int NQ, bool F2, bool SPLIT>
__global__ __launch_bounds__(256) void k_score_topk(
    const uint32_t* __restrict__ codes, const float* __restrict__ xnorm,
    const float* __restrict__ rnorm, int64_t n, int d, int nq, const float* __restrict__ qr,
    const float* __restrict__ u, KCodebook cb, int K, int nblk, int64_t span,
    float* __restrict__ part_vals, int64_t* __restrict__ part_ids) {
    extern __shared__ __align__(16) float2 s_qu[];  // [NQ][d]
    __shared__ float2 s_tab[SPLIT ? 32 : 16];
    __shared__ float s_lv[NQ][8][kMaxK];
    __shared__ uint32_t s_li[NQ][8][kMaxK];
    const int g = blockIdx.y;
    const int q0 = blockIdx.z * NQ;
    const int qn = min(NQ, nq - q0);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t kb0 = (int64_t)blockIdx.x * span;
    const int64_t kb1 = min(n, kb0 + span);
    load_score_smem<B, NQ, SPLIT>(cb, qr, u, (int64_t)g * nq + q0, qn, d, s_qu, s_tab);
    __syncthreads();
    const int W = SPLIT ? d / 64 * (2 * B - 1) : words_per_vector(d, B);
    const float k0 = kSqrtHalfPi / (float)d;
    WarpList<uint32_t> L[NQ];
#pragma unroll
    for (int qq = 0; qq < NQ; ++qq) L[qq].init();
    for (int64_t t0 = kb0; t0 < kb1; t0 += kCandTile) {
        const int64_t v = t0 + threadIdx.x;
        const bool ok = v < kb1;
        const int64_t gv = (int64_t)g * n + (ok ? v : kb0);
        const uint32_t* rec[1] = {codes + gv * W};
        float2 acc[1][NQ];
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq) acc[0][qq] = make_float2(0.f, 0.f);
        score_record<B, NQ, 1, F2, SPLIT>(rec, d, s_qu, s_tab, acc);
        const float xn = xnorm[gv];
        const float kap = k0 * rnorm[gv];
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq)
            L[qq].offer(ok && qq < qn, xn * (acc[0][qq].x + kap * acc[0][qq].y),
                        (uint32_t)(v - kb0), K, lane);
    }
#pragma unroll
    for (int qq = 0; qq < NQ; ++qq)
        if (lane < K) {
            s_lv[qq][warp][lane] = L[qq].v;
            s_li[qq][warp][lane] = L[qq].id;
        }
    __syncthreads();
    if (warp < qn) {
        WarpList<uint32_t> M;
        M.init();
        for (int w = 0; w < 8; ++w)
            M.offer(lane < K, s_lv[warp][w][lane], s_li[warp][w][lane], K, lane);
        const int64_t o = (((int64_t)g * nq + q0 + warp) * nblk + blockIdx.x) * K;
        if (lane < K) {
            const bool have = M.id != id_none<uint32_t>();
            part_vals[o + lane] = have ? M.v : -INFINITY;
            part_ids[o + lane] = have ? kb0 + (int64_t)M.id : INT64_MAX;
        }
    }
}

// Top-K of rows of materialised scores.  grid: (P blocks per row, rows); 256
// threads.  Every warp derives the same threshold t on its own: the chunk
// maxima (one per kTopkTile keys) are folded by max into 64 slots (two per
// lane), sorted across the warp, and t is the K-th largest slot -- K slots,
// hence K scores, are >= t, so the whole top K is.  Each block then scans its
// share of the row and appends the scores >= t to the row's candidate list in
// global memory.  The last block of a row to finish (a counter, no waiting)
// selects the best K from the list, or from the whole row if the list
// overflowed (massive ties).  The counters are zeroed by the score kernel that
// writes the row.
constexpr int kCandCapG = kTopkCandidates;  // candidate entries per row

// Descending bitonic sort of 64 values held two per lane (slot 2 * lane + h
// in v[h]).
__device__ __forceinline__ void warp_sort64_desc(float (&v)[2], int lane) {
    for (int k = 2; k <= 64; k <<= 1) {
        const bool desc = ((2 * lane) & k) == 0;  // direction of this slot's run
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 1) {  // partner slot in the same lane
                const float hi = fmaxf(v[0], v[1]), lo = fminf(v[0], v[1]);
                v[0] = desc ? hi : lo;
                v[1] = desc ? lo : hi;
            } else {
                const bool lower = (lane & (j >> 1)) == 0;  // bit j of the slot index
                const bool keep_max = lower == desc;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float o = __shfl_xor_sync(0xffffffffu, v[h], j >> 1);
                    v[h] = keep_max ? fmaxf(v[h], o) : fminf(v[h], o);
                }
            }
        }
    }
}

__global__ __launch_bounds__(256, 4) void k_topk_collect(const float* __restrict__ scores,
                                                      const float* __restrict__ cmax, int64_t n,
                                                      int nchunks, int K, int* cand_cnt, int* done,
                                                      float* cand_v, int* cand_i,
                                                      float* __restrict__ vals,
                                                      int64_t* __restrict__ ids, int64_t id0) {
    __shared__ int s_last;
    const int64_t row = blockIdx.y;
    const int P = gridDim.x;
    const int lane = threadIdx.x % 32;
    const float* sr = scores + row * n;
    const float* cm = cmax + row * nchunks;
    const int64_t per = (n + P - 1) / P;
    const int64_t e0 = (int64_t)blockIdx.x * per;
    const int64_t e1 = min(n, e0 + per);
    constexpr int U = 16;
    float v[U];
    auto load = [&](int64_t base) {
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t e = base + (int64_t)j * blockDim.x + threadIdx.x;
            v[j] = e < e1 ? sr[e] : -INFINITY;
        }
    };
    load(e0);  // the first pass's scores are in flight while the threshold is formed
    // slot s (0..63) = the maximum of the chunk maxima c = s (mod 64): the
    // block's 256 threads read the chunk maxima once (4 threads per slot),
    // warp 0 sorts the 64 slots and the K-th largest is the threshold
    __shared__ float s_slot[4][64];
    __shared__ float s_thr;
    {
        const int sl = threadIdx.x & 63, part = threadIdx.x >> 6;
        float m = -INFINITY;
#pragma unroll 4
        for (int c = sl + 64 * part; c < nchunks; c += 256) m = fmaxf(m, cm[c]);
        s_slot[part][sl] = m;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        float f[2];
        f[0] = fmaxf(fmaxf(s_slot[0][lane], s_slot[1][lane]), fmaxf(s_slot[2][lane], s_slot[3][lane]));
        f[1] = fmaxf(fmaxf(s_slot[0][lane + 32], s_slot[1][lane + 32]),
                     fmaxf(s_slot[2][lane + 32], s_slot[3][lane + 32]));
        warp_sort64_desc(f, lane);
        // the K-th largest slot (-inf when fewer than K chunks)
        const float t = __shfl_sync(0xffffffffu, ((K - 1) & 1) ? f[1] : f[0], (K - 1) >> 1);
        if (lane == 0) s_thr = t;
    }
    __syncthreads();
    const float thr = s_thr;
    float* cv = cand_v + row * kCandCapG;
    int* ci = cand_i + row * kCandCapG;
    for (int64_t base = e0; base < e1; base += (int64_t)U * blockDim.x) {
        if (base != e0) load(base);
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t e = base + (int64_t)j * blockDim.x + threadIdx.x;
            const bool pass = e < e1 && v[j] >= thr;
            const uint32_t m = __ballot_sync(0xffffffffu, pass);
            if (m) {
                const int leader = __ffs(m) - 1;
                int pos0 = 0;
                if (lane == leader) pos0 = atomicAdd(&cand_cnt[row], __popc(m));
                pos0 = __shfl_sync(0xffffffffu, pos0, leader);
                const int pos = pos0 + __popc(m & ((1u << lane) - 1u));
                if (pass && pos < kCandCapG) {
                    cv[pos] = v[j];
                    ci[pos] = (int)e;
                }
            }
        }
    }
    // the last block of the row selects
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&done[row], 1) == P - 1);
    __syncthreads();
    if (!s_last || threadIdx.x >= 32) return;
    __threadfence();
    const int cnt = __ldcg(&cand_cnt[row]);
    WarpList<int> L;
    L.init();
    if (cnt <= kCandCapG) {
        constexpr int C = 8;
        for (int c0 = 0; c0 < cnt; c0 += 32 * C) {
            float cvv[C];
            int cii[C];
#pragma unroll
            for (int j = 0; j < C; ++j) {
                const int c = c0 + 32 * j + lane;
                cvv[j] = c < cnt ? __ldcg(&cv[c]) : -INFINITY;
                cii[j] = c < cnt ? __ldcg(&ci[c]) : 0;
            }
#pragma unroll
            for (int j = 0; j < C; ++j) L.offer(c0 + 32 * j + lane < cnt, cvv[j], cii[j], K, lane);
        }
    } else {
        for (int64_t f0 = 0; f0 < n; f0 += 32) {
            const int64_t e = f0 + lane;
            L.offer(e < n, e < n ? sr[e] : -INFINITY, (int)e, K, lane);
        }
    }
    if (lane < K) {
        const bool have = L.id != id_none<int>();
        vals[row * K + lane] = have ? L.v : -INFINITY;
        ids[row * K + lane] = have ? id0 + (int64_t)L.id : INT64_MAX;
    }
}

// Plain score rows -> per-tile partial top-K (exact search path).
// grid: (tiles, rows); scores [rows][ncols] with column c having id col0 + c.
__global__ __launch_bounds__(256) void k_rows_topk_tile(const float* __restrict__ sc, int64_t ld,
                                                        int64_t ncols, int64_t col0, int K,
                                                        int ntiles_total, int tile0,
                                                        float* __restrict__ part_vals,
                                                        int64_t* __restrict__ part_ids) {
    __shared__ float s[kTopkTile];
    const int64_t row = blockIdx.y;
    const int64_t c0 = (int64_t)blockIdx.x * kTopkTile;
    for (int e = threadIdx.x; e < kTopkTile; e += blockDim.x)
        s[e] = (c0 + e < ncols) ? sc[row * ld + c0 + e] : -INFINITY;
    __syncthreads();
    if (threadIdx.x < 32) {
        const int64_t o = (row * ntiles_total + tile0 + blockIdx.x) * K;
        warp_select(s, kTopkTile, col0 + c0, K, part_vals + o, part_ids + o);
    }
}

// Merge partial lists of K entries (missing entries: id INT64_MAX) into the
// final K per row; list p of row r starts at r * row_stride + p * list_stride
// ([rows][nparts][K]: K * nparts, K; [nparts][rows][K]: K, rows * K).  One warp
// per row (4 rows per 128-thread block): the entries stream through a running
// best-K list, 16 per lane loaded ahead.
__global__ __launch_bounds__(128) void k_topk_merge(const float* __restrict__ part_vals,
                                                    const int64_t* __restrict__ part_ids,
                                                    int64_t rows, int nparts, int K,
                                                    float* __restrict__ vals,
                                                    int64_t* __restrict__ ids,
                                                    int64_t row_stride, int64_t list_stride) {
    constexpr int C = 16;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t row = (int64_t)blockIdx.x * 4 + warp;
    if (row >= rows) return;
    const float* pv = part_vals + row * row_stride;
    const int64_t* pi = part_ids + row * row_stride;
    const int64_t count = (int64_t)nparts * K;
    const bool packed = list_stride == K;
    WarpList<int64_t> L;
    L.init();
    for (int64_t base = 0; base < count; base += 32 * C) {
        float v[C];
        int64_t id[C];
#pragma unroll
        for (int j = 0; j < C; ++j) {
            const int64_t e = base + 32 * j + lane;
            const int64_t a = packed ? e : (e / K) * list_stride + e % K;
            v[j] = e < count ? pv[a] : -INFINITY;
            id[j] = e < count ? pi[a] : INT64_MAX;
        }
#pragma unroll
        for (int j = 0; j < C; ++j) L.offer(id[j] != INT64_MAX, v[j], id[j], K, lane);
    }
    if (lane < K) {
        vals[row * K + lane] = L.v;
        ids[row * K + lane] = L.id;
    }
}

// ---- dequantization -------------------------------------------------------
// T = 2z - 1 (fp32 rows) for the rows of a chunk.  SPLIT: records of a
// fractional width (the last d/64 blocks at width B - 1).
template <int B, bool SPLIT>
__global__ void k_signs(const uint32_t* __restrict__ codes, int64_t rows, int d,
                        float* __restrict__ T) {
    constexpr int BL = B > 1 ? B - 1 : 1;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= rows * (d / 32)) return;
    const int64_t row = e / (d / 32);
    const int blk = (int)(e % (d / 32));
    const int W = SPLIT ? d / 64 * (2 * B - 1) : words_per_vector(d, B);
    const uint32_t* rec = codes + row * W;
    float* t = T + row * d + blk * 32;
    uint32_t w[4];
    int cell;
    uint32_t z;
    if (SPLIT && blk >= d / 64) {
        load_block<BL, false>(rec + (d / 64) * B, blk - d / 64, w);
        for (int j = 0; j < 32; ++j) {
            field<BL>(w, j, cell, z);
            t[j] = z ? 1.f : -1.f;
        }
    } else {
        load_block<B, !SPLIT>(rec, blk, w);
        for (int j = 0; j < 32; ++j) {
            field<B>(w, j, cell, z);
            t[j] = z ? 1.f : -1.f;
        }
    }
}

// E = c[idx] + |r| sqrt(pi/2)/d * E  (E holds S^T (2z - 1) on entry); the
// second half of a fractional-width record takes c_lo.
template <int B, bool SPLIT>
__global__ void k_combine(const uint32_t* __restrict__ codes, const float* __restrict__ rnorm,
                          int64_t rows, int d, KCodebook cb, float* __restrict__ E) {
    constexpr int BL = B > 1 ? B - 1 : 1;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= rows * (d / 32)) return;
    const int64_t row = e / (d / 32);
    const int blk = (int)(e % (d / 32));
    const int W = SPLIT ? d / 64 * (2 * B - 1) : words_per_vector(d, B);
    const uint32_t* rec = codes + row * W;
    const float kap = kSqrtHalfPi / (float)d * rnorm[row];
    float* p = E + row * d + blk * 32;
    uint32_t w[4];
    int cell;
    uint32_t z;
    if (SPLIT && blk >= d / 64) {
        load_block<BL, false>(rec + (d / 64) * B, blk - d / 64, w);
        for (int j = 0; j < 32; ++j) {
            field<BL>(w, j, cell, z);
            p[j] = ((BL == 1) ? 0.f : cb.c_lo[cell]) + kap * p[j];
        }
        return;
    }
    load_block<B, !SPLIT>(rec, blk, w);
    for (int j = 0; j < 32; ++j) {
        field<B>(w, j, cell, z);
        if (cb.mse) {  // MSE-only variant: the b-bit cell is (idx | z << (b-1)); no QJL term
            p[j] = cb.c[(B == 1) ? (int)z : (cell | (int)(z << (B - 1)))];
        } else {
            const float yh = (B == 1) ? 0.f : cb.c[cell];
            p[j] = yh + kap * p[j];
        }
    }
}

// ---- unquantized fp32 logits ---------------------------------------------
// 8 lanes per key (4 keys per warp); each lane takes every 8th float4 of the
// key, fp32 products for QC queries held in shared memory, 3-step reduction.
template <int QC, typename TQ>
__global__ __launch_bounds__(256) void k_logits_fp32(const float* __restrict__ keys, int64_t n,
                                                     int d, int nq, const TQ* __restrict__ q,
                                                     float* __restrict__ out) {
    extern __shared__ __align__(16) float s_q[];  // [QC][d]
    const int g = blockIdx.y;
    const int q0 = blockIdx.z * QC;
    const int qn = min(QC, nq - q0);
    for (int e = threadIdx.x; e < QC * d; e += blockDim.x) {
        const int qq = e / d;
        s_q[e] = (qq < qn) ? load_f32(q, ((int64_t)g * nq + q0 + qq) * d + e % d) : 0.f;
    }
    __syncthreads();
    const int lane = threadIdx.x % 32;
    const int sub = lane % 8;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    const int64_t wid = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    for (int64_t base = wid * 4; base < n; base += warps * 4) {
        const int64_t v = base + lane / 8;
        float acc[QC];
#pragma unroll
        for (int qq = 0; qq < QC; ++qq) acc[qq] = 0.f;
        if (v < n) {
            const float4* kr = reinterpret_cast<const float4*>(keys + ((int64_t)g * n + v) * d);
            for (int f = sub; f < d / 4; f += 8) {
                const float4 kv = __ldg(kr + f);
#pragma unroll
                for (int qq = 0; qq < QC; ++qq) {
                    const float4 qv = *reinterpret_cast<const float4*>(s_q + qq * d + 4 * f);
                    acc[qq] = fmaf(kv.x, qv.x, acc[qq]);
                    acc[qq] = fmaf(kv.y, qv.y, acc[qq]);
                    acc[qq] = fmaf(kv.z, qv.z, acc[qq]);
                    acc[qq] = fmaf(kv.w, qv.w, acc[qq]);
                }
            }
        }
#pragma unroll
        for (int qq = 0; qq < QC; ++qq) {
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) acc[qq] += __shfl_xor_sync(0xffffffffu, acc[qq], o);
        }
        if (v < n && sub < QC) {
#pragma unroll
            for (int qq = 0; qq < QC; ++qq)
                if (qq == sub && qq < qn) out[((int64_t)g * nq + q0 + qq) * n + v] = acc[qq];
        }
    }
}

// ---- helpers ----------------------------------------------------------------

template <int B, int NQ, bool F2, bool SPLIT>
int launch_score2_t(const uint32_t* codes, const float* xn, const float* rn, int64_t n, int d,
                    int G, int nq, const float* qr, const float* u, const KCodebook& kc,
                    float* scores, float* cmax, int* zero_cnt, cudaStream_t s) {
    constexpr int KP = 2;
    static_assert(128 * KP == kTopkTile, "one score block per top-k chunk");
    const size_t smem = (size_t)NQ * d * sizeof(float2);
    TQ_TRY_CUDA(cudaFuncSetAttribute(k_score2<B, NQ, KP, F2, SPLIT>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    const int nchunks = (int)((n + 128 * KP - 1) / (128 * KP));
    dim3 grid((unsigned)nchunks, (unsigned)G, (unsigned)((nq + NQ - 1) / NQ));
    k_score2<B, NQ, KP, F2, SPLIT><<<grid, 128, smem, s>>>(codes, xn, rn, n, d, nq, qr, u, kc,
                                                           scores, cmax, nchunks, zero_cnt);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

// Queries per pass: as many as the group has, up to what shared memory holds.
int score_nq(int d, int nq) {
    const int cap = d <= 1536 ? 8 : (d <= 3072 ? 4 : 2);
    int p = 1;
    while (p < nq && p < cap) p <<= 1;
    return p;
}

template <int B>
int launch_score_b(const uint32_t* codes, const float* xn, const float* rn, int64_t n, int d,
                   int G, int nq, const float* qr, const float* u, const KCodebook& kc,
                   float* scores, float* cmax, int* zero_cnt, cudaStream_t s) {
#define TQ_SC(NQV)                                                                              \
    return (B >= 2 && kc.split)                                                                 \
               ? launch_score2_t<B, NQV, true, (B >= 2)>(codes, xn, rn, n, d, G, nq, qr, u, kc, \
                                                         scores, cmax, zero_cnt, s)             \
               : launch_score2_t<B, NQV, true, false>(codes, xn, rn, n, d, G, nq, qr, u, kc,    \
                                                      scores, cmax, zero_cnt, s)
    switch (score_nq(d, nq)) {
        case 1: TQ_SC(1);
        case 2: TQ_SC(2);
        case 4: TQ_SC(4);
        default: TQ_SC(8);
    }
#undef TQ_SC
}

// Key ranges per (group, query pass) for k_score_topk: enough blocks for one
// full wave of the device, each range a whole number of kCandTile passes.
struct TopkGrid {
    int nblk;
    int64_t span;
};

template <int B, int NQ, bool F2, bool SPLIT>
int launch_topk_t(const uint32_t* codes, const float* xn, const float* rn, int64_t n, int d,
                  int G, int nq, const float* qr, const float* u, const KCodebook& kc, int K,
                  float* pv, int64_t* pi, TopkGrid* out, cudaStream_t s) {
    const size_t smem = (size_t)NQ * d * sizeof(float2);
    auto kern = k_score_topk<B, NQ, F2, SPLIT>;
    TQ_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    int dev = 0, nsm = 0, occ = 0;
    TQ_TRY_CUDA(cudaGetDevice(&dev));
    TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    TQ_TRY_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 256, smem));
    const int npass = (nq + NQ - 1) / NQ;
    const int64_t passes = (n + kCandTile - 1) / kCandTile;  // kCandTile-key passes per group
    int64_t want = (int64_t)nsm * (occ > 0 ? occ : 1) / ((int64_t)G * npass);
    want = want < 1 ? 1 : (want > passes ? passes : want);
    const int64_t per = (passes + want - 1) / want;  // passes per block
    TopkGrid tg;
    tg.span = per * kCandTile;
    tg.nblk = (int)((n + tg.span - 1) / tg.span);
    *out = tg;
    dim3 grid((unsigned)tg.nblk, (unsigned)G, (unsigned)npass);
    kern<<<grid, 256, smem, s>>>(codes, xn, rn, n, d, nq, qr, u, kc, K, tg.nblk, tg.span, pv, pi);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

template <int B>
int launch_topk_b(const uint32_t* codes, const float* xn, const float* rn, int64_t n, int d,
                  int G, int nq, const float* qr, const float* u, const KCodebook& kc, int K,
                  float* pv, int64_t* pi, TopkGrid* tg, cudaStream_t s) {
#define TQ_TK(NQV)                                                                         \
    return (B >= 2 && kc.split)                                                            \
               ? launch_topk_t<B, NQV, true, (B >= 2)>(codes, xn, rn, n, d, G, nq, qr, u, kc, \
                                                       K, pv, pi, tg, s)                    \
               : launch_topk_t<B, NQV, true, false>(codes, xn, rn, n, d, G, nq, qr, u, kc, K, \
                                                    pv, pi, tg, s)
    switch (score_nq(d, nq)) {
        case 1: TQ_TK(1);
        case 2: TQ_TK(2);
        case 4: TQ_TK(4);
        default: TQ_TK(8);
    }
#undef TQ_TK
}

// qr = Pi_g q and u = S_g qr for one (query, group) per block: one warp per
// output row (coalesced row reads, shuffle reduction), qr kept in shared
// memory for the second product.  Used when there are few queries per group.
template <typename TQ>
__global__ __launch_bounds__(512) void k_query_prep(const float* __restrict__ Pi,
                                                    const float* __restrict__ S, int d, int nq,
                                                    const TQ* __restrict__ q,
                                                    float* __restrict__ qr,
                                                    float* __restrict__ u, int* err) {
    // the call's device status word starts clean (the scoring kernels after
    // this one on the stream may record a time-out in it)
    if (err && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *err = 0;
    extern __shared__ __align__(16) float sq[];  // [0, d): q   [d, 2d): qr
    constexpr int R = 8;  // rows per warp in flight
    const int g = blockIdx.y;
    // S of the group toward L2 while Pi q is formed (the second product then
    // reads it from L2), by one block of the group, for d <= 256
    if (S && blockIdx.x == 0 && d <= 256) {
        const char* sg = reinterpret_cast<const char*>(S + (size_t)g * d * d);
        for (int e = threadIdx.x; e * 128 < d * d * 4; e += blockDim.x)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(sg + (size_t)e * 128));
    }
    const int64_t row = (int64_t)g * nq + blockIdx.x;
    for (int j = threadIdx.x; j < d; j += blockDim.x) sq[j] = load_f32(q, row * d + j);
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        float* outg = (pass == 0 ? qr : u) + row * d;
        if (pass == 1 && !S) {  // MSE-only variant: no QJL vector
            for (int j = threadIdx.x; j < d; j += blockDim.x) outg[j] = 0.f;
            break;
        }
        const float* M = (pass == 0 ? Pi : S) + (size_t)g * d * d;
        const float* v = sq + pass * d;
        for (int i0 = warp * R; i0 < d; i0 += nw * R) {
            float acc[R];
#pragma unroll
            for (int r = 0; r < R; ++r) acc[r] = 0.f;
            for (int f = lane; f < d / 4; f += 32) {
                const float4 b = *reinterpret_cast<const float4*>(v + 4 * f);
                float4 a[R];
#pragma unroll
                for (int r = 0; r < R; ++r)
                    a[r] = __ldg(reinterpret_cast<const float4*>(M + (size_t)(i0 + r) * d) + f);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    acc[r] = fmaf(a[r].x, b.x, acc[r]);
                    acc[r] = fmaf(a[r].y, b.y, acc[r]);
                    acc[r] = fmaf(a[r].z, b.z, acc[r]);
                    acc[r] = fmaf(a[r].w, b.w, acc[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
            }
            if (lane < R) {
                float a = acc[0];
#pragma unroll
                for (int r = 1; r < R; ++r) a = (lane == r) ? acc[r] : a;
                outg[i0 + lane] = a;
                if (pass == 0) sq[d + i0 + lane] = a;
            }
        }
        __syncthreads();
    }
}

}  // namespace

// qr = Q Pi^T, u = qr S^T for every group: one fused launch for few queries,
// else two fp32 SIMT GEMMs per group.
int query_prep(const float* d_Pi, const float* d_S, int G, int d, int nq, const void* d_q,
               int q_dtype, float* qr, float* u, int* err, cudaStream_t s) {
    const size_t dd = (size_t)d * d;
    const size_t esz = (q_dtype == TQ_F32) ? 4 : 2;
    if (nq <= 32) {
        dim3 grid((unsigned)nq, (unsigned)G);
        const size_t smem = (size_t)2 * d * sizeof(float);
        if (q_dtype == TQ_F32) {
            TQ_TRY_CUDA(cudaFuncSetAttribute(k_query_prep<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
            k_query_prep<float><<<grid, 512, smem, s>>>(d_Pi, d_S, d, nq, (const float*)d_q, qr, u,
                                                        err);
        } else {
            TQ_TRY_CUDA(cudaFuncSetAttribute(k_query_prep<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
            k_query_prep<__nv_bfloat16><<<grid, 512, smem, s>>>(
                d_Pi, d_S, d, nq, (const __nv_bfloat16*)d_q, qr, u, err);
        }
        TQ_CHECK_LAUNCH();
        return TQ_OK;
    }
    if (err) TQ_TRY_CUDA(cudaMemsetAsync(err, 0, sizeof(int), s));
    for (int g = 0; g < G; ++g) {
        const void* qg = (const char*)d_q + (size_t)g * nq * d * esz;
        int rc = launch_sgemm(nq, d, d, qg, q_dtype, d, d_Pi + g * dd, true, d,
                              qr + (size_t)g * nq * d, d, nullptr, 0, s);
        if (rc) return rc;
        if (!d_S) {  // MSE-only variant: no QJL vector
            TQ_TRY_CUDA(cudaMemsetAsync(u + (size_t)g * nq * d, 0, (size_t)nq * d * 4, s));
            continue;
        }
        rc = launch_sgemm(nq, d, d, qr + (size_t)g * nq * d, TQ_F32, d, d_S + g * dd, true, d,
                          u + (size_t)g * nq * d, d, nullptr, 0, s);
        if (rc) return rc;
    }
    return TQ_OK;
}

int check_common(const tq_codebook_t* cb, int G, int64_t n, int nq, int q_dtype) {
    if (!cb || G < 1 || n < 0 || nq < 0) return TQ_ERR_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_ARG;
    if (!valid_db(cb->d, cb->b)) return TQ_ERR_UNSUPPORTED;
    if (cb->groups < G) return TQ_ERR_MISMATCH;
    return TQ_OK;
}

}  // namespace tq

using namespace tq;

extern "C" int tq_score(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G,
                        int64_t n, const uint32_t* d_codes, const float* d_xnorm,
                        const float* d_rnorm, int nq, const void* d_q, int q_dtype,
                        float* d_scores, void* d_ws, size_t ws_bytes, void* stream) {
    int rc = check_common(cb, G, n, nq, q_dtype);
    if (rc) return rc;
    if (n == 0 || nq == 0) return TQ_OK;
    if (!d_Pi || (!is_mse(cb) && !d_S) || !d_codes || !d_xnorm || !d_rnorm || !d_q || !d_scores)
        return TQ_ERR_ARG;
    if (is_mse(cb)) d_S = nullptr;
    const int d = cb->d, b = cb->b;
    if (!d_ws || ws_bytes < tq_workspace_bytes(TQ_OP_SCORE, d, b, G, n, nq, 0))
        return TQ_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    // [status word (256 B) | qr | u]
    int* err = (int*)d_ws;
    float* qr = (float*)((char*)d_ws + 256);
    float* u = (float*)((char*)qr + align256((size_t)G * nq * d * 4));
    rc = query_prep(d_Pi, d_S, G, d, nq, d_q, q_dtype, qr, u, err, s);
    if (rc) return rc;
    if (!is_split(cb) && score_gemm_supported(d, nq)) {  // many queries at d >= 256: decoded-key GEMM
        void* op = (char*)u + align256((size_t)G * nq * d * 4);
        return score_gemm(cb, G, n, d_codes, d_xnorm, d_rnorm, nq, qr, u, d_scores, nullptr, 0,
                          op, err, s);
    }
    if (score_i8_supported(cb, G, n, nq, d_codes))
        return launch_score_i8(cb, G, n, d_codes, d_xnorm, d_rnorm, nq, qr, u, d_scores, nullptr,
                               nullptr, err, s);
    if (!is_mse(cb) && !is_split(cb) && score_tc_supported(d, b, G, n, nq))
        return launch_score_tc(cb, G, n, d_codes, d_xnorm, d_rnorm, nq, qr, u, d_scores, nullptr,
                               nullptr, err, s);
    const KCodebook kc = make_kcodebook(cb);
    switch (b) {
        case 1: return launch_score_b<1>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, d_scores, nullptr, nullptr, s);
        case 2: return launch_score_b<2>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, d_scores, nullptr, nullptr, s);
        case 3: return launch_score_b<3>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, d_scores, nullptr, nullptr, s);
        default: return launch_score_b<4>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, d_scores, nullptr, nullptr, s);
    }
}

namespace tq {
// Blocks per score row of k_topk_collect: 16 scores per thread (one pass of
// loads), at least enough blocks for every SM; when that would take more than
// one wave of resident blocks (4 per SM), as many as one wave holds, each
// thread then taking several passes (the per-block threshold and the
// last-block selection are latency chains, paid once per wave).
static int64_t collect_blocks_per_row(int64_t n, int64_t rows, int nsm) {
    int64_t P = (n + 256 * 16 - 1) / (256 * 16);
    const int64_t pmin = ((int64_t)nsm + rows - 1) / rows;
    const int64_t pmax = (n + 255) / 256;
    const int64_t wave = 4 * (int64_t)nsm / rows;
    if (rows * P > 4 * (int64_t)nsm) P = wave;
    P = P < pmin ? pmin : P;
    P = P > pmax ? pmax : P;
    return P < 1 ? 1 : P;
}

int topk_run(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G, int64_t n,
             const uint32_t* d_codes, const float* d_xnorm, const float* d_rnorm, int nq,
             const void* d_q, int q_dtype, int k, float* d_vals, int64_t* d_ids, void* d_ws,
             size_t ws_bytes, bool materialize, cudaStream_t s, float* scores_out) {
    const int d = cb->d, b = cb->b;
    if (scores_out) materialize = true;
    if (!d_ws ||
        ws_bytes < topk_workspace_bytes(d, b, G, n, nq, k, materialize, scores_out == nullptr))
        return TQ_ERR_WORKSPACE;
    int rc;
    const int ntiles = (int)((n + kTopkTile - 1) / kTopkTile);
    // [status word (256 B) | qr | u | path-specific]
    int* err = (int*)d_ws;
    char* p = (char*)d_ws + 256;
    float* qr = (float*)p;
    p += align256((size_t)G * nq * d * 4);
    float* u = (float*)p;
    p += align256((size_t)G * nq * d * 4);
    rc = query_prep(d_Pi, is_mse(cb) ? nullptr : d_S, G, d, nq, d_q, q_dtype, qr, u, err, s);
    if (rc) return rc;
    const KCodebook kc = make_kcodebook(cb);
    const int64_t rows = (int64_t)G * nq;
    if (materialize) {
        // scores [G][nq][n], row maxima per chunk, counters, candidates; then
        // the per-row selection
        const bool tc = !is_mse(cb) && !is_split(cb) && score_tc_supported(d, b, G, n, nq);
        const int64_t ntm = (n + 127) / 128;
        float* sc = scores_out;  // the caller's score output, else the workspace
        if (!sc) {
            sc = (float*)p;
            p += align256((size_t)rows * n * 4);
        }
        float* cm = (float*)p;
        p += align256((size_t)rows * ntm * 4);
        int* cnt = (int*)p;  // [2][rows]: candidate counts, finished blocks
        p += align256((size_t)rows * 2 * 4);
        float* cv = (float*)p;
        p += align256((size_t)rows * kCandCapG * 4);
        int* ci = (int*)p;
        int nchunks;
        if (!is_split(cb) && score_gemm_supported(d, nq)) {  // decoded-key GEMM, maxima per 128-key tile
            p = (char*)ci + align256((size_t)rows * kCandCapG * 4);
            TQ_TRY_CUDA(cudaMemsetAsync(cnt, 0, (size_t)rows * 2 * 4, s));
            rc = score_gemm(cb, G, n, d_codes, d_xnorm, d_rnorm, nq, qr, u, sc, cm, ntm, p, err, s);
            nchunks = (int)ntm;
        } else if (score_i8_supported(cb, G, n, nq, d_codes)) {  // maxima per 128-key tile
            rc = launch_score_i8(cb, G, n, d_codes, d_xnorm, d_rnorm, nq, qr, u, sc, cm, cnt, err,
                                 s);
            nchunks = (int)ntm;
        } else if (tc) {  // maxima per 128-key tile
            rc = launch_score_tc(cb, G, n, d_codes, d_xnorm, d_rnorm, nq, qr, u, sc, cm, cnt, err,
                                 s);
            nchunks = (int)ntm;
        } else {  // maxima per 256-key block
            switch (b) {
                case 1: rc = launch_score_b<1>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, sc, cm, cnt, s); break;
                case 2: rc = launch_score_b<2>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, sc, cm, cnt, s); break;
                case 3: rc = launch_score_b<3>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, sc, cm, cnt, s); break;
                default: rc = launch_score_b<4>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, sc, cm, cnt, s); break;
            }
            nchunks = ntiles;
        }
        if (rc) return rc;
        int nsm = 0, dev = 0;
        TQ_TRY_CUDA(cudaGetDevice(&dev));
        TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
        // blocks per row: 16 scores per thread (one pass of loads), more when
        // the rows alone would leave most SMs idle
        dim3 grid((unsigned)collect_blocks_per_row(n, rows, nsm), (unsigned)rows);
        k_topk_collect<<<grid, 256, 0, s>>>(sc, cm, n, nchunks, k, cnt, cnt + rows, cv, ci, d_vals,
                                            d_ids, 0);
        TQ_CHECK_LAUNCH();
        return TQ_OK;
    }
    if (score_i8_supported(cb, G, n, nq, d_codes)) {
        // too many scores to hold at once: the same integer tensor-core scores
        // (so the lists equal tq_score_topk's) over chunks of keys sized to the
        // workspace, each chunk's top-k, then the merge of the chunks' lists
        const size_t avail = ws_bytes - (size_t)(p - (char*)d_ws);
        int64_t nc = 0, nch = 0;
        for (int64_t m = 1;; ++m) {
            const int64_t c = ((n + m - 1) / m + 127) / 128 * 128;
            const int64_t h = (n + c - 1) / c;
            const size_t need = align256((size_t)rows * c * 4) + align256((size_t)rows * (c / 128) * 4) +
                                align256((size_t)rows * 2 * 4) + 2 * align256((size_t)rows * kCandCapG * 4) +
                                align256((size_t)h * rows * k * 4) + align256((size_t)h * rows * k * 8);
            if (need <= avail) {
                nc = c;
                nch = h;
                break;
            }
            if (c <= 128) break;
        }
        if (nc > 0) {
            float* sc = (float*)p;
            p += align256((size_t)rows * nc * 4);
            float* cm = (float*)p;
            p += align256((size_t)rows * (nc / 128) * 4);
            int* cnt = (int*)p;
            p += align256((size_t)rows * 2 * 4);
            float* cv = (float*)p;
            p += align256((size_t)rows * kCandCapG * 4);
            int* ci = (int*)p;
            p += align256((size_t)rows * kCandCapG * 4);
            float* pv = (float*)p;
            p += align256((size_t)nch * rows * k * 4);
            int64_t* pi = (int64_t*)p;
            int nsm = 0, dev = 0;
            TQ_TRY_CUDA(cudaGetDevice(&dev));
            TQ_TRY_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
            for (int64_t h = 0; h < nch; ++h) {
                const int64_t k0 = h * nc;
                const int64_t len = (n - k0) < nc ? (n - k0) : nc;
                rc = launch_score_i8(cb, G, len, d_codes, d_xnorm, d_rnorm, nq, qr, u, sc, cm, cnt,
                                     err, s, n, k0);
                if (rc) return rc;
                dim3 grid((unsigned)collect_blocks_per_row(len, rows, nsm), (unsigned)rows);
                k_topk_collect<<<grid, 256, 0, s>>>(sc, cm, len, (int)((len + 127) / 128), k, cnt,
                                                    cnt + rows, cv, ci, pv + h * rows * k,
                                                    pi + h * rows * k, k0);
                TQ_CHECK_LAUNCH();
            }
            k_topk_merge<<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(pv, pi, rows, (int)nch, k, d_vals,
                                                                     d_ids, k, rows * k);
            TQ_CHECK_LAUNCH();
            return TQ_OK;
        }
    }
    // fused: per-range best-K lists [G][nq][nblk][K], then the merge
    float* pv = (float*)p;
    p += align256((size_t)rows * ntiles * k * 4);
    int64_t* pi = (int64_t*)p;
    TopkGrid tg;
    switch (b) {
        case 1: rc = launch_topk_b<1>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, k, pv, pi, &tg, s); break;
        case 2: rc = launch_topk_b<2>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, k, pv, pi, &tg, s); break;
        case 3: rc = launch_topk_b<3>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, k, pv, pi, &tg, s); break;
        default: rc = launch_topk_b<4>(d_codes, d_xnorm, d_rnorm, n, d, G, nq, qr, u, kc, k, pv, pi, &tg, s); break;
    }
    if (rc) return rc;
    k_topk_merge<<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(pv, pi, rows, tg.nblk, k, d_vals, d_ids,
                                                             (int64_t)tg.nblk * k, k);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}
}  // namespace tq

namespace tq {
int topk_validate(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G, int64_t n,
                  const uint32_t* d_codes, const float* d_xnorm, const float* d_rnorm, int nq,
                  const void* d_q, int q_dtype, int k, const float* d_vals,
                  const int64_t* d_ids) {
    int rc = check_common(cb, G, n, nq, q_dtype);
    if (rc) return rc;
    if (k < 1 || k > kMaxK || (int64_t)k > n) return (n == 0 && nq == 0) ? kTopkNothing : TQ_ERR_ARG;
    if (nq == 0) return kTopkNothing;
    if (!d_Pi || (!is_mse(cb) && !d_S) || !d_codes || !d_xnorm || !d_rnorm || !d_q || !d_vals ||
        !d_ids)
        return TQ_ERR_ARG;
    return TQ_OK;
}
}  // namespace tq

extern "C" int tq_topk(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G,
                       int64_t n, const uint32_t* d_codes, const float* d_xnorm,
                       const float* d_rnorm, int nq, const void* d_q, int q_dtype, int k,
                       float* d_vals, int64_t* d_ids, void* d_ws, size_t ws_bytes,
                       void* stream) {
    const int rc = topk_validate(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype,
                                 k, d_vals, d_ids);
    if (rc) return rc == kTopkNothing ? TQ_OK : rc;
    return topk_run(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype, k, d_vals,
                    d_ids, d_ws, ws_bytes, topk_materialized(cb->d, G, n, nq), (cudaStream_t)stream);
}

extern "C" int tq_score_topk(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G,
                             int64_t n, const uint32_t* d_codes, const float* d_xnorm,
                             const float* d_rnorm, int nq, const void* d_q, int q_dtype, int k,
                             float* d_scores, float* d_vals, int64_t* d_ids, void* d_ws,
                             size_t ws_bytes, void* stream) {
    const int rc = topk_validate(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype,
                                 k, d_vals, d_ids);
    if (rc) return rc == kTopkNothing ? TQ_OK : rc;
    if (!d_scores) return TQ_ERR_ARG;
    return topk_run(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype, k, d_vals,
                    d_ids, d_ws, ws_bytes, true, (cudaStream_t)stream, d_scores);
}

extern "C" int tq_decode(const tq_codebook_t* cb, const float* d_Pi, const float* d_S, int G,
                         int64_t n, const uint32_t* d_codes, const float* d_xnorm,
                         const float* d_rnorm, float* d_xhat, void* d_ws, size_t ws_bytes,
                         void* stream) {
    int rc = check_common(cb, G, n, 0, TQ_F32);
    if (rc) return rc;
    if (n == 0) return TQ_OK;
    const bool mse = is_mse(cb);
    if (!d_Pi || (!mse && !d_S) || !d_codes || !d_xnorm || !d_rnorm || !d_xhat) return TQ_ERR_ARG;
    const int d = cb->d, b = cb->b;
    if (!d_ws || ws_bytes < tq_workspace_bytes(TQ_OP_DECODE, d, b, G, n, 0, 0))
        return TQ_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const KCodebook kc = make_kcodebook(cb);
    const int64_t chunk = n < kEncodeChunk ? n : kEncodeChunk;
    float* T = (float*)d_ws;
    float* E = (float*)((char*)d_ws + align256((size_t)chunk * d * 4));
    const int W = record_words(cb);
    const bool split = is_split(cb);
    const size_t dd = (size_t)d * d;
    for (int g = 0; g < G; ++g) {
        for (int64_t r0 = 0; r0 < n; r0 += chunk) {
            const int64_t rows = (n - r0) < chunk ? (n - r0) : chunk;
            const int64_t off = (int64_t)g * n + r0;
            const uint32_t* cg = d_codes + off * W;
            const unsigned blocks = (unsigned)((rows * (d / 32) + 255) / 256);
            if (!mse) {
                if (split) {
                    switch (b) {
                        case 2: k_signs<2, true><<<blocks, 256, 0, s>>>(cg, rows, d, T); break;
                        case 3: k_signs<3, true><<<blocks, 256, 0, s>>>(cg, rows, d, T); break;
                        default: k_signs<4, true><<<blocks, 256, 0, s>>>(cg, rows, d, T); break;
                    }
                } else {
                    switch (b) {
                        case 1: k_signs<1, false><<<blocks, 256, 0, s>>>(cg, rows, d, T); break;
                        case 2: k_signs<2, false><<<blocks, 256, 0, s>>>(cg, rows, d, T); break;
                        case 3: k_signs<3, false><<<blocks, 256, 0, s>>>(cg, rows, d, T); break;
                        default: k_signs<4, false><<<blocks, 256, 0, s>>>(cg, rows, d, T); break;
                    }
                }
                TQ_CHECK_LAUNCH();
                // E = T S   (E[v][j] = sum_i T[v][i] S[i][j])
                rc = launch_sgemm((int)rows, d, d, T, TQ_F32, d, d_S + g * dd, false, d, E, d,
                                  nullptr, 0, s);
                if (rc) return rc;
            }
            if (split) {
                switch (b) {
                    case 2: k_combine<2, true><<<blocks, 256, 0, s>>>(cg, d_rnorm + off, rows, d, kc, E); break;
                    case 3: k_combine<3, true><<<blocks, 256, 0, s>>>(cg, d_rnorm + off, rows, d, kc, E); break;
                    default: k_combine<4, true><<<blocks, 256, 0, s>>>(cg, d_rnorm + off, rows, d, kc, E); break;
                }
            } else {
                switch (b) {
                    case 1: k_combine<1, false><<<blocks, 256, 0, s>>>(cg, d_rnorm + off, rows, d, kc, E); break;
                    case 2: k_combine<2, false><<<blocks, 256, 0, s>>>(cg, d_rnorm + off, rows, d, kc, E); break;
                    case 3: k_combine<3, false><<<blocks, 256, 0, s>>>(cg, d_rnorm + off, rows, d, kc, E); break;
                    default: k_combine<4, false><<<blocks, 256, 0, s>>>(cg, d_rnorm + off, rows, d, kc, E); break;
                }
            }
            TQ_CHECK_LAUNCH();
            // xhat = |x| E Pi   (xhat[v][j] = |x_v| sum_i E[v][i] Pi[i][j])
            rc = launch_sgemm((int)rows, d, d, E, TQ_F32, d, d_Pi + g * dd, false, d,
                              d_xhat + (size_t)off * d, d, d_xnorm + off, 2, s);
            if (rc) return rc;
        }
    }
    return TQ_OK;
}

template <typename TQ>
static int launch_logits(const float* keys, int64_t n, int d, int G, int nq, const TQ* q,
                         float* out, cudaStream_t s) {
    const int QC = nq >= 8 ? 8 : (nq >= 4 ? 4 : (nq >= 2 ? 2 : 1));
    const size_t smem = (size_t)QC * d * 4;
    const unsigned bx = (unsigned)std::min<int64_t>((n + 31) / 32, 148 * 16);
    dim3 grid(bx, (unsigned)G, (unsigned)((nq + QC - 1) / QC));
#define TQ_LG(QCV)                                                                           \
    do {                                                                                     \
        TQ_TRY_CUDA(cudaFuncSetAttribute(k_logits_fp32<QCV, TQ>,                             \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                                         (int)smem));                                        \
        k_logits_fp32<QCV, TQ><<<grid, 256, smem, s>>>(keys, n, d, nq, q, out);              \
    } while (0)
    switch (QC) {
        case 8: TQ_LG(8); break;
        case 4: TQ_LG(4); break;
        case 2: TQ_LG(2); break;
        default: TQ_LG(1); break;
    }
#undef TQ_LG
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

extern "C" int tq_logits_fp32(int d, int G, int64_t n, const float* d_keys, int nq,
                              const void* d_q, int q_dtype, float* d_out, void* stream) {
    if (G < 1 || n < 0 || nq < 0) return TQ_ERR_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_ARG;
    if (d < kMinD || d > kMaxD || d % 128) return TQ_ERR_UNSUPPORTED;
    if (n == 0 || nq == 0) return TQ_OK;
    if (!d_keys || !d_q || !d_out) return TQ_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (q_dtype == TQ_F32) return launch_logits<float>(d_keys, n, d, G, nq, (const float*)d_q, d_out, s);
    return launch_logits<__nv_bfloat16>(d_keys, n, d, G, nq, (const __nv_bfloat16*)d_q, d_out, s);
}

extern "C" int tq_exact_topk(int d, int G, int64_t n, const float* d_x, int nq, const void* d_q,
                             int q_dtype, int k, float* d_vals, int64_t* d_ids, void* d_ws,
                             size_t ws_bytes, void* stream) {
    if (G < 1 || n < 0 || nq < 0) return TQ_ERR_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_ARG;
    if (d < kMinD || d > kMaxD || d % 128) return TQ_ERR_UNSUPPORTED;
    if (nq == 0) return TQ_OK;
    if (k < 1 || k > kMaxK || (int64_t)k > n) return TQ_ERR_ARG;
    if (!d_x || !d_q || !d_vals || !d_ids) return TQ_ERR_ARG;
    if (!d_ws || ws_bytes < tq_workspace_bytes(TQ_OP_EXACT, d, 1, G, n, nq, k))
        return TQ_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const int ntiles = (int)((n + kTopkTile - 1) / kTopkTile);
    const int64_t chunk = n < kEncodeChunk ? n : kEncodeChunk;  // multiple of kTopkTile
    char* p = (char*)d_ws;
    float* sc = (float*)p;
    p += align256((size_t)nq * ((chunk + 3) & ~int64_t(3)) * 4);
    float* pv = (float*)p;
    p += align256((size_t)G * nq * ntiles * k * 4);
    int64_t* pi = (int64_t*)p;
    const size_t esz = (q_dtype == TQ_F32) ? 4 : 2;
    for (int g = 0; g < G; ++g) {
        const void* qg = (const char*)d_q + (size_t)g * nq * d * esz;
        for (int64_t c0 = 0; c0 < n; c0 += chunk) {
            const int64_t cols = (n - c0) < chunk ? (n - c0) : chunk;
            const int64_t ld = (cols + 3) & ~int64_t(3);
            int rc = launch_sgemm(nq, (int)cols, d, qg, q_dtype, d, d_x + ((size_t)g * n + c0) * d,
                                  true, d, sc, (int)ld, nullptr, 0, s);
            if (rc) return rc;
            const int tiles = (int)((cols + kTopkTile - 1) / kTopkTile);
            dim3 grid((unsigned)tiles, (unsigned)nq);
            k_rows_topk_tile<<<grid, 256, 0, s>>>(sc, ld, cols, c0, k, ntiles,
                                                  (int)(c0 / kTopkTile),
                                                  pv + (size_t)g * nq * ntiles * k,
                                                  pi + (size_t)g * nq * ntiles * k);
            TQ_CHECK_LAUNCH();
        }
    }
    const int64_t rows = (int64_t)G * nq;
    k_topk_merge<<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(pv, pi, rows, ntiles, k, d_vals, d_ids,
                                                             (int64_t)ntiles * k, k);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

// Merge of top-k lists computed on shards of a database (on one GPU or on
// several, gathered): every list already holds global ids.
extern "C" int tq_topk_merge(int64_t rows, int nlists, int k, const float* d_vals,
                             const int64_t* d_ids, float* d_out_vals, int64_t* d_out_ids,
                             void* stream) {
    if (rows < 0 || nlists < 1 || k < 1 || k > kMaxK) return TQ_ERR_ARG;
    if (rows == 0) return TQ_OK;
    if (!d_vals || !d_ids || !d_out_vals || !d_out_ids) return TQ_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    k_topk_merge<<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(d_vals, d_ids, rows, nlists, k,
                                                             d_out_vals, d_out_ids, k, rows * k);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

