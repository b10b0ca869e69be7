// Decode attention over quantized keys and values (d = 128): for every query
// row t of a group,
//   l_j = scale * s_tj,   s_tj = |x_j| ( <qr_t, c[idx_j]> + |r_j| sqrt(pi/2)/d <u_t, 2z_j - 1> )
//   out_t = sum_j softmax(l)_j v^_j,   v^_j = |v_j| Pi_v^T c_v[cell_j]
// with keys in the inner-product records (tq_encode, prod) and values in the
// MSE-only records (tq_encode, mse) of their own codebook.
//
// Pages: quant_prune_distill #674 (inner-product estimate from the codes;
// dequantization = inverse rotation and renormalisation); comuna.ru "Google
// speeds up LLMs 8x" (attention logits from 4-bit keys).  The softmax and the
// value sum are the standard attention those logits feed (the pages do not
// describe this step).
//
// Design: the logits come from tq_score itself (its scoring kernels for the
// group's query count) into the workspace; then split-K over the keys of a
// group (flash-decoding).  A block takes `split` keys in tiles of 256, keeps a
// running maximum and sum per query, and
// accumulates sum_j p_j |v_j| c_v[cell_j] in the rotated value domain: thread
// (coordinate pair, quarter of the tile) walks the tile's value records staged
// in shared memory and updates both coordinates with packed fp32x2 FMAs (at
// b_v = 4 one byte-indexed table load gives both centroids).  Because Pi_v^T
// is linear it is applied once per query, after the splits are merged
// (k_attn_combine), instead of once per value.
#include <cmath>

#include "tq_internal.cuh"
#include "tq_score_common.cuh"

namespace tq {
namespace {

using sc::ffma2;

constexpr int kAD = 128;         // head dimension
constexpr int kAT = 256;         // keys per tile = threads per block
constexpr int kAttnSplitMax = 4096;

// Value cell of coordinate j (0..31) of a block of the MSE-only layout (the
// index's top bit sits in the z position): the b-bit Lloyd-Max cell.
template <int BV>
__device__ __forceinline__ uint32_t value_cell(const uint32_t* blk, int j) {
    if (BV == 4) return (blk[j >> 3] >> (4 * (j & 7))) & 15u;
    if (BV == 3) return ((blk[j >> 4] >> (2 * (j & 15))) & 3u) | (((blk[2] >> j) & 1u) << 2);
    if (BV == 2) return (blk[j >> 4] >> (2 * (j & 15))) & 3u;
    return (blk[0] >> j) & 1u;
}

template <int BV, int NQ>
__global__ __launch_bounds__(kAT, 8) void k_attn_partial(
    const float* __restrict__ logits, const uint32_t* __restrict__ vcodes,
    const float* __restrict__ vxn, int64_t n, int nq, KCodebook vcb, float scale, int split,
    float* __restrict__ part_m, float* __restrict__ part_l, float* __restrict__ part_acc) {
    constexpr int WV = BV * kAD / 32;
    __shared__ float s_vc[16];
    __shared__ float2 s_vpair[256];  // b_v = 4: code byte -> (c_v[low nibble], c_v[high nibble])
    __shared__ uint32_t s_vcodes[kAT * WV];
    __shared__ __align__(16) float s_w[kAT][NQ];
    __shared__ float s_red[kAT / 32][NQ];
    __shared__ float2 s_part[3][NQ][kAD / 2];
    const int g = blockIdx.y, sp = blockIdx.x, nsplit = gridDim.x;
    const int q0 = blockIdx.z * NQ;
    const int qn = min(NQ, nq - q0);
    const int t = threadIdx.x, lane = t % 32, warp = t / 32;
    if (t < 16) {
        float c = 0.f;
        switch (t) {  // static indices keep the codebook in parameter space
#define TQ_VC(F) case F: c = vcb.c[F]; break;
            TQ_VC(0) TQ_VC(1) TQ_VC(2) TQ_VC(3) TQ_VC(4) TQ_VC(5) TQ_VC(6) TQ_VC(7)
            TQ_VC(8) TQ_VC(9) TQ_VC(10) TQ_VC(11) TQ_VC(12) TQ_VC(13) TQ_VC(14) TQ_VC(15)
#undef TQ_VC
        }
        s_vc[t] = c;
    }
    __syncthreads();
    if (BV == 4) s_vpair[t] = make_float2(s_vc[t & 15], s_vc[t >> 4]);

    const int64_t r_beg = (int64_t)sp * split;
    const int64_t r_end = min(n, r_beg + split);
    // value phase: coordinates 2 cp, 2 cp + 1 over quarter hq of every tile
    const int cp = t % (kAD / 2), hq = t / (kAD / 2);
    const int vblk = (2 * cp) / 32, vj = (2 * cp) % 32;
    float M[NQ], L[NQ];
    float2 accv[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        M[q] = -INFINITY;
        L[q] = 0.f;
        accv[q] = make_float2(0.f, 0.f);
    }
    for (int64_t r = r_beg; r < r_end; r += kAT) {
        const int cnt = (int)min((int64_t)kAT, r_end - r);
        const int64_t j = r + t;
        const bool ok = t < cnt;
        const int64_t gj = (int64_t)g * n + (ok ? j : r);
        // scaled logits of this thread's key
        float l[NQ];
#pragma unroll
        for (int q = 0; q < NQ; ++q)
            l[q] = (ok && q < qn) ? scale * logits[((int64_t)g * nq + q0 + q) * n + j] : -INFINITY;
        // the tile's value records, staged whole (coalesced)
        const uint32_t* vsrc = vcodes + ((int64_t)g * n + r) * WV;
        for (int e = t; e < cnt * WV; e += kAT) s_vcodes[e] = vsrc[e];
        const float vx = ok ? vxn[gj] : 0.f;
        // running maximum per query
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            float m = l[q];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) s_red[warp][q] = m;
        }
        __syncthreads();
        float alpha[NQ], p[NQ];
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            float mt = s_red[0][q];
#pragma unroll
            for (int w = 1; w < kAT / 32; ++w) mt = fmaxf(mt, s_red[w][q]);
            const float mn = fmaxf(M[q], mt);
            alpha[q] = (M[q] == -INFINITY) ? 0.f : __expf(M[q] - mn);
            M[q] = mn;
            p[q] = ok ? __expf(l[q] - mn) : 0.f;
            s_w[t][q] = p[q] * vx;
        }
        __syncthreads();  // every thread has read s_red (maxima) and written s_w
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            float ps = p[q];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            if (lane == 0) s_red[warp][q] = ps;
        }
        // value sums of this thread's coordinate pair over its quarter of the tile
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            accv[q].x *= alpha[q];
            accv[q].y *= alpha[q];
        }
        const int jj1 = min(cnt, kAT / 4 * (hq + 1));
        for (int jj = kAT / 4 * hq; jj < jj1; ++jj) {
            const uint32_t* blk = s_vcodes + jj * WV + vblk * BV;
            float2 c2;
            if (BV == 4) {
                c2 = s_vpair[__byte_perm(blk[vj >> 3], 0u, 0x4440u | ((vj >> 1) & 3))];
            } else {
                c2 = make_float2(s_vc[value_cell<BV>(blk, vj)], s_vc[value_cell<BV>(blk, vj + 1)]);
            }
            if (NQ == 4) {
                const float4 w4 = *reinterpret_cast<const float4*>(&s_w[jj][0]);
                accv[0] = ffma2(make_float2(w4.x, w4.x), c2, accv[0]);
                accv[1 % NQ] = ffma2(make_float2(w4.y, w4.y), c2, accv[1 % NQ]);
                accv[2 % NQ] = ffma2(make_float2(w4.z, w4.z), c2, accv[2 % NQ]);
                accv[3 % NQ] = ffma2(make_float2(w4.w, w4.w), c2, accv[3 % NQ]);
            } else {
#pragma unroll
                for (int q = 0; q < NQ; ++q)
                    accv[q] = ffma2(make_float2(s_w[jj][q], s_w[jj][q]), c2, accv[q]);
            }
        }
        __syncthreads();  // s_red holds the tile sums; s_vcodes / s_w may be reused
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            float ts = 0.f;
#pragma unroll
            for (int w = 0; w < kAT / 32; ++w) ts += s_red[w][q];
            L[q] = L[q] * alpha[q] + ts;
        }
        __syncthreads();  // s_red is rewritten by the next tile
    }
    // merge the four quarters of every coordinate pair and write the split's partials
    if (hq > 0) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) s_part[hq - 1][q][cp] = accv[q];
    }
    __syncthreads();
    if (hq == 0) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            if (q >= qn) continue;
            const int64_t row = (int64_t)g * nq + q0 + q;
            const float2 a1 = s_part[0][q][cp], a2 = s_part[1][q][cp], a3 = s_part[2][q][cp];
            const float2 sum = make_float2((accv[q].x + a1.x) + (a2.x + a3.x),
                                           (accv[q].y + a1.y) + (a2.y + a3.y));
            *reinterpret_cast<float2*>(&part_acc[(row * nsplit + sp) * kAD + 2 * cp]) = sum;
            if (cp == 0) {
                part_m[row * nsplit + sp] = M[q];
                part_l[row * nsplit + sp] = L[q];
            }
        }
    }
}

// Merge the splits of one (group, query) row and rotate back:
//   a = sum_s e^{m_s - M} acc_s / sum_s e^{m_s - M} l_s,   out = Pi_v^T a.
__global__ __launch_bounds__(kAD) void k_attn_combine(const float* __restrict__ part_m,
                                                      const float* __restrict__ part_l,
                                                      const float* __restrict__ part_acc,
                                                      int nsplit, int nq,
                                                      const float* __restrict__ Pi_v,
                                                      float* __restrict__ out) {
    __shared__ float s_a[kAD];
    const int q = blockIdx.x, g = blockIdx.y, k = threadIdx.x;
    const int64_t row = (int64_t)g * nq + q;
    const float* pm = part_m + row * nsplit;
    const float* pl = part_l + row * nsplit;
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, pm[s]);
    float L = 0.f, a = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const float e = __expf(pm[s] - M);
        L = fmaf(e, pl[s], L);
        a = fmaf(e, part_acc[(row * nsplit + s) * kAD + k], a);
    }
    s_a[k] = a / L;
    __syncthreads();
    const float* P = Pi_v + (size_t)g * kAD * kAD;
    float o = 0.f;
    for (int j = 0; j < kAD; ++j) o = fmaf(P[(size_t)j * kAD + k], s_a[j], o);
    out[row * kAD + k] = o;
}

template <int BV, int NQ>
int launch_partial(dim3 grid, const float* logits, const uint32_t* vc, const float* vx, int64_t n,
                   int nq, const KCodebook& vcb, float scale, int split, float* pm, float* pl,
                   float* pa, cudaStream_t s) {
    k_attn_partial<BV, NQ><<<grid, kAT, 0, s>>>(logits, vc, vx, n, nq, vcb, scale, split, pm, pl,
                                               pa);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}

template <int BV>
int launch_partial_nq(dim3 grid, int NQ, const float* logits, const uint32_t* vc, const float* vx,
                      int64_t n, int nq, const KCodebook& vcb, float scale, int split, float* pm,
                      float* pl, float* pa, cudaStream_t s) {
    if (NQ == 1) return launch_partial<BV, 1>(grid, logits, vc, vx, n, nq, vcb, scale, split, pm, pl, pa, s);
    return launch_partial<BV, 4>(grid, logits, vc, vx, n, nq, vcb, scale, split, pm, pl, pa, s);
}

}  // namespace

// Queries per pass and keys per split of the decode-attention kernels: enough
// blocks for eight per SM over all groups and passes (the tile loop waits on
// its loads; other blocks hide that), splits of whole tiles.
int attn_queries_per_pass(int nq) { return nq <= 1 ? 1 : 4; }

int64_t attn_split(int64_t n, int G, int nq) {
    const int64_t passes = (nq + attn_queries_per_pass(nq) - 1) / attn_queries_per_pass(nq);
    const int64_t want = 8 * 148;
    int64_t per = (n * G * passes + want - 1) / want;
    per = (per + kAT - 1) / kAT * kAT;
    return per < kAT ? kAT : (per > kAttnSplitMax ? kAttnSplitMax : per);
}

// [tq_score's workspace (its status word first) | logits [G][nq][n] |
//  split maxima | split sums | split value sums [G][nq][nsplit][d]]
size_t attn_workspace_bytes(int b, int G, int64_t n, int nq) {
    const int64_t split = attn_split(n, G, nq);
    const int64_t nsplit = (n + split - 1) / split;
    const size_t rows = (size_t)G * nq;
    return align256(tq_workspace_bytes(TQ_OP_SCORE, kAD, b, G, n, nq, 0)) +
           align256(rows * (size_t)n * 4) + 2 * align256(rows * nsplit * 4) +
           align256(rows * nsplit * kAD * 4);
}

}  // namespace tq

using namespace tq;

extern "C" int tq_attention_decode(const tq_codebook_t* cb_k, const float* d_Pi_k,
                                   const float* d_S_k, const tq_codebook_t* cb_v,
                                   const float* d_Pi_v, int G, int64_t n,
                                   const uint32_t* d_kcodes, const float* d_kxnorm,
                                   const float* d_krnorm, const uint32_t* d_vcodes,
                                   const float* d_vxnorm, int nq, const void* d_q, int q_dtype,
                                   float scale, float* d_out, void* d_ws, size_t ws_bytes,
                                   void* stream) {
    if (!cb_k || !cb_v || G < 1 || n < 1 || nq < 1) return TQ_ERR_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_ARG;
    if (is_mse(cb_k) || !is_mse(cb_v)) return TQ_ERR_ARG;
    if (cb_k->d != kAD || cb_v->d != kAD) return TQ_ERR_UNSUPPORTED;
    if (is_split(cb_k) || is_split(cb_v)) return TQ_ERR_UNSUPPORTED;
    if (!valid_db(cb_k->d, cb_k->b) || !valid_db(cb_v->d, cb_v->b)) return TQ_ERR_UNSUPPORTED;
    if (cb_k->groups < G || cb_v->groups < G) return TQ_ERR_MISMATCH;
    if (!d_Pi_k || !d_S_k || !d_Pi_v || !d_kcodes || !d_kxnorm || !d_krnorm || !d_vcodes ||
        !d_vxnorm || !d_q || !d_out || !std::isfinite(scale))
        return TQ_ERR_ARG;
    const size_t need = attn_workspace_bytes(cb_k->b, G, n, nq);
    if (!d_ws || ws_bytes < need) return TQ_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t split = attn_split(n, G, nq);
    const int64_t nsplit = (n + split - 1) / split;
    const size_t rows = (size_t)G * nq;
    const size_t score_ws = align256(tq_workspace_bytes(TQ_OP_SCORE, kAD, cb_k->b, G, n, nq, 0));
    float* logits = (float*)((char*)d_ws + score_ws);
    float* pm = (float*)((char*)logits + align256(rows * (size_t)n * 4));
    float* pl = (float*)((char*)pm + align256(rows * nsplit * 4));
    float* pa = (float*)((char*)pl + align256(rows * nsplit * 4));
    // the estimated inner products, by the scoring path tq_score takes for nq
    int rc = tq_score(cb_k, d_Pi_k, d_S_k, G, n, d_kcodes, d_kxnorm, d_krnorm, nq, d_q, q_dtype,
                      logits, d_ws, score_ws, stream);
    if (rc) return rc;
    const int NQ = attn_queries_per_pass(nq);
    const dim3 grid((unsigned)nsplit, (unsigned)G, (unsigned)((nq + NQ - 1) / NQ));
    const KCodebook vcb = make_kcodebook(cb_v);
    switch (cb_v->b) {
        case 1: rc = launch_partial_nq<1>(grid, NQ, logits, d_vcodes, d_vxnorm, n, nq, vcb, scale, (int)split, pm, pl, pa, s); break;
        case 2: rc = launch_partial_nq<2>(grid, NQ, logits, d_vcodes, d_vxnorm, n, nq, vcb, scale, (int)split, pm, pl, pa, s); break;
        case 3: rc = launch_partial_nq<3>(grid, NQ, logits, d_vcodes, d_vxnorm, n, nq, vcb, scale, (int)split, pm, pl, pa, s); break;
        default: rc = launch_partial_nq<4>(grid, NQ, logits, d_vcodes, d_vxnorm, n, nq, vcb, scale, (int)split, pm, pl, pa, s); break;
    }
    if (rc) return rc;
    k_attn_combine<<<dim3((unsigned)nq, (unsigned)G), kAD, 0, s>>>(pm, pl, pa, (int)nsplit, nq,
                                                                    d_Pi_v, d_out);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}
