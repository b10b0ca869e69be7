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
// group (flash-decoding).  A block takes `split` keys: the split's maximum per
// query first, then in tiles of 256 the weights e^(l - M) |v_j| and
// sum_j w_j c_v[cell_j] in the rotated value domain, a thread owning 8
// coordinates (one code word of every record) and a sixteenth of the keys.
// Because Pi_v^T is linear it is applied once per query, after the splits are
// merged (k_attn_combine), instead of once per value.
#include <cmath>

#include "tq_internal.cuh"
#include "tq_score_common.cuh"

namespace tq {
namespace {

using sc::ffma2;

constexpr int kAD = 128;         // head dimension
constexpr int kAT = 256;         // keys per tile = threads per block
constexpr int kAttnSplitMax = 4096;
constexpr int kPairCopies = 8;   // copies of the byte-pair centroid table (b_v = 4)

// Value cell of coordinate j (0..31) of a block of the MSE-only layout (the
// index's top bit sits in the z position): the b-bit Lloyd-Max cell.
template <int BV>
__device__ __forceinline__ uint32_t value_cell(const uint32_t* blk, int j) {
    if (BV == 4) return (blk[j >> 3] >> (4 * (j & 7))) & 15u;
    if (BV == 3) return ((blk[j >> 4] >> (2 * (j & 15))) & 3u) | (((blk[2] >> j) & 1u) << 2);
    if (BV == 2) return (blk[j >> 4] >> (2 * (j & 15))) & 3u;
    return (blk[0] >> j) & 1u;
}

// Asynchronous 16-byte global -> shared copies (completion per thread,
// cp.async.wait_all; a barrier then makes every thread's copies visible).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// One split of `split` keys of group g for queries q0 .. q0 + NQ - 1:
//   M_q = max_j l_qj over the split (one pass over its logits, so the
//         weights need no rescaling as the tiles go by),
//   w_qj = e^(l_qj - M_q) |v_j|,  L_q = sum_j e^(l_qj - M_q),
//   acc_q = sum_j w_qj c_v[cell_j]   (the rotated value domain).
// Tiles of 256 keys, software-pipelined: the value records of tile i + 1 are
// copied into shared memory (cp.async) and its logits loaded into registers
// while tile i is summed, so the sums never wait on HBM.  Per tile, thread t
// forms key t's weights (shared memory); then thread (8-coordinate word
// wi = t % 16, key lane kl = t / 16) walks keys kl, kl + 16, ... of the tile:
// one code word of the record (16 threads read one record: no bank
// conflicts), 8 centroids from a byte-pair table (b_v = 4) or the 16-entry
// table, 16 packed fp32x2 FMAs for the 4 queries.  The 16 key lanes' sums are
// merged once per split.
template <int BV, int NQ>
__global__ __launch_bounds__(kAT, 3) void k_attn_partial(
    const float* __restrict__ logits, const uint32_t* __restrict__ vcodes,
    const float* __restrict__ vxn, int64_t n, int nq, KCodebook vcb, float scale, int split,
    float* __restrict__ part_m, float* __restrict__ part_l, float* __restrict__ part_acc) {
    constexpr int WV = BV * kAD / 32;  // record words
    __shared__ float s_vc[16];
    // b_v = 4: code byte -> (c_v[low nibble], c_v[high nibble]), kPairCopies
    // copies side by side (dynamic shared memory); lane l reads copy l % 8,
    // so lanes of different copies never share a bank
    extern __shared__ float2 s_vpair[];
    __shared__ __align__(16) float s_w[2][kAT][4];
    __shared__ float s_red[kAT / 32][4];
    // two tiles' value records; after the tile loop, the key lanes' sums
    // [key lane][coordinate pair of the word][query][word] (float2)
    constexpr int kBufWords = (2 * kAT * WV > 16 * 4 * NQ * 16 * 2) ? 2 * kAT * WV : 16 * 4 * NQ * 16 * 2;
    __shared__ __align__(16) uint32_t s_buf[kBufWords];
    float2 (*s_acc)[4][NQ][16] = reinterpret_cast<float2 (*)[4][NQ][16]>(s_buf);
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
    if (BV == 4) {
        const float2 pv = make_float2(s_vc[t & 15], s_vc[t >> 4]);
#pragma unroll
        for (int r = 0; r < kPairCopies; ++r) s_vpair[t * kPairCopies + r] = pv;
    }
    const int pcopy = lane % kPairCopies;
    const int64_t r_beg = (int64_t)sp * split;
    const int64_t r_end = min(n, r_beg + split);
    const float* lg[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) lg[q] = logits + ((int64_t)g * nq + q0 + (q < qn ? q : 0)) * n;
    const uint32_t* vg = vcodes + (int64_t)g * n * WV;
    const float* vxg = vxn + (int64_t)g * n;
    const bool vec = ((reinterpret_cast<uintptr_t>(vg) & 15u) == 0);
    // the records of keys [r, r + cnt) into buffer b: 16-byte copies when the
    // records are 16-byte aligned (every record is 16 b_v bytes), else words
    auto stage = [&](int64_t r, int cnt, int b) {
        uint32_t* dst = s_buf + b * (kAT * WV);
        const uint32_t* src = vg + r * WV;
        if (vec) {
            for (int c = t; c < cnt * BV; c += kAT) cp_async16(dst + 4 * c, src + 4 * c);
            cp_async_commit();
        } else {
            for (int c = t; c < cnt * WV; c += kAT) dst[c] = __ldg(src + c);
        }
    };

    // ---- the split's maximum per query; the first tile's records in flight
    stage(r_beg, (int)min((int64_t)kAT, r_end - r_beg), 0);
    float M[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) M[q] = -INFINITY;
    for (int64_t j = r_beg + t; j < r_end; j += kAT)
#pragma unroll
        for (int q = 0; q < NQ; ++q)
            if (q < qn) M[q] = fmaxf(M[q], scale * lg[q][j]);
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M[q] = fmaxf(M[q], __shfl_xor_sync(0xffffffffu, M[q], o));
        if (lane == 0) s_red[warp][q] = M[q];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        float m = s_red[0][q];
#pragma unroll
        for (int w = 1; w < kAT / 32; ++w) m = fmaxf(m, s_red[w][q]);
        M[q] = m;
    }

    const int wi = t % 16, kl = t / 16;
    float2 acc[4][NQ];  // coordinates 8 wi + 2 e, 8 wi + 2 e + 1
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int q = 0; q < NQ; ++q) acc[e][q] = make_float2(0.f, 0.f);
    float Lp[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) Lp[q] = 0.f;
    // logits and value norm of key r + t of the next tile to weigh
    float lnext[NQ], vnext = 0.f;
    auto load_key = [&](int64_t r, int cnt) {
        const bool ok = t < cnt;
        vnext = ok ? vxg[r + t] : 0.f;
#pragma unroll
        for (int q = 0; q < NQ; ++q) lnext[q] = (ok && q < qn) ? lg[q][r + t] : -INFINITY;
    };
    load_key(r_beg, (int)min((int64_t)kAT, r_end - r_beg));
    int buf = 0;
    for (int64_t r = r_beg; r < r_end; r += kAT, buf ^= 1) {
        const int cnt = (int)min((int64_t)kAT, r_end - r);
        {  // the weights of key r + t
            float w4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const float pq = lnext[q] == -INFINITY ? 0.f : __expf(scale * lnext[q] - M[q]);
                Lp[q] += pq;
                w4[q] = pq * vnext;
            }
            *reinterpret_cast<float4*>(&s_w[buf][t][0]) = make_float4(w4[0], w4[1], w4[2], w4[3]);
        }
        const int64_t rn = r + kAT;
        const int cntn = rn < r_end ? (int)min((int64_t)kAT, r_end - rn) : 0;
        if (cntn > 0) load_key(rn, cntn);
        if (vec) cp_async_wait_all();
        __syncthreads();  // this tile's records and weights complete; the other buffers free
        if (cntn > 0) stage(rn, cntn, buf ^ 1);
        const uint32_t* rec = s_buf + buf * (kAT * WV);
#pragma unroll 4
        for (int kk = 0; kk < 16; ++kk) {
            const int key = kl + 16 * kk;
            if (key < cnt) {
                uint32_t cw[BV == 4 ? 1 : BV];
#pragma unroll
                for (int i = 0; i < (BV == 4 ? 1 : BV); ++i)
                    cw[i] = rec[key * WV + (BV == 4 ? wi : (wi >> 2) * BV + i)];
                const float4 w = *reinterpret_cast<const float4*>(&s_w[buf][key][0]);
                const float wq[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float2 c2;
                    if (BV == 4) {  // one code byte = one coordinate pair
                        c2 = s_vpair[__byte_perm(cw[0], 0u, 0x4440u | e) * kPairCopies + pcopy];
                    } else {
                        const int j = 8 * (wi & 3) + 2 * e;
                        c2 = make_float2(s_vc[value_cell<BV>(cw, j)], s_vc[value_cell<BV>(cw, j + 1)]);
                    }
#pragma unroll
                    for (int q = 0; q < NQ; ++q)
                        acc[e][q] = ffma2(make_float2(wq[q], wq[q]), c2, acc[e][q]);
                }
            }
        }
    }
    __syncthreads();  // every thread is done with the record buffers
    // ---- merge the 16 key lanes; the split's sums per query
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int q = 0; q < NQ; ++q) s_acc[kl][e][q][wi] = acc[e][q];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        float ls = Lp[q];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
        if (lane == 0) s_red[warp][q] = ls;
    }
    __syncthreads();
    // output o = ((q * 4 + e) * 16 + wi) * 2 + u is coordinate k = 8 wi + 2 e + u
    for (int o = t; o < kAD * NQ; o += kAT) {
        const int u = o & 1, wo = (o >> 1) & 15, e = (o >> 5) & 3, q = o >> 7;
        const int k = 8 * wo + 2 * e + u;
        if (q >= qn) continue;
        float a = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) {
            const float2 v = s_acc[l][e][q][wo];
            a += u ? v.y : v.x;
        }
        const int64_t row = (int64_t)g * nq + q0 + q;
        part_acc[(row * nsplit + sp) * kAD + k] = a;
        if (k == 0) {
            float ls = 0.f;
#pragma unroll
            for (int w = 0; w < kAT / 32; ++w) ls += s_red[w][q];
            part_m[row * nsplit + sp] = M[q];
            part_l[row * nsplit + sp] = ls;
        }
    }
}

// Merge the splits of one (group, query) row and rotate back:
//   a = sum_s e^{m_s - M} acc_s / sum_s e^{m_s - M} l_s,   out = Pi_v^T a.
// 256 threads: the split weights e^{m_s - M} go through shared memory in
// chunks of kCombChunk splits; warp w sums splits s = w mod 8 of a chunk for
// the 4 coordinates 4 lane .. 4 lane + 3 (float4 loads), the 8 warps' sums
// are added in shared memory, and the two halves of the block each apply
// half of the rows of Pi_v.
constexpr int kCombThreads = 256;
constexpr int kCombChunk = 1024;
__global__ __launch_bounds__(kCombThreads) void k_attn_combine(const float* __restrict__ part_m,
                                                               const float* __restrict__ part_l,
                                                               const float* __restrict__ part_acc,
                                                               int nsplit, int nq,
                                                               const float* __restrict__ Pi_v,
                                                               float* __restrict__ out) {
    __shared__ float s_e[kCombChunk];
    __shared__ float s_red[kCombThreads / 32];
    __shared__ __align__(16) float s_part[kCombThreads / 32][kAD];
    __shared__ float s_a[kAD];
    __shared__ float s_o[2][kAD];
    const int q = blockIdx.x, g = blockIdx.y, t = threadIdx.x, lane = t % 32, w = t / 32;
    constexpr int NW = kCombThreads / 32;
    const int64_t row = (int64_t)g * nq + q;
    const float* pm = part_m + row * nsplit;
    const float* pl = part_l + row * nsplit;
    const float* pa = part_acc + row * nsplit * kAD;
    // M = max_s m_s
    float M = -INFINITY;
    for (int s = t; s < nsplit; s += kCombThreads) M = fmaxf(M, pm[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) s_red[w] = M;
    __syncthreads();
    M = s_red[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) M = fmaxf(M, s_red[i]);
    __syncthreads();  // s_red is reused for L
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < nsplit; c0 += kCombChunk) {
        const int cn = min(kCombChunk, nsplit - c0);
        for (int s = t; s < cn; s += kCombThreads) {
            const float e = __expf(pm[c0 + s] - M);
            s_e[s] = e;
            L = fmaf(e, pl[c0 + s], L);
        }
        __syncthreads();
#pragma unroll 4
        for (int s = w; s < cn; s += NW) {
            const float e = s_e[s];
            const float4 v = reinterpret_cast<const float4*>(pa + (int64_t)(c0 + s) * kAD)[lane];
            acc.x = fmaf(e, v.x, acc.x);
            acc.y = fmaf(e, v.y, acc.y);
            acc.z = fmaf(e, v.z, acc.z);
            acc.w = fmaf(e, v.w, acc.w);
        }
        __syncthreads();  // s_e is rewritten by the next chunk
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) s_red[w] = L;
    reinterpret_cast<float4*>(s_part[w])[lane] = acc;
    __syncthreads();
    if (t < kAD) {
        float a = 0.f, Ls = 0.f;
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            a += s_part[i][t];
            Ls += s_red[i];
        }
        s_a[t] = a / Ls;
    }
    __syncthreads();
    // out = Pi_v^T a: thread (half h, coordinate k) sums rows j of its half
    const int k = t % kAD, h = t / kAD;
    const float* P = Pi_v + (size_t)g * kAD * kAD;
    float o = 0.f;
#pragma unroll 8
    for (int j = h * (kAD / 2); j < (h + 1) * (kAD / 2); ++j) o = fmaf(P[(size_t)j * kAD + k], s_a[j], o);
    s_o[h][k] = o;
    __syncthreads();
    if (t < kAD) out[row * kAD + t] = s_o[0][t] + s_o[1][t];
}

template <int BV, int NQ>
int launch_partial(dim3 grid, const float* logits, const uint32_t* vc, const float* vx, int64_t n,
                   int nq, const KCodebook& vcb, float scale, int split, float* pm, float* pl,
                   float* pa, cudaStream_t s) {
    const int dyn = BV == 4 ? 256 * kPairCopies * (int)sizeof(float2) : 0;
    if (dyn > 0)
        TQ_TRY_CUDA(cudaFuncSetAttribute(k_attn_partial<BV, NQ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, dyn));
    k_attn_partial<BV, NQ><<<grid, kAT, dyn, s>>>(logits, vc, vx, n, nq, vcb, scale, split, pm, pl,
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
    k_attn_combine<<<dim3((unsigned)nq, (unsigned)G), kCombThreads, 0, s>>>(pm, pl, pa, (int)nsplit,
                                                                            nq, d_Pi_v, d_out);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
}
