// Status strings and workspace sizing of the C ABI.
#include "tq_internal.cuh"

using namespace tq;

extern "C" const char* tq_status_str(int status) {
    switch (status) {
        case TQ_OK: return "ok";
        case TQ_ERR_ARG: return "invalid argument";
        case TQ_ERR_UNSUPPORTED: return "unsupported shape (d must be a multiple of 128 in [128, 4096], b in 1..4)";
        case TQ_ERR_WORKSPACE: return "workspace missing or smaller than tq_workspace_bytes()";
        case TQ_ERR_CUDA: return "CUDA error";
        case TQ_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case TQ_ERR_MISMATCH: return "codebook does not match the call";
        case TQ_ERR_SCRATCH_LIMIT: return "sizes need more scratch than tq_topk_noalloc's fixed 8 MiB array";
        default: return "unknown status";
    }
}

extern "C" size_t tq_workspace_bytes(int op, int d, int b, int G, int64_t n, int nq, int k) {
    if (d < kMinD || d > kMaxD || d % 128) return (size_t)-1;
    if (G < 1 || n < 0 || nq < 0 || k < 0) return (size_t)-1;
    const size_t dd = (size_t)d * d;
    const int64_t chunk = n < kEncodeChunk ? n : kEncodeChunk;
    const int64_t ntiles = (n + kTopkTile - 1) / kTopkTile;
    const size_t qbuf = align256((size_t)G * nq * d * 4);
    const size_t parts = align256((size_t)G * nq * ntiles * k * 4) +
                         align256((size_t)G * nq * ntiles * k * 8);
    switch (op) {
        case TQ_OP_BUILD:
            return 2 * align256(dd * 8) + 2 * align256((size_t)d * 8);
        case TQ_OP_ENCODE: {
            if (b < 1 || b > 4) return (size_t)-1;
            // status word, Y, P, cell bytes; for the tensor-core GEMMs the bf16
            // pieces of Pi, S and one operand chunk
            size_t bytes = 256 + 2 * align256((size_t)chunk * d * 4) + align256((size_t)chunk * d);
            if (encode_gemm_tc(d))
                bytes += 2 * align256(3 * dd * 2) + align256((size_t)3 * chunk * d * 2);
            return bytes;
        }
        case TQ_OP_SCORE:  // status word, transformed queries (, GEMM operands)
            return 256 + 2 * qbuf + (score_gemm_supported(d, nq) ? score_gemm_workspace(d, n, nq) : 0);
        case TQ_OP_TOPK:
            return tq::topk_workspace_bytes(d, b, G, n, nq, k, topk_materialized(d, G, n, nq));
        case TQ_OP_SCORE_TOPK:  // as TQ_OP_TOPK's materialised form, scores in the caller's output
            return tq::topk_workspace_bytes(d, b, G, n, nq, k, true, false);
        case TQ_OP_DECODE:
            return 2 * align256((size_t)chunk * d * 4);
        case TQ_OP_EXACT:
            return align256((size_t)nq * ((chunk + 3) & ~int64_t(3)) * 4) + parts;
        case TQ_OP_ATTENTION:  // d = 128 only; status word, queries, split partials
            if (d != 128 || n < 1 || nq < 1) return (size_t)-1;
            if (b < 1 || b > 4) return (size_t)-1;
            return attn_workspace_bytes(b, G, n, nq);
        default:
            return (size_t)-1;
    }
}

namespace tq {
size_t topk_workspace_bytes(int d, int b, int G, int64_t n, int nq, int k, bool materialize,
                            bool scores_in_ws) {
    (void)b;
    const size_t qbuf = align256((size_t)G * nq * d * 4);
    if (materialize) {
        // scores, maxima per 128-key tile, counters, candidate lists (, GEMM operands)
        const int64_t ntm = (n + 127) / 128;
        return 256 + 2 * qbuf + (scores_in_ws ? align256((size_t)G * nq * n * 4) : 0) +
               align256((size_t)G * nq * ntm * 4) + align256((size_t)G * nq * 8) +
               2 * align256((size_t)G * nq * kTopkCandidates * 4) +
               (score_gemm_supported(d, nq) ? score_gemm_workspace(d, n, nq) : 0);
    }
    const int64_t ntiles = (n + kTopkTile - 1) / kTopkTile;
    return 256 + 2 * qbuf + align256((size_t)G * nq * ntiles * k * 4) +
           align256((size_t)G * nq * ntiles * k * 8);
}
}  // namespace tq

extern "C" int tq_device_status(const void* d_ws, void* stream) {
    if (!d_ws) return TQ_ERR_ARG;
    int word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    TQ_TRY_CUDA(cudaMemcpyAsync(&word, d_ws, sizeof(int), cudaMemcpyDeviceToHost, s));
    TQ_TRY_CUDA(cudaStreamSynchronize(s));
    return word == 0 ? TQ_OK : TQ_ERR_DEVICE_TIMEOUT;
}
