// tq_topk_noalloc: tq_topk for callers that cannot allocate device memory.
//
// The scratch that tq_topk takes from the caller's workspace (the transformed
// queries and the per-tile candidate lists) comes here from one fixed array
// in the library's own device memory.  Nothing is allocated per call: the
// array is part of the module image and every GPU that loads the library
// holds it (TQ_NOALLOC_SCRATCH_BYTES) until the process exits.
#include <mutex>

#include "tq_internal.cuh"

namespace {

// Shared by every call on a device; keeps the previous call's contents.
static __device__ __align__(256) unsigned char g_topk_scratch[TQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_topk_scratch on the current device, looked up once per
// device.  In host code the symbol is only a host-side handle; the kernels
// must be given this address.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_topk_scratch);
        if (e != cudaSuccess || !p) return TQ_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return TQ_OK;
}

}  // namespace

extern "C" int tq_topk_noalloc(const tq_codebook_t* cb, const float* d_Pi, const float* d_S,
                               int G, int64_t n, const uint32_t* d_codes, const float* d_xnorm,
                               const float* d_rnorm, int nq, const void* d_q, int q_dtype, int k,
                               float* d_vals, int64_t* d_ids, void* stream) {
    const int v = tq::topk_validate(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q,
                                    q_dtype, k, d_vals, d_ids);
    if (v) return v == tq::kTopkNothing ? TQ_OK : v;
    const size_t need = tq_workspace_bytes(TQ_OP_TOPK, cb->d, cb->b, G, n, nq, k);
    // The materialised-score path when its scratch fits, else the fused path.
    bool materialize =
        tq::topk_materialized(cb->d, G, n, nq) && need <= (size_t)TQ_NOALLOC_SCRATCH_BYTES;
    if (!materialize && tq::topk_workspace_bytes(cb->d, cb->b, G, n, nq, k, false) >
                            (size_t)TQ_NOALLOC_SCRATCH_BYTES)
        return TQ_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc) return rc;
    return tq::topk_run(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype, k,
                        d_vals, d_ids, scratch, (size_t)TQ_NOALLOC_SCRATCH_BYTES, materialize,
                        (cudaStream_t)stream);
}
