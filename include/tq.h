/*
 * tq.h -- C ABI of the B200 (sm_100a) TurboQuant library, libtq.so.
 *
 * TurboQuant inner-product quantizer, as summarised on the reference pages
 * (page titles):
 *   quant_prune_distill #674 "TurboQuant": the two problem statements
 *     (MSE-optimal; inner-product-optimal and unbiased); the MSE quantizer
 *     rotates by a random orthogonal matrix (not Hadamard) and rounds on a
 *     Lloyd-Max grid; the inner-product quantizer spends b-1 bits on the MSE
 *     quantizer and 1 bit on a QJL sketch of the residual (random matrix,
 *     then the sign).
 *   RecSysChannel #256 "TurboQuant: Redefining AI efficiency with extreme
 *     compression": normalised vectors times a random matrix have nearly
 *     N(0, 1/d) coordinates; thresholds are precomputed; a 1-bit
 *     per-coordinate correction makes the inner-product estimate unbiased.
 *   seeallochnaya #3476: rotation spreads outliers; 1-D k-means boundaries,
 *     denser in the centre; residual -> random matrix -> sign; "parallelises
 *     well on a GPU".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All pointers named d_* are DEVICE pointers of the current CUDA device;
 *    the caller allocates and owns them.  The library allocates no memory
 *    and keeps no global state.  `stream` is a cudaStream_t (NULL = the
 *    legacy default stream); every call is asynchronous on it.
 *  - Return value: TQ_OK (0) or a negative TQ_ERR_* code; a call that
 *    returns an error has launched nothing that writes an output, except
 *    TQ_ERR_CUDA (a launch failed; the outputs are undefined).  Calls never
 *    abort the process.
 *  - Supported shapes: d a multiple of 128, 128 <= d <= 4096; b (total bits
 *    per coordinate) in 1..4; G (groups) >= 1; n, nq >= 0 (0 is a no-op).
 *  - Groups: group g has its own Pi_g and S_g, drawn from seed + g; arrays
 *    are group-major: x [G][n][d], codes [G][n][W], norms [G][n],
 *    queries [G][nq][d], scores [G][nq][n], top-k [G][nq][k].  For KV-cache
 *    keys a group is a KV head and its nq query heads share it (GQA).
 *  - W = b * d / 32 uint32 words per code record.  Layout (ours; the pages
 *    give none): d/32 blocks of b words, block w holding coordinates
 *    32w..32w+31 (j = coordinate - 32w):
 *      b = 1: word 0 bit j = z_j
 *      b = 2: word j/16, bits 2(j%16)+{0,1} = idx_j, z_j
 *      b = 3: word j/16, bits 2(j%16)+{0,1} = idx_j (2 bits); word 2 bit j = z_j
 *      b = 4: word j/8,  bits 4(j%8)+{0,1,2,3} = idx_j (3 bits), z_j
 *    idx_j = Lloyd-Max cell of the rotated coordinate, z_j = [(S r)_j >= 0].
 *    The two fp32 norms |x| and |r| are stored in separate arrays.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define TQ_OK                  0
#define TQ_ERR_ARG            -1  /* null pointer, negative size, bad enum   */
#define TQ_ERR_UNSUPPORTED    -2  /* d not a multiple of 128, b outside 1..4 */
#define TQ_ERR_WORKSPACE      -3  /* ws_bytes below tq_workspace_bytes()     */
#define TQ_ERR_CUDA           -4  /* a CUDA launch or API call failed        */
#define TQ_ERR_DEVICE_TIMEOUT -5  /* a bounded device-side wait gave up      */
#define TQ_ERR_MISMATCH       -6  /* codebook does not match the call's d/b  */
#define TQ_ERR_SCRATCH_LIMIT  -7  /* tq_topk_noalloc: sizes need more scratch
                                     than TQ_NOALLOC_SCRATCH_BYTES            */

/* element types of caller inputs */
#define TQ_F32  0
#define TQ_BF16 1

/* operation ids for tq_workspace_bytes */
#define TQ_OP_BUILD   0
#define TQ_OP_ENCODE  1
#define TQ_OP_SCORE   2
#define TQ_OP_TOPK    3
#define TQ_OP_DECODE  4
#define TQ_OP_EXACT   5
#define TQ_OP_ATTENTION 6
#define TQ_OP_SCORE_TOPK 7

/* codebook variants */
#define TQ_VARIANT_PROD 0  /* inner-product quantizer: (b-1)-bit Lloyd-Max index
                              + 1 QJL sign bit per coordinate (unbiased)        */
#define TQ_VARIANT_MSE  1  /* MSE-only quantizer: b-bit Lloyd-Max index, no QJL
                              (quant_prune_distill #674 "MSE-optimised";
                              biased inner products)                           */

/* Host-side codebook (quant_prune_distill #674: Lloyd-Max grid for the
 * target bit width; RecSysChannel #256 item 1: thresholds computed in
 * advance).  Filled by tq_build_codebook (TQ_VARIANT_PROD) or
 * tq_build_codebook_mse (TQ_VARIANT_MSE); plain data, caller-owned, may be
 * copied.  centroids[j] / boundaries[j] are the Lloyd-Max centroids and cell
 * boundaries of N(0,1) for `levels` levels, multiplied by 1/sqrt(d) and
 * rounded to fp32; unused entries are 0.  PROD: levels = 2^(b-1) (none for
 * b = 1).  MSE: levels = 2^b; its records use the layout below with the
 * b-bit index split into its low b-1 bits (the idx field) and its top bit
 * (the position of z), and store |r| = |y - c[idx]|. */
typedef struct tq_codebook {
    int32_t  d;            /* vector dimension                               */
    int32_t  b;            /* total bits per coordinate                      */
    int32_t  levels;       /* PROD: 2^(b-1), 0 for b = 1; MSE: 2^b           */
    int32_t  groups;       /* G: number of (Pi, S) pairs (MSE: Pi only) built */
    uint64_t seed;         /* group g uses seed + g                          */
    float    centroids[16];
    float    boundaries[16];
    double   distortion;   /* Lloyd-Max mean squared error for N(0,1)        */
    int32_t  variant;      /* TQ_VARIANT_PROD or TQ_VARIANT_MSE              */
    int32_t  reserved;     /* 0                                              */
    /* fractional widths (tq_build_codebook_split; all 0 otherwise): split = 1
     * when the last d/2 rotated coordinates use the tables below, of
     * levels_lo levels (0 when they keep only the sign) */
    int32_t  split;
    int32_t  levels_lo;
    float    centroids_lo[16];
    float    boundaries_lo[16];
} tq_codebook_t;

/* Bytes of device workspace an operation needs for the given sizes (0 when
 * it needs none).  op is a TQ_OP_*; arguments that do not apply are
 * ignored.  Never fails: returns (size_t)-1 for unsupported shapes. */
TQ_API size_t tq_workspace_bytes(int op, int d, int b, int G, int64_t n, int nq, int k);

/* Human-readable name of a status code (static string). */
TQ_API const char *tq_status_str(int status);

/* E0, parameters (once per (d, b, seed, G); not on the timed path).
 * quant_prune_distill #674: "random orthogonal matrix (not Hadamard)" and
 * the Lloyd-Max grid; seeallochnaya #3476 step 2 "a random matrix".
 *  - Pi_g = Q diag(sign R_jj) from the Householder QR (fp64, on the device)
 *    of the d x d Gaussian matrix G_g[i][j] = N_(seed+g, stream 0)[i*d+j];
 *    written row-major fp32 to d_Pi[g] so that y = Pi_g x.
 *  - S_g[i][j] = N_(seed+g, stream 1)[i*d+j] rounded to fp32 -> d_S[g].
 *  - N_(s, t)[m]: Box-Muller pairs over SplitMix64 stream t of seed s
 *    (counter form, state mix64(s XOR t*0x9E3779B97F4A7C15)).
 *  - cb (host) receives the fp32 codebook, computed on the host in fp64.
 * d_Pi, d_S: [G][d][d] fp32.  d_ws: >= tq_workspace_bytes(TQ_OP_BUILD,...).
 * Synchronous with respect to the host only in that it returns after
 * enqueueing; the matrices are ready once `stream` reaches this point. */
TQ_API int tq_build_codebook(int d, int b, uint64_t seed, int G, tq_codebook_t *cb,
                      float *d_Pi, float *d_S, void *d_ws, size_t ws_bytes,
                      void *stream);

/* E0 of the MSE-only quantizer (quant_prune_distill #674, "MSE-optimised
 * TurboQuant": random rotation, then every bit on the Lloyd-Max index):
 * Pi_g exactly as tq_build_codebook draws it (so a PROD and an MSE codebook of
 * one seed share their rotation) and the b-bit (2^b-level) Lloyd-Max tables;
 * no S.  cb->variant = TQ_VARIANT_MSE.  With such a codebook tq_encode,
 * tq_score, tq_topk and tq_decode take d_S = NULL and compute
 *   encode: idx_i = #{j : beta_j <= y_i} over 2^b levels, |r| = |y - c[idx]|;
 *   score:  s = |x| <Pi_g q, c[idx]>;      decode: xhat = |x| Pi_g^T c[idx].
 * Same arguments, sizes and errors as tq_build_codebook otherwise. */
TQ_API int tq_build_codebook_mse(int d, int b, uint64_t seed, int G, tq_codebook_t *cb,
                          float *d_Pi, void *d_ws, size_t ws_bytes, void *stream);

/* E0 of the fractional widths.  quant_prune_distill #674 (experiments) and
 * comuna.ru "Google speeds up LLMs 8x" report KV caches at 3.5 and 2.5 bits
 * per channel; the pages give only the average.  Here b - 1/2 bits a
 * coordinate: the first d/2 rotated coordinates take b total bits (b-1 index
 * bits and the QJL sign), the last d/2 take b - 1, each half rounded on the
 * Lloyd-Max grid of its own level count for the same N(0, 1/d) marginal:
 * centroids/boundaries hold 2^(b-1) levels, centroids_lo/boundaries_lo 2^(b-2)
 * (none for b = 2, whose second half keeps only the sign).  Pi_g and S_g are
 * tq_build_codebook's.  b in 2..4 (1.5, 2.5 and 3.5 bits); cb->split = 1.
 * Records hold W = d/64 (2b - 1) words: the first half's d/64 blocks in the
 * layout of width b (above), then the second half's in the layout of width
 * b - 1.  tq_encode, tq_score, tq_topk, tq_score_topk, tq_topk_noalloc and
 * tq_decode take such a codebook (same arguments; records of this layout);
 * tq_attention_decode returns TQ_ERR_UNSUPPORTED for it.  Same errors as
 * tq_build_codebook otherwise (b outside 2..4: TQ_ERR_UNSUPPORTED). */
TQ_API int tq_build_codebook_split(int d, int b, uint64_t seed, int G, tq_codebook_t *cb,
                                   float *d_Pi, float *d_S, void *d_ws, size_t ws_bytes,
                                   void *stream);

/* E1-E6, encode (quant_prune_distill #674 inner-product quantizer;
 * RecSysChannel #256 caveat 1: normalise, multiply by a random matrix):
 *   |x|, y = Pi_g x / |x| (y = 0 for x = 0), idx_i = #{j : beta_j <= y_i},
 *   r = y - c[idx], |r|, z_i = [(S_g r)_i >= 0], packed as above.
 * d_x: [G][n][d], element type x_dtype (TQ_F32 or TQ_BF16).
 * d_codes: [G][n][W] uint32; d_xnorm, d_rnorm: [G][n] fp32. */
TQ_API int tq_encode(const tq_codebook_t *cb, const float *d_Pi, const float *d_S,
              int G, int64_t n, const void *d_x, int x_dtype,
              uint32_t *d_codes, float *d_xnorm, float *d_rnorm,
              void *d_ws, size_t ws_bytes, void *stream);

/* Device status of the last tq_encode, tq_score or tq_topk that used d_ws
 * (its first 4 bytes): TQ_OK, or TQ_ERR_DEVICE_TIMEOUT when a bounded
 * device-side wait of a tensor-core kernel gave up (the kernel then drains its
 * in-flight copies and MMAs, releases tensor memory and exits; its outputs are
 * undefined).  Copies the word to the host and synchronises `stream`. */
TQ_API int tq_device_status(const void *d_ws, void *stream);

/* Self-test of the device-side time-out path (no counterpart on the pages):
 * one thread waits, with the same bounded wait the tensor-core kernels use,
 * on a barrier that nothing completes.  After limit_ns (1 .. 2e9) it gives up
 * and records TQ_ERR_DEVICE_TIMEOUT in the first 4 bytes of d_ws (>= 256
 * bytes), which tq_device_status(d_ws, stream) then reports; the context
 * stays usable.  TQ_ERR_ARG for a null d_ws or a limit out of range. */
TQ_API int tq_selftest_wait_timeout(void *d_ws, uint64_t limit_ns, void *stream);

/* S0 + S1, scores (quant_prune_distill #674: inner-product quantization with
 * an unbiased estimate; comuna.ru "8x faster attention logits"):
 *   qr = Pi_g q, u = S_g qr,
 *   s = |x| ( <qr, c[idx]> + |r| sqrt(pi/2)/d <u, 2z - 1> ).
 * d_q: [G][nq][d] (q_dtype); d_scores: [G][nq][n] fp32 (raw inner-product
 * estimates, no softmax scaling). */
TQ_API int tq_score(const tq_codebook_t *cb, const float *d_Pi, const float *d_S,
             int G, int64_t n, const uint32_t *d_codes, const float *d_xnorm,
             const float *d_rnorm, int nq, const void *d_q, int q_dtype,
             float *d_scores, void *d_ws, size_t ws_bytes, void *stream);

/* S2, top-k search over the codes (comuna.ru: vector search recall): the k
 * largest estimated scores per query, ordered by score descending then id
 * ascending.  1 <= k <= 32 and k <= n.  d_vals: [G][nq][k] fp32;
 * d_ids: [G][nq][k] int64 (index within the group). */
TQ_API int tq_topk(const tq_codebook_t *cb, const float *d_Pi, const float *d_S,
            int G, int64_t n, const uint32_t *d_codes, const float *d_xnorm,
            const float *d_rnorm, int nq, const void *d_q, int q_dtype, int k,
            float *d_vals, int64_t *d_ids, void *d_ws, size_t ws_bytes,
            void *stream);

/* S0-S2 in one call: the estimates of tq_score into d_scores and, from the
 * same scoring pass, the top-k of tq_topk into d_vals / d_ids (the queries
 * are transformed and scored once instead of once per call).  Arguments,
 * shapes, results and errors are those of tq_score and tq_topk; d_scores is
 * required.  d_ws: >= tq_workspace_bytes(TQ_OP_SCORE_TOPK, d, b, G, n, nq, k)
 * (no room for the scores: they live in d_scores). */
TQ_API int tq_score_topk(const tq_codebook_t *cb, const float *d_Pi, const float *d_S, int G,
                         int64_t n, const uint32_t *d_codes, const float *d_xnorm,
                         const float *d_rnorm, int nq, const void *d_q, int q_dtype, int k,
                         float *d_scores, float *d_vals, int64_t *d_ids, void *d_ws,
                         size_t ws_bytes, void *stream);

/* Dequantization (quant_prune_distill #674: "inverse rotation and
 * renormalisation"):  xhat = |x| Pi_g^T (c[idx] + |r| sqrt(pi/2)/d S_g^T (2z-1)).
 * d_xhat: [G][n][d] fp32.  Support path, not part of the timed step. */
TQ_API int tq_decode(const tq_codebook_t *cb, const float *d_Pi, const float *d_S,
              int G, int64_t n, const uint32_t *d_codes, const float *d_xnorm,
              const float *d_rnorm, float *d_xhat, void *d_ws, size_t ws_bytes,
              void *stream);

/* Unquantized baseline of the attention-logit comparison (comuna.ru:
 * "4-bit TurboQuant ... vs 32-bit unquantized keys"): exact fp32 logits
 *   out[g][t][v] = <q[g][t], keys[g][v]>  for fp32 keys [G][n][d] and
 * queries [G][nq][d] (q_dtype).  No workspace. */
TQ_API int tq_logits_fp32(int d, int G, int64_t n, const float *d_keys, int nq,
                   const void *d_q, int q_dtype, float *d_out, void *stream);

/* Exact fp32 inner-product top-k (ground truth for recall@k of the vector
 * search comparison on the pages), same ordering and shapes as tq_topk;
 * d_x: [G][n][d] fp32. */
TQ_API int tq_exact_topk(int d, int G, int64_t n, const float *d_x, int nq,
                  const void *d_q, int q_dtype, int k, float *d_vals,
                  int64_t *d_ids, void *d_ws, size_t ws_bytes, void *stream);

/* Merge of top-k lists computed on shards of one database (each shard's
 * tq_topk, ids made global by the caller, then one merge; the pages' vector
 * search is one top-k over all records, and sharding does not change it).
 * d_vals / d_ids: [nlists][rows][k] (the layout of an all-gather of every
 * shard's [rows][k] lists); missing entries carry id INT64_MAX.  Output:
 * [rows][k], values non-increasing, ties by smaller id (the tq_topk order).
 * 1 <= k <= 32 and nlists >= 1, else TQ_ERR_ARG.  No workspace. */
TQ_API int tq_topk_merge(int64_t rows, int nlists, int k, const float *d_vals,
                         const int64_t *d_ids, float *d_out_vals, int64_t *d_out_ids,
                         void *stream);

/* Decode attention over quantized keys and values (d = 128).  The pages stop
 * at the attention logits (comuna.ru "Google speeds up LLMs 8x": logits from
 * 4-bit keys; quant_prune_distill #674: the inner-product estimate and its
 * dequantization); this entry point takes the plain reading that those
 * logits feed standard softmax attention.  For every group g and query row t:
 *   l_j   = scale * s_tj      (s: the tq_score estimate of key record j)
 *   out_t = sum_j softmax_j(l) vhat_j,
 *   vhat_j = |v_j| Pi_v,g^T c_v[cell_j]   (the MSE-only dequantization).
 * Keys: inner-product records of cb_k (TQ_VARIANT_PROD) with d_Pi_k, d_S_k;
 * values: MSE-only records of cb_v (TQ_VARIANT_MSE) with d_Pi_v; both
 * [G][n] records (layout above) with their norms.  d_q: [G][nq][d] (q_dtype);
 * scale: finite (1/sqrt(d) for the usual attention); d_out: [G][nq][d] fp32.
 * d_ws: >= tq_workspace_bytes(TQ_OP_ATTENTION, 128, b, G, n, nq, 0).
 * n >= 1 and nq >= 1, else TQ_ERR_ARG; a variant other than PROD for cb_k or
 * MSE for cb_v is TQ_ERR_ARG; d != 128 is TQ_ERR_UNSUPPORTED.  Support path,
 * not part of the timed step. */
TQ_API int tq_attention_decode(const tq_codebook_t *cb_k, const float *d_Pi_k,
                               const float *d_S_k, const tq_codebook_t *cb_v,
                               const float *d_Pi_v, int G, int64_t n,
                               const uint32_t *d_kcodes, const float *d_kxnorm,
                               const float *d_krnorm, const uint32_t *d_vcodes,
                               const float *d_vxnorm, int nq, const void *d_q, int q_dtype,
                               float scale, float *d_out, void *d_ws, size_t ws_bytes,
                               void *stream);

/* Top-k without a caller workspace, for callers that cannot allocate device
 * memory.  The pages have no counterpart of this entry point; it exists for
 * the deployment, not for the method.
 *
 * Some callers of a KV-cache or vector-search library cannot call cudaMalloc
 * (or any allocator) at the point where they search: serving engines that
 * hand all device memory to their own pool at start-up and forbid libraries
 * from taking more, plugins that run inside another runtime's stream without
 * access to its allocator, and real-time paths where an allocation may block
 * on device synchronisation.  They still pass inputs and outputs; the scratch
 * that tq_topk would take from d_ws (transformed queries, per-tile candidate
 * lists) comes from one static device array of TQ_NOALLOC_SCRATCH_BYTES
 * (8 MiB) inside libtq, which every GPU that loads the library holds until
 * the process exits.
 *
 * Same arguments, results, ordering and errors as tq_topk, without d_ws and
 * ws_bytes.  Which scratch form it takes:
 *  - tq_topk's own choice when that fits the array (for searches up to 2^24
 *    scores, the full score matrix: tq_workspace_bytes(TQ_OP_TOPK, ...));
 *  - otherwise the form tq_topk takes beyond 2^24 scores, whose scratch holds
 *    the transformed queries and per-range candidate lists (at d = 128 with
 *    b >= 2 it scores chunks of keys sized to what is left of the array, with
 *    the same results as tq_topk);
 *  - TQ_ERR_SCRATCH_LIMIT, having launched nothing, only when that second
 *    form does not fit either (e.g. more than ~8000 queries, whose two
 *    transforms alone fill the array).  For d = 128, b = 4, 8 KV heads x 4
 *    query heads x 131072 tokens and k = 10 take the second form.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  A device reset (cudaDeviceReset) unloads the
 * library's module and invalidates the looked-up address: do not call this
 * entry point on a device after resetting it.  It allocates nothing: no
 * cudaMalloc, cudaFree or allocating library routine.  Every call on a device
 * shares the one array, which keeps the last call's contents (each call
 * overwrites all of the scratch it reads, nothing relies on it starting at
 * zero): calls that overlap on the GPU (different streams, or host threads)
 * race on it and must be serialised by the caller.  A bounded device-side
 * wait that gives up is recorded in the array, which the caller cannot read:
 * on this path such a time-out is not reported (tq_topk reports it through
 * tq_device_status). */
#define TQ_NOALLOC_SCRATCH_BYTES (8u << 20)
TQ_API int tq_topk_noalloc(const tq_codebook_t *cb, const float *d_Pi, const float *d_S,
                           int G, int64_t n, const uint32_t *d_codes, const float *d_xnorm,
                           const float *d_rnorm, int nq, const void *d_q, int q_dtype, int k,
                           float *d_vals, int64_t *d_ids, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H */
