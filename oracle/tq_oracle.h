/*
 * tq_oracle.h -- plain CPU oracle for the TurboQuant inner-product quantizer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * timed CPU baseline of the benchmark may load this library.  The CUDA
 * library never links, includes or calls it, and it includes nothing of the
 * CUDA library.
 *
 * Everything is computed in IEEE double (C `double`, no fast-math).  The
 * only fp32 values are the ones the method stores: the codebook tables, the
 * matrices Pi and S, and the two norms of a code record.
 *
 * Sources (page titles of the reference pages; see the .c file for each
 * function's passage):
 *   [QPD]  "quant_prune_distill post 674" (TurboQuant summary): problem
 *          statements, random orthogonal rotation (not Hadamard), Lloyd-Max
 *          grid, (b-1)-bit MSE quantizer plus 1-bit QJL on the residual.
 *   [RSC]  "RecSysChannel post 256": sphere -> near-Gaussian coordinates,
 *          precomputed thresholds, 1-bit correction, unbiasedness.
 *   [SEA]  "seeallochnaya post 3476": rotation, 1-D k-means thresholds
 *          denser in the centre, residual -> random matrix -> sign.
 *
 * Parity pins: every function below is pinned in tests/test_oracle_*.py
 * against something other than itself (published SplitMix64 outputs,
 * Max's 1960 table, LAPACK QR via numpy, numerical quadrature, brute force,
 * closed forms and the statistical unbiasedness of the estimator).
 */
#ifndef TQ_ORACLE_H
#define TQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- counter-based random numbers --------------------------------------- */
uint64_t tqo_mix64(uint64_t z);
uint64_t tqo_stream_key(uint64_t seed, uint64_t stream);
uint64_t tqo_u64(uint64_t seed, uint64_t stream, uint64_t i);
void     tqo_gaussian(uint64_t seed, uint64_t stream, int64_t count, double *out);

/* ---- parameters ---------------------------------------------------------- */
int tqo_lloyd_max(int levels, double *c, double *beta, double *distortion, int *iters);
int tqo_codebook(int d, int b, float *c, float *beta);
int tqo_rotation(int d, uint64_t seed, double *pi_d, float *pi_f, double *rdiag);
int tqo_qjl_matrix(int d, uint64_t seed, float *S);

/* ---- the quantizer -------------------------------------------------------- */
int64_t tqo_words_per_vector(int d, int b);
int tqo_encode(int d, int b, const float *c, const float *beta,
               const float *Pi, const float *S, int64_t n, const double *x,
               uint32_t *codes, float *xnorm, float *rnorm,
               double *y_out, double *p_out, int32_t *idx_out);
int tqo_unpack(int d, int b, int64_t n, const uint32_t *codes,
               int32_t *idx, int32_t *z);
int tqo_decode(int d, int b, const float *c, const float *Pi, const float *S,
               int64_t n, const uint32_t *codes, const float *xnorm,
               const float *rnorm, double *xhat);
int tqo_query(int d, const float *Pi, const float *S, int64_t nq,
              const double *q, double *qr, double *u);
int tqo_score(int d, int b, const float *c, int64_t n, const uint32_t *codes,
              const float *xnorm, const float *rnorm, int64_t nq,
              const double *qr, const double *u, double *scores);
int tqo_topk(int64_t nq, int64_t n, const double *scores, int k,
             double *vals, int64_t *ids);
int tqo_exact_scores(int d, int64_t n, const double *x, int64_t nq,
                     const double *q, double *out);
int tqo_mse_estimate(int d, int bits, const float *c, const float *beta,
                     const float *Pi, const double *x, const double *q,
                     double *estimate);

/* MSE-only quantizer stored as a code (b-bit Lloyd-Max index, no QJL). */
int tqo_mse_encode(int d, int b, const float *c, const float *beta, const float *Pi,
                   int64_t n, const double *x, uint32_t *codes, float *xnorm, float *rnorm,
                   double *y_out, int32_t *idx_out);
int tqo_mse_score(int d, int b, const float *c, int64_t n, const uint32_t *codes,
                  const float *xnorm, int64_t nq, const double *qr, double *scores);
int tqo_mse_decode(int d, int b, const float *c, const float *Pi, int64_t n,
                   const uint32_t *codes, const float *xnorm, double *out);

/* Fractional widths (b - 1/2 bits a coordinate): the first d/2 rotated
 * coordinates at b bits, the last d/2 at b - 1 (b = 2..4, d % 64 == 0). */
int64_t tqo_split_words_per_vector(int d, int b);
int tqo_split_encode(int d, int b, const float *c_hi, const float *beta_hi,
                     const float *c_lo, const float *beta_lo, const float *Pi,
                     const float *S, int64_t n, const double *x, uint32_t *codes,
                     float *xnorm, float *rnorm, double *y_out, double *p_out,
                     int32_t *idx_out);
int tqo_split_unpack(int d, int b, int64_t n, const uint32_t *codes, int32_t *idx, int32_t *z);
int tqo_split_decode(int d, int b, const float *c_hi, const float *c_lo, const float *Pi,
                     const float *S, int64_t n, const uint32_t *codes, const float *xnorm,
                     const float *rnorm, double *xhat);
int tqo_split_score(int d, int b, const float *c_hi, const float *c_lo, int64_t n,
                    const uint32_t *codes, const float *xnorm, const float *rnorm, int64_t nq,
                    const double *qr, const double *u, double *scores);

/* Decode attention: out_t = sum_j softmax_j(logits_t) values_j (fp64). */
int tqo_softmax_weighted_sum(int64_t nq, int64_t n, int d, const double *logits,
                             const double *values, double *out);

#ifdef __cplusplus
}
#endif

#endif
