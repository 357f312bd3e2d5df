/*
 * lrs_oracle.h -- plain CPU oracle for the quantized recurrent-state decode step.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path includes, links or calls
 * this code; only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg do. It shares no source, header, table or helper with the CUDA
 * library: everything here is written out independently, in the order in which
 * the method is stated, so that a reader can check it against the sources:
 *
 *   [LoReS]  "Quantizing Recurrent Language Models Is Easier Than You Think",
 *            abstract: value-axis scale grouping, decay-based mixed precision
 *            for slowly decaying heads, stochastic rounding against error
 *            accumulation under repeated requantization.
 *   [LRB/BDR] "Preserving Updates in Low-Bit Recurrent State Quantization",
 *            abstract: the state is updated and requantized at every step;
 *            Bounded Directional Rounding rounds an element that would move
 *            opposite to its update toward that update instead.
 *   [SplitMix64] Steele, Lea & Flood, "Fast Splittable Pseudorandom Number
 *            Generators", OOPSLA 2014 (the published generator and mixer).
 *
 * Arithmetic: IEEE binary32 with one round-to-nearest-even per written
 * operation; the only fused operations are the explicit fmaf() calls. Build
 * with -ffp-contract=off and without fast-math (see oracle/build.py).
 *
 * Data layout (logical, one code per byte, independent of any packed format):
 *   codes  int8  [ntiles][d_k][d_v]   code c_ij in [-qmax, qmax]
 *   scales float [ntiles][G][d_v]     G = d_k / group
 *   q, k   float [ntiles][d_k];  v, out float [ntiles][d_v]
 *   gates  float [ntiles][d_k] (per-key) or [ntiles] (scalar)
 *   beta   float [ntiles]       (delta rule only)
 * Tile t is head tile_h[t] of batch row tile_b[t]; (b, h) enter the hash and
 * select the precision prec_map[h] in {4, 8}.
 */
#ifndef LRS_ORACLE_H
#define LRS_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_ROUND_RTN = 0, ORC_ROUND_SR = 1, ORC_ROUND_BDR = 2 };
enum { ORC_UPDATE_GATED = 0, ORC_UPDATE_DELTA = 1 };
enum { ORC_GATE_SCALAR = 0, ORC_GATE_PER_KEY = 1 };

/* SplitMix64 output for generator state z: the state is advanced by the golden
 * gamma and then mixed. A generator seeded with s returns mix(s), mix(s+g), ... */
uint64_t orc_splitmix64(uint64_t z);

/* Counter hash of one state element: a chain of SplitMix64 mixes over
 * (seed, step, (b,h), (i,j)). */
uint64_t orc_hash(uint64_t seed, uint64_t step, uint32_t b, uint32_t h, uint32_t i, uint32_t j);

/* Uniform in [0,1) on the 2^-23 grid taken from the top 23 bits of r. */
float orc_uniform(uint64_t r);

/* One decode step, in place on codes and scales, writing out. Returns 0, or a
 * negative value for invalid arguments (nothing is written then). */
int orc_step(int ntiles, const int32_t *tile_b, const int32_t *tile_h,
             int d_k, int d_v, int group, int update_kind, int gate_kind, int mode,
             const uint8_t *prec_map, int8_t *codes, float *scales,
             const float *q, const float *k, const float *v, const float *gates,
             const float *beta, float *out, uint64_t seed, uint64_t step, int nthreads);

/* The same recurrence on an fp32 state S [ntiles][d_k][d_v], no quantization:
 * S <- x, out = x^T q. */
int orc_fp32_step(int ntiles, int d_k, int d_v, int update_kind, int gate_kind, float *S,
                  const float *q, const float *k, const float *v, const float *gates,
                  const float *beta, float *out, int nthreads);

/* Quantize an fp32 state with round-to-nearest into codes and scales. */
int orc_import(int ntiles, const int32_t *tile_h, int d_k, int d_v, int group,
               const uint8_t *prec_map, const float *S0, int8_t *codes, float *scales);

/* Dequantize codes and scales into S [ntiles][d_k][d_v]. */
int orc_dequant(int ntiles, int d_k, int d_v, int group, const int8_t *codes,
                const float *scales, float *S);

/* Mean decay per head, accumulated in binary64 in index order.
 * decay [outer][heads][inner]; means [heads]. */
void orc_decay_means(int64_t outer, int heads, int64_t inner, const float *decay, double *means);

/* Mixed precision: the n_int8 heads with the largest mean decay (ties to the
 * lower head index) get 8-bit codes, the rest 4-bit. */
int orc_precision_map(int heads, const double *means, int n_int8, uint8_t *prec_map);

/* Multi-token (chunked) update: the T tokens of each tile are applied one
 * after the other to the fp32 state, starting from the dequantized state, with
 * one output per token; the state is requantized once, after the last token.
 * Token t's inputs are those of a decode step, stacked on a leading token axis:
 * q, k [T][ntiles][d_k]; v, out [T][ntiles][d_v]; gates [T][ntiles][d_k] or
 * [T][ntiles]; beta [T][ntiles]. With T = 1 this is orc_step. */
int orc_chunk_step(int ntiles, const int32_t *tile_b, const int32_t *tile_h,
                   int d_k, int d_v, int group, int update_kind, int gate_kind, int mode,
                   const uint8_t *prec_map, int8_t *codes, float *scales, int T,
                   const float *q, const float *k, const float *v, const float *gates,
                   const float *beta, float *out, uint64_t seed, uint64_t step, int nthreads);

/* Per-channel precision: the same three entry points with one width per
 * (head, scale group) -- a block of `group` key channels -- in prec_map
 * [H][G] (G = d_k / group) instead of one per head. Group g of head h is
 * requantized with qmax of prec_map[h*G + g]. */
int orc_step_pg(int ntiles, const int32_t *tile_b, const int32_t *tile_h,
                int d_k, int d_v, int group, int update_kind, int gate_kind, int mode,
                const uint8_t *prec_map, int8_t *codes, float *scales,
                const float *q, const float *k, const float *v, const float *gates,
                const float *beta, float *out, uint64_t seed, uint64_t step, int nthreads);
int orc_chunk_step_pg(int ntiles, const int32_t *tile_b, const int32_t *tile_h,
                      int d_k, int d_v, int group, int update_kind, int gate_kind, int mode,
                      const uint8_t *prec_map, int8_t *codes, float *scales, int T,
                      const float *q, const float *k, const float *v, const float *gates,
                      const float *beta, float *out, uint64_t seed, uint64_t step, int nthreads);
int orc_import_pg(int ntiles, const int32_t *tile_h, int d_k, int d_v, int group,
                  const uint8_t *prec_map, const float *S0, int8_t *codes, float *scales);

/* Decode step with Low-Rank Bypass ([LRB/BDR] abstract): the step's rank-1
 * update goes into a rank-`rank` buffer (U [ntiles][rank][d_k], V
 * [ntiles][rank][d_v], updated in place; step mod rank components filled),
 * and every rank-th step the buffer's elements of at least half a
 * quantization step are merged into the state. The readings and the order of
 * operations are stated at the definition. x_out (NULL or [ntiles][d_k][d_v])
 * receives the values before rounding. Per-head widths. */
int orc_lrb_step(int ntiles, const int32_t *tile_b, const int32_t *tile_h,
                 int d_k, int d_v, int group, int update_kind, int gate_kind, int mode,
                 const uint8_t *prec_map, int8_t *codes, float *scales, int rank, float *U,
                 float *V, const float *q, const float *k, const float *v, const float *gates,
                 const float *beta, float *out, uint64_t seed, uint64_t step, float *x_out);

/* orc_lrb_step with one width per (head, scale group): prec_map [H][d_k/group]. */
int orc_lrb_step_pg(int ntiles, const int32_t *tile_b, const int32_t *tile_h,
                    int d_k, int d_v, int group, int update_kind, int gate_kind, int mode,
                    const uint8_t *prec_map, int8_t *codes, float *scales, int rank, float *U,
                    float *V, const float *q, const float *k, const float *v,
                    const float *gates, const float *beta, float *out, uint64_t seed,
                    uint64_t step, float *x_out);

/* A study of the Bounded Directional Rounding reading (not a step the
 * library implements). [LRB/BDR] says a stored element can move opposite to
 * "its update" and that BDR rounds such elements toward the update. The
 * library reads the update as the element's whole change x - deq this step.
 * This function takes the other reading, the additive term k_i w_j alone
 * (decay excluded), for the gated update with per-key gates and one code
 * width (qmax 127 or 7) for every tile: deq, x, out and the new scales as in
 * orc_step; then c0 = rint(y), move m = RN(RN(c0 s') - deq), and c = ceil(y)
 * when k_i w_j > 0 > m, floor(y) when k_i w_j < 0 < m, else c0; clamped.
 * Single-threaded. */
int orc_bdr_additive_step(int ntiles, int d_k, int d_v, int group, int qmax, int8_t *codes,
                          float *scales, const float *q, const float *k, const float *v,
                          const float *gates, float *out);

/* bfloat16 (the upper half of binary32: sign, 8 exponent bits, 7 fraction
 * bits) nearest to x, ties to the even fraction; NaN becomes a quiet NaN of the
 * same sign. Returns the 16-bit pattern. */
uint16_t orc_bf16_rne(float x);
void orc_bf16_rne_array(int64_t n, const float *x, uint16_t *out);

#ifdef __cplusplus
}
#endif
#endif
