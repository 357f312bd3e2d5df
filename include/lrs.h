/*
 * lrs.h -- C ABI of liblrs, the low-bit recurrent-state decode library for
 * NVIDIA B200 (sm_100a).
 *
 * The library keeps the recurrent state of linear-recurrence language models
 * (GLA, Gated DeltaNet, Mamba2-SSD style) in int8 or int4 codes with fp32
 * value-axis group scales, and advances it one decode step at a time with one
 * fused CUDA kernel: dequantize, gated or delta-rule update, output o = S^T q,
 * new scales, requantize.
 *
 * Sources of the operations (page title, part of the page):
 *   [LoReS]   "Quantizing Recurrent Language Models Is Easier Than You Think",
 *             abstract: value-axis scale grouping, decay-based mixed precision,
 *             stochastic rounding under repeated requantization.
 *   [LRB/BDR] "Preserving Updates in Low-Bit Recurrent State Quantization",
 *             abstract: a fixed-size state updated and requantized at every
 *             step; Bounded Directional Rounding.
 *
 * Conventions for every entry point:
 *   - All functions return lrs_status (LRS_OK = 0). No exception or signal
 *     crosses the ABI. On an error nothing is launched and nothing is written,
 *     and lrs_last_error() returns a message (thread-local).
 *   - "device" pointers are CUDA device pointers of the current device;
 *     "host" pointers are CPU pointers (pinned memory for asynchronous copies).
 *     Device pointers must be 16-byte aligned (LRS_ERR_ALIGNMENT otherwise).
 *   - Work is enqueued on the caller's CUDA stream (cudaStream_t passed as
 *     void*, NULL = the legacy default stream) and runs asynchronously.
 *     Errors found by a kernel (a wait that timed out, a layout that does not
 *     match the precision map, an out-of-range code) are recorded on the
 *     device and returned by lrs_sync().
 *   - The caller owns every buffer it passes; the library owns the buffers
 *     inside an lrs_state (allocated by lrs_state_alloc, released by
 *     lrs_state_free).
 *
 * Per (batch b, head h) the state S is d_k x d_v (row i = key index, column
 * j = value index). Input layouts (fp32, contiguous):
 *   q, k   [B][H][d_k]        v, out [B][H][d_v]
 *   gates  [B][H][d_k] (LRS_GATE_PER_KEY, decay per key channel) or
 *          [B][H] (LRS_GATE_SCALAR); multiplicative decay values
 *   beta   [B][H] (LRS_UPDATE_DELTA), otherwise ignored (may be NULL)
 */
#ifndef LRS_H
#define LRS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LRS_VERSION 2

typedef enum {
    LRS_OK = 0,
    LRS_ERR_INVALID_ARG = 1,    /* NULL pointer, bad size, bad enum value */
    LRS_ERR_ALIGNMENT = 2,      /* a device pointer is not 16-byte aligned */
    LRS_ERR_UNSUPPORTED = 3,    /* a shape outside the compiled kernels */
    LRS_ERR_OOM = 4,            /* device allocation failed */
    LRS_ERR_CUDA = 5,           /* a CUDA runtime call failed */
    LRS_ERR_DEVICE_TIMEOUT = 6, /* a kernel gave up waiting for its copies */
    LRS_ERR_DEVICE_LAYOUT = 7,  /* the precision map passed to a step does not
                                   fit the state's tile layout */
    LRS_ERR_DEVICE_RANGE = 8,   /* lrs_state_import_codes met a code outside
                                   [-qmax, qmax] */
    LRS_ERR_DEVICE_BOUNDS = 9   /* bounds-checked debug build only: a step
                                   kernel index fell outside its buffer (the
                                   access was skipped) */
} lrs_status;

typedef enum { LRS_ROUND_RTN = 0, LRS_ROUND_SR = 1, LRS_ROUND_BDR = 2 } lrs_round_mode;
typedef enum { LRS_UPDATE_GATED = 0, LRS_UPDATE_DELTA = 1 } lrs_update_kind;
typedef enum { LRS_GATE_SCALAR = 0, LRS_GATE_PER_KEY = 1 } lrs_gate_kind;

/* Shape of one layer's state.
 *   d_v   in {64, 128}
 *   d_k   a multiple of group, 16 <= d_k <= 256
 *   group key rows sharing one scale per value column: 16, 32 or 64, with
 *         group * d_v <= 4096 (group <= 32 at d_v = 128)
 *   update_kind / gate_kind: LRS_UPDATE_DELTA requires LRS_GATE_SCALAR. */
typedef struct {
    int32_t batch, heads, d_k, d_v, group;
    int32_t update_kind, gate_kind;
} lrs_shape;

/* A quantized state. All pointers are device memory owned by the library.
 *
 * Code layout. One batch row holds the heads' tiles in head order; head h's
 * tile starts at byte head_offsets[h] of the row and has d_k*d_v*bits/8 bytes
 * (bits = prec_map[h]) -- or, for a state with one width per scale group
 * (lrs_state_alloc_groups), the sum over its groups g of group*d_v*bits/8
 * bytes with bits = prec_map[h*G + g], the groups' blocks in order. Tile
 * (b, h) starts at b*batch_stride_bytes + head_offsets[h]. Inside a tile, lane t of 32 owns value columns
 * [t*C, t*C + C), C = d_v/32, for every key row. Its codes are ordered by
 * scale group, then by column pair p (columns t*C + 2p and t*C + 2p + 1),
 * then by key row, then by column within the pair; this byte stream is cut
 * into 16-byte units, and unit u of lane t sits at tile byte (u*32 + t)*16.
 * Within each 32-bit little-endian word of the stream: int8 holds 4
 * consecutive elements, byte n = element n; int4 holds 8 consecutive
 * elements e0..e7, byte n = e_n | e_(n+4) << 4. Codes are stored in offset
 * binary: the byte (nibble) is code + 128 (+ 8). The key rows of one scale
 * group are therefore one contiguous group*d_v*bits/8-byte block of the tile.
 *
 * Scale layout: fp32 [B][H][d_k/group][d_v]. A value dequantizes as
 * code * scale[b][h][i/group][j]. */
typedef struct {
    lrs_shape shape;
    void *state_codes;
    float *scales;
    uint8_t *prec_map;        /* [H], or [H][G] (lrs_state_alloc_groups); 4 or 8 */
    int64_t *head_offsets;    /* [H] */
    int64_t batch_stride_bytes;
    int64_t code_bytes;       /* batch * batch_stride_bytes */
    int64_t scale_count;      /* batch * heads * (d_k/group) * d_v */
    void *priv;               /* library-private host data */
} lrs_state;

/* Validate a shape and precision map and compute the code layout, on the
 * host only (no GPU needed). prec_map_host [H] of 4 or 8. head_offsets_host
 * may be NULL; otherwise it receives H offsets. */
lrs_status lrs_layout_query(const lrs_shape *shape, const uint8_t *prec_map_host,
                            int64_t *head_offsets_host, int64_t *batch_stride_bytes,
                            int64_t *scale_count);

/* Allocate a state on the current device and set it to zero (codes 0,
 * scales 0). prec_map_host [H] chooses int8 (8) or int4 (4) codes per head
 * ([LoReS] decay-based mixed precision; see lrs_precision_map).
 * Synchronous. On failure *out is left zeroed. */
lrs_status lrs_state_alloc(const lrs_shape *shape, const uint8_t *prec_map_host,
                           lrs_state *out);

/* Per-channel precision ([LoReS] abstract: the decay-based width choice can
 * protect slowly decaying heads or channels). The channel blocks are the
 * scale groups: prec_map_host [H][G], G = d_k/group, gives each group of
 * `group` key channels of each head its own width (4 or 8), so the tile's
 * groups have different widths. Everything else as lrs_layout_query and
 * lrs_state_alloc; every entry point that takes a prec_map then expects the
 * [H][G] form for this state. The widths of a state are normally chosen by
 * ranking the mean decay of each (head, key group) block: lrs_decay_head_means
 * and lrs_precision_map with heads = H*G and inner = group on a per-key decay
 * tensor [outer][H][d_k] (the same memory as [outer][H*G][group]). */
lrs_status lrs_layout_query_groups(const lrs_shape *shape, const uint8_t *prec_map_host,
                                   int64_t *head_offsets_host, int64_t *batch_stride_bytes,
                                   int64_t *scale_count);
lrs_status lrs_state_alloc_groups(const lrs_shape *shape, const uint8_t *prec_map_host,
                                  lrs_state *out);

/* Release everything lrs_state_alloc allocated and zero *st. NULL and
 * already-freed states are accepted. Synchronous. */
lrs_status lrs_state_free(lrs_state *st);

/* One decode step, in place ([LoReS] abstract; [LRB/BDR] abstract).
 * For every (b, h) tile, with old codes c and scales s:
 *   deq_ij = c_ij * s[i/group][j]
 *   gated: w = v;  delta: u_j = sum_i k_i deq_ij (i ascending, fused
 *          multiply-adds), w_j = beta * (v_j - alpha * u_j), alpha = gate
 *   x_ij   = fma(g_i, deq_ij, k_i * w_j)      (g_i per key, or the scalar)
 *   out_j  = sum_i q_i x_ij                    (i ascending, fused)
 *   A      = max |x_ij| over each group's rows, per column; scale' = A/qmax,
 *            inv = qmax/A (both 0 when A < 2^-100); qmax = 127 or 7
 *   y      = x_ij * inv taken exactly (the product is not rounded first);
 *            code' = an integer from y, clamped to [-qmax, qmax]:
 *     LRS_ROUND_RTN  nearest, ties to even
 *     LRS_ROUND_SR   floor(y) + [u < fr], fr = y - floor(y) rounded once to
 *                    binary32, u = top 23 bits of the
 *                    hash H(seed, step, b, h, i, j) times 2^-23, where
 *                    H = m(m(m(m(seed) ^ step) ^ (b<<32|h)) ^ (i<<32|j)) and
 *                    m is the SplitMix64 output function (add 0x9E3779B97F4A7C15,
 *                    then its 64-bit mixer)
 *     LRS_ROUND_BDR  nearest, except that when the update d = x - deq and the
 *                    move m = RN(RN(nearest*scale') - deq) have opposite signs
 *                    the code is ceil(y) (d > 0) or floor(y) (d < 0)
 * Every operation is binary32 with round-to-nearest-even; results are
 * deterministic and independent of the launch configuration.
 *
 * state_codes, scales, prec_map: device buffers laid out as st describes
 * (normally st->state_codes, st->scales, st->prec_map; another buffer set
 * allocated with the same shape and precision map, e.g. another layer's, is
 * also accepted). A prec_map whose tile sizes do not fit st's offsets is
 * detected per tile: that tile is skipped and LRS_ERR_DEVICE_LAYOUT is
 * recorded. q, k, v, gates, beta: device inputs (see the header comment);
 * out: device [B][H][d_v]. seed, step: the stochastic-rounding counters.
 * mode: lrs_round_mode. stream: cudaStream_t. */
lrs_status lrs_decode_step(const lrs_state *st, void *state_codes, float *scales,
                           const uint8_t *prec_map, const float *q, const float *k,
                           const float *v, const float *gates, const float *beta, float *out,
                           uint64_t seed, uint64_t step, int32_t mode, void *stream);

/* The step with bfloat16 q, k, v and out, as a model layer in bfloat16 feeds
 * and consumes it (the state, gates and beta are as in lrs_decode_step). The
 * method's sources fix no input precision; this variant reads each bfloat16
 * input as the float32 it denotes (exactly), runs the same fp32 step, and
 * writes each output element as the bfloat16 nearest to the fp32 o_j (ties to
 * even). q, k: [B][H][d_k], v, out: [B][H][d_v], bfloat16 bit patterns
 * (sign, 8 exponent bits, 7 fraction bits), device memory, 16-byte aligned.
 * Everything else -- layout, ownership, errors, asynchrony -- as
 * lrs_decode_step. */
lrs_status lrs_decode_step_bf16(const lrs_state *st, void *state_codes, float *scales,
                                const uint8_t *prec_map, const uint16_t *q, const uint16_t *k,
                                const uint16_t *v, const float *gates, const float *beta,
                                uint16_t *out, uint64_t seed, uint64_t step, int32_t mode,
                                void *stream);

/* Multi-token (chunked) update: T tokens applied to every tile in order, one
 * requantization at the end. The method's sources describe only the decode
 * step, where the state is requantized after every update; for the tokens
 * that precede decode (a prefill chunk, the tokens of a speculative-decoding
 * verification) this entry point keeps the fp32 state on chip across the T
 * updates and requantizes once, so repeated requantization happens once per
 * chunk. Per tile: S = dequantized state; for t = 0..T-1 in order, the same
 * update and output as lrs_decode_step with token t's inputs (S <- x,
 * out[t] = x^T q_t); then new scales and codes from S by `mode` -- for BDR the
 * update is S - (dequantized state at the chunk's start), for SR the counters
 * are (seed, step). T = 1 gives exactly lrs_decode_step.
 *   q, k: [T][B][H][d_k]; v, out: [T][B][H][d_v]; gates: [T][B][H][d_k]
 *   (per-key) or [T][B][H] (scalar); beta: [T][B][H] (delta rule, else NULL):
 *   token t's block is laid out exactly as one lrs_decode_step's inputs.
 *   All device memory, fp32, 16-byte aligned.
 *   Supported: d_k and d_v in {64, 128} (group as for the state); other
 *   shapes return LRS_ERR_UNSUPPORTED. T = 0 is a no-op.
 * Ownership, errors and asynchrony as lrs_decode_step. */
lrs_status lrs_chunk_step(const lrs_state *st, void *state_codes, float *scales,
                          const uint8_t *prec_map, int32_t T, const float *q, const float *k,
                          const float *v, const float *gates, const float *beta, float *out,
                          uint64_t seed, uint64_t step, int32_t mode, void *stream);

/* The decode step with a Low-Rank Bypass buffer ([LRB/BDR] abstract, Low-Rank
 * Bypass). The sources fix no rank, period or threshold; this entry point
 * keeps rank-r fp32 factors of the step's updates beside the quantized state,
 * merges them every r-th step with the threshold RN(s_old / 2), and takes:
 *   - buffer L = U V^T of rank `rank` (1..8): U [B][H][rank][d_k] and
 *     V [B][H][rank][d_v], fp32 device memory owned by the caller, zero at
 *     the start, updated in place; step mod rank components are filled before
 *     the call, so calls must pass consecutive steps (the buffer empties at
 *     every step with step mod rank == rank - 1);
 *   - each step appends its rank-1 update k w^T to the buffer instead of the
 *     quantized state, and the older components decay with the state;
 *   - the quantized state is decayed (x = RN(g deq)) and requantized as in
 *     lrs_decode_step; the delta rule's k^T S and the output read the
 *     effective state deq + U V^T;
 *   - at the step that fills the buffer, every element of U V^T whose
 *     magnitude is at least half of its quantization step (old scale / 2) is
 *     added to x before the requantization, and the buffer is emptied.
 * Other arguments, layouts, errors and asynchrony as lrs_decode_step, including
 * states with one width per (head, scale group) (lrs_state_alloc_groups); d_k
 * and d_v in {64, 128}. */
lrs_status lrs_lrb_step(const lrs_state *st, void *state_codes, float *scales,
                        const uint8_t *prec_map, int32_t rank, float *U, float *V,
                        const float *q, const float *k, const float *v, const float *gates,
                        const float *beta, float *out, uint64_t seed, uint64_t step,
                        int32_t mode, void *stream);

/* The same step with HOST inputs and output: copies q, k, v, gates, beta
 * from host memory into device staging buffers owned by the state (allocated
 * on first use), runs lrs_decode_step on the state's own buffers on stream,
 * and copies out back to host memory on stream. Consecutive calls on a state
 * alternate between two staging buffers and make their input copies on a
 * stream of the state's own, so the input copies of one call overlap the
 * kernel and output copy of the previous one; the kernel waits for its
 * inputs. The input copies wait only for the previous use of their staging
 * buffer, not for other work on `stream`: the host input buffers must not be
 * written by work still pending there. Pinned host memory makes the copies
 * asynchronous; the host buffers must stay valid until the stream reaches the
 * end of the step. */
lrs_status lrs_decode_step_host(const lrs_state *st, const float *q_host, const float *k_host,
                                const float *v_host, const float *gates_host,
                                const float *beta_host, float *out_host, uint64_t seed,
                                uint64_t step, int32_t mode, void *stream);

/* lrs_decode_step_host without any device allocation. This entry point has no
 * counterpart in the method's sources. It is for callers that must not
 * allocate device memory when they step: a process whose device memory is
 * owned by another allocator or by a fixed pool sized at start-up (an
 * allocation behind its back can fail for lack of room, or break the pool's
 * accounting), and code on a latency-critical path that must not pay for a
 * cudaMalloc, which can synchronize the device. Its scratch -- a device error
 * word and the staging of q, k, v, gates, beta and out -- is a 32 MiB array
 * inside the library's image. Each device takes those 32 MiB when the
 * library's device code is loaded there: at the latest on this entry point's
 * first call on that device (CUDA loads modules lazily by default), and they
 * stay taken until the process exits. It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *   - Limit: the staging must fit: 256 + 16-byte-padded sizes of q, k
 *     ([B][H][d_k]), v, out ([B][H][d_v]), gates and beta must not exceed
 *     32 MiB; a larger step is rejected with LRS_ERR_UNSUPPORTED and nothing
 *     is launched. (B=256, H=32, 128x128 with per-key gates needs 20 MiB.)
 *   - The first call on a device looks up the array's device address (and
 *     may load the library's device code there, taking the 32 MiB): make one
 *     call on each device before sizing a fixed pool from the free memory.
 *   - Every call shares the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other threads) race and
 *     corrupt each other's inputs and outputs. Serialize them.
 *   - device_error_host (may be NULL) receives, asynchronously on stream, the
 *     device error bits of this call's kernel: 0 when none, else bit 0 = a
 *     wait timed out, bit 1 = the precision map did not fit the layout. The
 *     word is cleared at the start of each call; lrs_sync does not see it.
 * Arguments otherwise as lrs_decode_step_host (the state's own buffers are
 * stepped; host buffers pinned for asynchronous copies); the launch is the
 * same as lrs_decode_step's. */
lrs_status lrs_decode_step_host_noalloc(const lrs_state *st, const float *q_host,
                                        const float *k_host, const float *v_host,
                                        const float *gates_host, const float *beta_host,
                                        float *out_host, uint32_t *device_error_host,
                                        uint64_t seed, uint64_t step, int32_t mode,
                                        void *stream);

/* Quantize an fp32 state S [B][H][d_k][d_v] (device) into st with
 * round-to-nearest (new scales and codes exactly as in a step with x = S). */
lrs_status lrs_state_import_fp32(const lrs_state *st, const float *S, void *stream);

/* Dequantize st into S [B][H][d_k][d_v] (device): code * scale. */
lrs_status lrs_state_export_fp32(const lrs_state *st, float *S, void *stream);

/* Signed codes of st, one int8 per element, [B][H][d_k][d_v] (device). */
lrs_status lrs_state_export_codes(const lrs_state *st, int8_t *codes, void *stream);

/* Set st from signed codes [B][H][d_k][d_v] and scales [B][H][d_k/group][d_v]
 * (device). A code outside [-qmax, qmax] of its head is stored clamped and
 * LRS_ERR_DEVICE_RANGE is recorded. */
lrs_status lrs_state_import_codes(const lrs_state *st, const int8_t *codes,
                                  const float *scales, void *stream);

/* Copy the raw packed codes (st->code_bytes bytes) and the scales
 * (st->scale_count floats) to host memory (to_host != 0) or from it
 * (to_host == 0): a checkpoint of the state. Synchronous on stream. */
lrs_status lrs_state_copy_raw(const lrs_state *st, void *codes_host, float *scales_host,
                              int32_t to_host, void *stream);

/* The same update and output on an fp32 state S [B][H][d_k][d_v] (device),
 * in place, with no quantization: S <- x, out = x^T q. The uncompressed
 * baseline the quantized state is compared with. shape->group is ignored. */
lrs_status lrs_fp32_decode_step(const lrs_shape *shape, float *S, const float *q,
                                const float *k, const float *v, const float *gates,
                                const float *beta, float *out, void *stream);

/* Mean decay per head ([LoReS] decay-based mixed precision): decay is a
 * device fp32 tensor [outer][heads][inner] (outer = steps * batch, inner =
 * d_k for per-key decay or 1); means receives [heads] doubles in device
 * memory, accumulated in binary64. */
lrs_status lrs_decay_head_means(const float *decay, int64_t outer, int32_t heads, int64_t inner,
                                double *means, void *stream);

/* Precision map from per-head mean decays (host arrays): the n_int8 heads
 * with the largest mean decay -- the most slowly decaying -- get 8, the rest
 * 4; equal means go to the lower head index first. */
lrs_status lrs_precision_map(int32_t heads, const double *means_host, int32_t n_int8,
                             uint8_t *prec_map_host);

/* Wait for stream, then return and clear the first error recorded on the
 * device by this library's kernels (LRS_ERR_DEVICE_*), or LRS_OK.
 *
 * State after a device timeout. A kernel records LRS_ERR_DEVICE_TIMEOUT when
 * a wait for its own copies runs out (2 s in normal operation: far above any
 * legitimate wait; it means the device stalled). The kernel then stops: tiles
 * it had not reached keep their old codes and scales, tiles it finished hold
 * the new ones, and the tile it was working on may hold new codes and scales
 * in its first scale groups and old ones in the rest (the delta rule reads a
 * whole tile before writing it, so there a tile is either old or new; the
 * gated forms write each group as they go). The step's outputs are not
 * valid. The state as a whole is therefore neither the old nor the new state:
 * restore it from a checkpoint (lrs_state_copy_raw) before stepping again. */
lrs_status lrs_sync(void *stream);

/* Fault injection for tests of the error path: when enabled (nonzero), the
 * next lrs_decode_step issues no copies and gives each of its waits
 * timeout_us microseconds, so the kernel records LRS_ERR_DEVICE_TIMEOUT and
 * returns without touching the state. Disarms itself after that launch. */
lrs_status lrs_debug_inject_timeout(int32_t enable, int32_t timeout_us);

/* The same with a later wait running out: the next lrs_decode_step (or
 * lrs_decode_step_bf16) copies in only the first items_copied (tile, scale
 * group) items of each warp of its launch, and the wait for the next item
 * runs out after timeout_us microseconds. items_copied < 0 disarms. With the
 * gated update a warp's first tile may then be left part-way: its first
 * items_copied groups hold the new codes and scales, the rest the old ones
 * (see "State after a device timeout" at lrs_sync). */
lrs_status lrs_debug_inject_timeout_after(int32_t items_copied, int32_t timeout_us);

/* Message of the last error returned on this thread ("" if none). */
const char *lrs_last_error(void);

/* Static name of a status code. */
const char *lrs_status_string(lrs_status s);

/* LRS_VERSION of the built library. */
int32_t lrs_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LRS_H */
