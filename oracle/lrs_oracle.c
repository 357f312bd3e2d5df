/*
 * lrs_oracle.c -- plain CPU oracle for the quantized recurrent-state decode step.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU baseline). Independent of
 * the CUDA library; see lrs_oracle.h for the sources and the data layout.
 *
 * One step for one (batch, head) tile, in the order the method states it:
 *   1. dequantize  deq_ij = c_ij * s[i/group][j]                     [LoReS]
 *   2. update      x = g (.) deq + k w^T, where w = v (gated form) or
 *                  w = beta (v - alpha k^T deq) (delta rule)          [LRB/BDR]
 *   3. output      o_j = sum_i q_i x_ij over the updated state
 *   4. new scales  per (group of key rows, value column): absmax / qmax
 *                                                      [LoReS value-axis grouping]
 *   5. requantize  x * qmax / absmax rounded to an integer: to nearest,
 *                  stochastically [LoReS], or by Bounded Directional
 *                  Rounding [LRB/BDR]
 */
#include "lrs_oracle.h"

#include <float.h>
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs binary32 evaluation of float expressions (SSE, not x87)"
#endif

/* A column group whose largest magnitude is below this is stored as zero.
 * (Reading: the sources are silent; without it qmax/A overflows.) */
#define ORC_TINY 0x1p-100f

/* ---------------------------------------------------------------- hash --- */

uint64_t orc_splitmix64(uint64_t z)
{
    /* [SplitMix64]: advance by the golden gamma, then the variant-13 mixer. */
    z += 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t orc_hash(uint64_t seed, uint64_t step, uint32_t b, uint32_t h, uint32_t i, uint32_t j)
{
    uint64_t k0 = orc_splitmix64(seed);
    uint64_t k1 = orc_splitmix64(k0 ^ step);
    uint64_t k2 = orc_splitmix64(k1 ^ (((uint64_t)b << 32) | (uint64_t)h));
    return orc_splitmix64(k2 ^ (((uint64_t)i << 32) | (uint64_t)j));
}

float orc_uniform(uint64_t r)
{
    /* 23-bit integer, exactly representable, times 2^-23 (exact). */
    return (float)(r >> 41) * 0x1p-23f;
}

/* ---------------------------------------------------------- rounding --- */

/* Code for one element. x: the updated value; deq: its value before the
 * update (dequantized old state); inv = qmax / A; s_new: the new scale.
 * The value to round is the exact product y = x * inv (a product of two
 * binary32 numbers is exact in binary64); it is rounded once, to an integer. */
static int round_element(int mode, float x, float deq, float inv, float s_new, int qmax,
                         uint64_t r)
{
    double y = (double)x * (double)inv;
    double c;
    if (mode == ORC_ROUND_SR) {
        /* [LoReS] stochastic rounding: up with probability equal to the
         * fractional part, here y - floor(y) rounded once to binary32. */
        double f = floor(y);
        float fr = fmaf(x, inv, (float)-f);
        float u = orc_uniform(r);
        c = (u < fr) ? f + 1.0 : f;
    } else if (mode == ORC_ROUND_BDR) {
        /* [LRB/BDR]: the update is delta = x - deq; the move the stored value
         * would make is m = c0*s_new - deq. When the two point in opposite
         * directions the element is rounded toward the update instead. */
        double c0 = rint(y);
        float delta = x - deq;
        float m = (float)c0 * s_new - deq;
        if (delta > 0.0f && m < 0.0f)
            c = ceil(y);
        else if (delta < 0.0f && m > 0.0f)
            c = floor(y);
        else
            c = c0;
    } else {
        c = rint(y); /* round half to even (default rounding mode) */
    }
    if (c > (double)qmax) c = (double)qmax;
    if (c < (double)-qmax) c = (double)-qmax;
    return (int)c;
}

/* Steps 4 and 5 for one tile: new scales from x, then codes. deq may be NULL
 * for RTN (import). */
static void requantize_tile(int d_k, int d_v, int group, const int *qmaxs, int mode, const float *x,
                            const float *deq, int8_t *codes, float *scales, uint64_t seed,
                            uint64_t step, uint32_t b, uint32_t h)
{
    int G = d_k / group;
    for (int g = 0; g < G; ++g) {
        int qmax = qmaxs[g];
        for (int j = 0; j < d_v; ++j) {
            float A = 0.0f;
            for (int i = g * group; i < (g + 1) * group; ++i) {
                float a = fabsf(x[i * d_v + j]);
                if (a > A) A = a;
            }
            float s_new, inv;
            if (A < ORC_TINY) {
                s_new = 0.0f;
                inv = 0.0f;
            } else {
                s_new = A / (float)qmax;
                inv = (float)qmax / A;
            }
            scales[g * d_v + j] = s_new;
            for (int i = g * group; i < (g + 1) * group; ++i) {
                float xv = x[i * d_v + j];
                uint64_t r = 0;
                if (mode == ORC_ROUND_SR) r = orc_hash(seed, step, b, h, (uint32_t)i, (uint32_t)j);
                float dv = deq ? deq[i * d_v + j] : 0.0f;
                codes[i * d_v + j] = (int8_t)round_element(mode, xv, dv, inv, s_new, qmax, r);
            }
        }
    }
}

/* ------------------------------------------------------------ update --- */

/* Steps 2 and 3 for one tile, shared by the quantized and the fp32 step.
 * S_old [d_k][d_v] is the state before the update (deq for the quantized
 * state). Writes x and out. gate points at d_k values (per key) or one. */
static void update_tile(int d_k, int d_v, int update_kind, int gate_kind, const float *S_old,
                        const float *q, const float *k, const float *v, const float *gate,
                        float beta, float *w, float *x, float *out)
{
    if (update_kind == ORC_UPDATE_DELTA) {
        /* Delta rule alpha (I - beta k k^T) S + beta k v^T, written as
         * alpha S + k w^T with w = beta (v - alpha k^T S). */
        float alpha = gate[0];
        for (int j = 0; j < d_v; ++j) {
            float u = 0.0f;
            for (int i = 0; i < d_k; ++i) u = fmaf(k[i], S_old[i * d_v + j], u);
            float t = alpha * u;
            float d = v[j] - t;
            w[j] = beta * d;
        }
    } else {
        for (int j = 0; j < d_v; ++j) w[j] = v[j];
    }
    for (int i = 0; i < d_k; ++i) {
        float gi = (gate_kind == ORC_GATE_PER_KEY) ? gate[i] : gate[0];
        for (int j = 0; j < d_v; ++j) {
            float kw = k[i] * w[j];
            x[i * d_v + j] = fmaf(gi, S_old[i * d_v + j], kw);
        }
    }
    for (int j = 0; j < d_v; ++j) {
        float acc = 0.0f;
        for (int i = 0; i < d_k; ++i) acc = fmaf(q[i], x[i * d_v + j], acc);
        out[j] = acc;
    }
}

/* ------------------------------------------------------------ checks --- */

static int check_shape(int d_k, int d_v, int group, int update_kind, int gate_kind)
{
    if (d_k <= 0 || d_v <= 0 || group <= 0 || d_k % group != 0) return -1;
    if (update_kind != ORC_UPDATE_GATED && update_kind != ORC_UPDATE_DELTA) return -1;
    if (gate_kind != ORC_GATE_SCALAR && gate_kind != ORC_GATE_PER_KEY) return -1;
    if (update_kind == ORC_UPDATE_DELTA && gate_kind != ORC_GATE_SCALAR) return -1;
    return 0;
}

static int qmax_of(uint8_t bits)
{
    return bits == 8 ? 127 : (bits == 4 ? 7 : -1);
}

/* qmax of each scale group of head h: prec_map holds one width per head
 * (prec_groups == 1) or one per (head, group) in [H][G] order (prec_groups ==
 * G). Returns -1 if a width is neither 4 nor 8. */
static int head_qmaxs(const uint8_t *prec_map, int prec_groups, int G, int h, int *qmaxs)
{
    for (int g = 0; g < G; ++g) {
        uint8_t bits = prec_groups > 1 ? prec_map[(size_t)h * G + g] : prec_map[h];
        qmaxs[g] = qmax_of(bits);
        if (qmaxs[g] < 0) return -1;
    }
    return 0;
}

/* ---------------------------------------------------- tile-parallel loop --- */

typedef struct {
    int ntiles, d_k, d_v, group, update_kind, gate_kind, mode, nthreads, tid;
    int T; /* tokens per call (chunked update); 1 for a decode step */
    int prec_groups; /* 1: prec_map [H]; G: prec_map [H][G] */
    const int32_t *tile_b, *tile_h;
    const uint8_t *prec_map;
    int8_t *codes;
    float *scales, *S;
    const float *q, *k, *v, *gates, *beta;
    float *out;
    uint64_t seed, step;
    int quantized;
} work_t;

static void *worker(void *arg)
{
    work_t *W = (work_t *)arg;
    int d_k = W->d_k, d_v = W->d_v, G = d_k / W->group;
    size_t n = (size_t)d_k * d_v;
    float *deq = (float *)malloc(n * sizeof(float));
    float *x = (float *)malloc(n * sizeof(float));
    float *w = (float *)malloc((size_t)d_v * sizeof(float));
    int *qm = (int *)malloc((size_t)G * sizeof(int));
    if (!deq || !x || !w || !qm) {
        free(deq); free(x); free(w); free(qm);
        return (void *)1;
    }
    size_t gate_len = (W->gate_kind == ORC_GATE_PER_KEY) ? (size_t)d_k : 1;
    if (W->T > 1) {
        float *cur = (float *)malloc(n * sizeof(float));
        if (!cur) {
            free(deq); free(x); free(w); free(qm);
            return (void *)1;
        }
        size_t NT = (size_t)W->ntiles;
        for (int t = W->tid; t < W->ntiles; t += W->nthreads) {
            int8_t *c = W->codes + (size_t)t * n;
            float *s = W->scales + (size_t)t * G * d_v;
            head_qmaxs(W->prec_map, W->prec_groups, G, W->tile_h[t], qm);
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_v; ++j)
                    deq[i * d_v + j] = (float)c[i * d_v + j] * s[(i / W->group) * d_v + j];
            memcpy(cur, deq, n * sizeof(float));
            /* the tokens in order, each an update of the fp32 state and its output */
            for (int tok = 0; tok < W->T; ++tok) {
                size_t row = (size_t)tok * NT + (size_t)t;
                update_tile(d_k, d_v, W->update_kind, W->gate_kind, cur, W->q + row * d_k,
                            W->k + row * d_k, W->v + row * d_v, W->gates + row * gate_len,
                            W->beta ? W->beta[row] : 0.0f, w, x, W->out + row * d_v);
                memcpy(cur, x, n * sizeof(float));
            }
            /* one requantization at the chunk's end; BDR compares with the
             * state at the chunk's start */
            requantize_tile(d_k, d_v, W->group, qm, W->mode, cur, deq, c, s, W->seed, W->step,
                            (uint32_t)W->tile_b[t], (uint32_t)W->tile_h[t]);
        }
        free(cur); free(deq); free(x); free(w); free(qm);
        return NULL;
    }
    for (int t = W->tid; t < W->ntiles; t += W->nthreads) {
        const float *q = W->q + (size_t)t * d_k;
        const float *k = W->k + (size_t)t * d_k;
        const float *v = W->v + (size_t)t * d_v;
        const float *gate = W->gates + (size_t)t * gate_len;
        float beta = W->beta ? W->beta[t] : 0.0f;
        float *out = W->out + (size_t)t * d_v;
        if (W->quantized) {
            int8_t *c = W->codes + (size_t)t * n;
            float *s = W->scales + (size_t)t * G * d_v;
            head_qmaxs(W->prec_map, W->prec_groups, G, W->tile_h[t], qm);
            /* 1. dequantize with the value-axis group scales */
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_v; ++j)
                    deq[i * d_v + j] = (float)c[i * d_v + j] * s[(i / W->group) * d_v + j];
            /* 2-3. update and output */
            update_tile(d_k, d_v, W->update_kind, W->gate_kind, deq, q, k, v, gate, beta, w, x, out);
            /* 4-5. new scales and codes */
            requantize_tile(d_k, d_v, W->group, qm, W->mode, x, deq, c, s, W->seed, W->step,
                            (uint32_t)W->tile_b[t], (uint32_t)W->tile_h[t]);
        } else {
            float *S = W->S + (size_t)t * n;
            update_tile(d_k, d_v, W->update_kind, W->gate_kind, S, q, k, v, gate, beta, w, x, out);
            memcpy(S, x, n * sizeof(float));
        }
    }
    free(deq); free(x); free(w); free(qm);
    return NULL;
}

static int run_tiles(work_t *proto, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > proto->ntiles) nthreads = proto->ntiles > 0 ? proto->ntiles : 1;
    work_t *ws = (work_t *)calloc((size_t)nthreads, sizeof(work_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!ws || !th) { free(ws); free(th); return -2; }
    int rc = 0;
    for (int t = 0; t < nthreads; ++t) {
        ws[t] = *proto;
        ws[t].tid = t;
        ws[t].nthreads = nthreads;
    }
    if (nthreads == 1) {
        if (worker(&ws[0]) != NULL) rc = -2;
    } else {
        int started = 0;
        for (int t = 0; t < nthreads; ++t) {
            if (pthread_create(&th[t], NULL, worker, &ws[t]) != 0) { rc = -2; break; }
            ++started;
        }
        for (int t = 0; t < started; ++t) {
            void *ret = NULL;
            pthread_join(th[t], &ret);
            if (ret != NULL) rc = -2;
        }
    }
    free(ws); free(th);
    return rc;
}

/* ------------------------------------------------------------ public --- */

/* Validation shared by the quantized entry points: every tile's head has
 * valid widths in prec_map (per head, or per (head, group)). */
static int check_prec(int ntiles, const int32_t *tile_h, const uint8_t *prec_map, int prec_groups,
                      int G)
{
    int *qm = (int *)malloc((size_t)G * sizeof(int));
    if (!qm) return -2;
    int rc = 0;
    for (int t = 0; t < ntiles && rc == 0; ++t)
        if (tile_h[t] < 0 || head_qmaxs(prec_map, prec_groups, G, tile_h[t], qm) != 0) rc = -1;
    free(qm);
    return rc;
}

static int step_impl(int ntiles, const int32_t *tile_b, const int32_t *tile_h, int d_k, int d_v,
                     int group, int update_kind, int gate_kind, int mode, const uint8_t *prec_map,
                     int prec_groups, int8_t *codes, float *scales, int T, const float *q,
                     const float *k, const float *v, const float *gates, const float *beta,
                     float *out, uint64_t seed, uint64_t step, int nthreads)
{
    if (T < 1) return -1;
    if (ntiles < 0 || check_shape(d_k, d_v, group, update_kind, gate_kind) != 0) return -1;
    if (mode != ORC_ROUND_RTN && mode != ORC_ROUND_SR && mode != ORC_ROUND_BDR) return -1;
    if (ntiles == 0) return 0;
    if (!tile_b || !tile_h || !prec_map || !codes || !scales || !q || !k || !v || !gates || !out)
        return -1;
    if (update_kind == ORC_UPDATE_DELTA && !beta) return -1;
    int rc = check_prec(ntiles, tile_h, prec_map, prec_groups, d_k / group);
    if (rc != 0) return rc;
    work_t W;
    memset(&W, 0, sizeof W);
    W.ntiles = ntiles; W.d_k = d_k; W.d_v = d_v; W.group = group;
    W.update_kind = update_kind; W.gate_kind = gate_kind; W.mode = mode; W.T = T;
    W.prec_groups = prec_groups;
    W.tile_b = tile_b; W.tile_h = tile_h; W.prec_map = prec_map;
    W.codes = codes; W.scales = scales;
    W.q = q; W.k = k; W.v = v; W.gates = gates; W.beta = beta; W.out = out;
    W.seed = seed; W.step = step; W.quantized = 1;
    return run_tiles(&W, nthreads);
}

int orc_step(int ntiles, const int32_t *tile_b, const int32_t *tile_h, int d_k, int d_v,
             int group, int update_kind, int gate_kind, int mode, const uint8_t *prec_map,
             int8_t *codes, float *scales, const float *q, const float *k, const float *v,
             const float *gates, const float *beta, float *out, uint64_t seed, uint64_t step,
             int nthreads)
{
    return step_impl(ntiles, tile_b, tile_h, d_k, d_v, group, update_kind, gate_kind, mode,
                     prec_map, 1, codes, scales, 1, q, k, v, gates, beta, out, seed, step,
                     nthreads);
}

int orc_step_pg(int ntiles, const int32_t *tile_b, const int32_t *tile_h, int d_k, int d_v,
                int group, int update_kind, int gate_kind, int mode, const uint8_t *prec_map,
                int8_t *codes, float *scales, const float *q, const float *k, const float *v,
                const float *gates, const float *beta, float *out, uint64_t seed, uint64_t step,
                int nthreads)
{
    if (group <= 0) return -1;
    return step_impl(ntiles, tile_b, tile_h, d_k, d_v, group, update_kind, gate_kind, mode,
                     prec_map, d_k / group, codes, scales, 1, q, k, v, gates, beta, out, seed,
                     step, nthreads);
}

int orc_chunk_step(int ntiles, const int32_t *tile_b, const int32_t *tile_h, int d_k, int d_v,
                   int group, int update_kind, int gate_kind, int mode, const uint8_t *prec_map,
                   int8_t *codes, float *scales, int T, const float *q, const float *k,
                   const float *v, const float *gates, const float *beta, float *out,
                   uint64_t seed, uint64_t step, int nthreads)
{
    return step_impl(ntiles, tile_b, tile_h, d_k, d_v, group, update_kind, gate_kind, mode,
                     prec_map, 1, codes, scales, T, q, k, v, gates, beta, out, seed, step,
                     nthreads);
}

int orc_chunk_step_pg(int ntiles, const int32_t *tile_b, const int32_t *tile_h, int d_k, int d_v,
                      int group, int update_kind, int gate_kind, int mode, const uint8_t *prec_map,
                      int8_t *codes, float *scales, int T, const float *q, const float *k,
                      const float *v, const float *gates, const float *beta, float *out,
                      uint64_t seed, uint64_t step, int nthreads)
{
    if (group <= 0) return -1;
    return step_impl(ntiles, tile_b, tile_h, d_k, d_v, group, update_kind, gate_kind, mode,
                     prec_map, d_k / group, codes, scales, T, q, k, v, gates, beta, out, seed,
                     step, nthreads);
}

/* ------------------------------------------------- Low-Rank Bypass --- */

/* [LRB/BDR] abstract, Low-Rank Bypass. The sources give neither the rank,
 * the merge period nor the threshold; the readings taken here (rank-r fp32
 * factors, a merge every r-th step, threshold RN(s_old / 2)):
 *   - buffer L = sum_l U_l V_l^T, l < r, U_l in R^{d_k}, V_l in R^{d_v}, fp32;
 *     the effective state is deq(S_q) + L;
 *   - each step appends the step's rank-1 update k w^T as the next component
 *     (U_m = k, V_m = w, m = step mod r components were already there) instead
 *     of adding it to the quantized state, and decays the older components
 *     with the state (U_l <- g * U_l, per key or scalar);
 *   - the quantized part is decayed and requantized every step as before;
 *   - every r-th step (when the buffer is full) the dense product M = U V^T
 *     is formed and every element with |M_ij| >= s_ij / 2 (half the element's
 *     quantization step before the step) is added to the state before it is
 *     requantized; the buffer is then emptied (the smaller elements, which
 *     rounding would have removed from the state too, are dropped);
 *   - the delta rule reads k^T of the effective state: u = k^T deq +
 *     sum_l (k . U_l) V_l;
 *   - the output is read from the effective state after the step:
 *     o = x^T q + sum_l (q . U_l) V_l, before any merge.
 * Order of operations (one rounding per operation, as in the decode step):
 *   e_l = sum_i k_i U_li (key order, undecayed U)      [delta rule only]
 *   u_j = sum_i k_i deq_ij (key order), then u_j = fma(e_l, V_lj, u_j), l order
 *   w_j = RN(beta RN(v_j - RN(alpha u_j)))  (gated: w = v)
 *   U_l <- RN(g_i U_li) for l < m;  U_m = k, V_m = w
 *   x_ij = RN(g_i deq_ij)
 *   o_j = sum_i q_i x_ij (key order), then f_l = sum_i q_i U_li (key order)
 *         and o_j = fma(f_l, V_lj, o_j), l order, l <= m
 *   merge (m + 1 == r): M_ij = fma chain over l of U_li V_lj from 0;
 *         if M_ij != 0 and |M_ij| >= RN(0.5 s_old): x_ij = RN(x_ij + M_ij);
 *         U, V <- 0
 *   then new scales and codes from x by the rounding mode (BDR: update x - deq).
 * x_out (may be NULL) receives x before rounding, for the pins. */
static void lrb_tile(int d_k, int d_v, int group, const int *qmaxs, int update_kind,
                     int gate_kind, int mode, int r, int m, int8_t *c, float *s, float *U,
                     float *V, const float *q, const float *k, const float *v, const float *gate,
                     float beta, float *out, float *deq, float *x, float *w, float *M,
                     uint64_t seed, uint64_t step, uint32_t b, uint32_t h, float *x_out)
{
    for (int i = 0; i < d_k; ++i)
        for (int j = 0; j < d_v; ++j)
            deq[i * d_v + j] = (float)c[i * d_v + j] * s[(i / group) * d_v + j];
    float alpha = gate[0];
    if (update_kind == ORC_UPDATE_DELTA) {
        for (int j = 0; j < d_v; ++j) {
            float u = 0.0f;
            for (int i = 0; i < d_k; ++i) u = fmaf(k[i], deq[i * d_v + j], u);
            w[j] = u;
        }
        for (int l = 0; l < m; ++l) {
            float e = 0.0f;
            for (int i = 0; i < d_k; ++i) e = fmaf(k[i], U[l * d_k + i], e);
            for (int j = 0; j < d_v; ++j) w[j] = fmaf(e, V[l * d_v + j], w[j]);
        }
        for (int j = 0; j < d_v; ++j) {
            float t = alpha * w[j];
            float d = v[j] - t;
            w[j] = beta * d;
        }
    } else {
        for (int j = 0; j < d_v; ++j) w[j] = v[j];
    }
    for (int l = 0; l < m; ++l)
        for (int i = 0; i < d_k; ++i) {
            float gi = (gate_kind == ORC_GATE_PER_KEY) ? gate[i] : alpha;
            U[l * d_k + i] = gi * U[l * d_k + i];
        }
    for (int i = 0; i < d_k; ++i) U[m * d_k + i] = k[i];
    for (int j = 0; j < d_v; ++j) V[m * d_v + j] = w[j];
    for (int i = 0; i < d_k; ++i) {
        float gi = (gate_kind == ORC_GATE_PER_KEY) ? gate[i] : alpha;
        for (int j = 0; j < d_v; ++j) x[i * d_v + j] = gi * deq[i * d_v + j];
    }
    for (int j = 0; j < d_v; ++j) {
        float acc = 0.0f;
        for (int i = 0; i < d_k; ++i) acc = fmaf(q[i], x[i * d_v + j], acc);
        out[j] = acc;
    }
    for (int l = 0; l <= m; ++l) {
        float f = 0.0f;
        for (int i = 0; i < d_k; ++i) f = fmaf(q[i], U[l * d_k + i], f);
        for (int j = 0; j < d_v; ++j) out[j] = fmaf(f, V[l * d_v + j], out[j]);
    }
    if (m + 1 == r) {
        for (int i = 0; i < d_k; ++i)
            for (int j = 0; j < d_v; ++j) {
                float acc = 0.0f;
                for (int l = 0; l < r; ++l) acc = fmaf(U[l * d_k + i], V[l * d_v + j], acc);
                M[i * d_v + j] = acc;
            }
        for (int i = 0; i < d_k; ++i)
            for (int j = 0; j < d_v; ++j) {
                float mij = M[i * d_v + j];
                float half = 0.5f * s[(i / group) * d_v + j];
                if (mij != 0.0f && fabsf(mij) >= half) x[i * d_v + j] = x[i * d_v + j] + mij;
            }
        memset(U, 0, (size_t)r * d_k * sizeof(float));
        memset(V, 0, (size_t)r * d_v * sizeof(float));
    }
    if (x_out) memcpy(x_out, x, (size_t)d_k * d_v * sizeof(float));
    requantize_tile(d_k, d_v, group, qmaxs, mode, x, deq, c, s, seed, step, b, h);
}

static int lrb_impl(int ntiles, const int32_t *tile_b, const int32_t *tile_h, int d_k, int d_v,
                    int group, int update_kind, int gate_kind, int mode, const uint8_t *prec_map,
                    int prec_groups, int8_t *codes, float *scales, int rank, float *U, float *V,
                    const float *q, const float *k, const float *v, const float *gates,
                    const float *beta, float *out, uint64_t seed, uint64_t step, float *x_out)
{
    if (ntiles < 0 || check_shape(d_k, d_v, group, update_kind, gate_kind) != 0) return -1;
    if (mode != ORC_ROUND_RTN && mode != ORC_ROUND_SR && mode != ORC_ROUND_BDR) return -1;
    if (rank < 1) return -1;
    if (ntiles == 0) return 0;
    if (!tile_b || !tile_h || !prec_map || !codes || !scales || !U || !V || !q || !k || !v ||
        !gates || !out)
        return -1;
    if (update_kind == ORC_UPDATE_DELTA && !beta) return -1;
    int G = d_k / group;
    int rc = check_prec(ntiles, tile_h, prec_map, prec_groups, G);
    if (rc != 0) return rc;
    size_t n = (size_t)d_k * d_v;
    float *deq = (float *)malloc(n * sizeof(float));
    float *x = (float *)malloc(n * sizeof(float));
    float *M = (float *)malloc(n * sizeof(float));
    float *w = (float *)malloc((size_t)d_v * sizeof(float));
    int *qm = (int *)malloc((size_t)G * sizeof(int));
    if (!deq || !x || !M || !w || !qm) {
        free(deq); free(x); free(M); free(w); free(qm);
        return -2;
    }
    int m = (int)(step % (uint64_t)rank);
    size_t gate_len = (gate_kind == ORC_GATE_PER_KEY) ? (size_t)d_k : 1;
    for (int t = 0; t < ntiles; ++t) {
        head_qmaxs(prec_map, prec_groups, G, tile_h[t], qm);
        lrb_tile(d_k, d_v, group, qm, update_kind, gate_kind, mode, rank, m, codes + t * n,
                 scales + (size_t)t * G * d_v, U + (size_t)t * rank * d_k,
                 V + (size_t)t * rank * d_v, q + (size_t)t * d_k, k + (size_t)t * d_k,
                 v + (size_t)t * d_v, gates + t * gate_len, beta ? beta[t] : 0.0f,
                 out + (size_t)t * d_v, deq, x, w, M, seed, step, (uint32_t)tile_b[t],
                 (uint32_t)tile_h[t], x_out ? x_out + t * n : NULL);
    }
    free(deq); free(x); free(M); free(w); free(qm);
    return 0;
}

int orc_lrb_step(int ntiles, const int32_t *tile_b, const int32_t *tile_h, int d_k, int d_v,
                 int group, int update_kind, int gate_kind, int mode, const uint8_t *prec_map,
                 int8_t *codes, float *scales, int rank, float *U, float *V, const float *q,
                 const float *k, const float *v, const float *gates, const float *beta,
                 float *out, uint64_t seed, uint64_t step, float *x_out)
{
    return lrb_impl(ntiles, tile_b, tile_h, d_k, d_v, group, update_kind, gate_kind, mode,
                    prec_map, 1, codes, scales, rank, U, V, q, k, v, gates, beta, out, seed, step,
                    x_out);
}

int orc_lrb_step_pg(int ntiles, const int32_t *tile_b, const int32_t *tile_h, int d_k, int d_v,
                    int group, int update_kind, int gate_kind, int mode, const uint8_t *prec_map,
                    int8_t *codes, float *scales, int rank, float *U, float *V, const float *q,
                    const float *k, const float *v, const float *gates, const float *beta,
                    float *out, uint64_t seed, uint64_t step, float *x_out)
{
    if (d_k <= 0 || group <= 0 || d_k % group != 0) return -1;
    return lrb_impl(ntiles, tile_b, tile_h, d_k, d_v, group, update_kind, gate_kind, mode,
                    prec_map, d_k / group, codes, scales, rank, U, V, q, k, v, gates, beta, out,
                    seed, step, x_out);
}

uint16_t orc_bf16_rne(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    uint32_t sign = u & 0x80000000u;
    if (isnan(x)) return (uint16_t)((sign >> 16) | 0x7FC0u);
    /* |x| lies between the bfloat16 values with patterns lo (the upper half
     * of x's pattern, i.e. x truncated toward zero) and lo + 1 (the next one
     * away from zero; past the largest finite value that is infinity). The
     * dropped half of the pattern says where: below 0x8000 nearer lo, above
     * nearer lo + 1, equal a tie, which goes to the even pattern. */
    uint32_t lo = u >> 16;
    uint32_t rest = u & 0xFFFFu;
    uint32_t r;
    if (rest < 0x8000u)
        r = lo;
    else if (rest > 0x8000u)
        r = lo + 1;
    else
        r = (lo & 1u) ? lo + 1 : lo;
    return (uint16_t)r;
}

void orc_bf16_rne_array(int64_t n, const float *x, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_rne(x[i]);
}

int orc_fp32_step(int ntiles, int d_k, int d_v, int update_kind, int gate_kind, float *S,
                  const float *q, const float *k, const float *v, const float *gates,
                  const float *beta, float *out, int nthreads)
{
    if (ntiles < 0 || check_shape(d_k, d_v, d_k, update_kind, gate_kind) != 0) return -1;
    if (ntiles == 0) return 0;
    if (!S || !q || !k || !v || !gates || !out) return -1;
    if (update_kind == ORC_UPDATE_DELTA && !beta) return -1;
    work_t W;
    memset(&W, 0, sizeof W);
    W.ntiles = ntiles; W.d_k = d_k; W.d_v = d_v; W.group = d_k;
    W.update_kind = update_kind; W.gate_kind = gate_kind;
    W.S = S; W.q = q; W.k = k; W.v = v; W.gates = gates; W.beta = beta; W.out = out;
    W.quantized = 0;
    return run_tiles(&W, nthreads);
}

static int import_impl(int ntiles, const int32_t *tile_h, int d_k, int d_v, int group,
                       const uint8_t *prec_map, int prec_groups, const float *S0, int8_t *codes,
                       float *scales)
{
    if (ntiles < 0 || check_shape(d_k, d_v, group, ORC_UPDATE_GATED, ORC_GATE_SCALAR) != 0)
        return -1;
    if (ntiles == 0) return 0;
    if (!tile_h || !prec_map || !S0 || !codes || !scales) return -1;
    size_t n = (size_t)d_k * d_v;
    int G = d_k / group;
    int *qm = (int *)malloc((size_t)G * sizeof(int));
    if (!qm) return -2;
    int rc = 0;
    for (int t = 0; t < ntiles && rc == 0; ++t) {
        if (tile_h[t] < 0 || head_qmaxs(prec_map, prec_groups, G, tile_h[t], qm) != 0) {
            rc = -1;
            break;
        }
        requantize_tile(d_k, d_v, group, qm, ORC_ROUND_RTN, S0 + (size_t)t * n, NULL,
                        codes + (size_t)t * n, scales + (size_t)t * G * d_v, 0, 0, 0, 0);
    }
    free(qm);
    return rc;
}

int orc_import(int ntiles, const int32_t *tile_h, int d_k, int d_v, int group,
               const uint8_t *prec_map, const float *S0, int8_t *codes, float *scales)
{
    return import_impl(ntiles, tile_h, d_k, d_v, group, prec_map, 1, S0, codes, scales);
}

int orc_import_pg(int ntiles, const int32_t *tile_h, int d_k, int d_v, int group,
                  const uint8_t *prec_map, const float *S0, int8_t *codes, float *scales)
{
    if (group <= 0) return -1;
    return import_impl(ntiles, tile_h, d_k, d_v, group, prec_map, d_k / group, S0, codes, scales);
}

int orc_dequant(int ntiles, int d_k, int d_v, int group, const int8_t *codes,
                const float *scales, float *S)
{
    if (ntiles < 0 || check_shape(d_k, d_v, group, ORC_UPDATE_GATED, ORC_GATE_SCALAR) != 0)
        return -1;
    size_t n = (size_t)d_k * d_v;
    int G = d_k / group;
    for (int t = 0; t < ntiles; ++t)
        for (int i = 0; i < d_k; ++i)
            for (int j = 0; j < d_v; ++j)
                S[t * n + (size_t)i * d_v + j] = (float)codes[t * n + (size_t)i * d_v + j] *
                                                 scales[(size_t)t * G * d_v + (i / group) * d_v + j];
    return 0;
}

void orc_decay_means(int64_t outer, int heads, int64_t inner, const float *decay, double *means)
{
    for (int h = 0; h < heads; ++h) {
        double sum = 0.0;
        for (int64_t o = 0; o < outer; ++o)
            for (int64_t c = 0; c < inner; ++c)
                sum += (double)decay[(o * heads + h) * inner + c];
        means[h] = sum / (double)(outer * inner);
    }
}

int orc_precision_map(int heads, const double *means, int n_int8, uint8_t *prec_map)
{
    if (heads <= 0 || n_int8 < 0 || n_int8 > heads) return -1;
    /* [LoReS] decay-based mixed precision: rank heads by mean decay, largest
     * first (slowest decay), ties to the lower index; selection by repeated
     * scan keeps this obviously correct for the head counts involved. */
    for (int h = 0; h < heads; ++h) prec_map[h] = 4;
    for (int n = 0; n < n_int8; ++n) {
        int best = -1;
        for (int h = 0; h < heads; ++h) {
            if (prec_map[h] == 8) continue;
            if (best < 0 || means[h] > means[best]) best = h;
        }
        prec_map[best] = 8;
    }
    return 0;
}

/* ------------------------------------------ BDR reading study (additive) --- */

int orc_bdr_additive_step(int ntiles, int d_k, int d_v, int group, int qmax, int8_t *codes,
                          float *scales, const float *q, const float *k, const float *v,
                          const float *gates, float *out)
{
    if (ntiles < 0 || d_k <= 0 || d_v <= 0 || group <= 0 || d_k % group != 0) return -1;
    if (qmax != 127 && qmax != 7) return -1;
    size_t n = (size_t)d_k * d_v;
    int G = d_k / group;
    float *deq = (float *)malloc(n * sizeof(float));
    float *kw = (float *)malloc(n * sizeof(float));
    float *x = (float *)malloc(n * sizeof(float));
    if (!deq || !kw || !x) {
        free(deq); free(kw); free(x);
        return -2;
    }
    for (int t = 0; t < ntiles; ++t) {
        int8_t *c = codes + (size_t)t * n;
        float *s = scales + (size_t)t * G * d_v;
        const float *qt = q + (size_t)t * d_k, *kt = k + (size_t)t * d_k;
        const float *vt = v + (size_t)t * d_v, *gt = gates + (size_t)t * d_k;
        /* dequantize, update (w = v), output -- as orc_step's gated form */
        for (int i = 0; i < d_k; ++i)
            for (int j = 0; j < d_v; ++j) {
                deq[i * d_v + j] = (float)c[i * d_v + j] * s[(i / group) * d_v + j];
                kw[i * d_v + j] = kt[i] * vt[j];
                x[i * d_v + j] = fmaf(gt[i], deq[i * d_v + j], kw[i * d_v + j]);
            }
        for (int j = 0; j < d_v; ++j) {
            float acc = 0.0f;
            for (int i = 0; i < d_k; ++i) acc = fmaf(qt[i], x[i * d_v + j], acc);
            out[(size_t)t * d_v + j] = acc;
        }
        /* new scales as orc_step; codes with the additive term as the update */
        for (int g = 0; g < G; ++g)
            for (int j = 0; j < d_v; ++j) {
                float A = 0.0f;
                for (int i = g * group; i < (g + 1) * group; ++i)
                    if (fabsf(x[i * d_v + j]) > A) A = fabsf(x[i * d_v + j]);
                float s_new = 0.0f, inv = 0.0f;
                if (A >= ORC_TINY) {
                    s_new = A / (float)qmax;
                    inv = (float)qmax / A;
                }
                s[g * d_v + j] = s_new;
                for (int i = g * group; i < (g + 1) * group; ++i) {
                    size_t e = (size_t)i * d_v + j;
                    double y = (double)x[e] * (double)inv;
                    double c0 = rint(y), cc = c0;
                    float m = (float)c0 * s_new - deq[e];
                    if (kw[e] > 0.0f && m < 0.0f)
                        cc = ceil(y);
                    else if (kw[e] < 0.0f && m > 0.0f)
                        cc = floor(y);
                    if (cc > qmax) cc = qmax;
                    if (cc < -qmax) cc = -qmax;
                    c[e] = (int8_t)cc;
                }
            }
    }
    free(deq); free(kw); free(x);
    return 0;
}

