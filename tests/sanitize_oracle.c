/*
 * sanitize_oracle.c -- test helper: drives every oracle entry point on small
 * seeded inputs (both update forms, both gate kinds, every rounding mode,
 * per-head and per-group widths, chunks of 1..3 tokens, bypass ranks 1..3,
 * shapes with ragged tile counts) so that a build with AddressSanitizer and
 * UndefinedBehaviorSanitizer can check the oracle's memory accesses and
 * integer arithmetic. Built and run by tests/test_sanitizers.py. Exits 0 when
 * every call accepted its arguments; the sanitizers abort on a finding.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "lrs_oracle.h"

static uint64_t rng = 0x243F6A8885A308D3ull;

static float frand(void)
{
    rng ^= rng << 13;
    rng ^= rng >> 7;
    rng ^= rng << 17;
    return (float)((double)(rng >> 11) * 0x1p-53) * 2.0f - 1.0f;
}

static float *fill(size_t n, float lo, float hi)
{
    float *a = (float *)malloc(n * sizeof(float) + 1);
    for (size_t i = 0; i < n; ++i) a[i] = lo + (hi - lo) * (0.5f + 0.5f * frand());
    return a;
}

static int fails = 0;

static void expect(int rc, const char *what)
{
    if (rc != 0) {
        fprintf(stderr, "%s returned %d\n", what, rc);
        ++fails;
    }
}

static void run_case(int B, int H, int d_k, int d_v, int group, int upd, int gate, int pergroup)
{
    const int n = B * H, G = d_k / group;
    const size_t nk = (size_t)n * d_k, nv = (size_t)n * d_v, ns = (size_t)n * d_k * d_v;
    int32_t *tb = (int32_t *)malloc(n * sizeof(int32_t));
    int32_t *th = (int32_t *)malloc(n * sizeof(int32_t));
    for (int t = 0; t < n; ++t) {
        tb[t] = t / H;
        th[t] = t % H;
    }
    const int npm = pergroup ? H * G : H;
    uint8_t *pm = (uint8_t *)malloc(npm);
    for (int i = 0; i < npm; ++i) pm[i] = (i % 3 == 1) ? 4 : 8;
    float *S0 = fill(ns, -0.05f, 0.05f);
    int8_t *codes = (int8_t *)malloc(ns);
    float *scales = (float *)malloc((size_t)n * G * d_v * sizeof(float));
    float *out = (float *)malloc(3 * nv * sizeof(float));
    const size_t ng = gate ? nk : (size_t)n;
    for (int mode = 0; mode < 3; ++mode) {
        expect((pergroup ? orc_import_pg : orc_import)(n, th, d_k, d_v, group, pm, S0, codes,
                                                       scales),
               "import");
        for (int T = 1; T <= 3; ++T) {
            float *q = fill(T * nk, -1, 1), *k = fill(T * nk, -1, 1), *v = fill(T * nv, -1, 1);
            float *g = fill(T * ng, 0.5f, 1.0f), *beta = fill((size_t)T * n, 0.1f, 0.9f);
            const float *bp = upd ? beta : NULL;
            if (T == 1)
                expect((pergroup ? orc_step_pg : orc_step)(n, tb, th, d_k, d_v, group, upd, gate,
                                                           mode, pm, codes, scales, q, k, v, g,
                                                           bp, out, 7, 3, 2),
                       "step");
            expect((pergroup ? orc_chunk_step_pg : orc_chunk_step)(
                       n, tb, th, d_k, d_v, group, upd, gate, mode, pm, codes, scales, T, q, k,
                       v, g, bp, out, 7, 4, 2),
                   "chunk");
            free(q); free(k); free(v); free(g); free(beta);
        }
        for (int rank = 1; rank <= 3; ++rank) {
            float *U = (float *)calloc((size_t)n * rank * d_k, sizeof(float));
            float *V = (float *)calloc((size_t)n * rank * d_v, sizeof(float));
            float *x = (float *)malloc(ns * sizeof(float));
            for (int step = 0; step < 2 * rank; ++step) {
                float *q = fill(nk, -1, 1), *k = fill(nk, -1, 1), *v = fill(nv, -1, 1);
                float *g = fill(ng, 0.5f, 1.0f), *beta = fill((size_t)n, 0.1f, 0.9f);
                expect((pergroup ? orc_lrb_step_pg : orc_lrb_step)(
                           n, tb, th, d_k, d_v, group, upd, gate, mode, pm, codes, scales, rank,
                           U, V, q, k, v, g, upd ? beta : NULL, out, 9, (uint64_t)step, x),
                       "lrb");
                free(q); free(k); free(v); free(g); free(beta);
            }
            free(U); free(V); free(x);
        }
    }
    if (!pergroup && gate) {
        float *q = fill(nk, -1, 1), *k = fill(nk, -1, 1), *v = fill(nv, -1, 1);
        float *g = fill(nk, 0.5f, 1.0f);
        int8_t *c = (int8_t *)malloc(ns);
        memcpy(c, codes, ns);
        for (int i = 0; i < n * G * d_v; ++i) scales[i] = scales[i] > 0 ? scales[i] : 0.01f;
        expect(orc_bdr_additive_step(n, d_k, d_v, group, 127, c, scales, q, k, v, g, out),
               "bdr_additive");
        free(q); free(k); free(v); free(g); free(c);
    }
    float *S = (float *)malloc(ns * sizeof(float));
    expect(orc_dequant(n, d_k, d_v, group, codes, scales, S), "dequant");
    float *q = fill(nk, -1, 1), *k = fill(nk, -1, 1), *v = fill(nv, -1, 1);
    float *g = fill(ng, 0.5f, 1.0f), *beta = fill((size_t)n, 0.1f, 0.9f);
    expect(orc_fp32_step(n, d_k, d_v, upd, gate, S, q, k, v, g, upd ? beta : NULL, out, 2),
           "fp32");
    free(S); free(q); free(k); free(v); free(g); free(beta);
    free(tb); free(th); free(pm); free(S0); free(codes); free(scales); free(out);
}

int main(void)
{
    /* shapes: ragged tile counts, small and large groups, d_v 64 and 128 */
    run_case(3, 5, 32, 64, 16, 0, 1, 0);
    run_case(2, 3, 64, 128, 32, 1, 0, 0);
    run_case(1, 7, 64, 64, 64, 0, 0, 0);
    run_case(2, 2, 64, 128, 16, 0, 1, 1);
    run_case(3, 2, 32, 64, 16, 1, 0, 1);
    /* the hash and the decay map */
    uint64_t acc = 0;
    for (uint32_t i = 0; i < 1000; ++i) acc ^= orc_hash(i, 2 * i, i, i + 1, i % 128, i % 64);
    float *decay = fill(6 * 5 * 8, 0.5f, 1.0f);
    double means[5];
    uint8_t pm[5];
    orc_decay_means(6, 5, 8, decay, means);
    expect(orc_precision_map(5, means, 2, pm), "precision_map");
    free(decay);
    printf("sanitized oracle run: %d failures (hash %llx)\n", fails, (unsigned long long)acc);
    return fails != 0;
}
