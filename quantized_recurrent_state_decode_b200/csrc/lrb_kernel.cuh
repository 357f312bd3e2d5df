// lrb_kernel.cuh -- the decode step with a Low-Rank Bypass buffer.
//
// "Preserving Updates in Low-Bit Recurrent State Quantization" (abstract,
// Low-Rank Bypass). The readings (the sources give neither rank, period nor
// threshold): each
// step's rank-1 update k w^T is appended to a rank-r fp32 buffer L = U V^T
// (U [r][d_k], V [r][d_v] per tile) instead of the quantized state; older
// components decay with the state; the delta rule and the output read the
// effective state deq + L; every r-th step (step mod r == r - 1) the elements
// of L of at least half a quantization step (|L_ij| >= s_ij / 2, old scale)
// are added to the state before it is requantized, and the buffer is emptied.
// The quantized part itself is only decayed and requantized every step.
//
// Mapping: the chunk kernel's (one CTA of d_v threads per tile, thread j
// holding value column j in registers). The per-component reductions over
// the key axis (k . U_l for the delta rule, q . U_l for the output) are one
// key-order chain each, run by threads l in parallel and shared through
// shared memory; thread j keeps V[l][j] for every component in registers.
#pragma once

#include "chunk_kernel.cuh"

namespace lrs {

constexpr int kLrbMaxRank = 8;

struct LrbParams {
    uint8_t* codes;
    float* scales;
    const uint8_t* prec_map;
    const int64_t* head_offsets;
    int64_t batch_stride;
    float* U;             // [ntiles][rank][d_k]
    float* V;             // [ntiles][rank][d_v]
    const float* q;
    const float* k;
    const float* v;
    const float* gates;
    const float* beta;
    float* out;
    uint64_t seed, step;
    unsigned* err;
    uint64_t timeout_ns;
    int32_t H, ntiles, rank, pgroups, inject;
};

// Shared memory of one CTA: two barriers, two stages (a tile is processed in
// one while the next tile's copies land in the other), then e and f:
//   stage: codes | scales | U (kLrbMaxRank rows) | q, k, [gate] (d_k fp32) | v
template <int DK, int DV, int GROUP, int GATE>
struct LrbSmem {
    static constexpr int G = DK / GROUP;
    static constexpr int kCodes = 0;
    static constexpr int kScales = kCodes + DK * DV;
    static constexpr int kU = kScales + G * DV * 4;
    static constexpr int kQ = kU + kLrbMaxRank * DK * 4;
    static constexpr int kK = kQ + DK * 4;
    static constexpr int kG = kK + DK * 4;
    static constexpr int kV = kG + (GATE == kGatePerKey ? DK * 4 : 0);
    static constexpr int kStage = (kV + DV * 4 + 127) / 128 * 128;
    static constexpr int kStage0 = 128;
    static constexpr int kE = kStage0 + 2 * kStage;
    static constexpr int kF = kE + kLrbMaxRank * 4;
    static constexpr int kBytes = kF + kLrbMaxRank * 4;
    static_assert(kU % 16 == 0 && kQ % 16 == 0 && kV % 16 == 0, "alignment");
};

// The copies of one tile into a stage (thread 0). A tile whose layout does
// not fit gets a bare arrival, so the stage's phase still completes.
template <int DK, int DV, int GROUP, int GATE>
__device__ __forceinline__ void lrb_issue(const LrbParams& p, uint64_t* bar, uint8_t* st,
                                          const TileLayout& tl, int tile, int m) {
    using S = LrbSmem<DK, DV, GROUP, GATE>;
    constexpr int G = DK / GROUP;
    if (!tl.ok) {
        mbar_arrive(bar);
        return;
    }
    fence_proxy_async_smem();                // earlier shared reads before the copies land
    const uint32_t cbytes = static_cast<uint32_t>(tl.goff(G, GROUP * DV / 2));
    const uint64_t pol = policy_evict_first();
    const int64_t row = static_cast<int64_t>(tile) * DK;
    uint32_t bytes = cbytes + G * DV * 4 + 2 * DK * 4 + DV * 4;
    if (GATE == kGatePerKey) bytes += DK * 4;
    if (m > 0) bytes += m * DK * 4;
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s(st + S::kCodes, p.codes + tl.code_off, cbytes, bar, pol);
    bulk_g2s(st + S::kScales, p.scales + static_cast<int64_t>(tile) * G * DV, G * DV * 4, bar, pol);
    if (m > 0)
        bulk_g2s(st + S::kU, p.U + static_cast<int64_t>(tile) * p.rank * DK, m * DK * 4, bar, pol);
    bulk_g2s(st + S::kQ, p.q + row, DK * 4, bar, pol);
    bulk_g2s(st + S::kK, p.k + row, DK * 4, bar, pol);
    if (GATE == kGatePerKey) bulk_g2s(st + S::kG, p.gates + row, DK * 4, bar, pol);
    bulk_g2s(st + S::kV, p.v + static_cast<int64_t>(tile) * DV, DV * 4, bar, pol);
}

__device__ __forceinline__ TileLayout lrb_layout(const LrbParams& p, int tile, int G, int gbytes8) {
    TileLayout tl;
    const int b = tile / p.H;
    tl.load(p.prec_map, p.head_offsets, p.batch_stride, p.H, p.pgroups, G, gbytes8, b,
            tile - b * p.H);
    return tl;
}

template <int DK, int DV, int GROUP, int UPD, int GATE, int MODE>
__global__ void __launch_bounds__(DV, (3 * 128) / DV) lrb_kernel(const LrbParams p) {
    using S = LrbSmem<DK, DV, GROUP, GATE>;
    constexpr int G = DK / GROUP;
    constexpr int C = DV / 32;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    float* es = reinterpret_cast<float*>(smem + S::kE);
    float* fs = reinterpret_cast<float*>(smem + S::kF);
    const int j = threadIdx.x;
    const ColumnPlace cp(j, C);
    const int r = p.rank;
    const int m = static_cast<int>(p.step % static_cast<uint64_t>(r));   // filled components
    const bool merge = m + 1 == r;

    if (j == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    bool ok = true;
    int issued = 0;              // tiles whose copies thread 0 has issued (for draining)

    // V[l][j] of the filled components of a tile (plain loads, coalesced across j)
    auto load_v = [&](int tile, float (&Vr)[kLrbMaxRank]) {
        const float* Vg = p.V + static_cast<int64_t>(tile) * r * DV;
#pragma unroll
        for (int l = 0; l < kLrbMaxRank; ++l) Vr[l] = l < m ? __ldcs(Vg + l * DV + j) : 0.0f;
    };

    const int first = blockIdx.x;
    float Vn[kLrbMaxRank];       // the next tile's V
    if (first < p.ntiles) {
        if (j == 0 && !p.inject) {
            lrb_issue<DK, DV, GROUP, GATE>(p, &bars[0], smem + S::kStage0,
                                           lrb_layout(p, first, G, GROUP * DV), first, m);
            issued = 1;
        }
        load_v(first, Vn);
    }
    int n = 0;
    for (int tile = first; tile < p.ntiles && ok; tile += gridDim.x, ++n) {
        const int stage = n & 1;
        uint8_t* st = smem + S::kStage0 + stage * S::kStage;
        uint8_t* cs = st + S::kCodes;
        float* ss = reinterpret_cast<float*>(st + S::kScales);
        float* Us = reinterpret_cast<float*>(st + S::kU);
        const float* qs = reinterpret_cast<const float*>(st + S::kQ);
        const float* ks = reinterpret_cast<const float*>(st + S::kK);
        const float* gs = reinterpret_cast<const float*>(st + S::kG);
        const float* vs = reinterpret_cast<const float*>(st + S::kV);
        float Vr[kLrbMaxRank];
#pragma unroll
        for (int l = 0; l < kLrbMaxRank; ++l) Vr[l] = Vn[l];
        // the next tile's copies go to the other stage, freed at the end of
        // the previous tile
        const int next = tile + gridDim.x;
        if (next < p.ntiles) {
            if (j == 0 && !p.inject) {
                lrb_issue<DK, DV, GROUP, GATE>(p, &bars[stage ^ 1],
                                               smem + S::kStage0 + (stage ^ 1) * S::kStage,
                                               lrb_layout(p, next, G, GROUP * DV), next, m);
                ++issued;
            }
            load_v(next, Vn);
        }
        const TileLayout tl = lrb_layout(p, tile, G, GROUP * DV);
        ok = __syncthreads_and(
            mbar_wait_bounded(&bars[stage], static_cast<uint32_t>((n >> 1) & 1), p.timeout_ns));
        if (!ok) break;
        if (!tl.ok) {
            if (j == 0) atomicOr(p.err, kErrLayout);
            __syncthreads();
            continue;
        }
        const int b = tile / p.H, h = tile - b * p.H;
        const uint32_t cbytes = static_cast<uint32_t>(tl.goff(G, GROUP * DV / 2));
        float* Ug = p.U + static_cast<int64_t>(tile) * r * DK;
        float* Vg = p.V + static_cast<int64_t>(tile) * r * DV;
        const float alpha = GATE == kGate ? __ldg(p.gates + tile) : 0.0f;

        float x[DK];
        decode_column<DK, DV, GROUP>(cs, ss, cp, j, tl, x);      // deq

        float w = vs[j];
        if (UPD == kDelta) {
            // e_l = k . U_l (undecayed buffer), one key-order chain per thread l
            if (j < m) {
                float e = 0.0f;
#pragma unroll 8
                for (int i = 0; i < DK; ++i) e = __fmaf_rn(ks[i], Us[j * DK + i], e);
                es[j] = e;
            }
            float u = 0.0f;
#pragma unroll
            for (int i = 0; i < DK; i += 4) {
                const float4 kv = lds4(ks + i);
                u = __fmaf_rn(kv.x, x[i], u);
                u = __fmaf_rn(kv.y, x[i + 1], u);
                u = __fmaf_rn(kv.z, x[i + 2], u);
                u = __fmaf_rn(kv.w, x[i + 3], u);
            }
            __syncthreads();
#pragma unroll
            for (int l = 0; l < kLrbMaxRank; ++l)
                if (l < m) u = __fmaf_rn(es[l], Vr[l], u);
            const float beta = __ldg(p.beta + tile);
            w = __fmul_rn(beta, __fsub_rn(w, __fmul_rn(alpha, u)));
        }
        // decay the buffer with the state and append the step's update k w^T
        for (int i = j; i < DK; i += DV) {
            const float gi = GATE == kGatePerKey ? gs[i] : alpha;
            for (int l = 0; l < m; ++l) Us[l * DK + i] = __fmul_rn(gi, Us[l * DK + i]);
            Us[m * DK + i] = ks[i];
        }
#pragma unroll
        for (int l = 0; l < kLrbMaxRank; ++l)
            if (l == m) Vr[l] = w;
        // the quantized part only decays: x = RN(g deq); o = x^T q, key order
        float o = 0.0f;
#pragma unroll
        for (int i = 0; i < DK; i += 4) {
            const float4 qv = lds4(qs + i);
            float4 gv = make_float4(alpha, alpha, alpha, alpha);
            if (GATE == kGatePerKey) gv = lds4(gs + i);
            x[i] = __fmul_rn(gv.x, x[i]);
            x[i + 1] = __fmul_rn(gv.y, x[i + 1]);
            x[i + 2] = __fmul_rn(gv.z, x[i + 2]);
            x[i + 3] = __fmul_rn(gv.w, x[i + 3]);
            o = __fmaf_rn(qv.x, x[i], o);
            o = __fmaf_rn(qv.y, x[i + 1], o);
            o = __fmaf_rn(qv.z, x[i + 2], o);
            o = __fmaf_rn(qv.w, x[i + 3], o);
        }
        __syncthreads();                    // U decayed and appended
        // f_l = q . U_l, one key-order chain per thread l <= m
        if (j <= m) {
            float f = 0.0f;
#pragma unroll 8
            for (int i = 0; i < DK; ++i) f = __fmaf_rn(qs[i], Us[j * DK + i], f);
            fs[j] = f;
        }
        __syncthreads();
#pragma unroll
        for (int l = 0; l < kLrbMaxRank; ++l)
            if (l <= m) o = __fmaf_rn(fs[l], Vr[l], o);
        p.out[static_cast<int64_t>(tile) * DV + j] = o;

        if (merge) {
            // add the buffer's elements of at least half a quantization step
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float half = __fmul_rn(0.5f, ss[g * DV + j]);
#pragma unroll
                for (int rr = 0; rr < GROUP; ++rr) {
                    const int i = g * GROUP + rr;
                    float mij = 0.0f;
#pragma unroll
                    for (int l = 0; l < kLrbMaxRank; ++l)
                        if (l < r) mij = __fmaf_rn(Us[l * DK + i], Vr[l], mij);
                    if (mij != 0.0f && fabsf(mij) >= half) x[i] = __fadd_rn(x[i], mij);
                }
            }
        }
        // write the buffer back (emptied after a merge)
        for (int idx = j; idx < (m + 1) * DK; idx += DV) Ug[idx] = merge ? 0.0f : Us[idx];
#pragma unroll
        for (int l = 0; l < kLrbMaxRank; ++l)
            if (l <= m) Vg[l * DV + j] = merge ? 0.0f : Vr[l];

        // requantize, pack, write back (as the chunked update)
        float snew[G];
        const uint64_t hkey = MODE == kSR ? tile_hash_key(p.seed, p.step, static_cast<uint32_t>(b),
                                                          static_cast<uint32_t>(h))
                                          : 0ull;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int gbase = static_cast<int>(tl.goff(g, GROUP * DV / 2));
            snew[g] = tl.bits(g) == 8
                          ? requantize_group<DK, DV, GROUP, MODE, 8>(x, g, cs, ss, cp, j, gbase, hkey)
                          : requantize_group<DK, DV, GROUP, MODE, 4>(x, g, cs, ss, cp, j, gbase, hkey);
        }
        __syncthreads();                    // old codes, scales and U no longer read
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int gbase = static_cast<int>(tl.goff(g, GROUP * DV / 2));
            if (tl.bits(g) == 8)
                store_group<DV, GROUP, 8>(cs, cp, gbase, x + g * GROUP);
            else
                store_group<DV, GROUP, 4>(cs, cp, gbase, x + g * GROUP);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) ss[g * DV + j] = snew[g];
        __syncthreads();
        uint8_t* gc = p.codes + tl.code_off;
        for (int off = j * 16; off < static_cast<int>(cbytes); off += DV * 16) {
            const uint4 vv = *reinterpret_cast<const uint4*>(cs + off);
            st_cs_u4(gc + off, vv.x, vv.y, vv.z, vv.w);
        }
        float* gsc = p.scales + static_cast<int64_t>(tile) * G * DV;
        for (int off = j * 4; off < G * DV; off += DV * 4)
            *reinterpret_cast<float4*>(gsc + off) = *reinterpret_cast<const float4*>(ss + off);
        __syncthreads();                    // the stage is free for the tile after next
    }
    if (!ok && j == 0) {
        // record the timeout, then wait (bounded) for copies still in flight
        atomicOr(p.err, kErrTimeout);
        for (int q = n; q < issued; ++q)
            mbar_wait_bounded(&bars[q & 1], static_cast<uint32_t>((q >> 1) & 1), p.timeout_ns);
    }
}

#define LRS_LRB_PICK(MODE, DK, DV, GROUP)                                                      \
    if (d_k == DK && d_v == DV && group == GROUP) {                                            \
        using S = LrbSmem<DK, DV, GROUP, kGatePerKey>;                                         \
        using S1 = LrbSmem<DK, DV, GROUP, kGate>;                                              \
        if (update_kind == kGated && gate_kind == kGatePerKey)                                 \
            return {reinterpret_cast<const void*>(                                             \
                        &lrb_kernel<DK, DV, GROUP, kGated, kGatePerKey, MODE>),                \
                    S::kBytes};                                                                \
        if (update_kind == kGated && gate_kind == kGate)                                       \
            return {reinterpret_cast<const void*>(                                             \
                        &lrb_kernel<DK, DV, GROUP, kGated, kGate, MODE>),                      \
                    S1::kBytes};                                                               \
        if (update_kind == kDelta && gate_kind == kGate)                                       \
            return {reinterpret_cast<const void*>(                                             \
                        &lrb_kernel<DK, DV, GROUP, kDelta, kGate, MODE>),                      \
                    S1::kBytes};                                                               \
        return {nullptr, 0};                                                                   \
    }
// Defines `ChunkKernel NAME(d_k, d_v, group, update_kind, gate_kind)` for the
// LRB kernel with rounding MODE.
#define LRS_LRB_VARIANTS(NAME, MODE)                                                           \
    ChunkKernel NAME(int d_k, int d_v, int group, int update_kind, int gate_kind) {            \
        LRS_LRB_PICK(MODE, 128, 128, 32)                                                       \
        LRS_LRB_PICK(MODE, 128, 128, 16)                                                       \
        LRS_LRB_PICK(MODE, 128, 64, 32)                                                        \
        LRS_LRB_PICK(MODE, 128, 64, 64)                                                        \
        LRS_LRB_PICK(MODE, 128, 64, 16)                                                        \
        LRS_LRB_PICK(MODE, 64, 64, 16)                                                         \
        LRS_LRB_PICK(MODE, 64, 64, 32)                                                         \
        LRS_LRB_PICK(MODE, 64, 64, 64)                                                         \
        LRS_LRB_PICK(MODE, 64, 128, 16)                                                        \
        LRS_LRB_PICK(MODE, 64, 128, 32)                                                        \
        return {nullptr, 0};                                                                   \
    }

}  // namespace lrs
