// lrb_stream.cuh -- the Low-Rank Bypass decode step on the step kernel's
// streaming design (ranks up to 4).
//
// The readings are those of lrb_kernel.cuh. The mapping is the decode step's:
// a warp owns a tile, lane t owns value columns [t*C, t*C + C) over all key
// rows, the tile streams through a ring of scale-group slots. What the bypass
// adds per tile:
//   - the buffer's U rows (filled components) arrive with the tile's first
//     group, in the tile-input buffer; each lane loads its columns of V;
//   - the per-component chains e_l = k . U_l (delta rule) and
//     f_l = q . RN(g U_l) (and f_m = q . k) run in key order on lanes 0..3
//     and 16..20 at once, then reach every lane by shuffles;
//   - U is decayed in place and k appended; the lane appends w to its V;
//   - the quantized part takes x = RN(g deq); at a merge step every element
//     adds its buffer value sum_l U'_l,i V'_l,j when it is at least half a
//     quantization step;
//   - the output adds sum_l f_l V'_l,j after the key-order chain;
//   - U' and V' (or zeros after a merge) go back to global memory.
// SR and BDR use the staged pair code (updated values in shared memory), RTN
// keeps a group's values in registers. Merge steps and the other steps are
// separate instantiations (MERGE), so the others carry no merge code.
#pragma once

#include "step_kernel.cuh"

namespace lrs {

constexpr int kLrbStreamMaxRank = 4;

struct LrbStreamParams {
    StepParams s;         // the decode step's parameters (state, inputs, ring)
    float* U;             // [ntiles][rank][d_k]
    float* V;             // [ntiles][rank][d_v]
    int32_t rank, m;      // rank, components filled before the step (step mod rank)
};

// Per-warp shared memory: barriers | two tile-input buffers | slots | x
// staging | SR row table.
// Tile-input buffer: q, k, [gate] (d_k fp32 each) | v (d_v) | U (4 rows of
// d_k) | V (4 rows of d_v).
template <int C, int GROUP, int GATE>
struct LrbSlot {
    static constexpr int DV = 32 * C;
    static constexpr int kCodes = GROUP * DV;
    static constexpr int kScales = kCodes;
    static constexpr int kBytes = kScales + DV * 4;
    static constexpr int kXsBytes = GROUP * 256;
    static constexpr int kTabBytes = GROUP * 8;    // SR: the group's row table of the hash
    __host__ __device__ static int in_k(int d_k) { return d_k * 4; }
    __host__ __device__ static int in_g(int d_k) { return 2 * d_k * 4; }
    __host__ __device__ static int in_v(int d_k) {
        return 2 * d_k * 4 + (GATE == kGatePerKey ? d_k * 4 : 0);
    }
    __host__ __device__ static int in_u(int d_k) { return in_v(d_k) + DV * 4; }
    __host__ __device__ static int in_vb(int d_k) { return in_u(d_k) + kLrbStreamMaxRank * d_k * 4; }
    __host__ __device__ static int tile_in_bytes(int d_k) {
        return (in_vb(d_k) + kLrbStreamMaxRank * DV * 4 + 15) / 16 * 16;
    }
    __host__ __device__ static int header(int d_k) { return 128 + 2 * tile_in_bytes(d_k); }
    static int warp_bytes(int slots, int d_k, bool staged, bool tab) {
        return (header(d_k) + slots * kBytes + (staged ? kXsBytes : 0) + (tab ? kTabBytes : 0) +
                127) / 128 * 128;
    }
};

// Group g of the cursor's tile into `slot` (lane 0); with the first group the
// tile's q, k, gates, v and filled U rows into `tin`.
template <int C, int GROUP, int GATE>
__device__ __forceinline__ void lrb_issue_item(const LrbStreamParams& lp, uint8_t* wsm, int slot,
                                               const TileCursor& tc, int g, uint8_t* tin,
                                               uint64_t pol_state, uint64_t pol_in) {
    using S = LrbSlot<C, GROUP, GATE>;
    constexpr int DV = 32 * C;
    const StepParams& p = lp.s;
    uint64_t* bar = reinterpret_cast<uint64_t*>(wsm) + slot;
    if (!tc.ok) {
        mbar_arrive(bar);
        return;
    }
    const int tile = tc.tile;
    const int dk = p.d_k;
    uint8_t* sm = wsm + S::header(dk) + slot * S::kBytes;
    const uint32_t cbytes = GROUP * DV * tc.bits(g) / 8;
    uint32_t total = cbytes + DV * 4;
    if (g == 0) total += S::in_u(dk) + lp.m * (dk + DV) * 4;
    mbar_arrive_expect_tx(bar, total);
    bulk_g2s(sm, p.codes + tc.code_off + tc.goff(g, GROUP * DV / 2), cbytes, bar, pol_state);
    bulk_g2s(sm + S::kScales, p.scales + (static_cast<int64_t>(tile) * p.G + g) * DV, DV * 4, bar,
             pol_state);
    if (g == 0) {
        const int64_t rowbase = static_cast<int64_t>(tile) * dk;
        bulk_g2s(tin, static_cast<const float*>(p.q) + rowbase, dk * 4, bar, pol_in);
        bulk_g2s(tin + S::in_k(dk), static_cast<const float*>(p.k) + rowbase, dk * 4, bar, pol_in);
        if (GATE == kGatePerKey) bulk_g2s(tin + S::in_g(dk), p.gates + rowbase, dk * 4, bar, pol_in);
        bulk_g2s(tin + S::in_v(dk), static_cast<const float*>(p.v) + static_cast<int64_t>(tile) * DV,
                 DV * 4, bar, pol_in);
        if (lp.m > 0) {
            bulk_g2s(tin + S::in_u(dk), lp.U + static_cast<int64_t>(tile) * lp.rank * dk,
                     lp.m * dk * 4, bar, pol_state);
            bulk_g2s(tin + S::in_vb(dk), lp.V + static_cast<int64_t>(tile) * lp.rank * DV,
                     lp.m * DV * 4, bar, pol_state);
        }
    }
}

// One column pair of one scale group with the bypass: x = RN(g deq), plus at
// a merge step the buffer's element where it reaches half a quantization
// step; then the output chain, new scales and codes as pair_step_xs.
// Ut: U' (decayed, appended; component-major, d_k floats per component) at
// the group's first row. vc0, vc1: V'[l] of the pair's two columns.
template <int GROUP, int GATE, int MODE, int BITS, bool STAGE>
__device__ __forceinline__ void pair_step_lrb(const uint8_t* __restrict__ cs, int ubase, float2 sc,
                                              const float* __restrict__ qs,
                                              const float* __restrict__ gs, float gscalar,
                                              float2& o, uint8_t* __restrict__ gcodes,
                                              float* __restrict__ gscale, uint64_t hkey, int row0,
                                              uint32_t j0, int lane, float4* __restrict__ xs,
                                              bool merge, int R, const float* __restrict__ Ut,
                                              int dk, const float (&vc0)[kLrbStreamMaxRank],
                                              const float (&vc1)[kLrbStreamMaxRank],
                                              const uint4* __restrict__ rtab, bool rowtab) {
    using G = PairGeo<GROUP, BITS>;
    constexpr float BIAS = Q<BITS>::kBias;
    constexpr int RPUH = G::RPU / 2;
    const float2 s0 = f2(sc.x), s1 = f2(sc.y);
    const float2 gsc = f2(gscalar);
    const float half0 = __fmul_rn(0.5f, sc.x), half1 = __fmul_rn(0.5f, sc.y);
    float a0 = 0.0f, b0 = 0.0f;
    float2 v0b[kLrbStreamMaxRank], v1b[kLrbStreamMaxRank];   // V' broadcast into pairs once
#pragma unroll
    for (int l = 0; l < kLrbStreamMaxRank; ++l) {
        v0b[l] = f2(vc0[l]);
        v1b[l] = f2(vc1[l]);
    }

#pragma unroll 1
    for (int un = 0; un < G::UNITS; ++un) {
        const uint4 raw = lds_unit(cs, ubase + un, lane);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
        float qq[G::RPU], gg[G::RPU];
        ld_smem_rows<G::RPU>(qs + un * G::RPU, qq);
        if constexpr (GATE == kGatePerKey) ld_smem_rows<G::RPU>(gs + un * G::RPU, gg);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            decode_word_biased<BITS>(wd[wi], f);
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int rl = wi * G::RPW + 2 * rp;
                const float2 qr = make_float2(qq[rl], qq[rl + 1]);
                const float2 gr = GATE == kGatePerKey ? make_float2(gg[rl], gg[rl + 1]) : gsc;
                const float2 c0 = add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-(kTwo23 + BIAS)));
                const float2 c1 = add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-(kTwo23 + BIAS)));
                float2 x0 = mul2(gr, mul2(c0, s0));
                float2 x1 = mul2(gr, mul2(c1, s1));
                // the output reads the state part before a merge (the buffer's
                // share is added from f_l after the tile)
                o.x = __fmaf_rn(qr.x, x0.x, o.x);
                o.x = __fmaf_rn(qr.y, x0.y, o.x);
                o.y = __fmaf_rn(qr.x, x1.x, o.y);
                o.y = __fmaf_rn(qr.y, x1.y, o.y);
                if (merge) {
                    // M = sum_l U'_l,i V'_l,j (fma chain in component order),
                    // added where |M| >= RN(s_old / 2). The rule's M != 0 is
                    // not tested: adding a zero M changes at most the sign of
                    // a zero x, which no code, scale or later output sees.
                    const int r = un * G::RPU + rl;
                    float2 m0 = f2(0.0f), m1 = f2(0.0f);
#pragma unroll
                    for (int l = 0; l < kLrbStreamMaxRank; ++l) {
                        if (l < R) {
                            const float2 u = *reinterpret_cast<const float2*>(Ut + l * dk + r);
                            m0 = fma2(u, v0b[l], m0);
                            m1 = fma2(u, v1b[l], m1);
                        }
                    }
                    const float2 y0 = add2(x0, m0), y1 = add2(x1, m1);
                    x0.x = fabsf(m0.x) >= half0 ? y0.x : x0.x;
                    x0.y = fabsf(m0.y) >= half0 ? y0.y : x0.y;
                    x1.x = fabsf(m1.x) >= half1 ? y1.x : x1.x;
                    x1.y = fabsf(m1.y) >= half1 ? y1.y : x1.y;
                }
                a0 = max_abs3(a0, x0.x, x0.y);
                b0 = max_abs3(b0, x1.x, x1.y);
                if constexpr (STAGE)
                    xs[(un * RPUH + rl / 2) * 32 + lane] = make_float4(x0.x, x0.y, x1.x, x1.y);
            }
        }
    }

    float2 snew, inv;
    new_scales<BITS>(a0, b0, snew, inv);
    st_cs_f2(gscale, snew);
    if constexpr (MODE == kSR) {
        // SR stages x: the decode step's rounding pass, with the row table of
        // the hash when the tile's carry allows it
        static_assert(STAGE, "SR stages x");
        if (rowtab)
            round_pass<GROUP, GATE, kSR, BITS, kIoF32, true, true>(
                cs, ubase, sc, nullptr, gs, gscalar, f2(0.0f), inv, snew, gcodes, hkey, row0, j0,
                lane, xs, rtab);
        else
            round_pass<GROUP, GATE, kSR, BITS, kIoF32, true, false>(
                cs, ubase, sc, nullptr, gs, gscalar, f2(0.0f), inv, snew, gcodes, hkey, row0, j0,
                lane, xs, rtab);
        return;
    }
    const float2 inv0 = f2(inv.x), inv1 = f2(inv.y);
    const float2 sn0 = f2(snew.x), sn1 = f2(snew.y);

    // Without a merge (STAGE false, BDR), x = RN(g deq) is recomputed from
    // the old codes the rounding decodes anyway, by the same operations.
    static_assert(STAGE || MODE == kBDR, "only BDR recomputes x");
#pragma unroll 1
    for (int un = 0; un < G::UNITS; ++un) {
        uint32_t ow[4];
        uint32_t wd[4] = {0u, 0u, 0u, 0u};
        if constexpr (MODE == kBDR) {
            const uint4 raw = lds_unit(cs, ubase + un, lane);
            wd[0] = raw.x; wd[1] = raw.y; wd[2] = raw.z; wd[3] = raw.w;
        }
        float gg[STAGE || GATE != kGatePerKey ? 1 : G::RPU];
        if constexpr (!STAGE && GATE == kGatePerKey) ld_smem_rows<G::RPU>(gs + un * G::RPU, gg);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            if constexpr (MODE == kBDR) decode_word_biased<BITS>(wd[wi], f);
            float t[G::EPW];
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int rl = wi * G::RPW + 2 * rp;
                float2 dq0 = f2(0.0f), dq1 = f2(0.0f);
                if constexpr (MODE == kBDR) {
                    dq0 = mul2(add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-(kTwo23 + BIAS))), s0);
                    dq1 = mul2(add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-(kTwo23 + BIAS))), s1);
                }
                float4 xv;
                if constexpr (STAGE) {
                    xv = xs[(un * RPUH + rl / 2) * 32 + lane];
                } else {
                    const float2 gr = GATE == kGatePerKey ? make_float2(gg[rl], gg[rl + 1]) : gsc;
                    const float2 x0 = mul2(gr, dq0), x1 = mul2(gr, dq1);
                    xv = make_float4(x0.x, x0.y, x1.x, x1.y);
                }
                const uint32_t i = static_cast<uint32_t>(row0 + un * G::RPU + rl);
                const float2 kb0 = make_float2(word_bias<BITS>(4 * rp), word_bias<BITS>(4 * rp + 2));
                const float2 kb1 = make_float2(word_bias<BITS>(4 * rp + 1), word_bias<BITS>(4 * rp + 3));
                const float2 t0 = round_rows<MODE, BITS>(make_float2(xv.x, xv.y), inv0, dq0, sn0,
                                                         kb0, hkey, i, j0);
                const float2 t1 = round_rows<MODE, BITS>(make_float2(xv.z, xv.w), inv1, dq1, sn1,
                                                         kb1, hkey, i, j0 + 1);
                t[4 * rp] = t0.x;
                t[4 * rp + 2] = t0.y;
                t[4 * rp + 1] = t1.x;
                t[4 * rp + 3] = t1.y;
            }
            ow[wi] = encode_word<BITS>(t);
        }
        st_cs_u4(gcodes + ((ubase + un) * 32 + lane) * 16, ow[0], ow[1], ow[2], ow[3]);
    }
}

// The RTN form of pair_step_lrb with the group's updated values in registers
// (the staged form's shared-memory round trip costs more than the longer
// per-element code of SR and BDR saves).
template <int GROUP, int GATE, int BITS>
__device__ __forceinline__ void pair_step_lrb_rtn(const uint8_t* __restrict__ cs, int ubase,
                                                  float2 sc, const float* __restrict__ qs,
                                                  const float* __restrict__ gs, float gscalar,
                                                  float2& o, uint8_t* __restrict__ gcodes,
                                                  float* __restrict__ gscale, int lane, bool merge,
                                                  int R, const float* __restrict__ Ut, int dk,
                                                  const float (&vc0)[kLrbStreamMaxRank],
                                                  const float (&vc1)[kLrbStreamMaxRank]) {
    using G = PairGeo<GROUP, BITS>;
    constexpr float BIAS = Q<BITS>::kBias;
    const float2 s0 = f2(sc.x), s1 = f2(sc.y);
    const float2 gsc = f2(gscalar);
    const float half0 = __fmul_rn(0.5f, sc.x), half1 = __fmul_rn(0.5f, sc.y);
    float2 x[GROUP / 2][2];

#pragma unroll
    for (int un = 0; un < G::UNITS; ++un) {
        const uint4 raw = lds_unit(cs, ubase + un, lane);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
        float qq[G::RPU], gg[G::RPU];
        ld_smem_rows<G::RPU>(qs + un * G::RPU, qq);
        if constexpr (GATE == kGatePerKey) ld_smem_rows<G::RPU>(gs + un * G::RPU, gg);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            decode_word_biased<BITS>(wd[wi], f);
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int rl = wi * G::RPW + 2 * rp;
                const int r = un * G::RPU + rl;
                const float2 qr = make_float2(qq[rl], qq[rl + 1]);
                const float2 gr = GATE == kGatePerKey ? make_float2(gg[rl], gg[rl + 1]) : gsc;
                const float2 c0 = add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-(kTwo23 + BIAS)));
                const float2 c1 = add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-(kTwo23 + BIAS)));
                float2 x0 = mul2(gr, mul2(c0, s0));
                float2 x1 = mul2(gr, mul2(c1, s1));
                o.x = __fmaf_rn(qr.x, x0.x, o.x);
                o.x = __fmaf_rn(qr.y, x0.y, o.x);
                o.y = __fmaf_rn(qr.x, x1.x, o.y);
                o.y = __fmaf_rn(qr.y, x1.y, o.y);
                x[r / 2][0] = x0;
                x[r / 2][1] = x1;
            }
        }
    }
    if (merge) {
        // a separate pass over the group, so the merge's values are not live
        // beside the decode's; four rows of each component per 16-byte load,
        // the columns' V' values broadcast into pairs once
        float2 v0b[kLrbStreamMaxRank], v1b[kLrbStreamMaxRank];
#pragma unroll
        for (int l = 0; l < kLrbStreamMaxRank; ++l) {
            v0b[l] = f2(vc0[l]);
            v1b[l] = f2(vc1[l]);
        }
#pragma unroll
        for (int rq = 0; rq < GROUP / 4; ++rq) {
            float2 m00 = f2(0.0f), m01 = f2(0.0f), m10 = f2(0.0f), m11 = f2(0.0f);
#pragma unroll
            for (int l = 0; l < kLrbStreamMaxRank; ++l) {
                if (l < R) {
                    const float4 u = *reinterpret_cast<const float4*>(Ut + l * dk + 4 * rq);
                    const float2 ua = make_float2(u.x, u.y), ub = make_float2(u.z, u.w);
                    m00 = fma2(ua, v0b[l], m00);
                    m01 = fma2(ua, v1b[l], m01);
                    m10 = fma2(ub, v0b[l], m10);
                    m11 = fma2(ub, v1b[l], m11);
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int rp = 2 * rq + h;
                const float2 m0 = h ? m10 : m00, m1 = h ? m11 : m01;
                const float2 x0 = x[rp][0], x1 = x[rp][1];
                const float2 y0 = add2(x0, m0), y1 = add2(x1, m1);
                x[rp][0].x = fabsf(m0.x) >= half0 ? y0.x : x0.x;
                x[rp][0].y = fabsf(m0.y) >= half0 ? y0.y : x0.y;
                x[rp][1].x = fabsf(m1.x) >= half1 ? y1.x : x1.x;
                x[rp][1].y = fabsf(m1.y) >= half1 ? y1.y : x1.y;
            }
        }
    }
    float a0 = 0.0f, a1 = 0.0f, b0 = 0.0f, b1 = 0.0f;
#pragma unroll
    for (int rp = 0; rp < GROUP / 2; rp += 2) {
        a0 = max_abs3(a0, x[rp][0].x, x[rp][0].y);
        a1 = max_abs3(a1, x[rp + 1][0].x, x[rp + 1][0].y);
        b0 = max_abs3(b0, x[rp][1].x, x[rp][1].y);
        b1 = max_abs3(b1, x[rp + 1][1].x, x[rp + 1][1].y);
    }
    float2 snew, inv;
    new_scales<BITS>(fmaxf(a0, a1), fmaxf(b0, b1), snew, inv);
    st_cs_f2(gscale, snew);
    const float2 inv0 = f2(inv.x), inv1 = f2(inv.y);
#pragma unroll
    for (int un = 0; un < G::UNITS; ++un) {
        uint32_t ow[4];
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float t[G::EPW];
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int r = un * G::RPU + wi * G::RPW + 2 * rp;
                const float2 kb0 = make_float2(word_bias<BITS>(4 * rp), word_bias<BITS>(4 * rp + 2));
                const float2 kb1 = make_float2(word_bias<BITS>(4 * rp + 1), word_bias<BITS>(4 * rp + 3));
                const float2 t0 = fma2(x[r / 2][0], inv0, kb0);
                const float2 t1 = fma2(x[r / 2][1], inv1, kb1);
                t[4 * rp] = t0.x;
                t[4 * rp + 2] = t0.y;
                t[4 * rp + 1] = t1.x;
                t[4 * rp + 3] = t1.y;
            }
            ow[wi] = encode_word<BITS>(t);
        }
        st_cs_u4(gcodes + ((ubase + un) * 32 + lane) * 16, ow[0], ow[1], ow[2], ow[3]);
    }
}

// One lane's key-order chain c = sum_i a_i * b'_i over n rows (n a multiple
// of 4), b'_i = RN(g_i * b_i) when `decay`, else b_i: every chain lane runs
// this one loop, each with its own operands, so the roles do not diverge.
__device__ __forceinline__ float lrb_chain(const float* a, const float* b, const float* g,
                                           bool decay, int n) {
    float c = 0.0f;
#pragma unroll 2
    for (int i = 0; i < n; i += 4) {
        const float4 av = *reinterpret_cast<const float4*>(a + i);
        float4 bv = *reinterpret_cast<const float4*>(b + i);
        const float4 gv = *reinterpret_cast<const float4*>(g + i);
        if (decay) {
            bv.x = __fmul_rn(gv.x, bv.x);
            bv.y = __fmul_rn(gv.y, bv.y);
            bv.z = __fmul_rn(gv.z, bv.z);
            bv.w = __fmul_rn(gv.w, bv.w);
        }
        c = __fmaf_rn(av.x, bv.x, c);
        c = __fmaf_rn(av.y, bv.y, c);
        c = __fmaf_rn(av.z, bv.z, c);
        c = __fmaf_rn(av.w, bv.w, c);
    }
    return c;
}

// The warp's items are (tile, group) pairs as in step_kernel.
// Launch bound in warps. A merge step (MERGE: step mod rank = rank - 1) and
// the staged rounding modes take 8, so up to 255 registers: the merge's
// buffer rows do not fit beside a register-resident group in 168. The other
// RTN and BDR steps with groups of up to 32 rows are compiled without the merge
// code and take up to 12 (shared memory leaves 10 for d_k = d_v = 128).
__host__ __device__ constexpr int lrb_max_warps(int mode, bool merge, int group) {
    return (mode != kSR && !merge && group <= 32) ? 12 : 8;
}
// Whether the pair code stages the updated values in shared memory: SR, and
// every merge step. A non-merge BDR step recomputes them (more warps fit).
__host__ __device__ constexpr bool lrb_staged(int mode, bool merge) {
    return mode == kSR || (mode == kBDR && merge);
}

template <int C, int GROUP, int UPD, int GATE, int MODE, bool MERGE>
__global__ void __launch_bounds__(lrb_max_warps(MODE, MERGE, GROUP) * 32, 1)
    lrb_step_kernel(const LrbStreamParams lp) {
    using S = LrbSlot<C, GROUP, GATE>;
    constexpr int DV = 32 * C;
    constexpr int P = C / 2;
    constexpr int MR = kLrbStreamMaxRank;
    const StepParams& p = lp.s;
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    const int W = gridDim.x * nw;
    // warp-major numbering: the tiles of the last round (ntiles mod W of
    // them) spread over every SM instead of filling the first CTAs
    const int gw = wib * gridDim.x + blockIdx.x;
    uint8_t* wsm = smem + wib * p.warp_smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsm);
    const int G = p.G, NS = p.slots, dk = p.d_k;
    const int hdr = S::header(dk), tib = S::tile_in_bytes(dk);
    const int in_k = S::in_k(dk), in_g = S::in_g(dk), in_v = S::in_v(dk), in_u = S::in_u(dk);
    float4* xs = reinterpret_cast<float4*>(wsm + hdr + NS * S::kBytes);
    uint2* rtab2 = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(xs) +
                                            (lrb_staged(MODE, MERGE) ? S::kXsBytes : 0));  // SR
    const uint4* rtab = reinterpret_cast<const uint4*>(rtab2);
    const int ntw = gw < p.ntiles ? (p.ntiles - gw + W - 1) / W : 0;
    const int64_t K = static_cast<int64_t>(ntw) * G;
    const int R = lp.rank, m = lp.m;
    constexpr bool merge = MERGE;   // the host launches this variant when m + 1 == R

    if (lane == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    const uint64_t pol_state = policy_evict_first();
    const uint64_t pol_in = policy_evict_first();
    Ring ic, is;
    int64_t kc = 0, ki = 0;
    int it_g = 0, it_n = 0;
    TileCursor itc;
    itc.init(p, gw, W);
    if (K > 0) itc.load(p, GROUP * DV);

    auto issue_next = [&]() {
        if (ki < K && !p.inject) {
            if (lane == 0)
                lrb_issue_item<C, GROUP, GATE>(lp, wsm, is.slot, itc, it_g,
                                               wsm + 128 + (it_n & 1) * tib, pol_state, pol_in);
            ++ki;
            is.advance(NS);
            if (++it_g == G) {
                it_g = 0;
                ++it_n;
                itc.advance(p, W);
                if (ki < K) itc.load(p, GROUP * DV);
            }
        }
    };
    for (int s = 0; s < NS; ++s) issue_next();

    bool ok = true;
    TileCursor ti;
    ti.init(p, gw, W);
    for (int n = 0; n < ntw && ok; ++n, ti.advance(p, W)) {
        const int tile = ti.tile;
        ti.load(p, GROUP * DV);
        uint8_t* tin = wsm + 128 + (n & 1) * tib;
        const float gscalar = GATE == kGate ? __ldg(p.gates + tile) : 0.0f;
        const float beta = UPD == kDelta ? __ldg(p.beta + tile) : 0.0f;
        const uint64_t hkey = MODE == kSR ? tile_hash_key(p.seed, p.step,
                                                          static_cast<uint32_t>(ti.b),
                                                          static_cast<uint32_t>(ti.h))
                                          : 0ull;
        uint32_t hcarry = 0;
        const bool rowtab = MODE == kSR && sr_tile_carry(hkey, DV, &hcarry);
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[ic.slot], ic.par, p.timeout_ns));
        if (!ok) break;
        if (!ti.ok) {
            if (lane == 0) atomicOr(p.err, kErrLayout);
            for (int g = 0; g < G; ++g) {
                if (g > 0) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait_bounded(&bars[ic.slot], ic.par, p.timeout_ns));
                    if (!ok) break;
                }
                ++kc;
                ic.advance(NS);
                __syncwarp();
                issue_next();
            }
            continue;
        }
        const float* qs_t = reinterpret_cast<const float*>(tin);
        const float* ks_t = reinterpret_cast<const float*>(tin + in_k);
        const float* gs_t = reinterpret_cast<const float*>(tin + in_g);
        const uint8_t* vs_t = tin + in_v;
        float* Ut = reinterpret_cast<float*>(tin + in_u);
        float* Vt = reinterpret_cast<float*>(tin + S::in_vb(dk)) + lane * C;   // this lane's V

        // the component chains, all lanes of one loop at once: e_l = k . U_l
        // (lanes 0..m-1, delta rule; undecayed U) and f_l = q . RN(g U_l) for
        // l < m, f_m = q . k (lanes 16..16+m). U_m = k is appended first.
        for (int i = lane; i < dk; i += 32) Ut[m * dk + i] = ks_t[i];
        __syncwarp();
        float chain = 0.0f;
        {
            const int le = lane, lf = lane - 16;
            const bool is_e = UPD == kDelta && le < m;
            const bool is_f = lf >= 0 && lf <= m;
            if (is_e || is_f) {
                const float* a = is_e ? ks_t : qs_t;
                const float* b = Ut + (is_e ? le : lf) * dk;
                // scalar decays multiply by the head's gate: a row of it is
                // not stored, so the per-key array stands in with a select
                const bool decay = is_f && lf < m;
                if (GATE == kGatePerKey) {
                    chain = lrb_chain(a, b, gs_t, decay, dk);
                } else {
                    float c = 0.0f;
#pragma unroll 2
                    for (int i = 0; i < dk; i += 4) {
                        const float4 av = *reinterpret_cast<const float4*>(a + i);
                        float4 bv = *reinterpret_cast<const float4*>(b + i);
                        if (decay) {
                            bv.x = __fmul_rn(gscalar, bv.x);
                            bv.y = __fmul_rn(gscalar, bv.y);
                            bv.z = __fmul_rn(gscalar, bv.z);
                            bv.w = __fmul_rn(gscalar, bv.w);
                        }
                        c = __fmaf_rn(av.x, bv.x, c);
                        c = __fmaf_rn(av.y, bv.y, c);
                        c = __fmaf_rn(av.z, bv.z, c);
                        c = __fmaf_rn(av.w, bv.w, c);
                    }
                    chain = c;
                }
            }
        }
        __syncwarp();
        // decay the buffer in place (k was appended above)
        for (int i = lane; i < dk; i += 32) {
            const float gi = GATE == kGatePerKey ? gs_t[i] : gscalar;
            for (int l = 0; l < m; ++l) Ut[l * dk + i] = __fmul_rn(gi, Ut[l * dk + i]);
        }
        __syncwarp();

        float2 w[P], o[P];
#pragma unroll
        for (int pc = 0; pc < P; ++pc) o[pc] = f2(0.0f);
        if (UPD == kDelta) {
            float2 u[P];
#pragma unroll
            for (int pc = 0; pc < P; ++pc) u[pc] = f2(0.0f);
            Ring r = ic;
            for (int g = 0; g < G && ok; ++g) {
                if (g > 0)
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait_bounded(&bars[r.slot], r.par, p.timeout_ns));
                if (!ok) break;
                const uint8_t* sm = wsm + hdr + r.slot * S::kBytes;
                const float* ss = reinterpret_cast<const float*>(sm + S::kScales) + lane * C;
                const uint8_t* ks = tin + in_k + g * GROUP * 4;
                float2 up = u[0], uq = u[P - 1];
#pragma unroll 1
                for (int pc = 0; pc < P; ++pc) {
                    const float2 sc = *reinterpret_cast<const float2*>(ss + 2 * pc);
                    if (ti.bits(g) == 8)
                        pair_ktS<GROUP, 8, kIoF32>(sm, pc * PairGeo<GROUP, 8>::UNITS, sc, ks, lane, up);
                    else
                        pair_ktS<GROUP, 4, kIoF32>(sm, pc * PairGeo<GROUP, 4>::UNITS, sc, ks, lane, up);
                    if constexpr (P == 2) {
                        const float2 t = up;
                        up = uq; uq = t;
                    }
                }
                u[0] = up;
                u[P - 1] = P == 2 ? uq : up;
                r.advance(NS);
            }
            if (!ok) break;
            // u += sum_l e_l V_l (undecayed buffer), component order
#pragma unroll
            for (int l = 0; l < MR; ++l) {
                const float el = __shfl_sync(0xffffffffu, chain, l);
                if (l < m) {
#pragma unroll
                    for (int pc = 0; pc < P; ++pc) {
                        u[pc].x = __fmaf_rn(el, Vt[l * DV + 2 * pc], u[pc].x);
                        u[pc].y = __fmaf_rn(el, Vt[l * DV + 2 * pc + 1], u[pc].y);
                    }
                }
            }
#pragma unroll
            for (int pc = 0; pc < P; ++pc) {
                const float2 vv = ld_pair<kIoF32>(vs_t, lane * C + 2 * pc);
                const float d0 = __fsub_rn(vv.x, __fmul_rn(gscalar, u[pc].x));
                const float d1 = __fsub_rn(vv.y, __fmul_rn(gscalar, u[pc].y));
                w[pc] = make_float2(__fmul_rn(beta, d0), __fmul_rn(beta, d1));
            }
        } else {
#pragma unroll
            for (int pc = 0; pc < P; ++pc) w[pc] = ld_pair<kIoF32>(vs_t, lane * C + 2 * pc);
        }
        // append w to V (the lane's own columns)
#pragma unroll
        for (int pc = 0; pc < P; ++pc)
            *reinterpret_cast<float2*>(Vt + m * DV + 2 * pc) = w[pc];

        uint8_t* gcodes_tile = p.codes + ti.code_off;
        for (int g = 0; g < G; ++g) {
            if (UPD != kDelta && g > 0) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait_bounded(&bars[ic.slot], ic.par, p.timeout_ns));
                if (!ok) break;
            }
            const uint8_t* sm = wsm + hdr + ic.slot * S::kBytes;
            const float* ss = reinterpret_cast<const float*>(sm + S::kScales) + lane * C;
            const float* qs = qs_t + g * GROUP;
            const float* gs = gs_t + g * GROUP;
            float* gscale = p.scales + (static_cast<int64_t>(tile) * G + g) * DV + lane * C;
            uint8_t* gcodes = gcodes_tile + ti.goff(g, GROUP * DV / 2);
            const bool int8g = ti.bits(g) == 8;
            const float* Ug = Ut + g * GROUP;
            if constexpr (MODE == kSR) {
                // the group's row table of the hash (the previous group's
                // readers finished at the warp barrier ending it)
                if (rowtab) {
                    for (int r = lane; r < GROUP; r += 32) {
                        const SrRow rr = sr_row(static_cast<uint32_t>(hkey >> 32),
                                                static_cast<uint32_t>(g * GROUP + r), hcarry);
                        rtab2[r] = make_uint2(rr.sh, rr.p);
                    }
                    __syncwarp();
                }
            }
            float2 op = o[0], oq = o[P - 1];
#pragma unroll 1
            for (int pc = 0; pc < P; ++pc) {
                const float2 sc = *reinterpret_cast<const float2*>(ss + 2 * pc);
                const uint32_t j0 = static_cast<uint32_t>(lane * C + 2 * pc);
                float vc0[MR], vc1[MR];
                if (merge) {
#pragma unroll
                    for (int l = 0; l < MR; ++l) {
                        const float2 vv = *reinterpret_cast<const float2*>(Vt + l * DV + 2 * pc);
                        vc0[l] = vv.x;
                        vc1[l] = vv.y;
                    }
                }
                if constexpr (MODE == kRTN) {
                    if (int8g)
                        pair_step_lrb_rtn<GROUP, GATE, 8>(sm, pc * PairGeo<GROUP, 8>::UNITS, sc, qs,
                                                          gs, gscalar, op, gcodes, gscale + 2 * pc,
                                                          lane, merge, R, Ug, dk, vc0, vc1);
                    else
                        pair_step_lrb_rtn<GROUP, GATE, 4>(sm, pc * PairGeo<GROUP, 4>::UNITS, sc, qs,
                                                          gs, gscalar, op, gcodes, gscale + 2 * pc,
                                                          lane, merge, R, Ug, dk, vc0, vc1);
                } else if (int8g)
                    pair_step_lrb<GROUP, GATE, MODE, 8, lrb_staged(MODE, MERGE)>(sm, pc * PairGeo<GROUP, 8>::UNITS, sc, qs, gs,
                                                        gscalar, op, gcodes, gscale + 2 * pc, hkey,
                                                        g * GROUP, j0, lane, xs, merge, R, Ug, dk,
                                                        vc0, vc1, rtab, rowtab);
                else
                    pair_step_lrb<GROUP, GATE, MODE, 4, lrb_staged(MODE, MERGE)>(sm, pc * PairGeo<GROUP, 4>::UNITS, sc, qs, gs,
                                                        gscalar, op, gcodes, gscale + 2 * pc, hkey,
                                                        g * GROUP, j0, lane, xs, merge, R, Ug, dk,
                                                        vc0, vc1, rtab, rowtab);
                if constexpr (P == 2) {
                    const float2 to = op;
                    op = oq; oq = to;
                }
            }
            o[0] = op;
            o[P - 1] = P == 2 ? oq : op;
            ++kc;
            ic.advance(NS);
            __syncwarp();
            if (lane == 0) fence_proxy_async_smem();
            issue_next();
        }
        if (!ok) break;
        // output: the state part's chain, then the buffer's share in component order
        float ov[C];
#pragma unroll
        for (int pc = 0; pc < P; ++pc) {
            ov[2 * pc] = o[pc].x;
            ov[2 * pc + 1] = o[pc].y;
        }
#pragma unroll
        for (int l = 0; l < MR; ++l) {
            const float fl = __shfl_sync(0xffffffffu, chain, 16 + l);
            if (l <= m)
#pragma unroll
                for (int c = 0; c < C; ++c) ov[c] = __fmaf_rn(fl, Vt[l * DV + c], ov[c]);
        }
        float* outp = static_cast<float*>(p.out) + static_cast<int64_t>(tile) * DV + lane * C;
#pragma unroll
        for (int c = 0; c < C; ++c) outp[c] = ov[c];
        // the buffer back to global memory (emptied after a merge)
        float* Ugl = lp.U + static_cast<int64_t>(tile) * R * dk;
        for (int idx = lane * 4; idx < (m + 1) * dk; idx += 128) {
            const float4 t = merge ? make_float4(0.f, 0.f, 0.f, 0.f)
                                   : *reinterpret_cast<const float4*>(Ut + idx);
            *reinterpret_cast<float4*>(Ugl + idx) = t;
        }
        float* Vgl = lp.V + static_cast<int64_t>(tile) * R * DV + lane * C;
        for (int l = 0; l <= m; ++l)
#pragma unroll
            for (int c = 0; c < C; ++c) Vgl[l * DV + c] = merge ? 0.0f : Vt[l * DV + c];
        __syncwarp();
    }
    if (!ok) {
        if (lane == 0) atomicOr(p.err, kErrTimeout);
        Ring r = ic;
        for (int64_t k = kc; k < ki; ++k) {
            mbar_wait_bounded(&bars[r.slot], r.par, p.timeout_ns);
            r.advance(NS);
        }
    }
}

// Defines `const void* NAME(C, group, update_kind, gate_kind, merge)`: the
// streaming bypass kernel with rounding MODE for a merge step or another step,
// or nullptr when that shape is not compiled.
#define LRS_LRB_STREAM_PICK2(MODE, CC, GG, MG)                                                 \
    if (update_kind == kGated && gate_kind == kGatePerKey)                                     \
        return reinterpret_cast<const void*>(                                                  \
            &lrb_step_kernel<CC, GG, kGated, kGatePerKey, MODE, MG>);                          \
    if (update_kind == kGated && gate_kind == kGate)                                           \
        return reinterpret_cast<const void*>(&lrb_step_kernel<CC, GG, kGated, kGate, MODE, MG>); \
    if (update_kind == kDelta && gate_kind == kGate)                                           \
        return reinterpret_cast<const void*>(&lrb_step_kernel<CC, GG, kDelta, kGate, MODE, MG>); \
    return nullptr;
#define LRS_LRB_STREAM_PICK1(MODE, CC, GG)                                                     \
    if (C == CC && group == GG) {                                                              \
        if (merge) {                                                                           \
            LRS_LRB_STREAM_PICK2(MODE, CC, GG, true)                                           \
        }                                                                                      \
        LRS_LRB_STREAM_PICK2(MODE, CC, GG, false)                                              \
    }
#define LRS_LRB_STREAM_VARIANTS(NAME, MODE)                                                    \
    const void* NAME(int C, int group, int update_kind, int gate_kind, bool merge) {           \
        LRS_LRB_STREAM_PICK1(MODE, 4, 16)                                                      \
        LRS_LRB_STREAM_PICK1(MODE, 4, 32)                                                      \
        LRS_LRB_STREAM_PICK1(MODE, 2, 16)                                                      \
        LRS_LRB_STREAM_PICK1(MODE, 2, 32)                                                      \
        LRS_LRB_STREAM_PICK1(MODE, 2, 64)                                                      \
        return nullptr;                                                                        \
    }

}  // namespace lrs
