// chunk_gated.cuh -- the multi-token (chunked) update for the gated forms
// (GLA per-key decay, scalar decay), with two threads per column pair.
//
// What it computes is chunk_kernel.cuh's: T tokens applied in order to the
// dequantized state in fp32, one output per token, one requantization at the
// end. The mapping differs. Thread (column pair cp, half h) holds columns
// 2cp and 2cp + 1 over key rows [h*d_k/2, (h+1)*d_k/2) in registers, so one
// broadcast shared-memory load of q, k or the gates feeds two columns, and
// each thread runs two independent output chains.
//
// The output o_j = sum_i q_i x_ij is one chain in key order: the lower half
// computes its rows' part and the upper half continues from it. The halves
// are skewed by one token: in iteration n the lower half applies token n and
// the upper half token n - 1, starting its chain from the lower half's
// partial sum of the previous iteration. Lanes 0-15 of a warp are lower
// halves and lanes 16-31 the upper halves of the same 16 column pairs, so the
// partial sums move by one shuffle. The gated update of a row needs only that
// row's state and the token's inputs, so the skew changes no value; the delta
// rule's u = k^T S needs the whole column before any row is updated, so it
// keeps chunk_kernel.cuh's mapping.
//
// Iteration n reads the ring slots of tokens n and n - 1; the slot of token
// n - 1 is refilled after the iteration. Requantization is per thread: a
// thread holds both columns of its pair for whole scale groups (group <= d_k/2)
// and writes its own 16-byte units of the state layout.
#pragma once

#include "chunk_kernel.cuh"

namespace lrs {

// Decode the thread's rows of one scale group (codes at gbase, scale row g)
// into row pairs of its two columns: xr[c][rp] = (x[2rp][c], x[2rp+1][c]).
template <int DV, int GROUP, int BITS>
__device__ __forceinline__ void gated_decode_group(const uint8_t* cs, const float* ss, int gbase,
                                                   int g, int pc, int own, int c0,
                                                   float2 (&x0)[GROUP / 2], float2 (&x1)[GROUP / 2]) {
    using PG = PairGeo<GROUP, BITS>;
    constexpr float K = kTwo23 + Q<BITS>::kBias;
    const float2 s0 = f2(ss[g * DV + c0]), s1 = f2(ss[g * DV + c0 + 1]);
#pragma unroll
    for (int un = 0; un < PG::UNITS; ++un) {
        const uint4 raw =
            *reinterpret_cast<const uint4*>(cs + unit_byte<GROUP, BITS>(gbase, pc, un, own));
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[PG::EPW];
            decode_word_biased<BITS>(wd[wi], f);
#pragma unroll
            for (int rp = 0; rp < PG::RPW / 2; ++rp) {
                const int r2 = (un * PG::RPU + wi * PG::RPW) / 2 + rp;   // row pair in the group
                x0[r2] = mul2(add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-K)), s0);
                x1[r2] = mul2(add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-K)), s1);
            }
        }
    }
}

// New scales and codes of one scale group of the thread's two columns: the
// codes replace the old ones in the thread's own units of cs (BDR reads each
// old word just before overwriting it), the scales are returned.
template <int DV, int GROUP, int MODE, int BITS>
__device__ __forceinline__ float2 gated_requantize_group(uint8_t* cs, const float* ss, int gbase,
                                                         int g, int pc, int own, int c0, int row0,
                                                         const float2 (&x0)[GROUP / 2],
                                                         const float2 (&x1)[GROUP / 2],
                                                         uint64_t hkey) {
    using PG = PairGeo<GROUP, BITS>;
    constexpr float K = kTwo23 + Q<BITS>::kBias;
    float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
    for (int r2 = 0; r2 < GROUP / 2; ++r2) {
        a0 = max_abs3(a0, x0[r2].x, x0[r2].y);
        a1 = max_abs3(a1, x1[r2].x, x1[r2].y);
    }
    float2 snew, inv;
    new_scales<BITS>(a0, a1, snew, inv);
    const float2 inv0 = f2(inv.x), inv1 = f2(inv.y);
    const float2 sn0 = f2(snew.x), sn1 = f2(snew.y);
    const float2 so0 = f2(ss[g * DV + c0]), so1 = f2(ss[g * DV + c0 + 1]);
#pragma unroll
    for (int un = 0; un < PG::UNITS; ++un) {
        uint32_t* up = reinterpret_cast<uint32_t*>(cs + unit_byte<GROUP, BITS>(gbase, pc, un, own));
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[PG::EPW];
            if constexpr (MODE == kBDR) decode_word_biased<BITS>(up[wi], f);
            float t[PG::EPW];
#pragma unroll
            for (int rp = 0; rp < PG::RPW / 2; ++rp) {
                const int r2 = (un * PG::RPU + wi * PG::RPW) / 2 + rp;
                float2 dq0 = f2(0.0f), dq1 = f2(0.0f);
                if constexpr (MODE == kBDR) {
                    dq0 = mul2(add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-K)), so0);
                    dq1 = mul2(add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-K)), so1);
                }
                const uint32_t i = static_cast<uint32_t>(row0 + 2 * r2);
                const float2 kb0 = make_float2(word_bias<BITS>(4 * rp), word_bias<BITS>(4 * rp + 2));
                const float2 kb1 = make_float2(word_bias<BITS>(4 * rp + 1), word_bias<BITS>(4 * rp + 3));
                const float2 t0 = round_rows<MODE, BITS, true>(x0[r2], inv0, dq0, sn0, kb0, hkey, i,
                                                               static_cast<uint32_t>(c0));
                const float2 t1 = round_rows<MODE, BITS, true>(x1[r2], inv1, dq1, sn1, kb1, hkey, i,
                                                               static_cast<uint32_t>(c0 + 1));
                t[4 * rp] = t0.x;
                t[4 * rp + 2] = t0.y;
                t[4 * rp + 1] = t1.x;
                t[4 * rp + 3] = t1.y;
            }
            up[wi] = encode_word<BITS>(t);
        }
    }
    return snew;
}

template <int DK, int DV, int GROUP, int GATE, int MODE>
__global__ void __launch_bounds__(DV, (3 * 128) / DV) chunk_gated_kernel(const ChunkParams p) {
    using S = ChunkSmem<DK, DV, GROUP, GATE>;
    constexpr int G = DK / GROUP;
    constexpr int C = DV / 32;
    constexpr int HK = DK / 2;                   // rows per half
    constexpr int GH = HK / GROUP;               // scale groups per half
    static_assert(GROUP <= HK && HK % GROUP == 0, "a scale group must lie in one half");
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bar_state = reinterpret_cast<uint64_t*>(smem);
    uint64_t* bar_tok = bar_state + 1;
    uint8_t* cs = smem + S::kCodes;
    float* ss = reinterpret_cast<float*>(smem + S::kScales);
    const int lane = threadIdx.x & 31;
    const int h = lane >> 4;                     // 0: lower rows, 1: upper rows
    const int cp = (threadIdx.x >> 5) * 16 + (lane & 15);
    const int c0 = 2 * cp;                       // the pair's first column
    const int own = c0 / C, pc = (c0 % C) / 2;   // its place in the state layout
    const int rbase = h * HK;

    if (threadIdx.x == 0) {
        mbar_init(bar_state, 1);
        for (int s = 0; s < kChunkSlots; ++s) mbar_init(&bar_tok[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    const int T = p.T;
    const int NS = T < kChunkSlots ? T : kChunkSlots;
    uint32_t par_state = 0;
    int64_t tok_base = 0;
    bool ok = true;
    int64_t issued_hi = 0;
    int64_t drain_lo = 0;
    bool state_pending = false;

    for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x) {
        TileLayout tl;
        tl.load(p.prec_map, p.head_offsets, p.batch_stride, p.H, p.pgroups, G, GROUP * DV,
                tile / p.H, tile % p.H);
        if (!tl.ok) {
            if (threadIdx.x == 0) atomicOr(p.err, kErrLayout);
            continue;
        }
        const int64_t code_off = tl.code_off;
        const uint32_t cbytes = static_cast<uint32_t>(tl.goff(G, GROUP * DV / 2));
        if (threadIdx.x == 0 && !p.inject) {
            fence_proxy_async_smem();
            const uint64_t pol = policy_evict_first();
            mbar_arrive_expect_tx(bar_state, cbytes + G * DV * 4);
            bulk_g2s(cs, p.codes + code_off, cbytes, bar_state, pol);
            bulk_g2s(ss, p.scales + static_cast<int64_t>(tile) * G * DV, G * DV * 4, bar_state,
                     pol);
            for (int t = 0; t < NS; ++t)
                issue_token<DK, DV, GROUP, GATE>(p, smem, static_cast<int>((tok_base + t) % NS),
                                                 tile, t);
            issued_hi = tok_base + NS;
        }
        ok = __syncthreads_and(mbar_wait_bounded(bar_state, par_state, p.timeout_ns));
        if (!ok) {
            state_pending = true;
            drain_lo = tok_base;
            break;
        }
        par_state ^= 1u;

        // the thread's rows of both columns, as row pairs
        float2 xa[HK / 2], xb[HK / 2];
#pragma unroll
        for (int gh = 0; gh < GH; ++gh) {
            const int g = h * GH + gh;
            const int gbase = static_cast<int>(tl.goff(g, GROUP * DV / 2));
            float2 ya[GROUP / 2], yb[GROUP / 2];
            if (tl.bits(g) == 8)
                gated_decode_group<DV, GROUP, 8>(cs, ss, gbase, g, pc, own, c0, ya, yb);
            else
                gated_decode_group<DV, GROUP, 4>(cs, ss, gbase, g, pc, own, c0, ya, yb);
#pragma unroll
            for (int r2 = 0; r2 < GROUP / 2; ++r2) {
                xa[gh * GROUP / 2 + r2] = ya[r2];
                xb[gh * GROUP / 2 + r2] = yb[r2];
            }
        }

        float2 carry = f2(0.0f);     // upper half: the lower half's partial sums
#pragma unroll 1
        for (int n = 0; n <= T; ++n) {
            if (n < T) {
                const int64_t u = tok_base + n;
                const bool good = mbar_wait_bounded(&bar_tok[u % NS],
                                                    static_cast<uint32_t>((u / NS) & 1), p.timeout_ns);
                if (__syncthreads_or(!good)) {
                    ok = false;
                    drain_lo = u;
                    break;
                }
            }
            const int t = n - h;                 // this half's token
            float2 o = h ? carry : f2(0.0f);
            if (t >= 0 && t < T) {
                const int slot = static_cast<int>((tok_base + t) % NS);
                const uint8_t* tb = smem + S::kRing + slot * S::kTok;
                const float* tq = reinterpret_cast<const float*>(tb + S::kQ) + rbase;
                const float* tkk = reinterpret_cast<const float*>(tb + S::kK) + rbase;
                const float* tg = reinterpret_cast<const float*>(tb + S::kG) + rbase;
                const float2 wv = *reinterpret_cast<const float2*>(tb + S::kV + c0 * 4);
                const float2 w0 = f2(wv.x), w1 = f2(wv.y);
                const int64_t row = static_cast<int64_t>(t) * p.ntiles + tile;
                const float2 gs2 = GATE == kGate ? f2(__ldg(p.gates + row)) : f2(0.0f);
#pragma unroll
                for (int r = 0; r < HK; r += 4) {
                    if (r % 16 == 0) asm volatile("" ::: "memory");   // bound the load hoisting
                    const float4 kv = lds4(tkk + r);
                    const float4 qv = lds4(tq + r);
                    float2 g0 = gs2, g1 = gs2;
                    if (GATE == kGatePerKey) {
                        const float4 gv = lds4(tg + r);
                        g0 = make_float2(gv.x, gv.y);
                        g1 = make_float2(gv.z, gv.w);
                    }
                    const float2 k0 = make_float2(kv.x, kv.y), k1 = make_float2(kv.z, kv.w);
                    // x = g * x + RN(k w), per column, row pairs
                    const float2 a0 = fma2(g0, xa[r / 2], mul2(k0, w0));
                    const float2 a1 = fma2(g1, xa[r / 2 + 1], mul2(k1, w0));
                    const float2 b0 = fma2(g0, xb[r / 2], mul2(k0, w1));
                    const float2 b1 = fma2(g1, xb[r / 2 + 1], mul2(k1, w1));
                    xa[r / 2] = a0; xa[r / 2 + 1] = a1;
                    xb[r / 2] = b0; xb[r / 2 + 1] = b1;
                    // the two output chains, key order
                    o.x = __fmaf_rn(qv.x, a0.x, o.x);
                    o.y = __fmaf_rn(qv.x, b0.x, o.y);
                    o.x = __fmaf_rn(qv.y, a0.y, o.x);
                    o.y = __fmaf_rn(qv.y, b0.y, o.y);
                    o.x = __fmaf_rn(qv.z, a1.x, o.x);
                    o.y = __fmaf_rn(qv.z, b1.x, o.y);
                    o.x = __fmaf_rn(qv.w, a1.y, o.x);
                    o.y = __fmaf_rn(qv.w, b1.y, o.y);
                }
                if (h == 1) *reinterpret_cast<float2*>(p.out + row * DV + c0) = o;
            }
            // the lower half's partial sums of token n go to the upper half
            const float ox = __shfl_up_sync(0xffffffffu, o.x, 16);
            const float oy = __shfl_up_sync(0xffffffffu, o.y, 16);
            carry = make_float2(ox, oy);
            __syncthreads();                     // every thread is done with token n - 1
            if (threadIdx.x == 0 && n >= 1 && n - 1 + NS < T) {
                const int64_t u = tok_base + n - 1;
                fence_proxy_async_smem();
                issue_token<DK, DV, GROUP, GATE>(p, smem, static_cast<int>(u % NS), tile,
                                                 n - 1 + NS);
                issued_hi = u + NS + 1;
            }
        }
        if (!ok) break;
        tok_base += T;

        // one requantization at the chunk's end, per thread and scale group
        const int b = tile / p.H, hh = tile - b * p.H;
        const uint64_t hkey = MODE == kSR ? tile_hash_key(p.seed, p.step,
                                                          static_cast<uint32_t>(b),
                                                          static_cast<uint32_t>(hh))
                                          : 0ull;
        float2 snew[GH];
#pragma unroll
        for (int gh = 0; gh < GH; ++gh) {
            const int g = h * GH + gh;
            const int gbase = static_cast<int>(tl.goff(g, GROUP * DV / 2));
            float2 ya[GROUP / 2], yb[GROUP / 2];
#pragma unroll
            for (int r2 = 0; r2 < GROUP / 2; ++r2) {
                ya[r2] = xa[gh * GROUP / 2 + r2];
                yb[r2] = xb[gh * GROUP / 2 + r2];
            }
            snew[gh] = tl.bits(g) == 8
                           ? gated_requantize_group<DV, GROUP, MODE, 8>(cs, ss, gbase, g, pc, own,
                                                                        c0, g * GROUP, ya, yb, hkey)
                           : gated_requantize_group<DV, GROUP, MODE, 4>(cs, ss, gbase, g, pc, own,
                                                                        c0, g * GROUP, ya, yb, hkey);
        }
#pragma unroll
        for (int gh = 0; gh < GH; ++gh)
            *reinterpret_cast<float2*>(ss + (h * GH + gh) * DV + c0) = snew[gh];
        __syncthreads();
        // write the tile back: 16-byte streaming stores
        uint8_t* gc = p.codes + code_off;
        for (int off = threadIdx.x * 16; off < static_cast<int>(cbytes); off += DV * 16) {
            const uint4 vv = *reinterpret_cast<const uint4*>(cs + off);
            st_cs_u4(gc + off, vv.x, vv.y, vv.z, vv.w);
        }
        float* gsc = p.scales + static_cast<int64_t>(tile) * G * DV;
        for (int off = threadIdx.x * 4; off < G * DV; off += DV * 4) {
            const float4 vv = *reinterpret_cast<const float4*>(ss + off);
            *reinterpret_cast<float4*>(gsc + off) = vv;
        }
        __syncthreads();                         // before the next tile's copies land
    }
    if (!ok && threadIdx.x == 0) {
        atomicOr(p.err, kErrTimeout);
        if (state_pending) mbar_wait_bounded(bar_state, par_state, p.timeout_ns);
        for (int64_t u = drain_lo; u < issued_hi; ++u)
            mbar_wait_bounded(&bar_tok[u % NS], static_cast<uint32_t>((u / NS) & 1),
                              p.timeout_ns);
    }
}

// The gated form's chunk kernel for a shape: this one where a scale group
// fits in half the key rows, chunk_kernel otherwise.
template <int DK, int DV, int GROUP, int GATE, int MODE>
inline const void* chunk_gated_pick() {
    if constexpr (GROUP <= DK / 2)
        return reinterpret_cast<const void*>(&chunk_gated_kernel<DK, DV, GROUP, GATE, MODE>);
    else
        return reinterpret_cast<const void*>(&chunk_kernel<DK, DV, GROUP, kGated, GATE, MODE>);
}

}  // namespace lrs
