// chunk_gated.cuh -- the multi-token (chunked) update for the gated forms
// (GLA per-key decay, scalar decay), with two threads per column pair.
//
// What it computes is chunk_kernel.cuh's: T tokens applied in order to the
// dequantized state in fp32, one output per token, one requantization at the
// end. The mapping differs. The key rows are cut into SEG segments (2 in the
// compiled variants); a thread holds SEG/2 column pairs over one segment's rows
// in registers, so one broadcast shared-memory load of q, k or the gates
// feeds SEG columns, and each thread runs SEG independent output chains. The
// description below is for SEG = 2; with more segments each passes its
// partial sums to the next, one token later.
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

template <int DK, int DV, int GROUP, int GATE, int MODE, int SEG>
__global__ void __launch_bounds__(DV, (3 * 128) / DV) chunk_gated_kernel(const ChunkParams p) {
    using S = ChunkSmem<DK, DV, GROUP, GATE>;
    constexpr int G = DK / GROUP;
    constexpr int C = DV / 32;
    constexpr int NP = SEG / 2;                  // column pairs per thread
    constexpr int CPL = 2 * NP;                  // columns per thread
    constexpr int LPS = 32 / SEG;                // lanes per row segment
    constexpr int RS = DK / SEG;                 // key rows per segment
    constexpr int GS = RS / GROUP;               // scale groups per segment
    static_assert(SEG == 2 || SEG == 4, "two or four row segments");
    static_assert(GROUP <= RS && RS % GROUP == 0 && RS % 4 == 0, "a scale group must lie in one segment");
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bar_state = reinterpret_cast<uint64_t*>(smem);
    uint64_t* bar_tok = bar_state + 1;
    uint8_t* cs = smem + S::kCodes;
    float* ss = reinterpret_cast<float*>(smem + S::kScales);
    const int lane = threadIdx.x & 31;
    const int seg = lane / LPS;                  // this thread's row segment
    const int cbase = (threadIdx.x >> 5) * 32 + (lane % LPS) * CPL;   // its first column
    const int rbase = seg * RS;
    int own[NP], pc[NP];                         // each pair's place in the state layout
#pragma unroll
    for (int q = 0; q < NP; ++q) {
        own[q] = (cbase + 2 * q) / C;
        pc[q] = ((cbase + 2 * q) % C) / 2;
    }

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

        // the thread's rows of its columns, as row pairs: x[pair][column][row pair]
        float2 x[NP][2][RS / 2];
#pragma unroll
        for (int gs = 0; gs < GS; ++gs) {
            const int g = seg * GS + gs;
            const int gbase = static_cast<int>(tl.goff(g, GROUP * DV / 2));
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                float2 ya[GROUP / 2], yb[GROUP / 2];
                if (tl.bits(g) == 8)
                    gated_decode_group<DV, GROUP, 8>(cs, ss, gbase, g, pc[q], own[q], cbase + 2 * q,
                                                     ya, yb);
                else
                    gated_decode_group<DV, GROUP, 4>(cs, ss, gbase, g, pc[q], own[q], cbase + 2 * q,
                                                     ya, yb);
#pragma unroll
                for (int r2 = 0; r2 < GROUP / 2; ++r2) {
                    x[q][0][gs * GROUP / 2 + r2] = ya[r2];
                    x[q][1][gs * GROUP / 2 + r2] = yb[r2];
                }
            }
        }

        float carry[CPL];            // the previous segment's partial sums
#pragma unroll
        for (int c = 0; c < CPL; ++c) carry[c] = 0.0f;
#pragma unroll 1
        for (int n = 0; n < T + SEG - 1; ++n) {
            // Token n: every thread waits on its barrier itself; a thread whose
            // wait runs out skips the work, and the one CTA barrier of the
            // iteration (below) ends the loop for all. The tokens of the other
            // segments passed that barrier in earlier iterations.
            bool good = true;
            if (n < T) {
                const int64_t u = tok_base + n;
                good = mbar_wait_bounded(&bar_tok[u % NS], static_cast<uint32_t>((u / NS) & 1),
                                         p.timeout_ns);
            }
            const int t = n - seg;               // this segment's token
            float o[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) o[c] = seg ? carry[c] : 0.0f;
            if (good && t >= 0 && t < T) {
                const int slot = static_cast<int>((tok_base + t) % NS);
                const uint8_t* tb = smem + S::kRing + slot * S::kTok;
                const float* tq = reinterpret_cast<const float*>(tb + S::kQ) + rbase;
                const float* tkk = reinterpret_cast<const float*>(tb + S::kK) + rbase;
                const float* tg = reinterpret_cast<const float*>(tb + S::kG) + rbase;
                float2 wc[CPL];                  // w of each column, both halves
                {
                    const float* tv = reinterpret_cast<const float*>(tb + S::kV) + cbase;
                    if constexpr (CPL == 2) {
                        const float2 v2 = *reinterpret_cast<const float2*>(tv);
                        wc[0] = f2(v2.x); wc[1] = f2(v2.y);
                    } else {
                        const float4 v4 = *reinterpret_cast<const float4*>(tv);
                        wc[0] = f2(v4.x); wc[1] = f2(v4.y); wc[2] = f2(v4.z); wc[3] = f2(v4.w);
                    }
                }
                const int64_t row = static_cast<int64_t>(t) * p.ntiles + tile;
                const float2 gs2 = GATE == kGate ? f2(__ldg(p.gates + row)) : f2(0.0f);
#pragma unroll
                for (int r = 0; r < RS; r += 4) {
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
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const int c = 2 * q + cc;
                            // x = g * x + RN(k w), row pairs
                            const float2 a = fma2(g0, x[q][cc][r / 2], mul2(k0, wc[c]));
                            const float2 b = fma2(g1, x[q][cc][r / 2 + 1], mul2(k1, wc[c]));
                            x[q][cc][r / 2] = a;
                            x[q][cc][r / 2 + 1] = b;
                            // this column's output chain, key order
                            o[c] = __fmaf_rn(qv.x, a.x, o[c]);
                            o[c] = __fmaf_rn(qv.y, a.y, o[c]);
                            o[c] = __fmaf_rn(qv.z, b.x, o[c]);
                            o[c] = __fmaf_rn(qv.w, b.y, o[c]);
                        }
                    }
                }
                if (seg == SEG - 1) {
                    float* op = p.out + row * DV + cbase;
                    if constexpr (CPL == 2)
                        *reinterpret_cast<float2*>(op) = make_float2(o[0], o[1]);
                    else
                        *reinterpret_cast<float4*>(op) = make_float4(o[0], o[1], o[2], o[3]);
                }
            }
            // each segment's partial sums go to the next segment
#pragma unroll
            for (int c = 0; c < CPL; ++c) carry[c] = __shfl_up_sync(0xffffffffu, o[c], LPS);
            // every thread is done with token n - SEG + 1; any wait that ran out
            if (__syncthreads_or(!good)) {
                ok = false;
                drain_lo = tok_base + n;
                break;
            }
            const int done = n - SEG + 1;        // the token no segment reads again
            if (threadIdx.x == 0 && done >= 0 && done + NS < T) {
                const int64_t u = tok_base + done;
                fence_proxy_async_smem();
                issue_token<DK, DV, GROUP, GATE>(p, smem, static_cast<int>(u % NS), tile, done + NS);
                issued_hi = u + NS + 1;
            }
        }
        if (!ok) break;
        tok_base += T;

        // one requantization at the chunk's end, per thread, pair and scale group
        const int b = tile / p.H, hh = tile - b * p.H;
        const uint64_t hkey = MODE == kSR ? tile_hash_key(p.seed, p.step,
                                                          static_cast<uint32_t>(b),
                                                          static_cast<uint32_t>(hh))
                                          : 0ull;
        float2 snew[GS][NP];
#pragma unroll
        for (int gs = 0; gs < GS; ++gs) {
            const int g = seg * GS + gs;
            const int gbase = static_cast<int>(tl.goff(g, GROUP * DV / 2));
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                float2 ya[GROUP / 2], yb[GROUP / 2];
#pragma unroll
                for (int r2 = 0; r2 < GROUP / 2; ++r2) {
                    ya[r2] = x[q][0][gs * GROUP / 2 + r2];
                    yb[r2] = x[q][1][gs * GROUP / 2 + r2];
                }
                snew[gs][q] =
                    tl.bits(g) == 8
                        ? gated_requantize_group<DV, GROUP, MODE, 8>(cs, ss, gbase, g, pc[q], own[q],
                                                                     cbase + 2 * q, g * GROUP, ya,
                                                                     yb, hkey)
                        : gated_requantize_group<DV, GROUP, MODE, 4>(cs, ss, gbase, g, pc[q], own[q],
                                                                     cbase + 2 * q, g * GROUP, ya,
                                                                     yb, hkey);
            }
        }
#pragma unroll
        for (int gs = 0; gs < GS; ++gs)
#pragma unroll
            for (int q = 0; q < NP; ++q)
                *reinterpret_cast<float2*>(ss + (seg * GS + gs) * DV + cbase + 2 * q) = snew[gs][q];
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
// (Four segments, each thread holding two pairs over a quarter of the rows,
// measured 3-5% slower than two on the throughput and int4 workloads: the
// three-token skew costs more than the extra chains per thread save.)
template <int DK, int DV, int GROUP, int GATE, int MODE>
inline const void* chunk_gated_pick() {
    if constexpr (GROUP <= DK / 2)
        return reinterpret_cast<const void*>(&chunk_gated_kernel<DK, DV, GROUP, GATE, MODE, 2>);
    else
        return reinterpret_cast<const void*>(&chunk_kernel<DK, DV, GROUP, kGated, GATE, MODE>);
}

}  // namespace lrs
