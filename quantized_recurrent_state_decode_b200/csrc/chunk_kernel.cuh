// chunk_kernel.cuh -- multi-token (chunked) update of the quantized state.
//
// T tokens are applied to each (batch, head) tile in order, in fp32, starting
// from the dequantized state, with one output per token; the state is
// requantized once, after the last token (BDR compares with the state at the
// chunk's start). This is the step before decode -- a prefill chunk, or the
// tokens of a speculative-decoding verification -- where requantizing after
// every token would repeat the error that the methods' sources attribute to
// repeated requantization ("Quantizing Recurrent Language Models Is Easier
// Than You Think", abstract; "Preserving Updates in Low-Bit Recurrent State
// Quantization", abstract).
//
// Mapping: one CTA of d_v threads works on one tile at a time; thread j owns
// value column j over all d_k key rows, held in registers for the whole
// chunk, so every key-axis reduction (u = k^T S for the delta rule, o = S^T q,
// the per-group absmax) runs inside one thread in key order. The tile's codes
// and scales arrive by one bulk copy; the tokens stream through a ring of
// shared-memory slots (q, k, v and per-key gates of one token each), refilled
// by thread 0 after every token. At the end the new codes are packed into the
// state's layout in shared memory (column pairs meet through one shuffle) and
// written back with 16-byte stores.
#pragma once

#include "lrs_internal.h"
#include "step_kernel.cuh"

namespace lrs {

constexpr int kChunkSlots = 8;

struct ChunkParams {
    uint8_t* codes;
    float* scales;
    const uint8_t* prec_map;
    const int64_t* head_offsets;
    int64_t batch_stride;
    const float* q;       // [T][ntiles][d_k]
    const float* k;       // [T][ntiles][d_k]
    const float* v;       // [T][ntiles][d_v]
    const float* gates;   // [T][ntiles][d_k] or [T][ntiles]
    const float* beta;    // [T][ntiles] (delta rule)
    float* out;           // [T][ntiles][d_v]
    uint64_t seed, step;
    unsigned* err;
    uint64_t timeout_ns;
    int32_t H, ntiles, T, inject;
    int32_t pgroups;      // widths in prec_map per head (1) or per (head, group) (G)
};

// Shared memory of one CTA: barriers | codes (int8 capacity) | scales |
// token slots (q, k, [gate], v as fp32). A slot is padded by 16 bytes so that
// the same row of two adjacent slots falls in different shared-memory banks
// (chunk_gated_kernel reads two tokens' rows at once).
template <int DK, int DV, int GROUP, int GATE>
struct ChunkSmem {
    static constexpr int G = DK / GROUP;
    static constexpr int kCodes = 128;
    static constexpr int kScales = kCodes + DK * DV;
    static constexpr int kRing = kScales + G * DV * 4;
    static constexpr int kQ = 0, kK = DK * 4, kG = 2 * DK * 4;
    static constexpr int kV = kG + (GATE == kGatePerKey ? DK * 4 : 0);
    static constexpr int kTok = kV + DV * 4 + 16;
    static constexpr int kBytes = kRing + kChunkSlots * kTok;
    static_assert(kTok % 16 == 0 && kRing % 16 == 0, "alignment");
};

// Column j's place in the state layout: lane l = j / C of a warp's walk owns
// columns [l*C, l*C + C); j is column cc of that lane's column pair pc.
struct ColumnPlace {
    int owner, pc, cc;
    __device__ ColumnPlace(int j, int C) : owner(j / C), pc((j % C) / 2), cc(j & 1) {}
};

// Byte offset, inside the tile's codes, of the 16-byte unit `un` of the pair
// `pc` of owner lane `owner` in the scale group whose codes start at gbase.
template <int GROUP, int BITS>
__device__ __forceinline__ int unit_byte(int gbase, int pc, int un, int owner) {
    using PG = PairGeo<GROUP, BITS>;
    return gbase + ((pc * PG::UNITS + un) * 32 + owner) * 16;
}

// Dequantize one scale group (codes at gbase, scale row g) of column j:
// y[r] = RN(code * s[g][j]) for the group's rows r.
template <int DV, int GROUP, int BITS>
__device__ __forceinline__ void decode_group(const uint8_t* cs, const float* ss,
                                             const ColumnPlace& cp, int j, int g, int gbase,
                                             float (&y)[GROUP]) {
    using PG = PairGeo<GROUP, BITS>;
    constexpr float K = kTwo23 + Q<BITS>::kBias;
    const float s = ss[g * DV + j];
#pragma unroll
    for (int un = 0; un < PG::UNITS; ++un) {
        const uint4 raw =
            *reinterpret_cast<const uint4*>(cs + unit_byte<GROUP, BITS>(gbase, cp.pc, un, cp.owner));
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int r = un * PG::RPU + w * PG::RPW;
            if constexpr (BITS == 8) {
                // bytes: (r, c0), (r, c1), (r+1, c0), (r+1, c1)
                y[r] = __fmul_rn(byte_to_biased_float(wd[w], cp.cc) - K, s);
                y[r + 1] = __fmul_rn(byte_to_biased_float(wd[w], 2 + cp.cc) - K, s);
            } else {
                // byte n holds elements n (low nibble) and n + 4 (high) of the
                // word's rows r..r+3 x 2 columns, element 2*(row - r) + column
                const uint32_t lo = wd[w] & 0x0F0F0F0Fu, hi = (wd[w] >> 4) & 0x0F0F0F0Fu;
                y[r] = __fmul_rn(byte_to_biased_float(lo, cp.cc) - K, s);
                y[r + 1] = __fmul_rn(byte_to_biased_float(lo, 2 + cp.cc) - K, s);
                y[r + 2] = __fmul_rn(byte_to_biased_float(hi, cp.cc) - K, s);
                y[r + 3] = __fmul_rn(byte_to_biased_float(hi, 2 + cp.cc) - K, s);
            }
        }
    }
}

// Dequantize column j: x[i] = RN(code_ij * s[g][j]), each group at its width.
template <int DK, int DV, int GROUP>
__device__ __forceinline__ void decode_column(const uint8_t* cs, const float* ss,
                                              const ColumnPlace& cp, int j, const TileLayout& tl,
                                              float (&x)[DK]) {
#pragma unroll
    for (int g = 0; g < DK / GROUP; ++g) {
        float y[GROUP];
        const int gbase = static_cast<int>(tl.goff(g, GROUP * DV / 2));
        if (tl.bits(g) == 8)
            decode_group<DV, GROUP, 8>(cs, ss, cp, j, g, gbase, y);
        else
            decode_group<DV, GROUP, 4>(cs, ss, cp, j, g, gbase, y);
#pragma unroll
        for (int r = 0; r < GROUP; ++r) x[g * GROUP + r] = y[r];
    }
}

// Stored bytes (int8) or nibbles (int4) of one group of column j, already
// rounded (t[r]: float whose low bits are the stored value), written into the
// tile's codes in the state layout. Columns c0 = 2m and c1 = 2m + 1 of a pair
// are adjacent threads: each packs four (int8) or eight (int4) of its rows,
// the two trade them with one shuffle, and each writes one of the two words
// that cover those rows.
template <int DV, int GROUP, int BITS>
__device__ __forceinline__ void store_group(uint8_t* cs, const ColumnPlace& cp, int gbase,
                                            const float* t) {
    using PG = PairGeo<GROUP, BITS>;
    constexpr int RPP = BITS == 8 ? 4 : 8;         // rows per packed word
#pragma unroll
    for (int r = 0; r < GROUP; r += RPP) {
        uint32_t m;
        if constexpr (BITS == 8) {
            m = pack_low_bytes(t[r], t[r + 1], t[r + 2], t[r + 3]);
        } else {
            // bytes: rows (r | r+2<<4), (r+1 | r+3<<4), (r+4 | r+6<<4), (r+5 | r+7<<4)
            uint32_t n[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) n[e] = __float_as_uint(t[r + e]) & 0xFu;
            m = (n[0] | n[2] << 4) | (n[1] | n[3] << 4) << 8 | (n[4] | n[6] << 4) << 16 |
                (n[5] | n[7] << 4) << 24;
        }
        const uint32_t p = __shfl_xor_sync(0xffffffffu, m, 1);
        // c0 writes the word of the first half of the rows, c1 of the second;
        // byte order within a word: (row, c0), (row, c1), (row+1, c0), ...
        const uint32_t word = cp.cc == 0 ? __byte_perm(m, p, 0x5140u) : __byte_perm(m, p, 0x3726u);
        const int rr = r + cp.cc * (RPP / 2);      // first row (in the group) of the word written
        const int un = rr / PG::RPU, w = (rr % PG::RPU) / PG::RPW;
        *reinterpret_cast<uint32_t*>(cs + unit_byte<GROUP, BITS>(gbase, cp.pc, un, cp.owner) +
                                     w * 4) = word;
    }
}

// New scale of one group of column j, and its codes (as floats kTwo23 + bias
// + code, in x[g*GROUP ...], replacing the values) by the rounding MODE. For
// BDR the group's old values are decoded again from the old codes and scales.
template <int DK, int DV, int GROUP, int MODE, int BITS>
__device__ __forceinline__ float requantize_group(float (&x)[DK], int g, const uint8_t* cs,
                                                  const float* ss, const ColumnPlace& cp, int j,
                                                  int gbase, uint64_t hkey) {
    constexpr float QMAX = Q<BITS>::kMax, BIAS = Q<BITS>::kBias;
    constexpr int QM = static_cast<int>(QMAX);
    float deq0[GROUP];
    if constexpr (MODE == kBDR) decode_group<DV, GROUP, BITS>(cs, ss, cp, j, g, gbase, deq0);
    float A = 0.0f;
#pragma unroll
    for (int r = g * GROUP; r < (g + 1) * GROUP; r += 2) A = max_abs3(A, x[r], x[r + 1]);
    const float s = A < kTiny ? 0.0f : div_by_qmax<QM>(A);
    const float inv = A < kTiny ? 0.0f : div_rn_fast(QMAX, A);
    const float2 inv2 = f2(inv), s2 = f2(s), kb = f2(kTwo23 + BIAS);
#pragma unroll
    for (int r = g * GROUP; r < (g + 1) * GROUP; r += 2) {
        const int rl = r - g * GROUP;
        const float2 d0 = MODE == kBDR ? make_float2(deq0[rl], deq0[rl + 1]) : f2(0.0f);
        const float2 tv = round_rows<MODE, BITS, false>(make_float2(x[r], x[r + 1]), inv2, d0, s2, kb,
                                                 hkey, static_cast<uint32_t>(r),
                                                 static_cast<uint32_t>(j));
        x[r] = tv.x;
        x[r + 1] = tv.y;
    }
    return s;
}

// Token t of the tile into ring slot `slot` (thread 0 only).
template <int DK, int DV, int GROUP, int GATE>
__device__ __forceinline__ void issue_token(const ChunkParams& p, uint8_t* smem, int slot,
                                            int tile, int t) {
    using S = ChunkSmem<DK, DV, GROUP, GATE>;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem) + 1 + slot;
    uint8_t* dst = smem + S::kRing + slot * S::kTok;
    const int64_t row = static_cast<int64_t>(t) * p.ntiles + tile;
    const uint64_t pol = policy_evict_first();
    uint32_t bytes = 2 * DK * 4 + DV * 4;
    if (GATE == kGatePerKey) bytes += DK * 4;
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s(dst + S::kQ, p.q + row * DK, DK * 4, bar, pol);
    bulk_g2s(dst + S::kK, p.k + row * DK, DK * 4, bar, pol);
    if (GATE == kGatePerKey) bulk_g2s(dst + S::kG, p.gates + row * DK, DK * 4, bar, pol);
    bulk_g2s(dst + S::kV, p.v + row * DV, DV * 4, bar, pol);
}

// Four floats of shared memory, loaded anew at every use (the delta rule reads
// k twice per token; keeping the first load's values live would cost 128
// registers).
__device__ __forceinline__ float4 lds4(const float* p) {
    float4 r;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "r"(smem_u32(p)));
    return r;
}

template <int DK, int DV, int GROUP, int UPD, int GATE, int MODE>
__global__ void __launch_bounds__(DV, (3 * 128) / DV) chunk_kernel(const ChunkParams p) {
    using S = ChunkSmem<DK, DV, GROUP, GATE>;
    constexpr int G = DK / GROUP;
    constexpr int C = DV / 32;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bar_state = reinterpret_cast<uint64_t*>(smem);
    uint64_t* bar_tok = bar_state + 1;
    uint8_t* cs = smem + S::kCodes;
    float* ss = reinterpret_cast<float*>(smem + S::kScales);
    const int j = threadIdx.x;
    const ColumnPlace cp(j, C);

    if (j == 0) {
        mbar_init(bar_state, 1);
        for (int s = 0; s < kChunkSlots; ++s) mbar_init(&bar_tok[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    const int T = p.T;
    const int NS = T < kChunkSlots ? T : kChunkSlots;
    uint32_t par_state = 0;
    int64_t tok_base = 0;        // tokens this CTA has consumed before the tile
    bool ok = true;
    int64_t issued_hi = 0;       // tokens issued (thread 0's count), for draining
    int64_t drain_lo = 0;        // first token whose copy may still be in flight
    bool state_pending = false;  // the state copy may still be in flight

    for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x) {
        TileLayout tl;
        tl.load(p.prec_map, p.head_offsets, p.batch_stride, p.H, p.pgroups, G, GROUP * DV,
                tile / p.H, tile % p.H);
        if (!tl.ok) {
            if (j == 0) atomicOr(p.err, kErrLayout);
            continue;
        }
        const int64_t code_off = tl.code_off;
        const uint32_t cbytes = static_cast<uint32_t>(tl.goff(G, GROUP * DV / 2));
        if (j == 0 && !p.inject) {
            // the previous tile's shared-memory reads come before these copies
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

        float x[DK];
        decode_column<DK, DV, GROUP>(cs, ss, cp, j, tl, x);

        // Delta rule: u_t = k_t^T S_{t-1} in key order. u_0 is taken here from
        // the dequantized state; u_{t+1} is accumulated while token t updates
        // the column (its rows come out in key order), so no pass over the
        // state waits on a whole reduction before it can start.
        float unext = 0.0f;
        if (UPD == kDelta) {
            const int64_t u0 = tok_base;
            ok = mbar_wait_bounded(&bar_tok[u0 % NS], static_cast<uint32_t>((u0 / NS) & 1),
                                   p.timeout_ns);
            if (__syncthreads_or(!ok)) {
                ok = false;
                drain_lo = u0;
                break;
            }
            const float* k0 = reinterpret_cast<const float*>(
                smem + S::kRing + static_cast<int>(u0 % NS) * S::kTok + S::kK);
#pragma unroll
            for (int r = 0; r < DK; r += 4) {
                const float4 kv = lds4(k0 + r);
                unext = __fmaf_rn(kv.x, x[r], unext);
                unext = __fmaf_rn(kv.y, x[r + 1], unext);
                unext = __fmaf_rn(kv.z, x[r + 2], unext);
                unext = __fmaf_rn(kv.w, x[r + 3], unext);
            }
        }

#pragma unroll 1
        for (int t = 0; t < T; ++t) {
            const int64_t u = tok_base + t;
            const int slot = static_cast<int>(u % NS);
            const uint32_t par = static_cast<uint32_t>((u / NS) & 1);
            bool good = mbar_wait_bounded(&bar_tok[slot], par, p.timeout_ns);
            // the delta rule also reads the next token's k
            const int nslot = static_cast<int>((u + 1) % NS);
            if (UPD == kDelta && t + 1 < T)
                good = good && mbar_wait_bounded(&bar_tok[nslot],
                                                 static_cast<uint32_t>(((u + 1) / NS) & 1),
                                                 p.timeout_ns);
            // A thread whose wait ran out skips the token; the one CTA barrier
            // of the iteration (below) ends the loop for all.
            if (good) {
            const uint8_t* tk = smem + S::kRing + slot * S::kTok;
            const float* tq = reinterpret_cast<const float*>(tk + S::kQ);
            const float* tkk = reinterpret_cast<const float*>(tk + S::kK);
            const float* tg = reinterpret_cast<const float*>(tk + S::kG);
            const float* tv = reinterpret_cast<const float*>(tk + S::kV);
            // k of the next token (the delta rule; the last token reads its own, unused)
            const float* tkn = UPD == kDelta && t + 1 < T
                                   ? reinterpret_cast<const float*>(smem + S::kRing +
                                                                    nslot * S::kTok + S::kK)
                                   : tkk;
            const int64_t row = static_cast<int64_t>(t) * p.ntiles + tile;
            float gsc = 0.0f;
            if (GATE == kGate) gsc = __ldg(p.gates + row);
            float w = tv[j];
            if (UPD == kDelta) {
                // w = beta (v - alpha u): three separate roundings
                const float beta = __ldg(p.beta + row);
                w = __fmul_rn(beta, __fsub_rn(w, __fmul_rn(gsc, unext)));
            }
            // x = g * x + RN(k w); o = x^T q and (delta) the next u, in key order
            const float2 w2 = f2(w), gs2 = f2(gsc);
            float o = 0.0f, un = 0.0f;
#pragma unroll
            for (int r = 0; r < DK; r += 4) {
                if (r % 16 == 0) asm volatile("" ::: "memory");   // bound the load hoisting
                const float4 kv = lds4(tkk + r);
                const float4 qv = lds4(tq + r);
                float2 g0 = gs2, g1 = gs2;
                if (GATE == kGatePerKey) {
                    const float4 gv = lds4(tg + r);
                    g0 = make_float2(gv.x, gv.y);
                    g1 = make_float2(gv.z, gv.w);
                }
                const float2 x0 = fma2(g0, make_float2(x[r], x[r + 1]),
                                       mul2(make_float2(kv.x, kv.y), w2));
                const float2 x1 = fma2(g1, make_float2(x[r + 2], x[r + 3]),
                                       mul2(make_float2(kv.z, kv.w), w2));
                x[r] = x0.x; x[r + 1] = x0.y; x[r + 2] = x1.x; x[r + 3] = x1.y;
                o = __fmaf_rn(qv.x, x0.x, o);
                o = __fmaf_rn(qv.y, x0.y, o);
                o = __fmaf_rn(qv.z, x1.x, o);
                o = __fmaf_rn(qv.w, x1.y, o);
                if (UPD == kDelta) {
                    const float4 kn = lds4(tkn + r);
                    un = __fmaf_rn(kn.x, x0.x, un);
                    un = __fmaf_rn(kn.y, x0.y, un);
                    un = __fmaf_rn(kn.z, x1.x, un);
                    un = __fmaf_rn(kn.w, x1.y, un);
                }
            }
            unext = un;
            p.out[row * DV + j] = o;
            }
            // every thread is done with the slot; any wait that ran out
            if (__syncthreads_or(!good)) {
                ok = false;
                drain_lo = u;
                break;
            }
            if (j == 0 && t + NS < T) {
                fence_proxy_async_smem();
                issue_token<DK, DV, GROUP, GATE>(p, smem, slot, tile, t + NS);
                issued_hi = u + NS + 1;
            }
        }
        if (!ok) break;
        tok_base += T;

        // one requantization at the chunk's end
        float snew[G];
        const int b = tile / p.H, h = tile - b * p.H;
        const uint64_t hkey = MODE == kSR ? tile_hash_key(p.seed, p.step,
                                                          static_cast<uint32_t>(b),
                                                          static_cast<uint32_t>(h))
                                          : 0ull;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int gbase = static_cast<int>(tl.goff(g, GROUP * DV / 2));
            snew[g] = tl.bits(g) == 8
                          ? requantize_group<DK, DV, GROUP, MODE, 8>(x, g, cs, ss, cp, j, gbase, hkey)
                          : requantize_group<DK, DV, GROUP, MODE, 4>(x, g, cs, ss, cp, j, gbase, hkey);
        }
        __syncthreads();                     // old codes and scales no longer read
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
        // write the tile back: 16-byte streaming stores
        uint8_t* gc = p.codes + code_off;
        for (int off = j * 16; off < static_cast<int>(cbytes); off += DV * 16) {
            const uint4 vv = *reinterpret_cast<const uint4*>(cs + off);
            st_cs_u4(gc + off, vv.x, vv.y, vv.z, vv.w);
        }
        float* gs = p.scales + static_cast<int64_t>(tile) * G * DV;
        for (int off = j * 4; off < G * DV; off += DV * 4) {
            const float4 vv = *reinterpret_cast<const float4*>(ss + off);
            *reinterpret_cast<float4*>(gs + off) = vv;
        }
        __syncthreads();                     // before the next tile's copies land
    }
    if (!ok && j == 0) {
        // record the timeout, then wait (bounded) for copies still in flight
        atomicOr(p.err, kErrTimeout);
        if (state_pending) mbar_wait_bounded(bar_state, par_state, p.timeout_ns);
        for (int64_t u = drain_lo; u < issued_hi; ++u)
            mbar_wait_bounded(&bar_tok[u % NS], static_cast<uint32_t>((u / NS) & 1),
                              p.timeout_ns);
    }
}

// Defines `ChunkKernel NAME(int d_k, int d_v, int group, int update_kind,
// int gate_kind)`: the chunk kernel with rounding MODE for that shape, with its
// shared-memory bytes, or {nullptr, 0} when it is not compiled. The gated
// forms take chunk_gated_kernel (chunk_gated.cuh, which the compiling file
// includes) where a scale group fits in half the key rows.
#define LRS_CHUNK_PICK(NAME, MODE, DK, DV, GROUP)                                              \
    if (d_k == DK && d_v == DV && group == GROUP) {                                            \
        using S = ChunkSmem<DK, DV, GROUP, kGatePerKey>;                                       \
        using S1 = ChunkSmem<DK, DV, GROUP, kGate>;                                            \
        if (update_kind == kGated && gate_kind == kGatePerKey)                                 \
            return {chunk_gated_pick<DK, DV, GROUP, kGatePerKey, MODE>(), S::kBytes};          \
        if (update_kind == kGated && gate_kind == kGate)                                       \
            return {chunk_gated_pick<DK, DV, GROUP, kGate, MODE>(), S1::kBytes};               \
        if (update_kind == kDelta && gate_kind == kGate)                                       \
            return {reinterpret_cast<const void*>(                                             \
                        &chunk_kernel<DK, DV, GROUP, kDelta, kGate, MODE>),                    \
                    S1::kBytes};                                                               \
        return {nullptr, 0};                                                                   \
    }
#define LRS_CHUNK_VARIANTS(NAME, MODE)                                                         \
    ChunkKernel NAME(int d_k, int d_v, int group, int update_kind, int gate_kind) {            \
        LRS_CHUNK_PICK(NAME, MODE, 128, 128, 32)                                               \
        LRS_CHUNK_PICK(NAME, MODE, 128, 128, 16)                                               \
        LRS_CHUNK_PICK(NAME, MODE, 128, 128, 64)                                               \
        LRS_CHUNK_PICK(NAME, MODE, 128, 64, 32)                                                \
        LRS_CHUNK_PICK(NAME, MODE, 128, 64, 16)                                                \
        LRS_CHUNK_PICK(NAME, MODE, 128, 64, 64)                                                \
        LRS_CHUNK_PICK(NAME, MODE, 64, 128, 32)                                                \
        LRS_CHUNK_PICK(NAME, MODE, 64, 128, 16)                                                \
        LRS_CHUNK_PICK(NAME, MODE, 64, 128, 64)                                                \
        LRS_CHUNK_PICK(NAME, MODE, 64, 64, 32)                                                 \
        LRS_CHUNK_PICK(NAME, MODE, 64, 64, 16)                                                 \
        LRS_CHUNK_PICK(NAME, MODE, 64, 64, 64)                                                 \
        return {nullptr, 0};                                                                   \
    }

}  // namespace lrs
