// step_kernel.cuh -- the fused quantized decode step (sm_100a).
//
// One warp owns one (batch, head) tile at a time; lane t owns value columns
// [t*C, t*C + C) (C = d_v / 32) over every key row, so every reduction the
// step needs over the key axis -- u = k^T deq (delta rule), o = x^T q and the
// per-(group, column) absmax -- runs inside one thread, in key order, with no
// shuffles. The tile streams through shared memory one scale group at a time:
// each group has its own slot and mbarrier; its codes, scales and the group's
// q, k (and per-key gate) rows arrive by 1-D bulk copies issued by lane 0, and
// as soon as a group is consumed its slot is refilled with the same group of
// the warp's next tile. New codes and scales are written straight back with
// 128-bit streaming stores, in place.
//
// Sources: "Quantizing Recurrent Language Models Is Easier Than You Think"
// (abstract: value-axis scale grouping, mixed precision by decay, stochastic
// rounding); "Preserving Updates in Low-Bit Recurrent State Quantization"
// (abstract: requantize after every update; Bounded Directional Rounding).
#pragma once

#include "lrs_device.cuh"

namespace lrs {

constexpr int kGate = 0, kGatePerKey = 1;        // matches lrs_gate_kind
constexpr int kGated = 0, kDelta = 1;            // matches lrs_update_kind
constexpr int kRTN = 0, kSR = 1, kBDR = 2;       // matches lrs_round_mode
constexpr int kMaxGroups = 16;
constexpr float kTiny = 0x1p-100f;               // absmax below this: stored as zero

struct StepParams {
    uint8_t* codes;
    float* scales;
    const uint8_t* prec_map;
    const int64_t* head_offsets;
    int64_t batch_stride;
    const float* q;
    const float* k;
    const float* v;
    const float* gates;
    const float* beta;
    float* out;
    uint64_t seed;
    uint64_t step;
    unsigned* err;
    uint64_t timeout_ns;
    int32_t H, d_k, G, ntiles;
    int32_t warp_smem;   // bytes of shared memory per warp
    int32_t inject;      // fault injection: issue no copies
};

// Shared-memory layout of one warp:
//   [0, 128)            mbarriers, one per group slot
//   [128, 128 + 4*d_v)  v of the current tile (arrives with slot 0)
//   then G slots of SlotBytes each:
//     codes (GROUP*d_v bytes: room for int8) | scales (d_v fp32) |
//     q, k, [gate] (GROUP fp32 each)
template <int C, int GROUP, int GATE>
struct Slot {
    static constexpr int DV = 32 * C;
    static constexpr int kCodes = GROUP * DV;                     // int8 capacity
    static constexpr int kScales = kCodes;
    static constexpr int kQ = kScales + DV * 4;
    static constexpr int kK = kQ + GROUP * 4;
    static constexpr int kG = kK + GROUP * 4;
    static constexpr int kBytes = kG + (GATE == kGatePerKey ? GROUP * 4 : 0);
    static constexpr int kHeader = 128 + DV * 4;
    static_assert(kBytes % 16 == 0, "slot alignment");
    static int warp_bytes(int G) { return (kHeader + G * kBytes + 127) / 128 * 128; }
};

template <int BITS>
__device__ __forceinline__ void decode_word(uint32_t w, float (&f)[32 / BITS]) {
    if constexpr (BITS == 8) {
#pragma unroll
        for (int n = 0; n < 4; ++n)
            f[n] = __fsub_rn(byte_to_biased_float(w, n), kTwo23 + 128.0f);
    } else {
        const uint32_t lo = w & 0x0F0F0F0Fu;
        const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            f[n] = __fsub_rn(byte_to_biased_float(lo, n), kTwo23 + 8.0f);
            f[n + 4] = __fsub_rn(byte_to_biased_float(hi, n), kTwo23 + 8.0f);
        }
    }
}

template <int BITS>
__device__ __forceinline__ uint32_t encode_word(const float (&t)[32 / BITS]) {
    if constexpr (BITS == 8) {
        return pack_low_bytes(t[0], t[1], t[2], t[3]);
    } else {
        const uint32_t lo = pack_low_bytes(t[0], t[1], t[2], t[3]);
        const uint32_t hi = pack_low_bytes(t[4], t[5], t[6], t[7]);
        return lo | (hi << 4);
    }
}

// Rounded code of y, returned as the float 1.5*2^23 + bias + code whose low
// byte is the stored offset-binary byte.
template <int MODE, int BITS>
__device__ __forceinline__ float round_code(float y, float x, float deq, float s_new,
                                            uint64_t hkey, uint32_t i, uint32_t j) {
    constexpr float QMAX = BITS == 8 ? 127.0f : 7.0f;
    constexpr float BIAS = BITS == 8 ? 128.0f : 8.0f;
    if constexpr (MODE == kRTN) {
        // |y| <= qmax (1 + 2^-24) because inv = RN(qmax/A) and |x| <= A, so
        // the nearest integer never leaves [-qmax, qmax]: no clamp needed.
        return __fadd_rn(y, kRound + BIAS);
    } else {
        const float rn = __fsub_rn(__fadd_rn(y, kRound), kRound);  // rint(y), exact
        float c;
        if constexpr (MODE == kSR) {
            const float f = rn > y ? __fsub_rn(rn, 1.0f) : rn;    // floor(y)
            const float fr = __fsub_rn(y, f);
            const float u = element_uniform(hkey, i, j);
            c = u < fr ? __fadd_rn(f, 1.0f) : f;
        } else {
            const float delta = __fsub_rn(x, deq);
            const float m = __fsub_rn(__fmul_rn(rn, s_new), deq);
            c = rn;
            if (delta > 0.0f && m < 0.0f)
                c = rn < y ? __fadd_rn(rn, 1.0f) : rn;            // ceil(y)
            else if (delta < 0.0f && m > 0.0f)
                c = rn > y ? __fsub_rn(rn, 1.0f) : rn;            // floor(y)
        }
        c = fminf(fmaxf(c, -QMAX), QMAX);
        return __fadd_rn(c, kRound + BIAS);
    }
}

__device__ __forceinline__ void st_cs_u4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

template <int C>
__device__ __forceinline__ void st_cs_f(float* p, const float (&s)[C]) {
    if constexpr (C == 4) {
        asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(s[0]), "f"(s[1]),
                     "f"(s[2]), "f"(s[3])
                     : "memory");
    } else {
        asm volatile("st.global.cs.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(s[0]), "f"(s[1])
                     : "memory");
    }
}

template <int C>
__device__ __forceinline__ void ld_smem_f(const float* p, float (&s)[C]) {
    if constexpr (C == 4) {
        const float4 t = *reinterpret_cast<const float4*>(p);
        s[0] = t.x; s[1] = t.y; s[2] = t.z; s[3] = t.w;
    } else {
        const float2 t = *reinterpret_cast<const float2*>(p);
        s[0] = t.x; s[1] = t.y;
    }
}

// Delta rule, first pass over the tile: u_j += k_i * deq_ij for the rows of
// one group, in key order.
template <int C, int GROUP, int BITS>
__device__ __forceinline__ void group_ktS(const uint8_t* __restrict__ cs,
                                          const float* __restrict__ ss,
                                          const float* __restrict__ ks, int lane, float (&u)[C]) {
    constexpr int EPW = 32 / BITS;
    constexpr int UNITS = GROUP * C * BITS / 8 / 16;
    float sc[C];
    ld_smem_f<C>(ss + lane * C, sc);
#pragma unroll
    for (int un = 0; un < UNITS; ++un) {
        const uint4 raw = *reinterpret_cast<const uint4*>(cs + (un * 32 + lane) * 16);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[EPW];
            decode_word<BITS>(wd[wi], f);
#pragma unroll
            for (int e = 0; e < EPW; ++e) {
                const int el = (un * 4 + wi) * EPW + e;
                const int r = el / C, c = el % C;
                const float deq = __fmul_rn(f[e], sc[c]);
                u[c] = __fmaf_rn(ks[r], deq, u[c]);
            }
        }
    }
}

// One scale group of one tile: dequantize, update, accumulate the output,
// new scales, requantize and store.
template <int C, int GROUP, int GATE, int MODE, int BITS>
__device__ __forceinline__ void group_step(const uint8_t* __restrict__ cs,
                                           const float* __restrict__ ss,
                                           const float* __restrict__ qs,
                                           const float* __restrict__ ks,
                                           const float* __restrict__ gs, float gscalar,
                                           const float (&w)[C], float (&o)[C],
                                           uint8_t* __restrict__ gcodes,
                                           float* __restrict__ gscales, uint64_t hkey, int row0,
                                           int lane) {
    constexpr int EPW = 32 / BITS;
    constexpr int UNITS = GROUP * C * BITS / 8 / 16;
    constexpr float QMAX = BITS == 8 ? 127.0f : 7.0f;

    float sc[C];
    ld_smem_f<C>(ss + lane * C, sc);
    float x[GROUP][C];
    float amax[C];
#pragma unroll
    for (int c = 0; c < C; ++c) amax[c] = 0.0f;

#pragma unroll
    for (int un = 0; un < UNITS; ++un) {
        const uint4 raw = *reinterpret_cast<const uint4*>(cs + (un * 32 + lane) * 16);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[EPW];
            decode_word<BITS>(wd[wi], f);
#pragma unroll
            for (int e = 0; e < EPW; ++e) {
                const int el = (un * 4 + wi) * EPW + e;
                const int r = el / C, c = el % C;
                const float deq = __fmul_rn(f[e], sc[c]);
                const float gi = GATE == kGatePerKey ? gs[r] : gscalar;
                const float kw = __fmul_rn(ks[r], w[c]);
                const float xv = __fmaf_rn(gi, deq, kw);
                o[c] = __fmaf_rn(qs[r], xv, o[c]);
                amax[c] = fmaxf(amax[c], fabsf(xv));
                x[r][c] = xv;
            }
        }
    }

    float snew[C], inv[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const float A = amax[c];
        const bool zero = A < kTiny;
        snew[c] = zero ? 0.0f : __fdiv_rn(A, QMAX);
        inv[c] = zero ? 0.0f : __fdiv_rn(QMAX, A);
    }
    st_cs_f<C>(gscales + lane * C, snew);

#pragma unroll
    for (int un = 0; un < UNITS; ++un) {
        uint32_t ow[4];
        uint32_t wd[4] = {0u, 0u, 0u, 0u};
        if constexpr (MODE == kBDR) {
            const uint4 raw = *reinterpret_cast<const uint4*>(cs + (un * 32 + lane) * 16);
            wd[0] = raw.x; wd[1] = raw.y; wd[2] = raw.z; wd[3] = raw.w;
        }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[EPW];
            if constexpr (MODE == kBDR) decode_word<BITS>(wd[wi], f);
            float t[EPW];
#pragma unroll
            for (int e = 0; e < EPW; ++e) {
                const int el = (un * 4 + wi) * EPW + e;
                const int r = el / C, c = el % C;
                const float y = __fmul_rn(x[r][c], inv[c]);
                float deq = 0.0f;
                if constexpr (MODE == kBDR) deq = __fmul_rn(f[e], sc[c]);
                t[e] = round_code<MODE, BITS>(y, x[r][c], deq, snew[c], hkey,
                                              static_cast<uint32_t>(row0 + r),
                                              static_cast<uint32_t>(lane * C + c));
            }
            ow[wi] = encode_word<BITS>(t);
        }
        st_cs_u4(gcodes + (un * 32 + lane) * 16, ow[0], ow[1], ow[2], ow[3]);
    }
}

// Layout of tile `tile`: byte offset of its codes and its precision, or
// prec = 0 when prec_map does not fit the offsets.
struct TileInfo {
    int64_t code_off;
    int prec;
};

__device__ __forceinline__ TileInfo tile_info(const StepParams& p, int tile, int dv) {
    const int h = tile % p.H;
    const int b = tile / p.H;
    const int prec = __ldg(p.prec_map + h);
    const int64_t off = __ldg(p.head_offsets + h);
    const int64_t end = (h + 1 < p.H) ? __ldg(p.head_offsets + h + 1) : p.batch_stride;
    const int64_t bytes = static_cast<int64_t>(p.d_k) * dv * prec / 8;
    TileInfo ti;
    ti.prec = ((prec == 4 || prec == 8) && off >= 0 && off + bytes <= end) ? prec : 0;
    ti.code_off = static_cast<int64_t>(b) * p.batch_stride + off;
    return ti;
}

template <int C, int GROUP, int GATE>
__device__ __forceinline__ void issue_slot(const StepParams& p, uint8_t* wsm, int tile, int g,
                                           const TileInfo& ti, uint64_t pol_state,
                                           uint64_t pol_in) {
    using S = Slot<C, GROUP, GATE>;
    constexpr int DV = 32 * C;
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsm);
    uint8_t* slot = wsm + S::kHeader + g * S::kBytes;
    const uint32_t cbytes = GROUP * DV * ti.prec / 8;
    uint32_t total = cbytes + DV * 4 + 2 * GROUP * 4;
    if (GATE == kGatePerKey) total += GROUP * 4;
    if (g == 0) total += DV * 4;
    mbar_arrive_expect_tx(&bars[g], total);
    bulk_g2s(slot, p.codes + ti.code_off + static_cast<int64_t>(g) * cbytes, cbytes, &bars[g],
             pol_state);
    bulk_g2s(slot + S::kScales, p.scales + (static_cast<int64_t>(tile) * p.G + g) * DV, DV * 4,
             &bars[g], pol_state);
    const int64_t rowbase = static_cast<int64_t>(tile) * p.d_k + g * GROUP;
    bulk_g2s(slot + S::kQ, p.q + rowbase, GROUP * 4, &bars[g], pol_in);
    bulk_g2s(slot + S::kK, p.k + rowbase, GROUP * 4, &bars[g], pol_in);
    if (GATE == kGatePerKey) bulk_g2s(slot + S::kG, p.gates + rowbase, GROUP * 4, &bars[g], pol_in);
    if (g == 0)
        bulk_g2s(wsm + 128, p.v + static_cast<int64_t>(tile) * DV, DV * 4, &bars[g], pol_in);
}

template <int C, int GROUP, int UPD, int GATE, int MODE>
__global__ void __launch_bounds__(256, 1) step_kernel(const StepParams p) {
    using S = Slot<C, GROUP, GATE>;
    constexpr int DV = 32 * C;
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    const int W = gridDim.x * nw;
    int tile = blockIdx.x * nw + wib;
    uint8_t* wsm = smem + wib * p.warp_smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsm);
    const float* v_s = reinterpret_cast<const float*>(wsm + 128);
    const int G = p.G;

    if (lane == 0) {
        for (int g = 0; g < G; ++g) mbar_init(&bars[g], 1);
        fence_mbar_init();
    }
    __syncwarp();

    const uint64_t pol_state = policy_evict_first();
    const uint64_t pol_in = policy_evict_first();
    // Every slot of a tile is issued once per tile, so all slots advance their
    // mbarrier phase together: the k-th tile issued by this warp completes
    // phase parity k & 1 in each slot.
    uint32_t issued = 0;    // tiles issued so far by this warp
    uint32_t cur_par = 0;   // phase parity of the current tile's copies
    uint32_t inflight = 0;  // slots with copies issued and not yet waited for
    uint32_t pend_par = 0;  // per slot: parity of the phase it is waiting for

    auto issue_tile_slot = [&](int t, int g, const TileInfo& tinfo, uint32_t par) {
        if (lane == 0) issue_slot<C, GROUP, GATE>(p, wsm, t, g, tinfo, pol_state, pol_in);
        inflight |= 1u << g;
        pend_par = (pend_par & ~(1u << g)) | (par << g);
    };

    if (tile < p.ntiles) {
        const TileInfo ti = tile_info(p, tile, DV);
        if (ti.prec != 0 && !p.inject) {
            cur_par = issued & 1u;
            for (int g = 0; g < G; ++g) issue_tile_slot(tile, g, ti, cur_par);
            ++issued;
        }
    }

    float nscal = 0.0f, nbeta = 0.0f;
    if (tile < p.ntiles) {
        if (GATE == kGate) nscal = __ldg(p.gates + tile);
        if (UPD == kDelta) nbeta = __ldg(p.beta + tile);
    }

    for (; tile < p.ntiles; tile += W) {
        const int next = tile + W;
        const TileInfo ti = tile_info(p, tile, DV);
        const TileInfo tn = next < p.ntiles ? tile_info(p, next, DV) : TileInfo{0, 0};
        const bool issue_next = tn.prec != 0 && !p.inject;
        const uint32_t nxt_par = issued & 1u;
        const float gscalar = nscal, beta = nbeta;
        if (next < p.ntiles) {
            if (GATE == kGate) nscal = __ldg(p.gates + next);
            if (UPD == kDelta) nbeta = __ldg(p.beta + next);
        }
        if (ti.prec == 0) {
            // No copies were issued for this tile: record the mismatch, skip
            // it, and start the next tile's copies in the free slots.
            if (lane == 0) atomicOr(p.err, kErrLayout);
            if (issue_next) {
                for (int g = 0; g < G; ++g) issue_tile_slot(next, g, tn, nxt_par);
                ++issued;
                cur_par = nxt_par;
            }
            continue;
        }
        const uint64_t hkey = MODE == kSR ? tile_hash_key(p.seed, p.step,
                                                          static_cast<uint32_t>(tile / p.H),
                                                          static_cast<uint32_t>(tile % p.H))
                                          : 0ull;
        bool ok = true;
        float w[C], o[C];
#pragma unroll
        for (int c = 0; c < C; ++c) o[c] = 0.0f;

        // ---- wait for the slots needed before the first group
        const int first_wait = UPD == kDelta ? G : 1;
        for (int g = 0; g < first_wait && ok; ++g) {
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[g], cur_par, p.timeout_ns));
            if (ok) inflight &= ~(1u << g);
        }
        if (ok) {
            if (UPD == kDelta) {
                float u[C];
#pragma unroll
                for (int c = 0; c < C; ++c) u[c] = 0.0f;
                for (int g = 0; g < G; ++g) {
                    const uint8_t* slot = wsm + S::kHeader + g * S::kBytes;
                    const float* ss = reinterpret_cast<const float*>(slot + S::kScales);
                    const float* ks = reinterpret_cast<const float*>(slot + S::kK);
                    if (ti.prec == 8)
                        group_ktS<C, GROUP, 8>(slot, ss, ks, lane, u);
                    else
                        group_ktS<C, GROUP, 4>(slot, ss, ks, lane, u);
                }
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    const float t = __fmul_rn(gscalar, u[c]);
                    const float d = __fsub_rn(v_s[lane * C + c], t);
                    w[c] = __fmul_rn(beta, d);
                }
            } else {
#pragma unroll
                for (int c = 0; c < C; ++c) w[c] = v_s[lane * C + c];
            }

            uint8_t* gcodes_tile = p.codes + ti.code_off;
            const uint32_t cbytes = GROUP * DV * ti.prec / 8;
            for (int g = 0; g < G; ++g) {
                if (UPD != kDelta && g > 0) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait_bounded(&bars[g], cur_par, p.timeout_ns));
                    if (!ok) break;
                    inflight &= ~(1u << g);
                }
                const uint8_t* slot = wsm + S::kHeader + g * S::kBytes;
                const float* ss = reinterpret_cast<const float*>(slot + S::kScales);
                const float* qs = reinterpret_cast<const float*>(slot + S::kQ);
                const float* ks = reinterpret_cast<const float*>(slot + S::kK);
                const float* gs = reinterpret_cast<const float*>(slot + S::kG);
                float* gscales = p.scales + (static_cast<int64_t>(tile) * G + g) * DV;
                uint8_t* gcodes = gcodes_tile + static_cast<int64_t>(g) * cbytes;
                if (ti.prec == 8)
                    group_step<C, GROUP, GATE, MODE, 8>(slot, ss, qs, ks, gs, gscalar, w, o,
                                                        gcodes, gscales, hkey, g * GROUP, lane);
                else
                    group_step<C, GROUP, GATE, MODE, 4>(slot, ss, qs, ks, gs, gscalar, w, o,
                                                        gcodes, gscales, hkey, g * GROUP, lane);
                __syncwarp();
                if (issue_next) {
                    if (lane == 0) fence_proxy_async_smem();
                    issue_tile_slot(next, g, tn, nxt_par);
                }
            }
        }
        if (!ok) {
            // Record the timeout, then wait (bounded) for this warp's copies
            // still in flight before leaving, so none lands after exit.
            if (lane == 0) atomicOr(p.err, kErrTimeout);
            for (int g = 0; g < G; ++g)
                if (inflight & (1u << g))
                    mbar_wait_bounded(&bars[g], (pend_par >> g) & 1u, p.timeout_ns);
            return;
        }
        if (issue_next) {
            ++issued;
            cur_par = nxt_par;
        }
        float* op = p.out + static_cast<int64_t>(tile) * DV + lane * C;
        if constexpr (C == 4) {
            *reinterpret_cast<float4*>(op) = make_float4(o[0], o[1], o[2], o[3]);
        } else {
            *reinterpret_cast<float2*>(op) = make_float2(o[0], o[1]);
        }
    }
}

}  // namespace lrs
