// step_kernel.cuh -- the fused quantized decode step (sm_100a).
//
// One warp owns one (batch, head) tile at a time; lane t owns value columns
// [t*C, t*C + C) (C = d_v / 32) over every key row, so every reduction the
// step needs over the key axis -- u = k^T deq (delta rule), o = x^T q and the
// per-(group, column) absmax -- runs inside one thread, in key order, with no
// shuffles. A lane works through its columns one adjacent pair at a time, so
// only one pair's updated values of one scale group are live in registers.
//
// The tile streams through shared memory one scale group at a time, through a
// ring of slots per warp, each with its own mbarrier: lane 0 fills a slot with
// 1-D bulk copies (the group's codes and scales, its q, k and per-key gate
// rows, and v with the tile's first group) and refills it with the warp's
// next item as soon as it is consumed. New codes and scales go back in place
// with 128-bit streaming stores.
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
constexpr int kIoF32 = 0, kIoBF16 = 1;           // element type of q, k, v and out
constexpr int kMaxSlots = 16;
// Variants that stage the group's updated values in shared memory for the
// rounding pass: SR, and BDR of the delta rule. Gated BDR recomputes them
// from the codes still in the slot instead (two two-wide operations per row
// pair), which saves the 8 KB buffer so that 12 warps fit beside the ring:
// measured 9% faster than staging at 8 warps. For SR the same change measured
// within 2% either way (its longer rounding keeps the issue slots busier), so
// SR keeps the buffer and its fewer instructions.
__host__ __device__ constexpr bool stage_x(int mode, int upd) {
    return mode == kSR || (mode == kBDR && upd == kDelta);
}
// SR of the gated forms runs a ring of one slot per warp, released early: its
// rounding loop reads only the staged values, so the slot is free for the
// next group's copy once the last column pair's first loop has read it. The
// one-slot ring leaves shared memory for 12 warps beside the staging buffer.
__host__ __device__ constexpr bool sr_early_release(int mode, int upd) {
    return mode == kSR && upd == kGated;
}
// Launch bound of a step variant in warps: 12 (at most 168 registers a thread)
// where the live state fits, 8 (255 registers) for the wider groups and for
// the other staging variants, whose buffer leaves shared memory for 8 warps
// beside a ring of several slots.
__host__ __device__ constexpr int step_max_warps(int group, int mode, int upd) {
    return ((stage_x(mode, upd) && !sr_early_release(mode, upd)) || group > 32) ? 8 : 12;
}
constexpr float kTiny = 0x1p-100f;               // absmax below this: stored as zero

struct StepParams {
    uint8_t* codes;
    float* scales;
    const uint8_t* prec_map;
    const int64_t* head_offsets;
    int64_t batch_stride;
    const void* q;       // fp32 or bfloat16 (the variant's IO)
    const void* k;
    const void* v;
    const float* gates;
    const float* beta;
    void* out;           // fp32 or bfloat16
    uint64_t seed;
    uint64_t step;
    unsigned* err;
    uint64_t timeout_ns;
    int32_t H, d_k, G, ntiles;
    int32_t pgroups;     // widths in prec_map per head: 1, or one per scale group: G
    int32_t slots;       // ring slots per warp, 1..min(G, 16); the delta rule needs G
    int32_t warp_smem;   // bytes of shared memory per warp
    int32_t inject;      // error-path tests: 0, or n + 1 to issue copies for n items per warp
    int64_t code_bytes;  // bytes of the code buffer and floats of the scale buffer
    int64_t scale_count; // (read by the bounds-checked build only)
};

// Shared-memory layout of one warp (ES = bytes of a q, k, v element).
// Gated forms (INS = false):
//   [0, 128)          mbarriers, one per slot
//   two tile-input buffers of tile_in_bytes(d_k) each, used by the warp's
//   tiles in turn (tile n in buffer n & 1):
//     q, k (d_k elements each) | [gate] (d_k fp32) | v (d_v elements)
//   then `slots` slots of kBytes each, one scale group per item:
//     codes (GROUP*d_v bytes: room for int8) | scales (d_v fp32)
// A tile's inputs come with its first group, in one bulk copy per array.
// Delta rule (INS = true; its ring holds a whole tile, and the shared memory
// of 8 warps leaves no room for two more tiles' inputs):
//   [0, 128) mbarriers | v (d_v elements, one buffer: read before the tile's
//   groups are, refilled with the next tile's first group) | slots of kBytes:
//     codes | scales (d_v fp32) | q, k (GROUP elements each)
// In both, the variants that stage x add the staging buffer after the slots
// (and the widened inputs), and SR adds its row table after that.
template <int C, int GROUP, int GATE, int IO = kIoF32, bool INS = false>
struct Slot {
    static constexpr int DV = 32 * C;
    static constexpr int ES = IO == kIoBF16 ? 2 : 4;
    static constexpr int kCodes = GROUP * DV;                     // int8 capacity
    static constexpr int kScales = kCodes;
    static constexpr int kQ = kScales + DV * 4;                   // INS only
    static constexpr int kK = kQ + GROUP * ES;                    // INS only
    static constexpr int kBytes = INS ? kK + GROUP * ES : kQ;
    static_assert(kBytes % 16 == 0, "slot alignment");
    static constexpr int kXsBytes = GROUP * 256;   // x staging: 16 B per row pair and lane
    static constexpr int kTabBytes = GROUP * 8;    // SR: the group's row table of the hash
    // offsets inside a tile-input buffer (!INS)
    __host__ __device__ static int in_k(int d_k) { return d_k * ES; }
    __host__ __device__ static int in_g(int d_k) { return 2 * d_k * ES; }
    __host__ __device__ static int in_v(int d_k) {
        return 2 * d_k * ES + (GATE == kGatePerKey ? d_k * 4 : 0);
    }
    __host__ __device__ static int tile_in_payload(int d_k) { return in_v(d_k) + DV * ES; }
    __host__ __device__ static int tile_in_bytes(int d_k) {
        return (tile_in_payload(d_k) + 15) / 16 * 16;
    }
    __host__ __device__ static int header(int d_k) {
        return INS ? 128 + DV * ES : 128 + 2 * tile_in_bytes(d_k);
    }
    // bfloat16 tile inputs (gated forms) are widened to fp32 once per tile
    // into a buffer after the slots: q, k (d_k each), v (d_v)
    static constexpr bool CVT = IO == kIoBF16 && !INS;
    __host__ __device__ static int cvt_bytes(int d_k) { return CVT ? (2 * d_k + DV) * 4 : 0; }
    // [header | slots | widened inputs (CVT) | x staging (xs) | row table (tab)]
    static int warp_bytes(int slots, bool xs, bool tab, int d_k) {
        return (header(d_k) + slots * kBytes + cvt_bytes(d_k) + (xs ? kXsBytes : 0) +
                (tab ? kTabBytes : 0) + 127) / 128 * 128;
    }
};


// ------------------------------------------------------- packed fp32 math ---
// Two consecutive key rows of one column go through the sm_100 two-wide fp32
// instructions;
// each half is an IEEE binary32 operation rounded to nearest even. They are
// written with an explicit .rn so that no multiply and add is ever fused into
// one rounding behind our back (results must follow the stated roundings).

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

// a + b rounded toward plus infinity, two-wide.
__device__ __forceinline__ float2 add2_rp(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rp.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

// 1.0f when a < b (a > b), else 0.0f: one comparison that writes a float.
__device__ __forceinline__ float set_lt(float a, float b) {
    float r;
    asm("set.lt.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float set_gt(float a, float b) {
    float r;
    asm("set.gt.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// fma with rounding toward minus infinity, two-wide.
__device__ __forceinline__ float2 fma2_rm(float2 a, float2 b, float2 c) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rm.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

// Three-input minimum and maximum.
__device__ __forceinline__ float min3(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// max(a, |b|, |c|): one three-input maximum.
__device__ __forceinline__ float max_abs3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}

// The stored bytes of one 32-bit word as floats 2^23 + byte (offset binary),
// in element order (int4: byte n holds elements n and n+4).
template <int BITS>
__device__ __forceinline__ void decode_word_biased(uint32_t w, float (&f)[32 / BITS]) {
    if constexpr (BITS == 8) {
#pragma unroll
        for (int n = 0; n < 4; ++n) f[n] = byte_to_biased_float(w, n);
    } else {
        const uint32_t lo = w & 0x0F0F0F0Fu;
        const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            f[n] = byte_to_biased_float(lo, n);
            f[n + 4] = byte_to_biased_float(hi, n);
        }
    }
}

// Rounded codes leave the rounding as floats 2^23 + B + code, whose bit
// patterns are 0x4B000000 + B + code with the stored byte (nibble) in their
// low byte: B is the offset-binary bias (128 for int8, 8 for int4), so the
// low byte is code + B in [1, 255] (int4: [1, 15], its high nibble 0). B is
// even, so rounding 2^23 + B + y to nearest-even breaks a tie of y the same
// way as rint. word_bias<BITS>(n) is 2^23 + B for element n of a word.
template <int BITS>
__host__ __device__ constexpr float word_bias(int) {
    return kTwo23 + (BITS == 8 ? 128.0f : 8.0f);
}

// Pack the stored bytes (nibbles) of 4 (8) rounded codes into one word with
// byte permutes on the integer pipe (the multiply-add pipe is the busier one
// in the step): int8 takes the low byte of each pattern; int4 gathers the
// low bytes of elements 0-3 and 4-7 and adds the second word shifted by 4
// (byte n = element n | element n+4 << 4).
template <int BITS>
__device__ __forceinline__ uint32_t encode_word(const float (&t)[32 / BITS]) {
    if constexpr (BITS == 8) {
        return pack_low_bytes(t[0], t[1], t[2], t[3]);
    } else {
        const uint32_t lo = pack_low_bytes(t[0], t[1], t[2], t[3]);
        const uint32_t hi = pack_low_bytes(t[4], t[5], t[6], t[7]);
        return lo + (hi << 4);
    }
}

template <int BITS> struct Q;
template <> struct Q<8> { static constexpr float kMax = 127.0f, kBias = 128.0f; };
template <> struct Q<4> { static constexpr float kMax = 7.0f, kBias = 8.0f; };

// New scales and their inverses for two columns of one group, from their
// absmax A: s' = RN(A/qmax), inv = RN(qmax/A), both 0 where A is below kTiny.
// The same remainder-corrected divisions as div_by_qmax and div_rn_fast
// (lrs_device.cuh), each step done for both columns in one two-wide
// instruction; above 2^100 the inverse falls back to IEEE division.
template <int BITS>
__device__ __forceinline__ void new_scales(float A0, float A1, float2& snew, float2& inv) {
    constexpr float QMAX = Q<BITS>::kMax;
    constexpr float Y = 1.0f / QMAX;                 // RN(1/qmax)
    const float2 A = make_float2(A0, A1);
    const float2 nA = neg2(A);
    // s' = A/qmax with the constant reciprocal
    const float2 q0 = mul2(A, f2(Y));
    const float2 s = fma2(fma2(q0, f2(-QMAX), A), f2(Y), q0);
    // inv = qmax/A with the refined hardware reciprocal
    float2 y0;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y0.x) : "f"(A0));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y0.y) : "f"(A1));
    const float2 y = fma2(fma2(nA, y0, f2(1.0f)), y0, y0);
    const float2 p0 = mul2(f2(QMAX), y);
    float2 iv = fma2(fma2(p0, nA, f2(QMAX)), y, p0);
    if (A0 > 0x1p100f) iv.x = __fdiv_rn(QMAX, A0);
    if (A1 > 0x1p100f) iv.y = __fdiv_rn(QMAX, A1);
    snew = make_float2(A0 < kTiny ? 0.0f : s.x, A1 < kTiny ? 0.0f : s.y);
    inv = make_float2(A0 < kTiny ? 0.0f : iv.x, A1 < kTiny ? 0.0f : iv.y);
}

// Stochastic rounding of two elements (key rows i, i+1 of one column), from
// their draws' `top` words (see hash_top). Returned as the floats kb + code
// (kb: word_bias of the elements' word positions).
//
// The floor comes straight out as kb + floor(y) from one fused multiply-add
// rounded toward minus infinity (y = x*inv exact inside it; kb is an integer
// in [2^23, 2^24), where the float spacing is 1). The floor is clamped to
// [-qmax, qmax - 1] first: the clamped cases then decide themselves -- below
// -qmax the fraction y - f is negative and never draws the step up, at or
// above qmax it is at least 1 and always does -- so no clamp is needed after
// the step, and everywhere else this is the plain floor. The fraction
// fr = RN(y - f) is rounded once, as defined. The draw u = (top >> 9) 2^-23 is
// on the 2^-23 grid, so u < fr exactly when 1 + u < RU(1 + fr): both sides
// are floats in the same binade or RU(1 + fr) has left it (fr >= 1 - 2^-24:
// always up; fr < 0: never). The comparison writes 1.0f or 0.0f, added to the
// floor.
template <int BITS>
__device__ __forceinline__ float2 sr_round(float2 x, float2 inv, float2 kb, uint32_t top0,
                                           uint32_t top1) {
    constexpr float QMAX = Q<BITS>::kMax;
    float2 tb = fma2_rm(x, inv, kb);
    tb.x = fminf(fmaxf(tb.x, kb.x - QMAX), kb.x + (QMAX - 1.0f));
    tb.y = fminf(fmaxf(tb.y, kb.y - QMAX), kb.y + (QMAX - 1.0f));
    const float2 fr = fma2(x, inv, sub2(kb, tb));       // y - f, one rounding (kb - tb = -f exactly)
    const float2 g = add2_rp(fr, f2(1.0f));
    return add2(tb, make_float2(set_lt(sr_unit1(top0), g.x), set_lt(sr_unit1(top1), g.y)));
}

// Bounded Directional Rounding of two elements (key rows i, i+1 of one
// column). deq: their values before the update; s_new: the new scale.
//
// n = rint(y) comes out biased (kb + n) from one multiply-add; -n = kb - nb
// exactly. The update a = RN(x - deq) and the move b = RN(p - deq),
// p = RN(n s'), enter only through their signs (a rounded difference of two
// floats is zero only when they are equal, and has their difference's sign),
// and so does d = RN(y - n). A reversal (a and b of opposite signs) takes
// ceil(y) when the update is positive and floor(y) when it is negative;
// ceil = n + 1 exactly when d > 0, floor = n - 1 exactly when d < 0. With
// e = RN(deq - p) = -b the code therefore moves up when min(a, e, d) > 0 and
// down when max(a, e, d) < 0: one three-input minimum and maximum, each
// compared into 1.0f or 0.0f.
//
// No clamp to [-qmax, qmax] is needed afterwards. A step up from n = qmax
// needs y > qmax, and only x = A itself (the column's absmax) reaches it,
// when A * inv > qmax; it also needs p < deq < x = A. For every significand
// of A where A * inv > qmax (qmax 7 and 127, all 2^23 of them; the
// quantities scale exactly with A's exponent over the range used), p is at
// least the float just below A, so no deq lies strictly between: the step
// never happens. Mirrored, the same holds for a step down from -qmax.
//
// deq and p are products. Their differences are taken with the scalar
// __fsub_rn / __fadd_rn, which the compiler never contracts with the
// multiply before them:
// a two-wide subtraction of a two-wide product was seen contracted into one
// fused multiply-add, which keeps the product unrounded and turns an exact
// tie (x == deq or deq == p, difference 0) into a nonzero sign.
template <int BITS>
__device__ __forceinline__ float2 bdr_round(float2 x, float2 inv, float2 deq, float2 s_new,
                                            float2 kb) {
    const float2 nb = fma2(x, inv, kb);
    const float2 nn = sub2(kb, nb);                     // -n
    const float2 d = fma2(x, inv, nn);
    const float2 mp = mul2(nn, s_new);                  // -p
    const float2 a = make_float2(__fsub_rn(x.x, deq.x), __fsub_rn(x.y, deq.y));
    const float2 e = make_float2(__fadd_rn(deq.x, mp.x), __fadd_rn(deq.y, mp.y));   // deq - p
    const float2 up = make_float2(set_gt(min3(a.x, e.x, d.x), 0.0f),
                                  set_gt(min3(a.y, e.y, d.y), 0.0f));
    const float2 dn = make_float2(set_lt(max3(a.x, e.x, d.x), 0.0f),
                                  set_lt(max3(a.y, e.y, d.y), 0.0f));
    return add2(nb, sub2(up, dn));
}

// Codes of two elements (key rows i, i+1 of value column j; i even), returned
// as the floats kb + code (kb: word_bias of the two elements' word positions)
// whose low bits are the stored byte (nibble). inv, s_new: the column's values
// in both halves. The value rounded is the exact product x*inv: one fused
// multiply-add rounds it straight to an integer. HASH64 selects the 64-bit
// form of the SR draw (identical bits).
template <int MODE, int BITS, bool HASH64 = false>
__device__ __forceinline__ float2 round_rows(float2 x, float2 inv, float2 deq, float2 s_new,
                                             float2 kb, uint64_t hkey, uint32_t i, uint32_t j) {
    if constexpr (MODE == kRTN) {
        // |x*inv| <= qmax (1 + 2^-24) since inv = RN(qmax/A) and |x| <= A:
        // the nearest integer never leaves [-qmax, qmax], no clamp needed.
        return fma2(x, inv, kb);
    } else if constexpr (MODE == kSR) {
        uint32_t t0, t1;
        if constexpr (HASH64) {
            t0 = element_top_u64(hkey, i, j);
            t1 = element_top_u64(hkey, i + 1, j);
        } else {
            const HashColumn hc = hash_column(hkey, j);
            const uint32_t khi = static_cast<uint32_t>(hkey >> 32) ^ i;
            t0 = hash_top(khi, hc);
            t1 = hash_top(khi ^ 1u, hc);                                // row i + 1 (i even)
        }
        return sr_round<BITS>(x, inv, kb, t0, t1);
    } else {
        return bdr_round<BITS>(x, inv, deq, s_new, kb);
    }
}

__device__ __forceinline__ void st_cs_u4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ void st_cs_f2(float* p, float2 s) {
    asm volatile("st.global.cs.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(s.x), "f"(s.y) : "memory");
}

// N consecutive floats of shared memory (N a multiple of 4) into registers.
template <int N>
__device__ __forceinline__ void ld_smem_rows(const float* p, float (&r)[N]) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
        const float4 t = reinterpret_cast<const float4*>(p)[i];
        r[4 * i] = t.x; r[4 * i + 1] = t.y; r[4 * i + 2] = t.z; r[4 * i + 3] = t.w;
    }
}

// bfloat16 pattern(s) -> float (exact: the pattern is the upper half of the
// binary32 pattern).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Rows [row0, row0 + N) of a q or k array in shared memory (element type IO),
// as floats. row0 and N multiples of 8.
template <int IO, int N>
__device__ __forceinline__ void ld_rows(const uint8_t* base, int row0, float (&r)[N]) {
    if constexpr (IO == kIoF32) {
        ld_smem_rows<N>(reinterpret_cast<const float*>(base) + row0, r);
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(base + row0 * 2);
#pragma unroll
        for (int i = 0; i < N / 8; ++i) {
            const uint4 t = p[i];
            const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                r[8 * i + 2 * e] = bf16_lo(w[e]);
                r[8 * i + 2 * e + 1] = bf16_hi(w[e]);
            }
        }
    }
}

// Two floats as the bfloat16 patterns nearest to them (ties to even), x in
// the low half of the word.
__device__ __forceinline__ uint32_t bf16x2_rn(float2 v) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(v.y), "f"(v.x));
    return r;
}

// Elements idx, idx + 1 (idx even) of a v array in shared memory.
template <int IO>
__device__ __forceinline__ float2 ld_pair(const uint8_t* base, int idx) {
    if constexpr (IO == kIoF32) {
        return *reinterpret_cast<const float2*>(base + idx * 4);
    } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(base + idx * 2);
        return make_float2(bf16_lo(w), bf16_hi(w));
    }
}

// Geometry of one lane's codes for one column pair of one scale group: a run
// of 16-byte units, each holding EPU consecutive elements of the pair's
// row-major (row, column) stream, i.e. RPU key rows; a 32-bit word holds RPW
// rows. The packed arithmetic works on two consecutive key rows of one
// column: in a word, the rows (r, r+1) of column c are elements 4p + c and
// 4p + 2 + c for row pair p of the word.
template <int GROUP, int BITS>
struct PairGeo {
    static constexpr int EPW = 32 / BITS;       // elements per 32-bit word
    static constexpr int RPW = EPW / 2;         // key rows per word
    static constexpr int EPU = 4 * EPW;         // elements per 16-byte unit
    static constexpr int RPU = EPU / 2;         // key rows per unit
    static constexpr int UNITS = GROUP / RPU;   // units per pair per group
    static_assert(RPU % 4 == 0 && GROUP % RPU == 0, "unit geometry");
};

__device__ __forceinline__ uint4 lds_unit(const uint8_t* cs, int unit, int lane) {
    return *reinterpret_cast<const uint4*>(cs + (unit * 32 + lane) * 16);
}

// Delta rule, first pass: u_c += k_i * deq_ic for the two columns of one
// pair over the rows of one group, in key order.
template <int GROUP, int BITS, int IO>
__device__ __forceinline__ void pair_ktS(const uint8_t* __restrict__ cs, int ubase, float2 sc,
                                         const uint8_t* __restrict__ ks, int lane, float2& u) {
    using G = PairGeo<GROUP, BITS>;
    constexpr float BIAS = Q<BITS>::kBias;
    const float2 s0 = f2(sc.x), s1 = f2(sc.y);
#pragma unroll
    for (int un = 0; un < G::UNITS; ++un) {
        const uint4 raw = lds_unit(cs, ubase + un, lane);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
        float kk[G::RPU];
        ld_rows<IO, G::RPU>(ks, un * G::RPU, kk);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            decode_word_biased<BITS>(wd[wi], f);
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int rl = wi * G::RPW + 2 * rp;
                const float2 kr = make_float2(kk[rl], kk[rl + 1]);
                const float2 c0 = add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-(kTwo23 + BIAS)));
                const float2 c1 = add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-(kTwo23 + BIAS)));
                const float2 d0 = mul2(c0, s0), d1 = mul2(c1, s1);
                u.x = __fmaf_rn(kr.x, d0.x, u.x);
                u.x = __fmaf_rn(kr.y, d0.y, u.x);
                u.y = __fmaf_rn(kr.x, d1.x, u.y);
                u.y = __fmaf_rn(kr.y, d1.y, u.y);
            }
        }
    }
}

// One column pair of one scale group: dequantize, update, accumulate the
// output, new scales, requantize and store. x[rp][c] holds rows (2rp, 2rp+1)
// of column c of the pair.
template <int GROUP, int GATE, int MODE, int BITS, int IO>
__device__ __forceinline__ void pair_step(const uint8_t* __restrict__ cs, int ubase, float2 sc,
                                          const uint8_t* __restrict__ qs,
                                          const uint8_t* __restrict__ ks,
                                          const float* __restrict__ gs, float gscalar, float2 w,
                                          float2& o, uint8_t* __restrict__ gcodes,
                                          float* __restrict__ gscale, uint64_t hkey, int row0,
                                          uint32_t j0, int lane) {
    using G = PairGeo<GROUP, BITS>;
    constexpr float BIAS = Q<BITS>::kBias;
    const float2 s0 = f2(sc.x), s1 = f2(sc.y);     // per-column constants as pairs
    const float2 w0 = f2(w.x), w1 = f2(w.y);
    const float2 gsc = f2(gscalar);
    float2 x[GROUP / 2][2];

#pragma unroll
    for (int un = 0; un < G::UNITS; ++un) {
        const uint4 raw = lds_unit(cs, ubase + un, lane);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
        float kk[G::RPU], qq[G::RPU], gg[G::RPU];
        ld_rows<IO, G::RPU>(ks, un * G::RPU, kk);
        ld_rows<IO, G::RPU>(qs, un * G::RPU, qq);
        if constexpr (GATE == kGatePerKey) ld_smem_rows<G::RPU>(gs + un * G::RPU, gg);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            decode_word_biased<BITS>(wd[wi], f);
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int rl = wi * G::RPW + 2 * rp;
                const int r = un * G::RPU + rl;
                const float2 kr = make_float2(kk[rl], kk[rl + 1]);
                const float2 qr = make_float2(qq[rl], qq[rl + 1]);
                const float2 gr = GATE == kGatePerKey ? make_float2(gg[rl], gg[rl + 1]) : gsc;
                const float2 c0 = add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-(kTwo23 + BIAS)));
                const float2 c1 = add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-(kTwo23 + BIAS)));
                const float2 x0 = fma2(gr, mul2(c0, s0), mul2(kr, w0));
                const float2 x1 = fma2(gr, mul2(c1, s1), mul2(kr, w1));
                o.x = __fmaf_rn(qr.x, x0.x, o.x);
                o.x = __fmaf_rn(qr.y, x0.y, o.x);
                o.y = __fmaf_rn(qr.x, x1.x, o.y);
                o.y = __fmaf_rn(qr.y, x1.y, o.y);
                x[r / 2][0] = x0;
                x[r / 2][1] = x1;
            }
        }
    }

    // absmax per column over the group's rows (order-free)
    float a0 = 0.0f, a1 = 0.0f, b0 = 0.0f, b1 = 0.0f;
#pragma unroll
    for (int rp = 0; rp < GROUP / 2; rp += 2) {
        a0 = max_abs3(a0, x[rp][0].x, x[rp][0].y);
        a1 = max_abs3(a1, x[rp + 1][0].x, x[rp + 1][0].y);
        b0 = max_abs3(b0, x[rp][1].x, x[rp][1].y);
        b1 = max_abs3(b1, x[rp + 1][1].x, x[rp + 1][1].y);
    }
    const float A0 = fmaxf(a0, a1), A1 = fmaxf(b0, b1);
    float2 snew, inv;
    new_scales<BITS>(A0, A1, snew, inv);
    st_cs_f2(gscale, snew);
    const float2 inv0 = f2(inv.x), inv1 = f2(inv.y);
    const float2 sn0 = f2(snew.x), sn1 = f2(snew.y);

#pragma unroll
    for (int un = 0; un < G::UNITS; ++un) {
        uint32_t ow[4];
        uint32_t wd[4] = {0u, 0u, 0u, 0u};
        if constexpr (MODE == kBDR) {
            const uint4 raw = lds_unit(cs, ubase + un, lane);
            wd[0] = raw.x; wd[1] = raw.y; wd[2] = raw.z; wd[3] = raw.w;
        }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            if constexpr (MODE == kBDR) decode_word_biased<BITS>(wd[wi], f);
            float t[G::EPW];
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int r = un * G::RPU + wi * G::RPW + 2 * rp;
                float2 dq0 = f2(0.0f), dq1 = f2(0.0f);
                if constexpr (MODE == kBDR) {
                    dq0 = mul2(add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-(kTwo23 + BIAS))), s0);
                    dq1 = mul2(add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-(kTwo23 + BIAS))), s1);
                }
                const uint32_t i = static_cast<uint32_t>(row0 + r);
                const float2 kb0 = make_float2(word_bias<BITS>(4 * rp), word_bias<BITS>(4 * rp + 2));
                const float2 kb1 = make_float2(word_bias<BITS>(4 * rp + 1), word_bias<BITS>(4 * rp + 3));
                const float2 t0 = round_rows<MODE, BITS>(x[r / 2][0], inv0, dq0, sn0, kb0, hkey, i, j0);
                const float2 t1 = round_rows<MODE, BITS>(x[r / 2][1], inv1, dq1, sn1, kb1, hkey, i,
                                                         j0 + 1);
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

// Where one tile's codes live and how wide each scale group's codes are.
// prec_map holds a width (4 or 8) per head (pgroups == 1) or per (head,
// group) in [H][G] order (pgroups == G); a head's groups are consecutive
// blocks of GROUP*d_v*width/8 bytes at head_offsets[h] within the batch row.
struct TileLayout {
    int64_t code_off;    // byte offset of the tile's codes
    uint32_t mask8;      // bit g set: group g is int8 (else int4); G <= 16
    bool ok;             // the widths are valid and fit the head's offsets

    __device__ __forceinline__ int bits(int g) const { return (mask8 >> g) & 1u ? 8 : 4; }
    // byte offset of group g inside the tile; half = GROUP*d_v/2 (an int4 group)
    __device__ __forceinline__ int64_t goff(int g, int half) const {
        return static_cast<int64_t>(half) * (g + __popc(mask8 & ((1u << g) - 1u)));
    }
    __device__ __forceinline__ void load(const uint8_t* prec_map, const int64_t* head_offsets,
                                         int64_t batch_stride, int H, int pgroups, int G,
                                         int group_bytes8, int b, int h) {
        const int64_t off = __ldg(head_offsets + h);
        const int64_t end = (h + 1 < H) ? __ldg(head_offsets + h + 1) : batch_stride;
        int64_t bytes = 0;
        bool valid = true;
        mask8 = 0;
        if (pgroups <= 1) {
            const int pr = __ldg(prec_map + h);
            valid = pr == 4 || pr == 8;
            mask8 = pr == 8 ? (G >= 32 ? 0xFFFFFFFFu : (1u << G) - 1u) : 0u;
            bytes = static_cast<int64_t>(G) * group_bytes8 * pr / 8;
        } else {
            for (int g = 0; g < G; ++g) {
                const int pr = __ldg(prec_map + static_cast<int64_t>(h) * G + g);
                valid = valid && (pr == 4 || pr == 8);
                if (pr == 8) mask8 |= 1u << g;
                bytes += static_cast<int64_t>(group_bytes8) * pr / 8;
            }
        }
        ok = valid && off >= 0 && off + bytes <= end;
        code_off = static_cast<int64_t>(b) * batch_stride + off;
    }
};

// A warp's walk over its tiles gw, gw + W, ...: the tile's batch row and
// head are advanced incrementally (no division per tile), and its layout
// read from the precision map and head offsets (ok = false when prec_map
// does not fit the offsets).
struct TileCursor : TileLayout {
    int tile, b, h;
    int db, dh;          // W / H and W % H

    __device__ __forceinline__ void init(const StepParams& p, int first, int W) {
        tile = first;
        b = first / p.H;
        h = first - b * p.H;
        db = W / p.H;
        dh = W - db * p.H;
    }
    __device__ __forceinline__ void advance(const StepParams& p, int W) {
        tile += W;
        b += db;
        h += dh;
        if (h >= p.H) {
            h -= p.H;
            ++b;
        }
    }
    __device__ __forceinline__ void load(const StepParams& p, int group_bytes8) {
        TileLayout::load(p.prec_map, p.head_offsets, p.batch_stride, p.H, p.pgroups, p.G,
                         group_bytes8, b, h);
    }
};

// The same step for modes whose per-element rounding is long (SR, BDR): two
// short loops over 16-byte units, so the kernel's code stays small enough for
// the instruction cache. The first computes x, the output and the absmax; the
// second rounds. Between them, the group's updated values are either staged
// in the warp's shared-memory x buffer (STAGE; xs holds (x[r][c0],
// x[r+1][c0], x[r][c1], x[r+1][c1]) per row pair r and lane) or recomputed
// from the codes, scales, k, gates and w, by the same operations in the same
// order, so bit for bit the same values.
//
// SR draws come from the group's row table (rtab: per row pair of the group
// the SrRow values of its two rows) when the tile's low-sum carry is the same
// for all columns (rowtab), else from the whole per-element hash.
template <int GROUP, int GATE, int MODE, int BITS, int IO, bool STAGE, bool ROWTAB>
__device__ __forceinline__ void round_pass(const uint8_t* __restrict__ cs, int ubase, float2 sc,
                                           const uint8_t* __restrict__ ks,
                                           const float* __restrict__ gs, float gscalar, float2 w,
                                           float2 inv, float2 snew, uint8_t* __restrict__ gcodes,
                                           uint64_t hkey, int row0, uint32_t j0, int lane,
                                           const float4* __restrict__ xs,
                                           const uint4* __restrict__ rtab) {
    using G = PairGeo<GROUP, BITS>;
    constexpr float BIAS = Q<BITS>::kBias;
    constexpr int RPUH = G::RPU / 2;              // row pairs per unit
    const float2 s0 = f2(sc.x), s1 = f2(sc.y);
    const float2 w0 = f2(w.x), w1 = f2(w.y);
    const float2 gsc = f2(gscalar);
    const float2 inv0 = f2(inv.x), inv1 = f2(inv.y);
    const float2 sn0 = f2(snew.x), sn1 = f2(snew.y);
    // SR column parts of the draw: row-table form (clo only) or the whole hash
    const uint32_t khi = static_cast<uint32_t>(hkey >> 32);
    const HashColumn hc0 = hash_column(hkey, j0), hc1 = hash_column(hkey, j0 + 1);

    constexpr bool DECODE = MODE == kBDR || !STAGE;   // this pass reads the old codes
#pragma unroll 1
    for (int un = 0; un < G::UNITS; ++un) {
        uint32_t ow[4];
        uint32_t wd[4] = {0u, 0u, 0u, 0u};
        if constexpr (DECODE) {
            const uint4 raw = lds_unit(cs, ubase + un, lane);
            wd[0] = raw.x; wd[1] = raw.y; wd[2] = raw.z; wd[3] = raw.w;
        }
        float kk[STAGE ? 1 : G::RPU], gg[STAGE || GATE != kGatePerKey ? 1 : G::RPU];
        if constexpr (!STAGE) {
            ld_rows<IO, G::RPU>(ks, un * G::RPU, kk);
            if constexpr (GATE == kGatePerKey) ld_smem_rows<G::RPU>(gs + un * G::RPU, gg);
        }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            if constexpr (DECODE) decode_word_biased<BITS>(wd[wi], f);
            float t[G::EPW];
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int rl = wi * G::RPW + 2 * rp;
                float2 dq0 = f2(0.0f), dq1 = f2(0.0f);
                if constexpr (DECODE) {
                    dq0 = mul2(add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-(kTwo23 + BIAS))), s0);
                    dq1 = mul2(add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-(kTwo23 + BIAS))), s1);
                }
                float4 xv;
                if constexpr (STAGE) {
                    xv = xs[(un * RPUH + rl / 2) * 32 + lane];
                } else {
                    // the first loop's x, recomputed by the same operations
                    const float2 kr = make_float2(kk[rl], kk[rl + 1]);
                    const float2 gr = GATE == kGatePerKey ? make_float2(gg[rl], gg[rl + 1]) : gsc;
                    const float2 x0 = fma2(gr, dq0, mul2(kr, w0));
                    const float2 x1 = fma2(gr, dq1, mul2(kr, w1));
                    xv = make_float4(x0.x, x0.y, x1.x, x1.y);
                }
                const float2 kb0 = make_float2(word_bias<BITS>(4 * rp), word_bias<BITS>(4 * rp + 2));
                const float2 kb1 = make_float2(word_bias<BITS>(4 * rp + 1), word_bias<BITS>(4 * rp + 3));
                float2 t0, t1;
                if constexpr (MODE == kSR) {
                    uint32_t a0, a1, b0, b1;          // tops: column 0 rows i, i+1; column 1
                    if constexpr (ROWTAB) {
                        const uint4 rt = rtab[un * RPUH + rl / 2];
                        a0 = hash_top_row(hc0.clo, rt.x, rt.y);
                        a1 = hash_top_row(hc0.clo, rt.z, rt.w);
                        b0 = hash_top_row(hc1.clo, rt.x, rt.y);
                        b1 = hash_top_row(hc1.clo, rt.z, rt.w);
                    } else {
                        const uint32_t ki = khi ^ static_cast<uint32_t>(row0 + un * G::RPU + rl);
                        a0 = hash_top(ki, hc0);
                        a1 = hash_top(ki ^ 1u, hc0);
                        b0 = hash_top(ki, hc1);
                        b1 = hash_top(ki ^ 1u, hc1);
                    }
                    t0 = sr_round<BITS>(make_float2(xv.x, xv.y), inv0, kb0, a0, a1);
                    t1 = sr_round<BITS>(make_float2(xv.z, xv.w), inv1, kb1, b0, b1);
                } else {
                    t0 = round_rows<MODE, BITS>(make_float2(xv.x, xv.y), inv0, dq0, sn0, kb0, 0ull,
                                                0u, 0u);
                    t1 = round_rows<MODE, BITS>(make_float2(xv.z, xv.w), inv1, dq1, sn1, kb1, 0ull,
                                                0u, 0u);
                }
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

// The first loop of pair_step_xs: x, the output, the absmax (and the staged
// x); then the new scales, stored, and their inverses.
template <int GROUP, int GATE, int MODE, int BITS, int IO, bool STAGE>
__device__ __forceinline__ void pair_pass1_xs(const uint8_t* __restrict__ cs, int ubase, float2 sc,
                                              const uint8_t* __restrict__ qs,
                                              const uint8_t* __restrict__ ks,
                                              const float* __restrict__ gs, float gscalar,
                                              float2 w, float2& o, float* __restrict__ gscale,
                                              int lane, float4* __restrict__ xs, float2& snew,
                                              float2& inv) {
    using G = PairGeo<GROUP, BITS>;
    constexpr float BIAS = Q<BITS>::kBias;
    constexpr int RPUH = G::RPU / 2;              // row pairs per unit
    const float2 s0 = f2(sc.x), s1 = f2(sc.y);
    const float2 w0 = f2(w.x), w1 = f2(w.y);
    const float2 gsc = f2(gscalar);
    float a0 = 0.0f, b0 = 0.0f;

#pragma unroll 1
    for (int un = 0; un < G::UNITS; ++un) {
        const uint4 raw = lds_unit(cs, ubase + un, lane);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
        float kk[G::RPU], qq[G::RPU], gg[G::RPU];
        ld_rows<IO, G::RPU>(ks, un * G::RPU, kk);
        ld_rows<IO, G::RPU>(qs, un * G::RPU, qq);
        if constexpr (GATE == kGatePerKey) ld_smem_rows<G::RPU>(gs + un * G::RPU, gg);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            decode_word_biased<BITS>(wd[wi], f);
#pragma unroll
            for (int rp = 0; rp < G::RPW / 2; ++rp) {
                const int rl = wi * G::RPW + 2 * rp;
                const float2 kr = make_float2(kk[rl], kk[rl + 1]);
                const float2 qr = make_float2(qq[rl], qq[rl + 1]);
                const float2 gr = GATE == kGatePerKey ? make_float2(gg[rl], gg[rl + 1]) : gsc;
                const float2 c0 = add2(make_float2(f[4 * rp], f[4 * rp + 2]), f2(-(kTwo23 + BIAS)));
                const float2 c1 = add2(make_float2(f[4 * rp + 1], f[4 * rp + 3]), f2(-(kTwo23 + BIAS)));
                const float2 x0 = fma2(gr, mul2(c0, s0), mul2(kr, w0));
                const float2 x1 = fma2(gr, mul2(c1, s1), mul2(kr, w1));
                o.x = __fmaf_rn(qr.x, x0.x, o.x);
                o.x = __fmaf_rn(qr.y, x0.y, o.x);
                o.y = __fmaf_rn(qr.x, x1.x, o.y);
                o.y = __fmaf_rn(qr.y, x1.y, o.y);
                a0 = max_abs3(a0, x0.x, x0.y);
                b0 = max_abs3(b0, x1.x, x1.y);
                if constexpr (STAGE)
                    xs[(un * RPUH + rl / 2) * 32 + lane] = make_float4(x0.x, x0.y, x1.x, x1.y);
            }
        }
    }

    new_scales<BITS>(a0, b0, snew, inv);
    st_cs_f2(gscale, snew);
}

// The rounding loop of pair_step_xs, from the first loop's snew and inv.
template <int GROUP, int GATE, int MODE, int BITS, int IO, bool STAGE>
__device__ __forceinline__ void pair_round_xs(const uint8_t* __restrict__ cs, int ubase, float2 sc,
                                              const uint8_t* __restrict__ ks,
                                              const float* __restrict__ gs, float gscalar,
                                              float2 w, float2 snew, float2 inv,
                                              uint8_t* __restrict__ gcodes, uint64_t hkey,
                                              int row0, uint32_t j0, int lane,
                                              const float4* __restrict__ xs,
                                              const uint4* __restrict__ rtab, bool rowtab) {
    if (MODE == kSR && rowtab)
        round_pass<GROUP, GATE, MODE, BITS, IO, STAGE, true>(cs, ubase, sc, ks, gs, gscalar, w,
                                                            inv, snew, gcodes, hkey, row0, j0,
                                                            lane, xs, rtab);
    else
        round_pass<GROUP, GATE, MODE, BITS, IO, STAGE, false>(cs, ubase, sc, ks, gs, gscalar, w,
                                                             inv, snew, gcodes, hkey, row0, j0,
                                                             lane, xs, rtab);
}

template <int GROUP, int GATE, int MODE, int BITS, int IO, bool STAGE>
__device__ __forceinline__ void pair_step_xs(const uint8_t* __restrict__ cs, int ubase, float2 sc,
                                             const uint8_t* __restrict__ qs,
                                             const uint8_t* __restrict__ ks,
                                             const float* __restrict__ gs, float gscalar,
                                             float2 w, float2& o, uint8_t* __restrict__ gcodes,
                                             float* __restrict__ gscale, uint64_t hkey, int row0,
                                             uint32_t j0, int lane, float4* __restrict__ xs,
                                             const uint4* __restrict__ rtab, bool rowtab) {
    float2 snew, inv;
    pair_pass1_xs<GROUP, GATE, MODE, BITS, IO, STAGE>(cs, ubase, sc, qs, ks, gs, gscalar, w, o,
                                                      gscale, lane, xs, snew, inv);
    pair_round_xs<GROUP, GATE, MODE, BITS, IO, STAGE>(cs, ubase, sc, ks, gs, gscalar, w, snew, inv,
                                                      gcodes, hkey, row0, j0, lane, xs, rtab,
                                                      rowtab);
}

// Fill `slot` with group g of the cursor's tile (lane 0 only); with the
// first group, also the tile's inputs (into `tin`, or for INS into the
// header's v and the slot's q, k rows). A tile whose layout does not fit gets
// a bare arrival, so the slot's phase still completes.
template <int C, int GROUP, int GATE, int IO, bool INS>
__device__ __forceinline__ void issue_item(const StepParams& p, uint8_t* wsm, int slot,
                                           const TileCursor& tc, int g, uint8_t* tin,
                                           uint64_t pol_state, uint64_t pol_in) {
    using S = Slot<C, GROUP, GATE, IO, INS>;
    constexpr int DV = 32 * C;
    constexpr int ES = S::ES;
    uint64_t* bar = reinterpret_cast<uint64_t*>(wsm) + slot;
    if (!tc.ok) {
        mbar_arrive(bar);
        return;
    }
    const int tile = tc.tile;
    const int dk = p.d_k;
    uint8_t* sm = wsm + S::header(dk) + slot * S::kBytes;
    const uint32_t cbytes = GROUP * DV * tc.bits(g) / 8;
    const int64_t rowbase = static_cast<int64_t>(tile) * dk;
    uint32_t total = cbytes + DV * 4;
    if (INS) {
        total += 2 * GROUP * ES;
        if (g == 0) total += DV * ES;
    } else if (g == 0) {
        total += S::tile_in_payload(dk);
    }
    if constexpr (kBoundsCheck) {
        // the slot and the tile-input buffer inside the warp's shared memory;
        // the group's codes and scales and the tile's rows inside their buffers
        const int64_t coff = tc.code_off + tc.goff(g, GROUP * DV / 2);
        const bool ok =
            in_bounds(sm + S::kBytes <= wsm + p.warp_smem && (INS || slot < p.slots) &&
                          (INS || tin + S::tile_in_payload(dk) <= wsm + S::header(dk)) &&
                          coff >= 0 && coff + cbytes <= p.code_bytes &&
                          (static_cast<int64_t>(tile) * p.G + g + 1) * DV <= p.scale_count &&
                          tile < p.ntiles,
                      p.err);
        if (!ok) {
            mbar_arrive(bar);
            return;
        }
    }
    mbar_arrive_expect_tx(bar, total);
    bulk_g2s(sm, p.codes + tc.code_off + tc.goff(g, GROUP * DV / 2), cbytes, bar, pol_state);
    bulk_g2s(sm + S::kScales, p.scales + (static_cast<int64_t>(tile) * p.G + g) * DV, DV * 4, bar,
             pol_state);
    const uint8_t* vsrc = static_cast<const uint8_t*>(p.v) + static_cast<int64_t>(tile) * DV * ES;
    if (INS) {
        const int64_t r0 = rowbase + g * GROUP;
        bulk_g2s(sm + S::kQ, static_cast<const uint8_t*>(p.q) + r0 * ES, GROUP * ES, bar, pol_in);
        bulk_g2s(sm + S::kK, static_cast<const uint8_t*>(p.k) + r0 * ES, GROUP * ES, bar, pol_in);
        if (g == 0) bulk_g2s(wsm + 128, vsrc, DV * ES, bar, pol_in);
    } else if (g == 0) {
        bulk_g2s(tin, static_cast<const uint8_t*>(p.q) + rowbase * ES, dk * ES, bar, pol_in);
        bulk_g2s(tin + S::in_k(dk), static_cast<const uint8_t*>(p.k) + rowbase * ES, dk * ES, bar,
                 pol_in);
        if (GATE == kGatePerKey)
            bulk_g2s(tin + S::in_g(dk), p.gates + rowbase, dk * 4, bar, pol_in);
        bulk_g2s(tin + S::in_v(dk), vsrc, DV * ES, bar, pol_in);
    }
}

// Position in a warp's ring: item k lives in slot k % slots and completes
// phase parity (k / slots) & 1 of that slot's mbarrier.
struct Ring {
    int slot = 0;
    uint32_t par = 0;
    __device__ __forceinline__ void advance(int slots) {
        if (++slot == slots) {
            slot = 0;
            par ^= 1u;
        }
    }
};

// The warp's items are (tile, group) pairs in order: item k is group k % G of
// the warp's tile k / G (tiles gw, gw + W, ...).
template <int C, int GROUP, int UPD, int GATE, int MODE, int IO>
__global__ void __launch_bounds__(step_max_warps(GROUP, MODE, UPD) * 32, 1)
    step_kernel(const StepParams p) {
    constexpr bool INS = UPD == kDelta;
    using S = Slot<C, GROUP, GATE, IO, INS>;
    constexpr int DV = 32 * C;
    constexpr int P = C / 2;
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
    const int G = p.G, NS = p.slots;
    const int hdr = S::header(p.d_k), tib = S::tile_in_bytes(p.d_k);
    const int in_k = S::in_k(p.d_k), in_g = S::in_g(p.d_k), in_v = S::in_v(p.d_k);
    float* cvt = reinterpret_cast<float*>(wsm + hdr + NS * S::kBytes);   // bf16 widened (CVT)
    float4* xs = reinterpret_cast<float4*>(wsm + hdr + NS * S::kBytes +
                                           S::cvt_bytes(p.d_k));              // staging variants
    uint2* rtab2 = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(xs) +
                                            (stage_x(MODE, UPD) ? S::kXsBytes : 0));  // SR
    const uint4* rtab = reinterpret_cast<const uint4*>(rtab2);
    constexpr int IOR = S::CVT ? kIoF32 : IO;     // element type the pair code reads
    constexpr int ESR = IOR == kIoBF16 ? 2 : 4;
    const int ntw = gw < p.ntiles ? (p.ntiles - gw + W - 1) / W : 0;   // this warp's tiles
    const int64_t K = static_cast<int64_t>(ntw) * G;                    // this warp's items

    if (lane == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    const uint64_t pol_state = policy_evict_first();
    const uint64_t pol_in = policy_evict_first();
    Ring ic, is;                 // consumer and issuer positions
    int64_t kc = 0, ki = 0;      // items consumed, items issued
    int it_g = 0;                // group of item ki
    int it_n = 0;                // warp-local tile number of item ki
    TileCursor itc;              // tile of item ki
    itc.init(p, gw, W);
    if (K > 0) itc.load(p, GROUP * DV);

    // p.inject (error-path tests): n + 1 issues copies for the warp's first n
    // items only, so a later wait runs out
    const int64_t kmax = p.inject ? static_cast<int64_t>(p.inject - 1) : K;
    auto issue_next = [&]() {
        if (ki < K && ki < kmax) {
            if (lane == 0)
                issue_item<C, GROUP, GATE, IO, INS>(p, wsm, is.slot, itc, it_g,
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
    // the consumer is done with its slot: hand it to the next item's copy
    auto release_slot = [&]() {
        ++kc;
        ic.advance(NS);
        __syncwarp();
        if (lane == 0) fence_proxy_async_smem();
        issue_next();
    };

    float nscal = 0.0f, nbeta = 0.0f;
    if (ntw > 0) {
        if (GATE == kGate) nscal = __ldg(p.gates + gw);
        if (UPD == kDelta) nbeta = __ldg(p.beta + gw);
    }

    bool ok = true;
    TileCursor ti;               // the consumer's tile
    ti.init(p, gw, W);
    for (int n = 0; n < ntw && ok; ++n, ti.advance(p, W)) {
        const int tile = ti.tile;
        ti.load(p, GROUP * DV);
        const uint8_t* tin = wsm + 128 + (n & 1) * tib;   // this tile's q, k, gates, v (!INS)
        const uint8_t* v_s = INS ? wsm + 128 : tin + in_v;
        const float gscalar = nscal, beta = nbeta;
        if (n + 1 < ntw) {
            if (GATE == kGate) nscal = __ldg(p.gates + tile + W);
            if (UPD == kDelta) nbeta = __ldg(p.beta + tile + W);
        }
        const uint64_t hkey = MODE == kSR ? tile_hash_key(p.seed, p.step,
                                                          static_cast<uint32_t>(ti.b),
                                                          static_cast<uint32_t>(ti.h))
                                          : 0ull;
        uint32_t hcarry = 0;
        const bool rowtab = MODE == kSR && sr_tile_carry(hkey, DV, &hcarry);

        // the tile's first group
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[ic.slot], ic.par, p.timeout_ns));
        if (!ok) break;

        // where this tile's q, k, v are read from (widened to fp32 for CVT)
        const uint8_t* tq = tin;
        const uint8_t* tk = tin + in_k;
        const uint8_t* tv = v_s;
        if constexpr (S::CVT) {
            if (ti.ok) {
                const int dk = p.d_k;
                __syncwarp();                 // the previous tile is done with cvt
                for (int e = 2 * lane; e < dk; e += 64) {
                    const uint32_t wq = *reinterpret_cast<const uint32_t*>(tin + e * 2);
                    const uint32_t wk = *reinterpret_cast<const uint32_t*>(tin + in_k + e * 2);
                    cvt[e] = bf16_lo(wq);
                    cvt[e + 1] = bf16_hi(wq);
                    cvt[dk + e] = bf16_lo(wk);
                    cvt[dk + e + 1] = bf16_hi(wk);
                }
                for (int e = 2 * lane; e < DV; e += 64) {
                    const uint32_t wv = *reinterpret_cast<const uint32_t*>(v_s + e * 2);
                    cvt[2 * dk + e] = bf16_lo(wv);
                    cvt[2 * dk + e + 1] = bf16_hi(wv);
                }
                __syncwarp();
                tq = reinterpret_cast<const uint8_t*>(cvt);
                tk = reinterpret_cast<const uint8_t*>(cvt + dk);
                tv = reinterpret_cast<const uint8_t*>(cvt + 2 * dk);
            }
        }

        bool inside = true;      // the tile's codes and scales inside their buffers
        if constexpr (kBoundsCheck) {
            const int64_t tbytes = ti.goff(G, GROUP * DV / 2);
            inside = !ti.ok || in_bounds(ti.code_off >= 0 && ti.code_off + tbytes <= p.code_bytes &&
                                             (static_cast<int64_t>(tile) + 1) * G * DV <=
                                                 p.scale_count,
                                         p.err);
        }
        if (!ti.ok || !inside) {
            // a layout mismatch (no copies were made) or, in the bounds-checked
            // build, a tile outside its buffers: record it and skip the tile
            if (lane == 0 && !ti.ok) atomicOr(p.err, kErrLayout);
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

        float2 w[P], o[P];
#pragma unroll
        for (int pc = 0; pc < P; ++pc) o[pc] = f2(0.0f);
        if (UPD == kDelta) {
            float2 u[P];
#pragma unroll
            for (int pc = 0; pc < P; ++pc) u[pc] = f2(0.0f);
            // the first pass takes the groups as they arrive (the ring holds
            // the whole tile), the second pass finds them all resident
            Ring r = ic;
            for (int g = 0; g < G && ok; ++g) {
                if (g > 0)
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait_bounded(&bars[r.slot], r.par, p.timeout_ns));
                if (!ok) break;
                const uint8_t* sm = wsm + hdr + r.slot * S::kBytes;
                const float* ss = reinterpret_cast<const float*>(sm + S::kScales) + lane * C;
                const uint8_t* ks = INS ? sm + S::kK : tk + g * GROUP * ESR;
                float2 up = u[0], uq = u[P - 1];
#pragma unroll 1
                for (int pc = 0; pc < P; ++pc) {
                    const float2 sc = *reinterpret_cast<const float2*>(ss + 2 * pc);
                    if (ti.bits(g) == 8)
                        pair_ktS<GROUP, 8, IOR>(sm, pc * PairGeo<GROUP, 8>::UNITS, sc, ks, lane, up);
                    else
                        pair_ktS<GROUP, 4, IOR>(sm, pc * PairGeo<GROUP, 4>::UNITS, sc, ks, lane, up);
                    if constexpr (P == 2) {
                        const float2 t = up;
                        up = uq; uq = t;
                    }
                }
                u[0] = up;
                u[P - 1] = P == 2 ? uq : up;
                r.advance(NS);
            }
#pragma unroll
            for (int pc = 0; pc < P; ++pc) {
                const float2 vv = ld_pair<IOR>(tv, lane * C + 2 * pc);
                // w = beta (v - alpha u): three separate roundings
                const float d0 = __fsub_rn(vv.x, __fmul_rn(gscalar, u[pc].x));
                const float d1 = __fsub_rn(vv.y, __fmul_rn(gscalar, u[pc].y));
                w[pc] = make_float2(__fmul_rn(beta, d0), __fmul_rn(beta, d1));
            }
        } else {
#pragma unroll
            for (int pc = 0; pc < P; ++pc)
                w[pc] = ld_pair<IOR>(tv, lane * C + 2 * pc);
        }

        if (!ok) break;
        uint8_t* gcodes_tile = p.codes + ti.code_off;
        for (int g = 0; g < G; ++g) {
            if (UPD != kDelta && g > 0) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait_bounded(&bars[ic.slot], ic.par, p.timeout_ns));
                if (!ok) break;
            }
            const uint8_t* sm = wsm + hdr + ic.slot * S::kBytes;
            const float* ss = reinterpret_cast<const float*>(sm + S::kScales) + lane * C;
            const uint8_t* qs = INS ? sm + S::kQ : tq + g * GROUP * ESR;
            const uint8_t* ks = INS ? sm + S::kK : tk + g * GROUP * ESR;
            const float* gs = reinterpret_cast<const float*>(tin + in_g) + g * GROUP;
            float* gscale = p.scales + (static_cast<int64_t>(tile) * G + g) * DV + lane * C;
            uint8_t* gcodes = gcodes_tile + ti.goff(g, GROUP * DV / 2);
            const bool int8g = ti.bits(g) == 8;
            if constexpr (MODE == kSR) {
                // the group's row table of the element hash (the previous
                // group's readers finished at the warp barrier ending it)
                if (rowtab) {
                    for (int r = lane; r < GROUP; r += 32) {
                        const SrRow rr = sr_row(static_cast<uint32_t>(hkey >> 32),
                                                static_cast<uint32_t>(g * GROUP + r), hcarry);
                        rtab2[r] = make_uint2(rr.sh, rr.p);
                    }
                    __syncwarp();
                }
            }
            // The column pairs run one after the other through one copy of the
            // (large) pair code; the pairs' w and o rotate through (wp, op).
            float2 wp = w[0], op = o[0], wq = w[P - 1], oq = o[P - 1];
            constexpr bool EARLY = sr_early_release(MODE, UPD);
            bool released = false;   // the slot, after the last pair's first loop (EARLY)
#pragma unroll 1
            for (int pc = 0; pc < P; ++pc) {
                const float2 sc = *reinterpret_cast<const float2*>(ss + 2 * pc);
                const uint32_t j0 = static_cast<uint32_t>(lane * C + 2 * pc);
                if constexpr (kBoundsCheck) {
                    // this pair's units of the slot and of the state, and its scales
                    const int units = int8g ? PairGeo<GROUP, 8>::UNITS : PairGeo<GROUP, 4>::UNITS;
                    const int64_t end = (static_cast<int64_t>(pc) + 1) * units * 512;
                    if (!in_bounds(end <= S::kCodes &&
                                       (gcodes - p.codes) + end <= p.code_bytes &&
                                       (gscale - p.scales) + 2 * pc + 2 <= p.scale_count &&
                                       j0 + 2 <= static_cast<uint32_t>(DV),
                                   p.err)) {
                        if constexpr (P == 2) {
                            const float2 tw = wp, to = op;
                            wp = wq; op = oq; wq = tw; oq = to;
                        }
                        continue;
                    }
                }
                if constexpr (EARLY) {
                    // first loop; the slot's last reader done, the next copy
                    // is issued; then the rounding loop on the staged values
                    float2 snew, inv;
                    if (int8g)
                        pair_pass1_xs<GROUP, GATE, MODE, 8, IOR, true>(
                            sm, pc * PairGeo<GROUP, 8>::UNITS, sc, qs, ks, gs, gscalar, wp, op,
                            gscale + 2 * pc, lane, xs, snew, inv);
                    else
                        pair_pass1_xs<GROUP, GATE, MODE, 4, IOR, true>(
                            sm, pc * PairGeo<GROUP, 4>::UNITS, sc, qs, ks, gs, gscalar, wp, op,
                            gscale + 2 * pc, lane, xs, snew, inv);
                    if (pc == P - 1) {
                        release_slot();
                        released = true;
                    }
                    if (int8g)
                        pair_round_xs<GROUP, GATE, MODE, 8, IOR, true>(
                            sm, pc * PairGeo<GROUP, 8>::UNITS, sc, ks, gs, gscalar, wp, snew, inv,
                            gcodes, hkey, g * GROUP, j0, lane, xs, rtab, rowtab);
                    else
                        pair_round_xs<GROUP, GATE, MODE, 4, IOR, true>(
                            sm, pc * PairGeo<GROUP, 4>::UNITS, sc, ks, gs, gscalar, wp, snew, inv,
                            gcodes, hkey, g * GROUP, j0, lane, xs, rtab, rowtab);
                } else if constexpr (MODE != kRTN) {
                    constexpr bool ST = stage_x(MODE, UPD);
                    if (int8g)
                        pair_step_xs<GROUP, GATE, MODE, 8, IOR, ST>(sm, pc * PairGeo<GROUP, 8>::UNITS, sc,
                                                               qs, ks, gs, gscalar, wp, op, gcodes,
                                                               gscale + 2 * pc, hkey, g * GROUP, j0,
                                                               lane, xs, rtab, rowtab);
                    else
                        pair_step_xs<GROUP, GATE, MODE, 4, IOR, ST>(sm, pc * PairGeo<GROUP, 4>::UNITS, sc,
                                                               qs, ks, gs, gscalar, wp, op, gcodes,
                                                               gscale + 2 * pc, hkey, g * GROUP, j0,
                                                               lane, xs, rtab, rowtab);
                } else {
                    if (int8g)
                        pair_step<GROUP, GATE, MODE, 8, IOR>(sm, pc * PairGeo<GROUP, 8>::UNITS, sc, qs, ks,
                                                        gs, gscalar, wp, op, gcodes,
                                                        gscale + 2 * pc, hkey, g * GROUP, j0, lane);
                    else
                        pair_step<GROUP, GATE, MODE, 4, IOR>(sm, pc * PairGeo<GROUP, 4>::UNITS, sc, qs, ks,
                                                        gs, gscalar, wp, op, gcodes,
                                                        gscale + 2 * pc, hkey, g * GROUP, j0, lane);
                }
                if constexpr (P == 2) {
                    const float2 tw = wp, to = op;
                    wp = wq; op = oq; wq = tw; oq = to;
                }
            }
            o[0] = op;
            o[P - 1] = P == 2 ? oq : op;
            if (!released) release_slot();
        }
        if (!ok) break;
        const int64_t oi = static_cast<int64_t>(tile) * DV + lane * C;
        if (!in_bounds(oi + C <= static_cast<int64_t>(p.ntiles) * DV, p.err)) continue;
        if constexpr (IO == kIoF32) {
            float* op = static_cast<float*>(p.out) + oi;
            if constexpr (P == 2) {
                *reinterpret_cast<float4*>(op) = make_float4(o[0].x, o[0].y, o[1].x, o[1].y);
            } else {
                *reinterpret_cast<float2*>(op) = o[0];
            }
        } else {
            // nearest bfloat16, ties to even
            uint16_t* op = static_cast<uint16_t*>(p.out) + oi;
            const uint32_t w0 = bf16x2_rn(o[0]);
            if constexpr (P == 2) {
                *reinterpret_cast<uint2*>(op) = make_uint2(w0, bf16x2_rn(o[1]));
            } else {
                *reinterpret_cast<uint32_t*>(op) = w0;
            }
        }
    }
    if (!ok) {
        // Record the timeout, then wait (bounded) for this warp's copies
        // still in flight before leaving, so none lands after exit.
        if (lane == 0) atomicOr(p.err, kErrTimeout);
        Ring r = ic;
        for (int64_t k = kc; k < ki; ++k) {
            mbar_wait_bounded(&bars[r.slot], r.par, p.timeout_ns);
            r.advance(NS);
        }
    }
}

}  // namespace lrs
