// aux_kernels.cu -- the state's set-up and inspection kernels, the fp32-state
// decode step used as the uncompressed baseline, and the per-head mean decay.
//
// The quantizing kernels here share the step kernel's rounding and packing
// (round_rows / encode_word), so an imported state is exactly the state a step
// with x = S would produce.
#include "lrs_internal.h"
#include "step_kernel.cuh"

namespace lrs {

namespace {

constexpr int kAuxWarps = 8;

// Byte offset, inside a group block, of the 16-byte unit `u` of lane `lane`.
__device__ __forceinline__ int unit_offset(int u, int lane) { return (u * 32 + lane) * 16; }

// Layout of tile `tile` (b = tile / H, h = tile % H).
__device__ __forceinline__ TileLayout tile_layout(const LayoutArgs& a, int tile) {
    TileLayout t;
    t.load(a.prec_map, a.head_offsets, a.batch_stride, a.H, a.pgroups, a.d_k / a.group,
           a.group * a.d_v, tile / a.H, tile % a.H);
    return t;
}

// Round x * inv (inv = 1 for given integer codes) to nearest for one column
// pair of one group and store the pair's units (same rounding and packing as
// the step kernel).
template <int GROUP, int BITS>
__device__ void encode_pair_rtn(const float2 (&x)[GROUP], float2 inv, uint8_t* gcodes, int pc,
                                int lane) {
    using G = PairGeo<GROUP, BITS>;
#pragma unroll
    for (int un = 0; un < G::UNITS; ++un) {
        uint32_t ow[4];
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float t[G::EPW];
#pragma unroll
            for (int e = 0; e < G::EPW; e += 2) {
                const int r = un * G::RPU + (wi * G::EPW + e) / 2;
                const float2 kb = make_float2(word_bias<BITS>(e), word_bias<BITS>(e + 1));
                const float2 tv = round_rows<kRTN, BITS>(x[r], inv, f2(0.f), f2(0.f), kb, 0ull, 0u, 0u);
                t[e] = tv.x;
                t[e + 1] = tv.y;
            }
            ow[wi] = encode_word<BITS>(t);
        }
        *reinterpret_cast<uint4*>(gcodes + unit_offset(pc * G::UNITS + un, lane)) =
            make_uint4(ow[0], ow[1], ow[2], ow[3]);
    }
}

// Signed codes of one column pair of one group block.
template <int GROUP, int BITS>
__device__ void decode_pair(const uint8_t* gcodes, int pc, int lane, float2 (&code)[GROUP]) {
    using G = PairGeo<GROUP, BITS>;
    constexpr float BIAS = Q<BITS>::kBias;
#pragma unroll
    for (int un = 0; un < G::UNITS; ++un) {
        const uint4 raw =
            *reinterpret_cast<const uint4*>(gcodes + unit_offset(pc * G::UNITS + un, lane));
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            float f[G::EPW];
            decode_word_biased<BITS>(wd[wi], f);
#pragma unroll
            for (int e = 0; e < G::EPW; e += 2)
                code[un * G::RPU + (wi * G::EPW + e) / 2] =
                    make_float2(__fsub_rn(f[e], kTwo23 + BIAS), __fsub_rn(f[e + 1], kTwo23 + BIAS));
        }
    }
}

enum { kOpFillZero, kOpImportFp32, kOpExportFp32, kOpExportCodes, kOpImportCodes };

// One scale group g of one tile, codes of width BITS at gcodes.
template <int C, int GROUP, int BITS>
__device__ void layout_op_group(const LayoutArgs& a, int op, int tile, int g, uint8_t* gcodes,
                                const float* S, float* So, int8_t* Co, const int8_t* Ci,
                                const float* Si, int lane) {
    constexpr int DV = 32 * C;
    constexpr int P = C / 2;
    constexpr int QMAX = BITS == 8 ? 127 : 7;
    const int G = a.d_k / GROUP;
    const int64_t tile_elems = static_cast<int64_t>(a.d_k) * DV;
    {
        float* gscales = a.scales + (static_cast<int64_t>(tile) * G + g) * DV;
        for (int pc = 0; pc < P; ++pc) {
            const int j = lane * C + 2 * pc;
            const int64_t base = tile * tile_elems + static_cast<int64_t>(g) * GROUP * DV + j;
            float2 x[GROUP];
            if (op == kOpImportFp32) {
                float A0 = 0.0f, A1 = 0.0f;
#pragma unroll
                for (int r = 0; r < GROUP; ++r) {
                    x[r] = make_float2(S[base + r * DV], S[base + r * DV + 1]);
                    A0 = fmaxf(A0, fabsf(x[r].x));
                    A1 = fmaxf(A1, fabsf(x[r].y));
                }
                constexpr float QF = static_cast<float>(QMAX);
                const float2 snew = make_float2(A0 < kTiny ? 0.0f : div_by_qmax<QMAX>(A0),
                                                A1 < kTiny ? 0.0f : div_by_qmax<QMAX>(A1));
                const float2 inv = make_float2(A0 < kTiny ? 0.0f : div_rn_fast(QF, A0),
                                               A1 < kTiny ? 0.0f : div_rn_fast(QF, A1));
                gscales[j] = snew.x;
                gscales[j + 1] = snew.y;
                encode_pair_rtn<GROUP, BITS>(x, inv, gcodes, pc, lane);
            } else if (op == kOpFillZero || op == kOpImportCodes) {
                // zero state, or given codes: the codes are written as they are
                // (clamped), the scales copied.
#pragma unroll
                for (int r = 0; r < GROUP; ++r) {
                    float cv[2] = {0.0f, 0.0f};
                    if (op == kOpImportCodes) {
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            int ci = Ci[base + r * DV + c];
                            if (ci > QMAX || ci < -QMAX) {
                                atomicOr(a.err, kErrRange);
                                ci = ci > QMAX ? QMAX : -QMAX;
                            }
                            cv[c] = static_cast<float>(ci);
                        }
                    }
                    x[r] = make_float2(cv[0], cv[1]);
                }
                encode_pair_rtn<GROUP, BITS>(x, f2(1.0f), gcodes, pc, lane);
                const int64_t si = (static_cast<int64_t>(tile) * G + g) * DV + j;
                gscales[j] = op == kOpImportCodes ? Si[si] : 0.0f;
                gscales[j + 1] = op == kOpImportCodes ? Si[si + 1] : 0.0f;
            } else {
                decode_pair<GROUP, BITS>(gcodes, pc, lane, x);
#pragma unroll
                for (int r = 0; r < GROUP; ++r) {
                    if (op == kOpExportFp32) {
                        So[base + r * DV] = __fmul_rn(x[r].x, gscales[j]);
                        So[base + r * DV + 1] = __fmul_rn(x[r].y, gscales[j + 1]);
                    } else {
                        Co[base + r * DV] = static_cast<int8_t>(static_cast<int>(x[r].x));
                        Co[base + r * DV + 1] = static_cast<int8_t>(static_cast<int>(x[r].y));
                    }
                }
            }
        }
    }
}

template <int C, int GROUP>
__device__ void layout_op_tile(const LayoutArgs& a, int op, int tile, const TileLayout& tl,
                               const float* S, float* So, int8_t* Co, const int8_t* Ci,
                               const float* Si, int lane) {
    constexpr int DV = 32 * C;
    for (int g = 0; g < a.d_k / GROUP; ++g) {
        uint8_t* gcodes = a.codes + tl.code_off + tl.goff(g, GROUP * DV / 2);
        if (tl.bits(g) == 8)
            layout_op_group<C, GROUP, 8>(a, op, tile, g, gcodes, S, So, Co, Ci, Si, lane);
        else
            layout_op_group<C, GROUP, 4>(a, op, tile, g, gcodes, S, So, Co, Ci, Si, lane);
    }
}

template <int C, int GROUP>
__global__ void __launch_bounds__(kAuxWarps * 32) layout_kernel(const LayoutArgs a, int op,
                                                                 const float* S, float* So,
                                                                 int8_t* Co, const int8_t* Ci,
                                                                 const float* Si) {
    const int lane = threadIdx.x & 31;
    const int ntiles = a.B * a.H;
    for (int tile = blockIdx.x * kAuxWarps + (threadIdx.x >> 5); tile < ntiles;
         tile += gridDim.x * kAuxWarps) {
        const TileLayout t = tile_layout(a, tile);
        if (!t.ok) {
            if (lane == 0) atomicOr(a.err, kErrLayout);
            continue;
        }
        layout_op_tile<C, GROUP>(a, op, tile, t, S, So, Co, Ci, Si, lane);
    }
}

cudaError_t launch_layout(const LayoutArgs& a, int op, const float* S, float* So, int8_t* Co,
                          const int8_t* Ci, const float* Si, cudaStream_t s) {
    const int ntiles = a.B * a.H;
    if (ntiles == 0) return cudaSuccess;
    const int grid = (ntiles + kAuxWarps - 1) / kAuxWarps;
    const int C = a.d_v / 32;
#define LRS_LAYOUT_CASE(CC, GG)                                                              \
    if (C == CC && a.group == GG) {                                                          \
        layout_kernel<CC, GG><<<grid, kAuxWarps * 32, 0, s>>>(a, op, S, So, Co, Ci, Si);     \
        return cudaGetLastError();                                                           \
    }
    LRS_LAYOUT_CASE(4, 16)
    LRS_LAYOUT_CASE(4, 32)
    LRS_LAYOUT_CASE(2, 16)
    LRS_LAYOUT_CASE(2, 32)
    LRS_LAYOUT_CASE(2, 64)
#undef LRS_LAYOUT_CASE
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------------ fp32 step ---

// One warp per tile, lane t owns columns [t*C, t*C + C) of every row, rows in
// key order: the same arithmetic, in the same order, as the quantized step
// with deq replaced by the fp32 state.
template <int C, int UPD, int GATE>
__global__ void __launch_bounds__(kAuxWarps * 32) fp32_step_kernel(
    int ntiles, int d_k, float* S, const float* q, const float* k, const float* v,
    const float* gates, const float* beta, float* out) {
    constexpr int DV = 32 * C;
    constexpr int UNR = 8;
    const int lane = threadIdx.x & 31;
    for (int tile = blockIdx.x * kAuxWarps + (threadIdx.x >> 5); tile < ntiles;
         tile += gridDim.x * kAuxWarps) {
        float* St = S + static_cast<int64_t>(tile) * d_k * DV + lane * C;
        const float* qt = q + static_cast<int64_t>(tile) * d_k;
        const float* kt = k + static_cast<int64_t>(tile) * d_k;
        const float* gt = gates + (GATE == kGatePerKey ? static_cast<int64_t>(tile) * d_k : tile);
        float w[C], o[C];
        const float alpha = GATE == kGate ? __ldg(gt) : 0.0f;
        if (UPD == kDelta) {
            float u[C];
#pragma unroll
            for (int c = 0; c < C; ++c) u[c] = 0.0f;
            for (int i0 = 0; i0 < d_k; i0 += UNR) {
                float s[UNR][C];
#pragma unroll
                for (int r = 0; r < UNR; ++r) {
                    const float* row = St + static_cast<int64_t>(i0 + r) * DV;
                    if constexpr (C == 4) {
                        const float4 t = *reinterpret_cast<const float4*>(row);
                        s[r][0] = t.x; s[r][1] = t.y; s[r][2] = t.z; s[r][3] = t.w;
                    } else {
                        const float2 t = *reinterpret_cast<const float2*>(row);
                        s[r][0] = t.x; s[r][1] = t.y;
                    }
                }
#pragma unroll
                for (int r = 0; r < UNR; ++r) {
                    const float ki = __ldg(kt + i0 + r);
#pragma unroll
                    for (int c = 0; c < C; ++c) u[c] = __fmaf_rn(ki, s[r][c], u[c]);
                }
            }
            const float b = __ldg(beta + tile);
#pragma unroll
            for (int c = 0; c < C; ++c) {
                const float t = __fmul_rn(alpha, u[c]);
                const float d = __fsub_rn(__ldg(v + static_cast<int64_t>(tile) * DV + lane * C + c), t);
                w[c] = __fmul_rn(b, d);
            }
        } else {
#pragma unroll
            for (int c = 0; c < C; ++c) w[c] = __ldg(v + static_cast<int64_t>(tile) * DV + lane * C + c);
        }
#pragma unroll
        for (int c = 0; c < C; ++c) o[c] = 0.0f;
        for (int i0 = 0; i0 < d_k; i0 += UNR) {
            float s[UNR][C];
#pragma unroll
            for (int r = 0; r < UNR; ++r) {
                const float* row = St + static_cast<int64_t>(i0 + r) * DV;
                if constexpr (C == 4) {
                    const float4 t = __ldcs(reinterpret_cast<const float4*>(row));
                    s[r][0] = t.x; s[r][1] = t.y; s[r][2] = t.z; s[r][3] = t.w;
                } else {
                    const float2 t = __ldcs(reinterpret_cast<const float2*>(row));
                    s[r][0] = t.x; s[r][1] = t.y;
                }
            }
#pragma unroll
            for (int r = 0; r < UNR; ++r) {
                const int i = i0 + r;
                const float gi = GATE == kGatePerKey ? __ldg(gt + i) : alpha;
                const float ki = __ldg(kt + i), qi = __ldg(qt + i);
                float x[C];
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    x[c] = __fmaf_rn(gi, s[r][c], __fmul_rn(ki, w[c]));
                    o[c] = __fmaf_rn(qi, x[c], o[c]);
                }
                float* row = St + static_cast<int64_t>(i) * DV;
                if constexpr (C == 4)
                    __stcs(reinterpret_cast<float4*>(row), make_float4(x[0], x[1], x[2], x[3]));
                else
                    __stcs(reinterpret_cast<float2*>(row), make_float2(x[0], x[1]));
            }
        }
        float* op = out + static_cast<int64_t>(tile) * DV + lane * C;
#pragma unroll
        for (int c = 0; c < C; ++c) op[c] = o[c];
    }
}

// ----------------------------------------------------------- decay mean ---

// One block per head; a fixed assignment of elements to threads and a fixed
// reduction tree make the binary64 sum deterministic.
__global__ void decay_mean_kernel(const float* decay, int64_t outer, int heads, int64_t inner,
                                  double* means) {
    __shared__ double part[256];
    const int h = blockIdx.x;
    const int64_t n = outer * inner;
    double acc = 0.0;
    for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
        const int64_t o = e / inner, c = e % inner;
        acc += static_cast<double>(decay[(o * heads + h) * inner + c]);
    }
    part[threadIdx.x] = acc;
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if (threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) means[h] = part[0] / static_cast<double>(n);
}

}  // namespace

bool layout_kernels_support(int d_v, int group) {
    const int C = d_v / 32;
    return (C == 4 && (group == 16 || group == 32)) ||
           (C == 2 && (group == 16 || group == 32 || group == 64));
}

cudaError_t launch_fill_zero(const LayoutArgs& a, cudaStream_t s) {
    return launch_layout(a, kOpFillZero, nullptr, nullptr, nullptr, nullptr, nullptr, s);
}
cudaError_t launch_import_fp32(const LayoutArgs& a, const float* S, cudaStream_t s) {
    return launch_layout(a, kOpImportFp32, S, nullptr, nullptr, nullptr, nullptr, s);
}
cudaError_t launch_export_fp32(const LayoutArgs& a, float* S, cudaStream_t s) {
    return launch_layout(a, kOpExportFp32, nullptr, S, nullptr, nullptr, nullptr, s);
}
cudaError_t launch_export_codes(const LayoutArgs& a, int8_t* codes, cudaStream_t s) {
    return launch_layout(a, kOpExportCodes, nullptr, nullptr, codes, nullptr, nullptr, s);
}
cudaError_t launch_import_codes(const LayoutArgs& a, const int8_t* codes, const float* scales,
                                cudaStream_t s) {
    return launch_layout(a, kOpImportCodes, nullptr, nullptr, nullptr, codes, scales, s);
}

cudaError_t launch_fp32_step(int B, int H, int d_k, int d_v, int update_kind, int gate_kind,
                             float* S, const float* q, const float* k, const float* v,
                             const float* gates, const float* beta, float* out, cudaStream_t s) {
    const int ntiles = B * H;
    if (ntiles == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int grid = (ntiles + kAuxWarps - 1) / kAuxWarps;
    grid = grid < sms * 8 ? grid : sms * 8;
    const int C = d_v / 32;
#define LRS_FP32_CASE(CC, UU, GG)                                                           \
    if (C == CC && update_kind == UU && gate_kind == GG) {                                  \
        fp32_step_kernel<CC, UU, GG><<<grid, kAuxWarps * 32, 0, s>>>(ntiles, d_k, S, q, k, v, \
                                                                    gates, beta, out);      \
        return cudaGetLastError();                                                          \
    }
    LRS_FP32_CASE(4, kGated, kGatePerKey)
    LRS_FP32_CASE(4, kGated, kGate)
    LRS_FP32_CASE(4, kDelta, kGate)
    LRS_FP32_CASE(2, kGated, kGatePerKey)
    LRS_FP32_CASE(2, kGated, kGate)
    LRS_FP32_CASE(2, kDelta, kGate)
#undef LRS_FP32_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decay_means(const float* decay, int64_t outer, int heads, int64_t inner,
                               double* means, cudaStream_t s) {
    if (heads == 0) return cudaSuccess;
    decay_mean_kernel<<<heads, 256, 0, s>>>(decay, outer, heads, inner, means);
    return cudaGetLastError();
}

}  // namespace lrs
