// lrb_api.cu -- C ABI of the decode step with a Low-Rank Bypass buffer
// (lrs_lrb_step).
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <string>
#include <cstdint>
#include <mutex>
#include <vector>

#include "lrs.h"
#include "lrs_internal.h"
#include "lrb_kernel.cuh"
#include "lrb_stream.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lrs::ChunkKernel find_lrb(int d_k, int d_v, int group, int update_kind, int gate_kind, int mode) {
    switch (mode) {
        case LRS_ROUND_RTN: return lrs::find_lrb_kernel_rtn(d_k, d_v, group, update_kind, gate_kind);
        case LRS_ROUND_SR: return lrs::find_lrb_kernel_sr(d_k, d_v, group, update_kind, gate_kind);
        case LRS_ROUND_BDR: return lrs::find_lrb_kernel_bdr(d_k, d_v, group, update_kind, gate_kind);
        default: return {nullptr, 0};
    }
}

lrs_status lrb_ctas_per_sm(const lrs::ChunkKernel& k, int threads, int* per_sm) {
    struct Entry { const void* fn; int dev; int per_sm; };
    static std::mutex mu;
    static std::vector<Entry> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return lrs::api_cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(mu);
    for (const Entry& c : cache)
        if (c.fn == k.fn && c.dev == dev) {
            *per_sm = c.per_sm;
            return LRS_OK;
        }
    e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, k.fn, threads, k.smem);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return lrs::api_cuda_fail(e, "preparing the low-rank-bypass kernel");
    }
    if (*per_sm < 1) return lrs::api_fail(LRS_ERR_UNSUPPORTED, "kernel does not fit on an SM");
    cache.push_back({k.fn, dev, *per_sm});
    return LRS_OK;
}

const void* find_lrb_stream(int C, int group, int update_kind, int gate_kind, int mode,
                            bool merge) {
    switch (mode) {
        case LRS_ROUND_RTN: return lrs::find_lrb_stream_rtn(C, group, update_kind, gate_kind, merge);
        case LRS_ROUND_SR: return lrs::find_lrb_stream_sr(C, group, update_kind, gate_kind, merge);
        case LRS_ROUND_BDR: return lrs::find_lrb_stream_bdr(C, group, update_kind, gate_kind, merge);
        default: return nullptr;
    }
}

int lrb_stream_warp_smem(int C, int group, int gate_kind, int slots, int d_k, bool staged,
                         bool tab) {
#define LRS_LRB_SLOT(CC, GG)                                                                       \
    if (C == CC && group == GG)                                                                    \
        return gate_kind == lrs::kGatePerKey                                                       \
                   ? lrs::LrbSlot<CC, GG, lrs::kGatePerKey>::warp_bytes(slots, d_k, staged, tab)    \
                   : lrs::LrbSlot<CC, GG, lrs::kGate>::warp_bytes(slots, d_k, staged, tab);
    LRS_LRB_SLOT(4, 16)
    LRS_LRB_SLOT(4, 32)
    LRS_LRB_SLOT(2, 16)
    LRS_LRB_SLOT(2, 32)
    LRS_LRB_SLOT(2, 64)
#undef LRS_LRB_SLOT
    return -1;
}

// The streaming bypass step (ranks up to 4): the decode step's launch shape
// with the bypass kernel's shared memory. Returns LRS_ERR_UNSUPPORTED (and
// launches nothing) when no streaming kernel covers the shape.
lrs_status launch_lrb_stream(const lrs_state* st, void* state_codes, float* scales,
                             const uint8_t* prec_map, int32_t rank, float* U, float* V,
                             const float* q, const float* k, const float* v, const float* gates,
                             const float* beta, float* out, uint64_t seed, uint64_t step,
                             int32_t mode, unsigned* err, int sms, void* stream) {
    const lrs_shape& sh = st->shape;
    const int C = sh.d_v / 32, G = sh.d_k / sh.group;
    if (rank > lrs::kLrbStreamMaxRank) return LRS_ERR_UNSUPPORTED;
    const int m = static_cast<int>(step % static_cast<uint64_t>(rank));   // components filled
    const bool merge = m + 1 == rank;
    const void* fn = find_lrb_stream(C, sh.group, sh.update_kind, sh.gate_kind, mode, merge);
    if (!fn) return LRS_ERR_UNSUPPORTED;
    int slots = sh.update_kind == LRS_UPDATE_DELTA ? G : std::min(2, G);
    slots = std::max(1, std::min(slots, lrs::kMaxSlots));
    const int warp_smem =
        lrb_stream_warp_smem(C, sh.group, sh.gate_kind, slots, sh.d_k, lrs::lrb_staged(mode, merge),
                             mode == LRS_ROUND_SR);
    constexpr int kSmemLimit = 227 * 1024;
    const int warps = std::min(lrs::lrb_max_warps(mode, merge, sh.group), kSmemLimit / warp_smem);
    if (warps < 1) return LRS_ERR_UNSUPPORTED;
    const int smem = warps * warp_smem;
    static std::mutex mu;
    struct Entry { const void* fn; int dev; int smem; int per_sm; };
    static std::vector<Entry> cache;
    int dev = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return lrs::api_cuda_fail(e, "cudaGetDevice");
    {
        std::lock_guard<std::mutex> lk(mu);
        for (const Entry& c : cache)
            if (c.fn == fn && c.dev == dev && c.smem == smem) per_sm = c.per_sm;
        if (per_sm == 0) {
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, warps * 32, smem);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return lrs::api_cuda_fail(e, "preparing the streaming bypass kernel");
            }
            if (per_sm < 1) return LRS_ERR_UNSUPPORTED;
            cache.push_back({fn, dev, smem, per_sm});
        }
    }
    const int ntiles = sh.batch * sh.heads;
    const int grid = std::min(sms * per_sm, (ntiles + warps - 1) / warps);
    lrs::LrbStreamParams lp;
    memset(&lp, 0, sizeof lp);
    lrs::StepParams& p = lp.s;
    p.codes = static_cast<uint8_t*>(state_codes);
    p.scales = scales;
    p.prec_map = prec_map;
    p.head_offsets = st->head_offsets;
    p.batch_stride = st->batch_stride_bytes;
    p.q = q;
    p.k = k;
    p.v = v;
    p.gates = gates;
    p.beta = beta;
    p.out = out;
    p.seed = seed;
    p.step = step;
    p.err = err;
    p.timeout_ns = 2000000000ull;
    p.H = sh.heads;
    p.d_k = sh.d_k;
    p.G = G;
    p.ntiles = ntiles;
    p.pgroups = lrs::state_prec_groups(st);
    p.warp_smem = warp_smem;
    p.slots = slots;
    p.inject = lrs::take_injected_timeout(&p.timeout_ns) ? 1 : 0;
    p.code_bytes = st->code_bytes;
    p.scale_count = st->scale_count;
    lp.U = U;
    lp.V = V;
    lp.rank = rank;
    lp.m = m;
    void* args[] = {&lp};
    e = cudaLaunchKernel(fn, dim3(grid), dim3(warps * 32), args, smem,
                         static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return lrs::api_cuda_fail(e, "launch of the streaming bypass kernel");
    }
    return lrs::api_ok();
}

}  // namespace

extern "C" {

lrs_status lrs_lrb_step(const lrs_state* st, void* state_codes, float* scales,
                        const uint8_t* prec_map, int32_t rank, float* U, float* V, const float* q,
                        const float* k, const float* v, const float* gates, const float* beta,
                        float* out, uint64_t seed, uint64_t step, int32_t mode, void* stream) {
    lrs_status s = lrs::api_check_state(st);
    if (s != LRS_OK) return s;
    const lrs_shape& sh = st->shape;
    if (rank < 1 || rank > lrs::kLrbMaxRank)
        return lrs::api_fail(LRS_ERR_INVALID_ARG, "rank must be in [1, 8]");
    if (mode != LRS_ROUND_RTN && mode != LRS_ROUND_SR && mode != LRS_ROUND_BDR)
        return lrs::api_fail(LRS_ERR_INVALID_ARG, "mode is not an lrs_round_mode");
    const void* ptrs[] = {state_codes, scales, U, V, q, k, v, gates, out};
    for (const void* p : ptrs) {
        if (!p) return lrs::api_fail(LRS_ERR_INVALID_ARG, "a buffer is NULL");
        if (!aligned16(p)) return lrs::api_fail(LRS_ERR_ALIGNMENT, "a buffer is not 16-byte aligned");
    }
    if (!prec_map) return lrs::api_fail(LRS_ERR_INVALID_ARG, "prec_map is NULL");
    if (sh.update_kind == LRS_UPDATE_DELTA && !beta)
        return lrs::api_fail(LRS_ERR_INVALID_ARG, "beta is NULL");
    const int64_t ntiles0 = static_cast<int64_t>(sh.batch) * sh.heads;
    if (ntiles0 == 0) return lrs::api_ok();
    if (rank <= lrs::kLrbStreamMaxRank) {
        unsigned* err = nullptr;
        int sms = 0;
        s = lrs::device_error_word(&err, &sms);
        if (s != LRS_OK) return s;
        s = launch_lrb_stream(st, state_codes, scales, prec_map, rank, U, V, q, k, v, gates, beta,
                              out, seed, step, mode, err, sms, stream);
        if (s != LRS_ERR_UNSUPPORTED) return s;
    }
    const lrs::ChunkKernel kern =
        find_lrb(sh.d_k, sh.d_v, sh.group, sh.update_kind, sh.gate_kind, mode);
    if (!kern.fn)
        return lrs::api_fail(LRS_ERR_UNSUPPORTED,
                             "no compiled bypass kernel for this shape (d_k, d_v in {64, 128})");
    const int64_t ntiles = static_cast<int64_t>(sh.batch) * sh.heads;
    if (ntiles == 0) return lrs::api_ok();
    unsigned* err = nullptr;
    int sms = 0;
    s = lrs::device_error_word(&err, &sms);
    if (s != LRS_OK) return s;
    int per_sm = 0;
    s = lrb_ctas_per_sm(kern, sh.d_v, &per_sm);
    if (s != LRS_OK) return s;

    lrs::LrbParams p;
    p.codes = static_cast<uint8_t*>(state_codes);
    p.scales = scales;
    p.prec_map = prec_map;
    p.head_offsets = st->head_offsets;
    p.batch_stride = st->batch_stride_bytes;
    p.U = U;
    p.V = V;
    p.q = q;
    p.k = k;
    p.v = v;
    p.gates = gates;
    p.beta = beta;
    p.out = out;
    p.seed = seed;
    p.step = step;
    p.err = err;
    p.timeout_ns = 2000000000ull;   // 2 s: far above any legitimate wait
    p.H = sh.heads;
    p.ntiles = static_cast<int32_t>(ntiles);
    p.rank = rank;
    p.pgroups = lrs::state_prec_groups(st);
    p.inject = lrs::take_injected_timeout(&p.timeout_ns) ? 1 : 0;
    const int grid = static_cast<int>(std::min<int64_t>(ntiles, int64_t(sms) * per_sm));
    void* args[] = {&p};
    cudaError_t e = cudaLaunchKernel(kern.fn, dim3(grid), dim3(sh.d_v), args, kern.smem,
                                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return lrs::api_cuda_fail(e, "launch of the low-rank-bypass kernel");
    }
    return lrs::api_ok();
}

}  // extern "C"
