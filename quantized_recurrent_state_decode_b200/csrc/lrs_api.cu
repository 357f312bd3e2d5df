// lrs_api.cu -- the C ABI of liblrs (declared in include/lrs.h): argument
// validation, the state's layout and memory, kernel selection and launch.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "lrs.h"
#include "lrs_internal.h"
#include "step_kernel.cuh"

namespace {

thread_local std::string g_last_error;

lrs_status fail(lrs_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = std::string(lrs_status_string(s)) + ": " + buf;
    return s;
}

lrs_status ok() {
    g_last_error.clear();
    return LRS_OK;
}

lrs_status cuda_fail(cudaError_t e, const char* what) {
    return fail(e == cudaErrorMemoryAllocation ? LRS_ERR_OOM : LRS_ERR_CUDA, "%s: %s", what,
                cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------- per-device context ---

constexpr int kMaxDevices = 64;

struct DeviceCtx {
    unsigned* err = nullptr;  // device error word
    int sms = 0;
};

std::mutex g_ctx_mu;
DeviceCtx g_ctx[kMaxDevices];

lrs_status device_ctx(DeviceCtx** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(LRS_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_ctx_mu);
    DeviceCtx& c = g_ctx[dev];
    if (!c.err) {
        e = cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        unsigned* p = nullptr;
        e = cudaMalloc(&p, 256);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(error word)");
        e = cudaMemset(p, 0, 256);
        if (e != cudaSuccess) {
            cudaFree(p);
            return cuda_fail(e, "cudaMemset(error word)");
        }
        c.err = p;
    }
    *out = &c;
    return LRS_OK;
}

// Fault injection (tests of the error path only): the next step launch
// issues copies for only its first g_inject_items items per warp (0: none)
// and gives its waits g_inject_timeout_ns.
std::mutex g_inject_mu;
bool g_inject = false;
int32_t g_inject_items = 0;
uint64_t g_inject_timeout_ns = 0;

constexpr int kDefaultWarps = 12;
constexpr int kDefaultSlots = 2;
constexpr int kSmemLimit = 227 * 1024;

struct StatePriv {
    int device = -1;
    int pgroups = 1;    // widths per head (1) or per (head, scale group) (G)
    std::vector<uint8_t> prec_host;
    std::vector<int64_t> offsets_host;
    // lrs_decode_step_host (set up on first use): two staging buffers used by
    // alternate calls, a stream for their input copies, and per buffer the
    // events "inputs copied" and "buffer free again" (after the output copy)
    float* stage[2] = {nullptr, nullptr};
    size_t stage_floats = 0;
    cudaStream_t copy_stream = nullptr;
    cudaEvent_t h2d_done[2] = {nullptr, nullptr};
    cudaEvent_t free_again[2] = {nullptr, nullptr};
    uint64_t host_calls = 0;
};

// ------------------------------------------------------------- layout ---

lrs_status check_shape(const lrs_shape* s) {
    if (!s) return fail(LRS_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 0 || s->heads < 1 || s->d_k < 1 || s->d_v < 1 || s->group < 1)
        return fail(LRS_ERR_INVALID_ARG, "non-positive dimension (B=%d H=%d d_k=%d d_v=%d group=%d)",
                    s->batch, s->heads, s->d_k, s->d_v, s->group);
    if (s->update_kind != LRS_UPDATE_GATED && s->update_kind != LRS_UPDATE_DELTA)
        return fail(LRS_ERR_INVALID_ARG, "update_kind %d", s->update_kind);
    if (s->gate_kind != LRS_GATE_SCALAR && s->gate_kind != LRS_GATE_PER_KEY)
        return fail(LRS_ERR_INVALID_ARG, "gate_kind %d", s->gate_kind);
    if (s->update_kind == LRS_UPDATE_DELTA && s->gate_kind != LRS_GATE_SCALAR)
        return fail(LRS_ERR_UNSUPPORTED, "the delta rule takes a scalar decay");
    if (s->d_v != 64 && s->d_v != 128)
        return fail(LRS_ERR_UNSUPPORTED, "d_v=%d (supported: 64, 128)", s->d_v);
    if (s->group != 16 && s->group != 32 && s->group != 64)
        return fail(LRS_ERR_UNSUPPORTED, "group=%d (supported: 16, 32, 64)", s->group);
    if (s->group * s->d_v > 4096)
        return fail(LRS_ERR_UNSUPPORTED, "group*d_v=%d exceeds 4096", s->group * s->d_v);
    if (s->d_k % s->group != 0 || s->d_k < 16 || s->d_k > 256)
        return fail(LRS_ERR_UNSUPPORTED, "d_k=%d (a multiple of group=%d in [16, 256])", s->d_k,
                    s->group);
    if (static_cast<int64_t>(s->batch) * s->heads > INT32_MAX / 2)
        return fail(LRS_ERR_UNSUPPORTED, "batch*heads too large");
    return LRS_OK;
}

// Head offsets within a batch row for widths per head (pgroups == 1,
// prec [H]) or per (head, scale group) (pgroups == G, prec [H][G]).
lrs_status compute_layout(const lrs_shape* s, const uint8_t* prec, int pgroups, int64_t* offsets,
                          int64_t* stride, int64_t* scale_count) {
    lrs_status st = check_shape(s);
    if (st != LRS_OK) return st;
    if (!prec) return fail(LRS_ERR_INVALID_ARG, "prec_map is NULL");
    const int G = s->d_k / s->group;
    if (pgroups != 1 && pgroups != G)
        return fail(LRS_ERR_INVALID_ARG, "widths per head or per scale group only");
    int64_t off = 0;
    for (int h = 0; h < s->heads; ++h) {
        if (offsets) offsets[h] = off;
        for (int g = 0; g < G; ++g) {
            const int w = pgroups == 1 ? prec[h] : prec[static_cast<int64_t>(h) * G + g];
            if (w != 4 && w != 8)
                return fail(LRS_ERR_INVALID_ARG, "prec_map width %d at head %d group %d "
                            "(must be 4 or 8)", w, h, g);
            off += static_cast<int64_t>(s->group) * s->d_v * w / 8;
        }
    }
    if (stride) *stride = off;
    if (scale_count)
        *scale_count = static_cast<int64_t>(s->batch) * s->heads * (s->d_k / s->group) * s->d_v;
    return LRS_OK;
}

lrs_status check_state(const lrs_state* st) {
    if (!st || !st->priv) return fail(LRS_ERR_INVALID_ARG, "state is NULL or not allocated");
    const StatePriv* pv = static_cast<const StatePriv*>(st->priv);
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != pv->device)
        return fail(LRS_ERR_INVALID_ARG, "state lives on device %d, current device is %d",
                    pv->device, dev);
    return check_shape(&st->shape);
}

lrs::LayoutArgs layout_args(const lrs_state* st, unsigned* err) {
    lrs::LayoutArgs a;
    a.codes = static_cast<uint8_t*>(st->state_codes);
    a.scales = st->scales;
    a.prec_map = st->prec_map;
    a.head_offsets = st->head_offsets;
    a.batch_stride = st->batch_stride_bytes;
    a.B = st->shape.batch;
    a.H = st->shape.heads;
    a.d_k = st->shape.d_k;
    a.d_v = st->shape.d_v;
    a.group = st->shape.group;
    a.pgroups = static_cast<const StatePriv*>(st->priv)->pgroups;
    a.err = err;
    return a;
}

#define LRS_REQUIRE_PTR(p)                                                          \
    do {                                                                            \
        if (!(p)) return fail(LRS_ERR_INVALID_ARG, "%s is NULL", #p);               \
        if (!aligned16(p)) return fail(LRS_ERR_ALIGNMENT, "%s is not 16-byte aligned", #p); \
    } while (0)

}  // namespace

namespace lrs {

const void* find_step_kernel(int C, int group, int update_kind, int gate_kind, int mode, int io) {
    if (io == kStepIoBF16) {
        switch (mode) {
            case kRTN: return find_step_kernel_rtn_bf16(C, group, update_kind, gate_kind);
            case kSR: return find_step_kernel_sr_bf16(C, group, update_kind, gate_kind);
            case kBDR: return find_step_kernel_bdr_bf16(C, group, update_kind, gate_kind);
            default: return nullptr;
        }
    }
    if (io != kStepIoF32) return nullptr;
    switch (mode) {
        case kRTN: return find_step_kernel_rtn(C, group, update_kind, gate_kind);
        case kSR: return find_step_kernel_sr(C, group, update_kind, gate_kind);
        case kBDR: return find_step_kernel_bdr(C, group, update_kind, gate_kind);
        default: return nullptr;
    }
}

int step_warp_smem(int C, int group, int update_kind, int gate_kind, int slots, int mode, int io,
                   int d_k) {
    const bool xs = stage_x(mode, update_kind), tab = mode == kSR;
#define LRS_SLOT_IO(CC, GG, IO)                                                                   \
    if (update_kind == kDelta)                                                                  \
        return Slot<CC, GG, kGate, IO, true>::warp_bytes(slots, xs, tab, d_k);                  \
    return gate_kind == kGatePerKey                                                             \
               ? Slot<CC, GG, kGatePerKey, IO>::warp_bytes(slots, xs, tab, d_k)                 \
               : Slot<CC, GG, kGate, IO>::warp_bytes(slots, xs, tab, d_k);
#define LRS_SLOT(CC, GG)                                                                     \
    if (C == CC && group == GG) {                                                            \
        if (io == kStepIoBF16) {                                                             \
            LRS_SLOT_IO(CC, GG, kIoBF16)                                                     \
        }                                                                                    \
        LRS_SLOT_IO(CC, GG, kIoF32)                                                          \
    }
    LRS_SLOT(4, 16)
    LRS_SLOT(4, 32)
    LRS_SLOT(2, 16)
    LRS_SLOT(2, 32)
    LRS_SLOT(2, 64)
#undef LRS_SLOT
#undef LRS_SLOT_IO
    return -1;
}

// One launch shape per (kernel, device), prepared on its first use: the
// dynamic shared-memory limit raised once (the attribute belongs to the
// function and is never lowered again) and the CTAs that fit on an SM.
lrs_status step_launch_shape(const lrs_shape& sh, int mode, int io, int device, int sms,
                             StepLaunch* out) {
    const int C = sh.d_v / 32, G = sh.d_k / sh.group;
    const void* fn = find_step_kernel(C, sh.group, sh.update_kind, sh.gate_kind, mode, io);
    if (!fn) return fail(LRS_ERR_UNSUPPORTED, "no compiled kernel for this shape and mode");
    // ring slots per warp: the delta rule keeps a whole tile resident; the
    // gated forms stream a few groups ahead (at most G, so that the single v
    // buffer is never overwritten before it is read); gated SR streams one
    // group ahead through a single slot released early (sr_early_release)
    int slots = sh.update_kind == LRS_UPDATE_DELTA
                    ? G
                    : std::min(sr_early_release(mode, sh.update_kind) ? 1 : kDefaultSlots, G);
    slots = std::max(1, std::min(slots, kMaxSlots));
    const int warp_smem = step_warp_smem(C, sh.group, sh.update_kind, sh.gate_kind, slots, mode,
                                         io, sh.d_k);
    if (warp_smem <= 0) return fail(LRS_ERR_UNSUPPORTED, "no shared-memory layout for this shape");
    int warps = std::min(kDefaultWarps, std::max(1, kSmemLimit / warp_smem));
    warps = std::min(warps, step_max_warps(sh.group, mode, sh.update_kind));
    const int smem = warps * warp_smem;

    struct Prepared { const void* fn; int dev; int smem; int per_sm; };
    static std::mutex mu;
    static std::vector<Prepared> prepared;
    int per_sm = 0;
    std::lock_guard<std::mutex> lk(mu);
    bool attr = false;
    for (const Prepared& c : prepared) {
        if (c.fn != fn || c.dev != device) continue;
        attr = true;
        if (c.smem == smem) per_sm = c.per_sm;
    }
    if (per_sm == 0) {
        cudaError_t e = cudaSuccess;
        if (!attr)
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e, "cudaFuncSetAttribute");
        }
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, warps * 32, smem);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
        }
        if (per_sm < 1) return fail(LRS_ERR_UNSUPPORTED, "step kernel does not fit on an SM");
        prepared.push_back({fn, device, smem, per_sm});
    }
    *out = {fn, slots, warps, warp_smem, smem, sms * per_sm};
    return LRS_OK;
}

}  // namespace lrs

extern "C" {

const char* lrs_status_string(lrs_status s) {
    switch (s) {
        case LRS_OK: return "LRS_OK";
        case LRS_ERR_INVALID_ARG: return "LRS_ERR_INVALID_ARG";
        case LRS_ERR_ALIGNMENT: return "LRS_ERR_ALIGNMENT";
        case LRS_ERR_UNSUPPORTED: return "LRS_ERR_UNSUPPORTED";
        case LRS_ERR_OOM: return "LRS_ERR_OOM";
        case LRS_ERR_CUDA: return "LRS_ERR_CUDA";
        case LRS_ERR_DEVICE_TIMEOUT: return "LRS_ERR_DEVICE_TIMEOUT";
        case LRS_ERR_DEVICE_LAYOUT: return "LRS_ERR_DEVICE_LAYOUT";
        case LRS_ERR_DEVICE_RANGE: return "LRS_ERR_DEVICE_RANGE";
        case LRS_ERR_DEVICE_BOUNDS: return "LRS_ERR_DEVICE_BOUNDS";
    }
    return "LRS_ERR_UNKNOWN";
}

const char* lrs_last_error(void) { return g_last_error.c_str(); }

int32_t lrs_version(void) { return LRS_VERSION; }

lrs_status lrs_layout_query(const lrs_shape* shape, const uint8_t* prec_map_host,
                            int64_t* head_offsets_host, int64_t* batch_stride_bytes,
                            int64_t* scale_count) {
    lrs_status s = compute_layout(shape, prec_map_host, 1, head_offsets_host, batch_stride_bytes,
                                  scale_count);
    return s == LRS_OK ? ok() : s;
}

lrs_status lrs_layout_query_groups(const lrs_shape* shape, const uint8_t* prec_map_host,
                                   int64_t* head_offsets_host, int64_t* batch_stride_bytes,
                                   int64_t* scale_count) {
    lrs_status s = check_shape(shape);
    if (s != LRS_OK) return s;
    s = compute_layout(shape, prec_map_host, shape->d_k / shape->group, head_offsets_host,
                       batch_stride_bytes, scale_count);
    return s == LRS_OK ? ok() : s;
}

}  // extern "C"

static lrs_status state_alloc(const lrs_shape* shape, const uint8_t* prec_map_host, int pgroups,
                              lrs_state* out) {
    if (!out) return fail(LRS_ERR_INVALID_ARG, "out is NULL");
    memset(out, 0, sizeof *out);
    lrs_status s = check_shape(shape);
    if (s != LRS_OK) return s;
    std::vector<int64_t> offs(shape->heads);
    int64_t stride = 0, nscales = 0;
    s = compute_layout(shape, prec_map_host, pgroups, offs.data(), &stride, &nscales);
    if (s != LRS_OK) return s;
    DeviceCtx* ctx = nullptr;
    s = device_ctx(&ctx);
    if (s != LRS_OK) return s;
    const int nprec = shape->heads * pgroups;

    StatePriv* pv = new StatePriv;
    cudaGetDevice(&pv->device);
    pv->pgroups = pgroups;
    pv->prec_host.assign(prec_map_host, prec_map_host + nprec);
    pv->offsets_host = offs;

    lrs_state st;
    memset(&st, 0, sizeof st);
    st.shape = *shape;
    st.batch_stride_bytes = stride;
    st.code_bytes = stride * shape->batch;
    st.scale_count = nscales;
    st.priv = pv;
    auto cleanup = [&](cudaError_t e, const char* what) {
        cudaFree(st.state_codes);
        cudaFree(st.scales);
        cudaFree(st.prec_map);
        cudaFree(st.head_offsets);
        delete pv;
        return cuda_fail(e, what);
    };
    cudaError_t e;
    if ((e = cudaMalloc(&st.state_codes, std::max<int64_t>(st.code_bytes, 16))) != cudaSuccess)
        return cleanup(e, "cudaMalloc(codes)");
    if ((e = cudaMalloc(&st.scales, std::max<int64_t>(nscales, 4) * sizeof(float))) != cudaSuccess)
        return cleanup(e, "cudaMalloc(scales)");
    if ((e = cudaMalloc(&st.prec_map, std::max(nprec, 16))) != cudaSuccess)
        return cleanup(e, "cudaMalloc(prec_map)");
    if ((e = cudaMalloc(&st.head_offsets, shape->heads * sizeof(int64_t))) != cudaSuccess)
        return cleanup(e, "cudaMalloc(head_offsets)");
    if ((e = cudaMemcpy(st.prec_map, prec_map_host, nprec, cudaMemcpyHostToDevice)) !=
        cudaSuccess)
        return cleanup(e, "cudaMemcpy(prec_map)");
    if ((e = cudaMemcpy(st.head_offsets, offs.data(), shape->heads * sizeof(int64_t),
                        cudaMemcpyHostToDevice)) != cudaSuccess)
        return cleanup(e, "cudaMemcpy(head_offsets)");
    if ((e = lrs::launch_fill_zero(layout_args(&st, ctx->err), nullptr)) != cudaSuccess)
        return cleanup(e, "zero fill");
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cleanup(e, "zero fill");
    *out = st;
    return ok();
}

extern "C" {

lrs_status lrs_state_alloc(const lrs_shape* shape, const uint8_t* prec_map_host, lrs_state* out) {
    return state_alloc(shape, prec_map_host, 1, out);
}

lrs_status lrs_state_alloc_groups(const lrs_shape* shape, const uint8_t* prec_map_host,
                                  lrs_state* out) {
    if (!shape) return fail(LRS_ERR_INVALID_ARG, "shape is NULL");
    if (!out) return fail(LRS_ERR_INVALID_ARG, "out is NULL");
    memset(out, 0, sizeof *out);
    lrs_status s = check_shape(shape);
    if (s != LRS_OK) return s;
    return state_alloc(shape, prec_map_host, shape->d_k / shape->group, out);
}

lrs_status lrs_state_free(lrs_state* st) {
    if (!st || !st->priv) return ok();
    StatePriv* pv = static_cast<StatePriv*>(st->priv);
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != pv->device) cudaSetDevice(pv->device);
    cudaDeviceSynchronize();
    cudaFree(st->state_codes);
    cudaFree(st->scales);
    cudaFree(st->prec_map);
    cudaFree(st->head_offsets);
    cudaFree(pv->stage[0]);
    cudaFree(pv->stage[1]);
    for (int b = 0; b < 2; ++b) {
        if (pv->h2d_done[b]) cudaEventDestroy(pv->h2d_done[b]);
        if (pv->free_again[b]) cudaEventDestroy(pv->free_again[b]);
    }
    if (pv->copy_stream) cudaStreamDestroy(pv->copy_stream);
    if (prev != pv->device && prev >= 0) cudaSetDevice(prev);
    delete pv;
    memset(st, 0, sizeof *st);
    return ok();
}

}  // extern "C"

// The step with q, k, v and out of element type io (lrs::StepIo).
static lrs_status decode_step_io(const lrs_state* st, void* state_codes, float* scales,
                                 const uint8_t* prec_map, const void* q, const void* k,
                                 const void* v, const float* gates, const float* beta, void* out,
                                 uint64_t seed, uint64_t step, int32_t mode, int io,
                                 void* stream) {
    lrs_status s = check_state(st);
    if (s != LRS_OK) return s;
    const lrs_shape& sh = st->shape;
    LRS_REQUIRE_PTR(state_codes);
    LRS_REQUIRE_PTR(scales);
    if (!prec_map) return fail(LRS_ERR_INVALID_ARG, "prec_map is NULL");
    LRS_REQUIRE_PTR(q);
    LRS_REQUIRE_PTR(k);
    LRS_REQUIRE_PTR(v);
    LRS_REQUIRE_PTR(gates);
    LRS_REQUIRE_PTR(out);
    if (sh.update_kind == LRS_UPDATE_DELTA) LRS_REQUIRE_PTR(beta);
    if (mode != LRS_ROUND_RTN && mode != LRS_ROUND_SR && mode != LRS_ROUND_BDR)
        return fail(LRS_ERR_INVALID_ARG, "mode %d", mode);
    const int G = sh.d_k / sh.group;
    DeviceCtx* ctx = nullptr;
    s = device_ctx(&ctx);
    if (s != LRS_OK) return s;
    const int ntiles = sh.batch * sh.heads;
    if (ntiles == 0) return ok();

    lrs::StepLaunch ls;
    s = lrs::step_launch_shape(sh, mode, io, static_cast<const StatePriv*>(st->priv)->device,
                               ctx->sms, &ls);
    if (s != LRS_OK) return s;
    const int grid = std::min(ls.grid, (ntiles + ls.warps - 1) / ls.warps);
    lrs::StepParams p;
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
    p.err = ctx->err;
    p.timeout_ns = 2000000000ull;  // 2 s: far above any legitimate wait
    p.H = sh.heads;
    p.d_k = sh.d_k;
    p.G = G;
    p.ntiles = ntiles;
    p.pgroups = static_cast<const StatePriv*>(st->priv)->pgroups;
    p.warp_smem = ls.warp_smem;
    p.slots = ls.slots;
    p.inject = 0;
    p.code_bytes = st->code_bytes;
    p.scale_count = st->scale_count;
    {
        std::lock_guard<std::mutex> lk(g_inject_mu);
        if (g_inject) {
            p.inject = 1 + g_inject_items;
            p.timeout_ns = g_inject_timeout_ns;
            g_inject = false;
        }
    }
    void* args[] = {&p};
    cudaError_t e = cudaLaunchKernel(ls.fn, dim3(grid), dim3(ls.warps * 32), args, ls.smem,
                                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();  // a failed launch must not surface again in a later call
        return cuda_fail(e, "launch of the step kernel");
    }
    return ok();
}

extern "C" {

lrs_status lrs_decode_step(const lrs_state* st, void* state_codes, float* scales,
                           const uint8_t* prec_map, const float* q, const float* k,
                           const float* v, const float* gates, const float* beta, float* out,
                           uint64_t seed, uint64_t step, int32_t mode, void* stream) {
    return decode_step_io(st, state_codes, scales, prec_map, q, k, v, gates, beta, out, seed,
                          step, mode, lrs::kStepIoF32, stream);
}

lrs_status lrs_decode_step_bf16(const lrs_state* st, void* state_codes, float* scales,
                                const uint8_t* prec_map, const uint16_t* q, const uint16_t* k,
                                const uint16_t* v, const float* gates, const float* beta,
                                uint16_t* out, uint64_t seed, uint64_t step, int32_t mode,
                                void* stream) {
    return decode_step_io(st, state_codes, scales, prec_map, q, k, v, gates, beta, out, seed,
                          step, mode, lrs::kStepIoBF16, stream);
}

lrs_status lrs_decode_step_host(const lrs_state* st, const float* q_host, const float* k_host,
                                const float* v_host, const float* gates_host,
                                const float* beta_host, float* out_host, uint64_t seed,
                                uint64_t step, int32_t mode, void* stream) {
    lrs_status s = check_state(st);
    if (s != LRS_OK) return s;
    const lrs_shape& sh = st->shape;
    if (!q_host || !k_host || !v_host || !gates_host || !out_host)
        return fail(LRS_ERR_INVALID_ARG, "a host buffer is NULL");
    const bool delta = sh.update_kind == LRS_UPDATE_DELTA;
    if (delta && !beta_host) return fail(LRS_ERR_INVALID_ARG, "beta_host is NULL");
    const size_t T = static_cast<size_t>(sh.batch) * sh.heads;
    // staging: q, k [T][d_k] | v, out [T][d_v] | gates [T][d_k or 1] | beta [T]
    auto rnd = [](size_t n) { return (n + 3) / 4 * 4; };  // keep 16-byte alignment
    const size_t nq = rnd(T * sh.d_k), nv = rnd(T * sh.d_v);
    const size_t ng = rnd(sh.gate_kind == LRS_GATE_PER_KEY ? T * sh.d_k : T), nb = rnd(T);
    const size_t need = 2 * nq + 2 * nv + ng + nb;
    StatePriv* pv = static_cast<StatePriv*>(st->priv);
    cudaError_t e;
    if (!pv->copy_stream) {
        if ((e = cudaStreamCreateWithFlags(&pv->copy_stream, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamCreate(copies)");
        for (int b = 0; b < 2; ++b)
            if ((e = cudaEventCreateWithFlags(&pv->h2d_done[b], cudaEventDisableTiming)) !=
                    cudaSuccess ||
                (e = cudaEventCreateWithFlags(&pv->free_again[b], cudaEventDisableTiming)) !=
                    cudaSuccess)
                return cuda_fail(e, "cudaEventCreate(staging)");
    }
    if (pv->stage_floats < need) {
        // no staging buffer may be in use when it is replaced
        if ((e = cudaStreamSynchronize(pv->copy_stream)) != cudaSuccess ||
            (e = cudaEventSynchronize(pv->free_again[0])) != cudaSuccess ||
            (e = cudaEventSynchronize(pv->free_again[1])) != cudaSuccess)
            return cuda_fail(e, "waiting for the staging buffers");
        for (int b = 0; b < 2; ++b) {
            cudaFree(pv->stage[b]);
            pv->stage[b] = nullptr;
        }
        pv->stage_floats = 0;
        for (int b = 0; b < 2; ++b)
            if ((e = cudaMalloc(&pv->stage[b], need * sizeof(float))) != cudaSuccess)
                return cuda_fail(e, "cudaMalloc(staging)");
        pv->stage_floats = need;
    }
    // Alternate calls use alternate buffers, so the input copies of one call
    // overlap the kernel and output copy of the previous one. The copies of a
    // buffer wait for its previous use to end (its output copy); they are not
    // ordered after other work on `stream`.
    const int b = static_cast<int>(pv->host_calls++ & 1);
    float* dq = pv->stage[b];
    float* dk = dq + nq;
    float* dv = dk + nq;
    float* dout = dv + nv;
    float* dg = dout + nv;
    float* db = dg + ng;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaStream_t cp = pv->copy_stream;
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice;
    if ((e = cudaStreamWaitEvent(cp, pv->free_again[b], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dq, q_host, T * sh.d_k * 4, h2d, cp)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dk, k_host, T * sh.d_k * 4, h2d, cp)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dv, v_host, T * sh.d_v * 4, h2d, cp)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dg, gates_host,
                             (sh.gate_kind == LRS_GATE_PER_KEY ? T * sh.d_k : T) * 4, h2d, cp)) !=
            cudaSuccess ||
        (delta && (e = cudaMemcpyAsync(db, beta_host, T * 4, h2d, cp)) != cudaSuccess) ||
        (e = cudaEventRecord(pv->h2d_done[b], cp)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(cs, pv->h2d_done[b], 0)) != cudaSuccess)
        return cuda_fail(e, "host-to-device copy of the step inputs");
    s = lrs_decode_step(st, st->state_codes, st->scales, st->prec_map, dq, dk, dv, dg,
                        delta ? db : nullptr, dout, seed, step, mode, stream);
    if (s != LRS_OK) return s;
    if ((e = cudaMemcpyAsync(out_host, dout, T * sh.d_v * 4, cudaMemcpyDeviceToHost, cs)) !=
            cudaSuccess ||
        (e = cudaEventRecord(pv->free_again[b], cs)) != cudaSuccess)
        return cuda_fail(e, "device-to-host copy of the output");
    return ok();
}

}  // extern "C"

template <class Fn>
static lrs_status layout_op(const lrs_state* st, void* stream, Fn&& fn) {
    lrs_status s = check_state(st);
    if (s != LRS_OK) return s;
    DeviceCtx* ctx = nullptr;
    s = device_ctx(&ctx);
    if (s != LRS_OK) return s;
    cudaError_t e = fn(layout_args(st, ctx->err), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "layout kernel launch");
}

extern "C" {

lrs_status lrs_state_import_fp32(const lrs_state* st, const float* S, void* stream) {
    LRS_REQUIRE_PTR(S);
    return layout_op(st, stream, [&](const lrs::LayoutArgs& a, cudaStream_t s) {
        return lrs::launch_import_fp32(a, S, s);
    });
}

lrs_status lrs_state_export_fp32(const lrs_state* st, float* S, void* stream) {
    LRS_REQUIRE_PTR(S);
    return layout_op(st, stream, [&](const lrs::LayoutArgs& a, cudaStream_t s) {
        return lrs::launch_export_fp32(a, S, s);
    });
}

lrs_status lrs_state_export_codes(const lrs_state* st, int8_t* codes, void* stream) {
    LRS_REQUIRE_PTR(codes);
    return layout_op(st, stream, [&](const lrs::LayoutArgs& a, cudaStream_t s) {
        return lrs::launch_export_codes(a, codes, s);
    });
}

lrs_status lrs_state_import_codes(const lrs_state* st, const int8_t* codes, const float* scales,
                                  void* stream) {
    LRS_REQUIRE_PTR(codes);
    LRS_REQUIRE_PTR(scales);
    return layout_op(st, stream, [&](const lrs::LayoutArgs& a, cudaStream_t s) {
        return lrs::launch_import_codes(a, codes, scales, s);
    });
}

lrs_status lrs_state_copy_raw(const lrs_state* st, void* codes_host, float* scales_host,
                              int32_t to_host, void* stream) {
    lrs_status s = check_state(st);
    if (s != LRS_OK) return s;
    if (!codes_host || !scales_host) return fail(LRS_ERR_INVALID_ARG, "a host buffer is NULL");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (to_host) {
        if ((e = cudaMemcpyAsync(codes_host, st->state_codes, st->code_bytes,
                                 cudaMemcpyDeviceToHost, cs)) != cudaSuccess ||
            (e = cudaMemcpyAsync(scales_host, st->scales, st->scale_count * sizeof(float),
                                 cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
            return cuda_fail(e, "copy to host");
    } else {
        if ((e = cudaMemcpyAsync(st->state_codes, codes_host, st->code_bytes,
                                 cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
            (e = cudaMemcpyAsync(st->scales, scales_host, st->scale_count * sizeof(float),
                                 cudaMemcpyHostToDevice, cs)) != cudaSuccess)
            return cuda_fail(e, "copy from host");
    }
    if ((e = cudaStreamSynchronize(cs)) != cudaSuccess) return cuda_fail(e, "synchronize");
    return ok();
}

lrs_status lrs_fp32_decode_step(const lrs_shape* shape, float* S, const float* q, const float* k,
                                const float* v, const float* gates, const float* beta,
                                float* out, void* stream) {
    if (!shape) return fail(LRS_ERR_INVALID_ARG, "shape is NULL");
    const lrs_shape& sh = *shape;
    if (sh.batch < 0 || sh.heads < 1 || sh.d_k < 1)
        return fail(LRS_ERR_INVALID_ARG, "non-positive dimension");
    if (sh.update_kind != LRS_UPDATE_GATED && sh.update_kind != LRS_UPDATE_DELTA)
        return fail(LRS_ERR_INVALID_ARG, "update_kind %d", sh.update_kind);
    if (sh.gate_kind != LRS_GATE_SCALAR && sh.gate_kind != LRS_GATE_PER_KEY)
        return fail(LRS_ERR_INVALID_ARG, "gate_kind %d", sh.gate_kind);
    if (sh.update_kind == LRS_UPDATE_DELTA && sh.gate_kind != LRS_GATE_SCALAR)
        return fail(LRS_ERR_UNSUPPORTED, "the delta rule takes a scalar decay");
    if (sh.d_v != 64 && sh.d_v != 128)
        return fail(LRS_ERR_UNSUPPORTED, "d_v=%d (supported: 64, 128)", sh.d_v);
    if (sh.d_k % 8 != 0 || sh.d_k > 1024)
        return fail(LRS_ERR_UNSUPPORTED, "d_k=%d (a multiple of 8, at most 1024)", sh.d_k);
    LRS_REQUIRE_PTR(S);
    LRS_REQUIRE_PTR(q);
    LRS_REQUIRE_PTR(k);
    LRS_REQUIRE_PTR(v);
    LRS_REQUIRE_PTR(gates);
    LRS_REQUIRE_PTR(out);
    if (sh.update_kind == LRS_UPDATE_DELTA) LRS_REQUIRE_PTR(beta);
    cudaError_t e = lrs::launch_fp32_step(sh.batch, sh.heads, sh.d_k, sh.d_v, sh.update_kind,
                                          sh.gate_kind, S, q, k, v, gates, beta, out,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "launch of the fp32 step kernel");
}

lrs_status lrs_decay_head_means(const float* decay, int64_t outer, int32_t heads, int64_t inner,
                                double* means, void* stream) {
    if (outer < 1 || heads < 1 || inner < 1)
        return fail(LRS_ERR_INVALID_ARG, "outer=%lld heads=%d inner=%lld", (long long)outer, heads,
                    (long long)inner);
    LRS_REQUIRE_PTR(decay);
    LRS_REQUIRE_PTR(means);
    cudaError_t e = lrs::launch_decay_means(decay, outer, heads, inner, means,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "launch of the decay-mean kernel");
}

lrs_status lrs_precision_map(int32_t heads, const double* means_host, int32_t n_int8,
                             uint8_t* prec_map_host) {
    if (heads < 1 || !means_host || !prec_map_host || n_int8 < 0 || n_int8 > heads)
        return fail(LRS_ERR_INVALID_ARG, "heads=%d n_int8=%d", heads, n_int8);
    std::vector<int> order(heads);
    for (int h = 0; h < heads; ++h) order[h] = h;
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return means_host[a] > means_host[b]; });
    for (int h = 0; h < heads; ++h) prec_map_host[h] = 4;
    for (int n = 0; n < n_int8; ++n) prec_map_host[order[n]] = 8;
    return ok();
}

lrs_status lrs_sync(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    DeviceCtx* ctx = nullptr;
    lrs_status s = device_ctx(&ctx);
    if (s != LRS_OK) return s;
    unsigned flags = 0;
    e = cudaMemcpy(&flags, ctx->err, sizeof flags, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "read of the device error word");
    if (flags == 0) return ok();
    e = cudaMemset(ctx->err, 0, sizeof flags);
    if (e != cudaSuccess) return cuda_fail(e, "reset of the device error word");
    if (flags & lrs::kErrTimeout)
        return fail(LRS_ERR_DEVICE_TIMEOUT, "a step kernel timed out waiting for its copies");
    if (flags & lrs::kErrLayout)
        return fail(LRS_ERR_DEVICE_LAYOUT, "prec_map does not fit the state's tile layout");
    if (flags & lrs::kErrBounds)
        return fail(LRS_ERR_DEVICE_BOUNDS, "a step kernel index fell outside its buffer "
                    "(bounds-checked build)");
    return fail(LRS_ERR_DEVICE_RANGE, "an imported code was outside [-qmax, qmax]");
}

lrs_status lrs_debug_inject_timeout(int32_t enable, int32_t timeout_us) {
    return lrs_debug_inject_timeout_after(enable ? 0 : -1, timeout_us);
}

lrs_status lrs_debug_inject_timeout_after(int32_t items_copied, int32_t timeout_us) {
    if (items_copied >= 0 && timeout_us < 1)
        return fail(LRS_ERR_INVALID_ARG, "timeout_us=%d", timeout_us);
    std::lock_guard<std::mutex> lk(g_inject_mu);
    g_inject = items_copied >= 0;
    g_inject_items = items_copied < 0 ? 0 : items_copied;
    g_inject_timeout_ns = static_cast<uint64_t>(timeout_us) * 1000ull;
    return ok();
}

}  // extern "C"

namespace lrs {

// Status helpers for entry points defined in other translation units: they
// set and clear the same thread-local message as the functions above.
lrs_status device_error_word(unsigned** err, int* sms) {
    DeviceCtx* ctx = nullptr;
    lrs_status s = device_ctx(&ctx);
    if (s != LRS_OK) return s;
    *err = ctx->err;
    *sms = ctx->sms;
    return LRS_OK;
}

bool take_injected_timeout(uint64_t* timeout_ns) {
    std::lock_guard<std::mutex> lk(g_inject_mu);
    if (!g_inject) return false;
    g_inject = false;
    *timeout_ns = g_inject_timeout_ns;
    return true;
}

int sm_count(int device) {
    static std::mutex mu;
    static int sms[kMaxDevices];
    if (device < 0 || device >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (sms[device] == 0 &&
        cudaDeviceGetAttribute(&sms[device], cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
        cudaGetLastError();
        sms[device] = 0;
    }
    return sms[device];
}

lrs_status api_fail(lrs_status s, const char* msg) { return fail(s, "%s", msg); }
lrs_status api_cuda_fail(cudaError_t e, const char* what) { return cuda_fail(e, what); }
lrs_status api_ok() { return ok(); }
lrs_status api_check_state(const lrs_state* st) { return check_state(st); }

int state_prec_groups(const lrs_state* st) {
    return static_cast<const StatePriv*>(st->priv)->pgroups;
}

}  // namespace lrs
