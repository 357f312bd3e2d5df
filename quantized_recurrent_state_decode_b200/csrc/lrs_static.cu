// lrs_static.cu -- the decode step on host buffers with no device allocation.
//
// lrs_decode_step_host stages the step's inputs and output in device buffers
// that it allocates on first use, and its kernels record errors in a device
// word allocated by the library. Some callers must not allocate device memory
// when they step: processes whose device memory belongs to another allocator
// or to a fixed pool sized at start-up (an allocation behind its back can fail
// or break its accounting), and latency-critical paths that cannot afford a
// cudaMalloc, which may synchronize the device. lrs_decode_step_host_noalloc
// serves them: its scratch (the error word and the staging of inputs and
// output) is the file-scope array below, part of the library's device image.
// Each device takes it when that image is loaded there -- at the latest on the
// first call on the device, since CUDA loads modules lazily -- and keeps it
// until the process exits.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "lrs.h"
#include "lrs_internal.h"
#include "step_kernel.cuh"

namespace {

// Layout of the scratch: [0, 256) the device error word; then the staging of
// q, k, v, out, gates and beta, each padded to a multiple of 16 bytes.
constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr size_t kNoallocErrBytes = 256;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];   // device address of the array, per device

// Device address of the scratch array on the current device. The first call
// on a device looks the address up (the name of the array in host code is a
// stand-in, not a device address); later calls reuse it.
lrs_status scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return lrs::api_cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return lrs::api_fail(LRS_ERR_UNSUPPORTED, "device index");
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return lrs::api_cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LRS_OK;
}

size_t pad16(size_t bytes) { return (bytes + 15) / 16 * 16; }

}  // namespace

extern "C" lrs_status lrs_decode_step_host_noalloc(const lrs_state* st, const float* q_host,
                                                   const float* k_host, const float* v_host,
                                                   const float* gates_host,
                                                   const float* beta_host, float* out_host,
                                                   uint32_t* device_error_host, uint64_t seed,
                                                   uint64_t step, int32_t mode, void* stream) {
    lrs_status s = lrs::api_check_state(st);
    if (s != LRS_OK) return s;
    const lrs_shape& sh = st->shape;
    if (!q_host || !k_host || !v_host || !gates_host || !out_host)
        return lrs::api_fail(LRS_ERR_INVALID_ARG, "a host buffer is NULL");
    const bool delta = sh.update_kind == LRS_UPDATE_DELTA;
    if (delta && !beta_host) return lrs::api_fail(LRS_ERR_INVALID_ARG, "beta_host is NULL");
    if (mode != LRS_ROUND_RTN && mode != LRS_ROUND_SR && mode != LRS_ROUND_BDR)
        return lrs::api_fail(LRS_ERR_INVALID_ARG, "mode is not an lrs_round_mode");
    const int G = sh.d_k / sh.group;

    const size_t T = static_cast<size_t>(sh.batch) * sh.heads;
    const size_t bq = T * sh.d_k * 4, bv = T * sh.d_v * 4;
    const size_t bg = (sh.gate_kind == LRS_GATE_PER_KEY ? T * sh.d_k : T) * 4;
    const size_t bb = delta ? T * 4 : 0;
    const size_t need = kNoallocErrBytes + 2 * pad16(bq) + 2 * pad16(bv) + pad16(bg) + pad16(bb);
    if (need > kNoallocScratchBytes) {
        char msg[160];
        snprintf(msg, sizeof msg,
                 "this step needs %zu bytes of static scratch; the maximum is %zu bytes (32 MiB)",
                 need, kNoallocScratchBytes);
        return lrs::api_fail(LRS_ERR_UNSUPPORTED, msg);
    }
    if (T == 0) return lrs::api_ok();

    void* base = nullptr;
    s = scratch_address(&base);
    if (s != LRS_OK) return s;
    unsigned char* sp = static_cast<unsigned char*>(base);
    unsigned* err = reinterpret_cast<unsigned*>(sp);
    float* dq = reinterpret_cast<float*>(sp + kNoallocErrBytes);
    float* dk = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(dq) + pad16(bq));
    float* dv = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(dk) + pad16(bq));
    float* dout = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(dv) + pad16(bv));
    float* dg = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(dout) + pad16(bv));
    float* db = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(dg) + pad16(bg));

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice;
    cudaError_t e;
    if ((e = cudaMemsetAsync(err, 0, sizeof(unsigned), cs)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dq, q_host, bq, h2d, cs)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dk, k_host, bq, h2d, cs)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dv, v_host, bv, h2d, cs)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dg, gates_host, bg, h2d, cs)) != cudaSuccess ||
        (delta && (e = cudaMemcpyAsync(db, beta_host, bb, h2d, cs)) != cudaSuccess)) {
        cudaGetLastError();
        return lrs::api_cuda_fail(e, "host-to-device copy into the static scratch");
    }

    // the launch shape of lrs_decode_step (one shared, cached helper)
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return lrs::api_cuda_fail(e, "cudaGetDevice");
    lrs::StepLaunch ls;
    s = lrs::step_launch_shape(sh, mode, lrs::kStepIoF32, dev, lrs::sm_count(dev), &ls);
    if (s != LRS_OK) return s;
    const int ntiles = static_cast<int>(T);
    const int grid = std::min(ls.grid, (ntiles + ls.warps - 1) / ls.warps);

    lrs::StepParams p;
    memset(&p, 0, sizeof p);
    p.codes = static_cast<uint8_t*>(st->state_codes);
    p.scales = st->scales;
    p.prec_map = st->prec_map;
    p.head_offsets = st->head_offsets;
    p.batch_stride = st->batch_stride_bytes;
    p.q = dq;
    p.k = dk;
    p.v = dv;
    p.gates = dg;
    p.beta = delta ? db : nullptr;
    p.out = dout;
    p.seed = seed;
    p.step = step;
    p.err = err;
    p.timeout_ns = 2000000000ull;
    p.H = sh.heads;
    p.d_k = sh.d_k;
    p.G = G;
    p.ntiles = ntiles;
    p.pgroups = lrs::state_prec_groups(st);
    p.slots = ls.slots;
    p.warp_smem = ls.warp_smem;
    p.inject = 0;
    p.code_bytes = st->code_bytes;
    p.scale_count = st->scale_count;
    void* args[] = {&p};
    if ((e = cudaLaunchKernel(ls.fn, dim3(grid), dim3(ls.warps * 32), args, ls.smem, cs)) !=
        cudaSuccess) {
        cudaGetLastError();
        return lrs::api_cuda_fail(e, "launch of the step kernel");
    }
    if ((e = cudaMemcpyAsync(out_host, dout, bv, cudaMemcpyDeviceToHost, cs)) != cudaSuccess ||
        (device_error_host &&
         (e = cudaMemcpyAsync(device_error_host, err, sizeof(unsigned), cudaMemcpyDeviceToHost,
                              cs)) != cudaSuccess)) {
        cudaGetLastError();
        return lrs::api_cuda_fail(e, "device-to-host copy from the static scratch");
    }
    return lrs::api_ok();
}
