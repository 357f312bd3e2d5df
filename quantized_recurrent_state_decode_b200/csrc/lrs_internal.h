// lrs_internal.h -- declarations shared by liblrs's translation units (host side).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "lrs.h"

namespace lrs {

// Element type of q, k, v and out.
enum StepIo { kStepIoF32 = 0, kStepIoBF16 = 1 };

// Kernel entry of one compiled step variant, or nullptr when the combination
// (columns per lane C = d_v/32, group rows, update kind, gate kind, rounding
// mode, I/O element type) is not compiled.
const void* find_step_kernel(int C, int group, int update_kind, int gate_kind, int mode,
                             int io = kStepIoF32);
const void* find_step_kernel_rtn(int C, int group, int update_kind, int gate_kind);
const void* find_step_kernel_sr(int C, int group, int update_kind, int gate_kind);
const void* find_step_kernel_bdr(int C, int group, int update_kind, int gate_kind);
const void* find_step_kernel_rtn_bf16(int C, int group, int update_kind, int gate_kind);
const void* find_step_kernel_sr_bf16(int C, int group, int update_kind, int gate_kind);
const void* find_step_kernel_bdr_bf16(int C, int group, int update_kind, int gate_kind);

// Bytes of shared memory one warp of the step kernel uses with `slots` ring
// slots in rounding mode `mode` with I/O element type `io` and d_k key rows.
int step_warp_smem(int C, int group, int update_kind, int gate_kind, int slots, int mode, int io,
                   int d_k);

// Launch shape of the step kernel for one state shape, rounding mode and I/O
// type on `device` with `sms` SMs: kernel, ring slots per warp, warps per
// CTA, shared memory per warp and per CTA, and the grid (CTAs that fit on all
// SMs; a launch takes at most one warp per tile). Prepared once per (kernel,
// device). The one launcher of every entry point that runs the step kernel.
struct StepLaunch {
    const void* fn;
    int slots, warps, warp_smem, smem, grid;
};
lrs_status step_launch_shape(const lrs_shape& sh, int mode, int io, int device, int sms,
                             StepLaunch* out);

// SM count of a device (queried once; 0 when the query fails).
int sm_count(int device);

// The chunked-update kernel for one shape and rounding mode, with the bytes
// of shared memory it takes per CTA ({nullptr, 0} when not compiled).
struct ChunkKernel {
    const void* fn;
    int smem;
};
ChunkKernel find_chunk_kernel_rtn(int d_k, int d_v, int group, int update_kind, int gate_kind);
ChunkKernel find_chunk_kernel_sr(int d_k, int d_v, int group, int update_kind, int gate_kind);
ChunkKernel find_chunk_kernel_bdr(int d_k, int d_v, int group, int update_kind, int gate_kind);

ChunkKernel find_lrb_kernel_rtn(int d_k, int d_v, int group, int update_kind, int gate_kind);
ChunkKernel find_lrb_kernel_sr(int d_k, int d_v, int group, int update_kind, int gate_kind);
ChunkKernel find_lrb_kernel_bdr(int d_k, int d_v, int group, int update_kind, int gate_kind);

// The streaming bypass kernels (ranks up to 4), by (C = d_v/32, group,
// update kind, gate kind); nullptr when not compiled.
const void* find_lrb_stream_rtn(int C, int group, int update_kind, int gate_kind,
                                 bool merge);
const void* find_lrb_stream_sr(int C, int group, int update_kind, int gate_kind,
                                 bool merge);
const void* find_lrb_stream_bdr(int C, int group, int update_kind, int gate_kind,
                                 bool merge);

struct LayoutArgs {
    uint8_t* codes;
    float* scales;
    const uint8_t* prec_map;
    const int64_t* head_offsets;
    int64_t batch_stride;
    int32_t B, H, d_k, d_v, group;
    int32_t pgroups;        // widths in prec_map per head (1) or per (head, group) (G)
    unsigned* err;
};

cudaError_t launch_fill_zero(const LayoutArgs& a, cudaStream_t s);
cudaError_t launch_import_fp32(const LayoutArgs& a, const float* S, cudaStream_t s);
cudaError_t launch_export_fp32(const LayoutArgs& a, float* S, cudaStream_t s);
cudaError_t launch_export_codes(const LayoutArgs& a, int8_t* codes, cudaStream_t s);
cudaError_t launch_import_codes(const LayoutArgs& a, const int8_t* codes, const float* scales,
                                cudaStream_t s);
cudaError_t launch_fp32_step(int B, int H, int d_k, int d_v, int update_kind, int gate_kind,
                             float* S, const float* q, const float* k, const float* v,
                             const float* gates, const float* beta, float* out, cudaStream_t s);
cudaError_t launch_decay_means(const float* decay, int64_t outer, int heads, int64_t inner,
                               double* means, cudaStream_t s);
bool layout_kernels_support(int d_v, int group);

// The current device's error word (read and cleared by lrs_sync) and SM count.
lrs_status device_error_word(unsigned** err, int* sms);

// Consumes an armed lrs_debug_inject_timeout: returns true (and the wait limit
// to use) for the one launch that must issue no copies.
bool take_injected_timeout(uint64_t* timeout_ns);

// Status helpers shared by the C-ABI translation units (lrs_api.cu).
lrs_status api_fail(lrs_status s, const char* msg);
lrs_status api_cuda_fail(cudaError_t e, const char* what);
lrs_status api_ok();
lrs_status api_check_state(const lrs_state* st);

// Widths per head (1) or per (head, scale group) (G) of an allocated state.
int state_prec_groups(const lrs_state* st);

}  // namespace lrs
