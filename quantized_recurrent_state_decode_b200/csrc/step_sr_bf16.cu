// step_sr_bf16.cu -- compiled variants of the fused decode step: SR rounding,
// bfloat16 q, k, v and out.
#include "step_instances.cuh"

namespace lrs {
LRS_STEP_VARIANTS(find_step_kernel_sr_bf16, kSR, kIoBF16)
}  // namespace lrs
