// step_rtn_bf16.cu -- compiled variants of the fused decode step: RTN rounding,
// bfloat16 q, k, v and out.
#include "step_instances.cuh"

namespace lrs {
LRS_STEP_VARIANTS(find_step_kernel_rtn_bf16, kRTN, kIoBF16)
}  // namespace lrs
