// step_bdr_bf16.cu -- compiled variants of the fused decode step: BDR rounding,
// bfloat16 q, k, v and out.
#include "step_instances.cuh"

namespace lrs {
LRS_STEP_VARIANTS(find_step_kernel_bdr_bf16, kBDR, kIoBF16)
}  // namespace lrs
