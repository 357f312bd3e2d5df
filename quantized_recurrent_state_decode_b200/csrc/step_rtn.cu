// step_rtn.cu -- compiled variants of the fused decode step: RTN rounding,
// fp32 q, k, v and out.
#include "step_instances.cuh"

namespace lrs {
LRS_STEP_VARIANTS(find_step_kernel_rtn, kRTN, kIoF32)
}  // namespace lrs
