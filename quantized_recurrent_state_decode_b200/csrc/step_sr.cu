// step_sr.cu -- compiled variants of the fused decode step: SR rounding,
// fp32 q, k, v and out.
#include "step_instances.cuh"

namespace lrs {
LRS_STEP_VARIANTS(find_step_kernel_sr, kSR, kIoF32)
}  // namespace lrs
