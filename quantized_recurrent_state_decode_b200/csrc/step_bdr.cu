// step_bdr.cu -- compiled variants of the fused decode step: BDR rounding,
// fp32 q, k, v and out.
#include "step_instances.cuh"

namespace lrs {
LRS_STEP_VARIANTS(find_step_kernel_bdr, kBDR, kIoF32)
}  // namespace lrs
