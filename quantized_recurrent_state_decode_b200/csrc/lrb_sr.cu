// lrb_sr.cu -- compiled variants of the decode step with a Low-Rank Bypass
// buffer, SR rounding.
#include "lrb_kernel.cuh"

namespace lrs {
LRS_LRB_VARIANTS(find_lrb_kernel_sr, kSR)
}  // namespace lrs
