// lrb_rtn.cu -- compiled variants of the decode step with a Low-Rank Bypass
// buffer, RTN rounding.
#include "lrb_kernel.cuh"

namespace lrs {
LRS_LRB_VARIANTS(find_lrb_kernel_rtn, kRTN)
}  // namespace lrs
