// lrb_bdr.cu -- compiled variants of the decode step with a Low-Rank Bypass
// buffer, BDR rounding.
#include "lrb_kernel.cuh"

namespace lrs {
LRS_LRB_VARIANTS(find_lrb_kernel_bdr, kBDR)
}  // namespace lrs
