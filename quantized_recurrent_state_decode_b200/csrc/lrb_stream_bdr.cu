// lrb_stream_bdr.cu -- compiled variants of the streaming Low-Rank Bypass
// decode step, BDR rounding.
#include "lrb_stream.cuh"
#include "lrs_internal.h"

namespace lrs {
LRS_LRB_STREAM_VARIANTS(find_lrb_stream_bdr, kBDR)
}  // namespace lrs
