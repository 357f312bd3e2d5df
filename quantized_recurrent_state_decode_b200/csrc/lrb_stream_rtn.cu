// lrb_stream_rtn.cu -- compiled variants of the streaming Low-Rank Bypass
// decode step, RTN rounding.
#include "lrb_stream.cuh"
#include "lrs_internal.h"

namespace lrs {
LRS_LRB_STREAM_VARIANTS(find_lrb_stream_rtn, kRTN)
}  // namespace lrs
