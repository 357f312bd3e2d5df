// chunk_sr.cu -- compiled variants of the chunked (multi-token) update with
// SR rounding at the chunk's end.
#include "chunk_gated.cuh"

namespace lrs {
LRS_CHUNK_VARIANTS(find_chunk_kernel_sr, kSR)
}  // namespace lrs
