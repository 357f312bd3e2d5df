// step_sr.cu -- compiled variants of the fused decode step with
// the SR rounding mode (one translation unit per mode to build in parallel).
#include "lrs_internal.h"
#include "step_kernel.cuh"

namespace lrs {

template <int C, int GROUP>
static const void* pick(int update_kind, int gate_kind) {
    if (update_kind == kGated && gate_kind == kGatePerKey)
        return reinterpret_cast<const void*>(&step_kernel<C, GROUP, kGated, kGatePerKey, kSR>);
    if (update_kind == kGated && gate_kind == kGate)
        return reinterpret_cast<const void*>(&step_kernel<C, GROUP, kGated, kGate, kSR>);
    if (update_kind == kDelta && gate_kind == kGate)
        return reinterpret_cast<const void*>(&step_kernel<C, GROUP, kDelta, kGate, kSR>);
    return nullptr;
}

const void* find_step_kernel_sr(int C, int group, int update_kind, int gate_kind) {
    if (C == 4 && group == 16) return pick<4, 16>(update_kind, gate_kind);
    if (C == 4 && group == 32) return pick<4, 32>(update_kind, gate_kind);
    if (C == 2 && group == 16) return pick<2, 16>(update_kind, gate_kind);
    if (C == 2 && group == 32) return pick<2, 32>(update_kind, gate_kind);
    if (C == 2 && group == 64) return pick<2, 64>(update_kind, gate_kind);
    return nullptr;
}

}  // namespace lrs
