// step_instances.cuh -- the compiled variants of the fused decode step: one
// translation unit per (rounding mode, I/O element type) includes this and
// defines its lookup with LRS_STEP_VARIANTS, so the variants build in
// parallel.
#pragma once

#include "lrs_internal.h"
#include "step_kernel.cuh"

// Defines `const void* NAME(int C, int group, int update_kind, int gate_kind)`
// returning the kernel for (C = d_v / 32, group rows) with rounding MODE and
// element type IO, or nullptr when that combination is not compiled.
#define LRS_STEP_VARIANTS(NAME, MODE, IO)                                                        \
    namespace {                                                                                  \
    template <int C, int GROUP>                                                                  \
    const void* NAME##_pick(int update_kind, int gate_kind) {                                    \
        if (update_kind == kGated && gate_kind == kGatePerKey)                                   \
            return reinterpret_cast<const void*>(                                                \
                &step_kernel<C, GROUP, kGated, kGatePerKey, MODE, IO>);                          \
        if (update_kind == kGated && gate_kind == kGate)                                         \
            return reinterpret_cast<const void*>(&step_kernel<C, GROUP, kGated, kGate, MODE, IO>); \
        if (update_kind == kDelta && gate_kind == kGate)                                         \
            return reinterpret_cast<const void*>(&step_kernel<C, GROUP, kDelta, kGate, MODE, IO>); \
        return nullptr;                                                                          \
    }                                                                                            \
    }                                                                                            \
    const void* NAME(int C, int group, int update_kind, int gate_kind) {                         \
        if (C == 4 && group == 16) return NAME##_pick<4, 16>(update_kind, gate_kind);            \
        if (C == 4 && group == 32) return NAME##_pick<4, 32>(update_kind, gate_kind);            \
        if (C == 2 && group == 16) return NAME##_pick<2, 16>(update_kind, gate_kind);            \
        if (C == 2 && group == 32) return NAME##_pick<2, 32>(update_kind, gate_kind);            \
        if (C == 2 && group == 64) return NAME##_pick<2, 64>(update_kind, gate_kind);            \
        return nullptr;                                                                          \
    }
