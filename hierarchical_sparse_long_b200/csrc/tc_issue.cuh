// MMA issue helper shared by the tcgen05 attention kernels.
#pragma once

#include <cstdint>

namespace hga {
namespace tc {

// One lane of a converged warp (the same lane on every call with the full mask).  An
// MMA-issuing warp runs its loop (waits included) converged and elects one lane for
// each tcgen05.mma and for the commits that track those MMAs, so every MMA and its
// commit come from the same thread.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile("{\n\t.reg .b32 rx;\n\t.reg .pred px;\n\telect.sync rx|px, %1;\n\t@px mov.s32 %0, 1;\n\t}"
                 : "+r"(pred)
                 : "r"(0xffffffffu));
    return pred != 0;
}

}  // namespace tc
}  // namespace hga
