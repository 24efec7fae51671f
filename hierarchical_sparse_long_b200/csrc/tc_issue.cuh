// MMA issue helper shared by the tcgen05 attention kernels.
#pragma once

#include <cstdint>

namespace hga {
namespace tc {

// One lane of a converged warp (the same lane on every call with the full mask).  A
// single thread issues a tcgen05.mma only about every 110-120 cycles, while an
// M128 N64 K16 MMA with both operands in shared memory occupies the tensor pipe for
// ~55: the pipe is fed by several issuing warps, each running its loop converged and
// electing one lane per MMA and for the commits that track those MMAs.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile("{\n\t.reg .b32 rx;\n\t.reg .pred px;\n\telect.sync rx|px, %1;\n\t@px mov.s32 %0, 1;\n\t}"
                 : "+r"(pred)
                 : "r"(0xffffffffu));
    return pred != 0;
}

}  // namespace tc
}  // namespace hga
