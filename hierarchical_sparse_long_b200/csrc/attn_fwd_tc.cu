// tcgen05 forward kernel (in progress).
#include "common.cuh"

namespace hga {
bool attn_fwd_tc_supported(const hga_params_t &) { return false; }
hga_status_t launch_attn_fwd_tc(const hga_params_t &, const void *, const void *, const void *, const void *,
                                const void *, const int32_t *, void *, float *, unsigned *, cudaStream_t) {
    return HGA_ERR_UNSUPPORTED;
}
}  // namespace hga
