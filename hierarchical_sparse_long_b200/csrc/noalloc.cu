// hga_attn_bwd_noalloc: the HGA backward for callers that cannot allocate.
//
// hga_attn_bwd needs a small device workspace (one fp32 row term per query
// row) that the caller allocates.  Some callers cannot do that: a plugin or
// serving runtime that hands this library its tensors and a stream but owns
// every byte of device memory through its own pool, or a hot path where a
// cudaMalloc (which may synchronise the device) is not allowed.  This entry
// point keeps that workspace in a fixed array inside the library instead, so
// the call allocates nothing; the caller still passes every input and output.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its 4 MiB until the process exits.  Its host-side name is
// only a stand-in, so its device address is looked up once per device, with
// that device current, on the first call made on that device.
#include <mutex>

#include "common.cuh"

namespace {

// fp32 row terms for up to 1,048,576 query rows (batch * q heads * segment length)
constexpr size_t kScratchFloats = size_t(1) << 20;

__device__ __align__(256) float g_bwd_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
float *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of this device's copy of the array (nullptr on failure).
float *scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
        if (e != cudaSuccess) {
            hga::record_cuda(e);
            return nullptr;
        }
        g_scratch_addr[dev] = static_cast<float *>(ptr);
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" hga_status_t hga_attn_bwd_noalloc(const hga_params_t *p, const void *q, const void *k_hist,
                                             const void *v_hist, const void *k_seg, const void *v_seg,
                                             const int32_t *idx, const void *out, const float *lse,
                                             const void *dout, void *dq, void *dk_seg, void *dv_seg,
                                             cudaStream_t stream) {
    const size_t need = hga_attn_bwd_workspace_size(p);
    // a shape hga_attn_bwd rejects gets hga_attn_bwd's own status (its checks run
    // before anything is enqueued)
    if (need == 0)
        return hga_attn_bwd(p, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, dout, dq, dk_seg, dv_seg, nullptr, 0,
                            stream);
    if (need > kScratchFloats * sizeof(float)) {
        hga::record_error("hga_attn_bwd_noalloc: batch * n_q_heads * seg_len exceeds the built-in "
                          "scratch of 1048576 rows; use hga_attn_bwd with a caller-allocated workspace");
        return HGA_ERR_INVALID_ARG;
    }
    float *scratch = scratch_for_current_device();
    if (!scratch) return HGA_ERR_CUDA;
    // The row terms are fully rewritten before they are read, so the array
    // needs no clearing between calls.
    return hga_attn_bwd(p, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, dout, dq, dk_seg, dv_seg, scratch,
                        kScratchFloats * sizeof(float), stream);
}
