// C ABI of the HGA library: argument validation, kernel selection and the
// device status word.  Every check runs on the host before anything is
// enqueued, so a rejected call leaves the stream untouched.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace {

// An NVTX range named after the entry point around every C-ABI call (the
// host-side validation and the launches), for timelines taken with a
// profiler; without one attached a push/pop is a call through a no-op stub.
struct CallRange {
    explicit CallRange(const char *name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange &) = delete;
    CallRange &operator=(const CallRange &) = delete;
};

__device__ unsigned int g_status_word;

thread_local std::string t_last_error;

constexpr int kMaxDevices = 64;
std::atomic<unsigned *> g_status_ptr[kMaxDevices];
std::mutex g_status_mu;

// Address of this device's status word (looked up once per device with the
// device current, as the symbol's host-side name is not a device address).
unsigned *status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (unsigned *p = g_status_ptr[dev].load(std::memory_order_acquire)) return p;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_ptr[dev].load(std::memory_order_relaxed)) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev].store(static_cast<unsigned *>(ptr), std::memory_order_release);
    }
    return g_status_ptr[dev].load(std::memory_order_relaxed);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by route / fwd / bwd / fetch.
hga_status_t check_params(const hga_params_t *p) {
    if (!p) return HGA_ERR_INVALID_ARG;
    if (p->batch < 1 || p->n_q_heads < 1 || p->n_kv_heads < 1) return HGA_ERR_INVALID_ARG;
    if (p->n_q_heads % p->n_kv_heads) return HGA_ERR_INVALID_ARG;
    if (p->dtype != HGA_BF16 && p->dtype != HGA_FP32) return HGA_ERR_INVALID_ARG;
    if (p->head_dim != 64 && p->head_dim != 128) return HGA_ERR_UNSUPPORTED;
    // query blocks of 64, or a one-token segment (decode: seg_len = q_block = 1)
    if (p->chunk != 64 || !(p->q_block == 64 || (p->q_block == 1 && p->seg_len == 1))) return HGA_ERR_UNSUPPORTED;
    if (p->topk < 1 || p->topk > 64) return HGA_ERR_INVALID_ARG;
    if (p->sink_chunks < 0 || p->sink_chunks > p->topk) return HGA_ERR_INVALID_ARG;
    if (p->seg_len < 1 || p->seg_len % p->q_block || (p->q_block > 1 && p->seg_len % p->chunk))
        return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks < 0) return HGA_ERR_INVALID_ARG;
    if (p->seg_head_stride < p->seg_len) return HGA_ERR_INVALID_ARG;
    if (p->hist_head_stride < 0) return HGA_ERR_INVALID_ARG;
    if (p->hist_head_stride != 0 && p->hist_head_stride < (long long)p->n_hist_chunks * p->chunk)
        return HGA_ERR_INVALID_ARG;
    const int nqb = p->seg_len / p->q_block;
    if (!(p->qblock_begin == 0 && p->qblock_end == 0)) {
        if (p->qblock_begin < 0 || p->qblock_end <= p->qblock_begin || p->qblock_end > nqb)
            return HGA_ERR_INVALID_ARG;
    }
    return HGA_OK;
}

}  // namespace

namespace hga {
hga_status_t record_cuda(cudaError_t e) {
    if (e == cudaSuccess) return HGA_OK;
    t_last_error = cudaGetErrorString(e);
    return HGA_ERR_CUDA;
}
void record_error(const char *msg) { t_last_error = msg; }
}  // namespace hga

extern "C" {

const char *hga_status_string(hga_status_t s) {
    switch (s) {
    case HGA_OK: return "HGA_OK";
    case HGA_ERR_INVALID_ARG: return "HGA_ERR_INVALID_ARG";
    case HGA_ERR_UNSUPPORTED: return "HGA_ERR_UNSUPPORTED";
    case HGA_ERR_CUDA: return "HGA_ERR_CUDA";
    case HGA_ERR_DEVICE_CHECK: return "HGA_ERR_DEVICE_CHECK";
    case HGA_ERR_TIMEOUT: return "HGA_ERR_TIMEOUT";
    }
    return "HGA_ERR_UNKNOWN";
}

const char *hga_last_error(void) { return t_last_error.c_str(); }

hga_status_t hga_build_summaries(const void *k, long long head_stride, int batch, int n_kv_heads, int head_dim,
                                 int chunk, int first_chunk, int n_chunks, hga_dtype_t dtype, float *summ,
                                 int summ_cap_chunks, cudaStream_t stream) {
    CallRange range("hga_build_summaries");
    if (batch < 1 || n_kv_heads < 1 || n_chunks < 0 || first_chunk < 0 || chunk < 1) return HGA_ERR_INVALID_ARG;
    if (dtype != HGA_BF16 && dtype != HGA_FP32) return HGA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return HGA_ERR_UNSUPPORTED;
    if ((long long)first_chunk + n_chunks > summ_cap_chunks) return HGA_ERR_INVALID_ARG;
    if (head_stride < (long long)(first_chunk + n_chunks) * chunk) return HGA_ERR_INVALID_ARG;
    if (n_chunks == 0) return HGA_OK;
    if (!k || !summ || !aligned16(k) || !aligned16(summ)) return HGA_ERR_INVALID_ARG;
    return hga::launch_summaries(k, head_stride, batch * n_kv_heads, head_dim, chunk, first_chunk, n_chunks, dtype,
                                 summ, summ_cap_chunks, stream);
}

hga_status_t hga_route(const hga_params_t *p, const void *q, const float *summ, int summ_cap_chunks, int32_t *idx,
                       cudaStream_t stream) {
    CallRange range("hga_route");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (summ_cap_chunks < p->n_hist_chunks) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 16384) return HGA_ERR_UNSUPPORTED;
    if (!q || !idx || !aligned16(q)) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 0 && (!summ || !aligned16(summ))) return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    return hga::launch_route(*p, q, summ, summ_cap_chunks, idx, status, stream);
}

hga_status_t hga_route_groups(const hga_params_t *p, const void *q, const float *gsumm, int gsumm_cap_groups,
                              const int32_t *idx, int group, int topg, int32_t *gidx, cudaStream_t stream) {
    CallRange range("hga_route_groups");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (group != 8 && group != 16 && group != 32) return HGA_ERR_INVALID_ARG;
    const int gpc = p->chunk / group;
    if (topg < 1 || topg > p->topk * gpc) return HGA_ERR_INVALID_ARG;
    if ((long long)gsumm_cap_groups < (long long)p->n_hist_chunks * gpc) return HGA_ERR_INVALID_ARG;
    if (!q || !idx || !gidx || !aligned16(q)) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 0 && (!gsumm || !aligned16(gsumm))) return HGA_ERR_INVALID_ARG;
    return hga::launch_route_groups(*p, q, gsumm, gsumm_cap_groups, idx, group, topg, gidx, stream);
}

hga_status_t hga_route_groups_tiered(const hga_params_t *p, const void *q, const float *host_gsumm,
                                     int gsumm_cap_groups, const int32_t *idx, int group, int topg, int32_t *gidx,
                                     float *stage_gsumm, int stage_slots, int32_t *scratch, int32_t *idx_remapped,
                                     int32_t *n_fetched, cudaStream_t stream) {
    CallRange range("hga_route_groups_tiered");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (p->q_block != 64) return HGA_ERR_UNSUPPORTED;
    if (group != 8 && group != 16 && group != 32) return HGA_ERR_INVALID_ARG;
    const int gpc = p->chunk / group;
    if (topg < 1 || topg > p->topk * gpc) return HGA_ERR_INVALID_ARG;
    if ((long long)gsumm_cap_groups < (long long)p->n_hist_chunks * gpc) return HGA_ERR_INVALID_ARG;
    // the cache's tiles are (b, g, chunk) of the group-summary history
    if (p->hist_head_stride != (long long)gsumm_cap_groups * group || gsumm_cap_groups % gpc) {
        hga::record_error("hga_route_groups_tiered: hist_head_stride must be gsumm_cap_groups * group "
                          "(a whole number of chunks)");
        return HGA_ERR_INVALID_ARG;
    }
    if (!q || !idx || !gidx || !host_gsumm || !stage_gsumm || !scratch || !idx_remapped || stage_slots < 1)
        return HGA_ERR_INVALID_ARG;
    for (const void *ptr : {q, (const void *)host_gsumm, (const void *)stage_gsumm})
        if (!aligned16(ptr)) return HGA_ERR_INVALID_ARG;
    const int keff = p->topk < p->n_hist_chunks ? p->topk : p->n_hist_chunks;
    const long long worst = 2ll * (p->seg_len / p->q_block) * p->batch * p->n_kv_heads * keff;
    const long long distinct = (long long)p->batch * p->n_kv_heads * p->n_hist_chunks;
    if ((worst < distinct ? worst : distinct) > stage_slots) {
        hga::record_error("hga_route_groups_tiered: stage_slots below twice the chunks one call can route "
                          "(or every routable chunk)");
        return HGA_ERR_INVALID_ARG;
    }
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    if (p->n_hist_chunks > 0) {
        st = hga::launch_fetch_group_summaries(*p, host_gsumm, group, idx, stage_gsumm, stage_slots, scratch,
                                               idx_remapped, n_fetched, status, stream);
        if (st != HGA_OK) return st;
    }
    return hga::launch_route_groups(*p, q, stage_gsumm, 0, idx, group, topg, gidx, stream, idx_remapped);
}

hga_status_t hga_route_causal(const hga_params_t *p, const void *q, const float *summ, int summ_cap_chunks,
                              int32_t *idx, cudaStream_t stream) {
    CallRange range("hga_route_causal");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (summ_cap_chunks < p->n_hist_chunks) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 16384) return HGA_ERR_UNSUPPORTED;
    if (!q || !idx || !aligned16(q)) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 0 && (!summ || !aligned16(summ))) return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    return hga::launch_route_causal(*p, q, summ, summ_cap_chunks, idx, status, stream);
}

hga_status_t hga_attn_fwd(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                          const void *k_seg, const void *v_seg, const int32_t *idx, void *out, float *lse,
                          cudaStream_t stream) {
    CallRange range("hga_attn_fwd");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (p->q_block != 64) return HGA_ERR_UNSUPPORTED;  // one-token segments go through hga_attn_decode
    if (!q || !k_seg || !v_seg || !idx || !out || !lse) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 0 && (!k_hist || !v_hist)) return HGA_ERR_INVALID_ARG;
    for (const void *ptr : {q, k_hist, v_hist, k_seg, v_seg, (const void *)out})
        if (ptr && !aligned16(ptr)) return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    // bf16 with head_dim 128 runs on the tcgen05 kernel and nowhere else; fp32
    // (and bf16 with head_dim 64) on the CUDA-core kernel
    if (hga::attn_fwd_tc_shape(*p)) {
        if (!hga::attn_fwd_tc_supported(*p)) {
            hga::record_error("hga_attn_fwd: the tcgen05 kernel cannot take this call (no TMA tensor-map "
                              "encoder in the driver, or a row coordinate beyond 32 bits)");
            return HGA_ERR_UNSUPPORTED;
        }
        return hga::launch_attn_fwd_tc(*p, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, status, stream);
    }
    return hga::launch_attn_fwd_simt(*p, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, status, stream);
}

hga_status_t hga_route_attn_fwd(const hga_params_t *p, const void *q, const float *summ, int summ_cap_chunks,
                                int32_t *idx, const void *k_hist, const void *v_hist, const void *k_seg,
                                const void *v_seg, void *out, float *lse, cudaStream_t stream) {
    CallRange range("hga_route_attn_fwd");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (p->q_block != 64) return HGA_ERR_UNSUPPORTED;  // one-token segments go through hga_attn_decode
    if (summ_cap_chunks < p->n_hist_chunks) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 16384) return HGA_ERR_UNSUPPORTED;
    if (!q || !idx || !k_seg || !v_seg || !out || !lse) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 0 && (!summ || !k_hist || !v_hist)) return HGA_ERR_INVALID_ARG;
    for (const void *ptr : {q, (const void *)summ, k_hist, v_hist, k_seg, v_seg, (const void *)out})
        if (ptr && !aligned16(ptr)) return HGA_ERR_INVALID_ARG;
    const bool tc = hga::attn_fwd_tc_shape(*p);
    if (tc && !hga::attn_fwd_tc_supported(*p)) {
        hga::record_error("hga_route_attn_fwd: the tcgen05 kernel cannot take this call (no TMA tensor-map "
                          "encoder in the driver, or a row coordinate beyond 32 bits)");
        return HGA_ERR_UNSUPPORTED;
    }
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    hga_params_t pr = *p;  // every block is routed
    pr.qblock_begin = pr.qblock_end = 0;
    st = hga::launch_route(pr, q, summ, summ_cap_chunks, idx, status, stream);
    if (st != HGA_OK) return st;
    if (tc) return hga::launch_attn_fwd_tc_after_route(*p, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, status,
                                                        stream);
    return hga::launch_attn_fwd_simt(*p, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, status, stream);
}

size_t hga_attn_bwd_workspace_size(const hga_params_t *p) {
    if (check_params(p) != HGA_OK) return 0;
    const size_t rows = (size_t)p->batch * p->n_q_heads * p->seg_len;
    return ((rows * sizeof(float)) + 255) & ~(size_t)255;
}

hga_status_t hga_attn_bwd(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                          const void *k_seg, const void *v_seg, const int32_t *idx, const void *out,
                          const float *lse, const void *dout, void *dq, void *dk_seg, void *dv_seg, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
    CallRange range("hga_attn_bwd");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (p->q_block != 64) return HGA_ERR_UNSUPPORTED;  // one-token segments go through hga_attn_decode
    if (p->qblock_begin != 0 || p->qblock_end != 0) return HGA_ERR_INVALID_ARG;
    if (!q || !k_seg || !v_seg || !idx || !out || !lse || !dout || !dq || !dk_seg || !dv_seg || !workspace)
        return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 0 && (!k_hist || !v_hist)) return HGA_ERR_INVALID_ARG;
    if (workspace_bytes < hga_attn_bwd_workspace_size(p)) return HGA_ERR_INVALID_ARG;
    for (const void *ptr : {q, k_hist, v_hist, k_seg, v_seg, out, dout, (const void *)dq, (const void *)dk_seg,
                            (const void *)dv_seg, (const void *)workspace, (const void *)lse})
        if (ptr && !aligned16(ptr)) return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    float *delta = static_cast<float *>(workspace);
    if (hga::attn_fwd_tc_shape(*p)) {
        if (!hga::attn_bwd_tc_supported(*p)) {
            hga::record_error("hga_attn_bwd: the tcgen05 kernel cannot take this call (no TMA tensor-map "
                              "encoder in the driver, or a row coordinate beyond 32 bits)");
            return HGA_ERR_UNSUPPORTED;
        }
        st = hga::launch_bwd_delta(*p, out, dout, delta, stream);
        if (st != HGA_OK) return st;
        return hga::launch_attn_bwd_tc(*p, q, k_hist, v_hist, k_seg, v_seg, idx, lse, delta, dout,
                                       static_cast<float *>(dq), static_cast<float *>(dk_seg),
                                       static_cast<float *>(dv_seg), status, stream);
    }
    return hga::launch_attn_bwd_simt(*p, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, dout, dq, dk_seg, dv_seg,
                                     delta, status, stream);
}

namespace {

// Checks shared by the group-routed and token-masked attention calls: the
// tcgen05 shape only (bf16, head_dim 128), every block, pointers as in
// hga_attn_fwd / hga_attn_bwd.
hga_status_t check_routed_attn(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                               const void *k_seg, const void *v_seg, const void *routes, const void *out,
                               const float *lse) {
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (p->q_block != 64) return HGA_ERR_UNSUPPORTED;
    if (!hga::attn_fwd_tc_shape(*p)) {
        hga::record_error("group-routed and token-masked attention run on the tcgen05 kernels only "
                          "(bf16, head_dim 128)");
        return HGA_ERR_UNSUPPORTED;
    }
    if (!hga::attn_fwd_tc_supported(*p)) {
        hga::record_error("the tcgen05 kernel cannot take this call (no TMA tensor-map encoder in the "
                          "driver, or a row coordinate beyond 32 bits)");
        return HGA_ERR_UNSUPPORTED;
    }
    if (!q || !k_seg || !v_seg || !routes || !out || !lse) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 0 && (!k_hist || !v_hist)) return HGA_ERR_INVALID_ARG;
    for (const void *ptr : {q, k_hist, v_hist, k_seg, v_seg, out})
        if (ptr && !aligned16(ptr)) return HGA_ERR_INVALID_ARG;
    return HGA_OK;
}

hga_status_t check_group_args(const hga_params_t *p, int group, int topg) {
    if (group != 8 && group != 16 && group != 32) return HGA_ERR_INVALID_ARG;
    const int gpc = p->chunk / group;
    if (topg < 1 || topg > p->topk * gpc || topg > 512) return HGA_ERR_INVALID_ARG;
    return HGA_OK;
}

hga_status_t check_bwd_outputs(const hga_params_t *p, const void *dout, const void *dq, const void *dk,
                               const void *dv) {
    if (p->qblock_begin != 0 || p->qblock_end != 0) return HGA_ERR_INVALID_ARG;
    if (!dout || !dq || !dk || !dv) return HGA_ERR_INVALID_ARG;
    for (const void *ptr : {dout, dq, dk, dv})
        if (!aligned16(ptr)) return HGA_ERR_INVALID_ARG;
    return HGA_OK;
}

size_t delta_bytes(const hga_params_t &p) {
    const size_t rows = (size_t)p.batch * p.n_q_heads * p.seg_len;
    return ((rows * sizeof(float)) + 255) & ~(size_t)255;
}

}  // namespace

hga_status_t hga_attn_fwd_groups(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                                 const void *k_seg, const void *v_seg, const int32_t *gidx, int group, int topg,
                                 void *out, float *lse, cudaStream_t stream) {
    CallRange range("hga_attn_fwd_groups");
    hga_status_t st = check_routed_attn(p, q, k_hist, v_hist, k_seg, v_seg, gidx, out, lse);
    if (st == HGA_OK) st = check_group_args(p, group, topg);
    if (st != HGA_OK) return st;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    const hga::FwdRoutes rt{gidx, topg, group, nullptr, nullptr};
    return hga::launch_attn_fwd_tc_routes(*p, q, k_hist, v_hist, k_seg, v_seg, rt, out, lse, status, stream);
}

hga_status_t hga_attn_bwd_groups(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                                 const void *k_seg, const void *v_seg, const int32_t *gidx, int group, int topg,
                                 const void *out, const float *lse, const void *dout, void *dq, void *dk_seg,
                                 void *dv_seg, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    CallRange range("hga_attn_bwd_groups");
    hga_status_t st = check_routed_attn(p, q, k_hist, v_hist, k_seg, v_seg, gidx, out, lse);
    if (st == HGA_OK) st = check_group_args(p, group, topg);
    if (st == HGA_OK) st = check_bwd_outputs(p, dout, dq, dk_seg, dv_seg);
    if (st != HGA_OK) return st;
    if (!workspace || !aligned16(workspace) || workspace_bytes < delta_bytes(*p)) return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    float *delta = static_cast<float *>(workspace);
    st = hga::launch_bwd_delta(*p, out, dout, delta, stream);
    if (st != HGA_OK) return st;
    const hga::FwdRoutes rt{gidx, topg, group, nullptr, nullptr};
    return hga::launch_attn_bwd_tc_routes(*p, q, k_hist, v_hist, k_seg, v_seg, rt, lse, delta, dout,
                                          static_cast<float *>(dq), static_cast<float *>(dk_seg),
                                          static_cast<float *>(dv_seg), status, stream);
}

size_t hga_attn_causal_workspace_size(const hga_params_t *p, int backward) {
    if (check_params(p) != HGA_OK || p->q_block != 64) return 0;
    return hga::route_union_bytes(*p) + (backward ? delta_bytes(*p) : 0);
}

hga_status_t hga_attn_fwd_causal(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                                 const void *k_seg, const void *v_seg, const int32_t *idx_tok, void *out, float *lse,
                                 void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    CallRange range("hga_attn_fwd_causal");
    hga_status_t st = check_routed_attn(p, q, k_hist, v_hist, k_seg, v_seg, idx_tok, out, lse);
    if (st != HGA_OK) return st;
    if (p->n_hist_chunks > 16384) return HGA_ERR_UNSUPPORTED;
    if (!workspace || !aligned16(workspace) || workspace_bytes < hga::route_union_bytes(*p))
        return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    const hga::UnionView u = hga::route_union_view(*p, workspace);
    st = hga::launch_route_union(*p, idx_tok, u, status, stream);
    if (st != HGA_OK) return st;
    const hga::FwdRoutes rt{u.list, u.cap, 0, u.count, u.mask};
    return hga::launch_attn_fwd_tc_routes(*p, q, k_hist, v_hist, k_seg, v_seg, rt, out, lse, status, stream);
}

hga_status_t hga_attn_bwd_causal(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                                 const void *k_seg, const void *v_seg, const int32_t *idx_tok, const void *out,
                                 const float *lse, const void *dout, void *dq, void *dk_seg, void *dv_seg,
                                 void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    CallRange range("hga_attn_bwd_causal");
    hga_status_t st = check_routed_attn(p, q, k_hist, v_hist, k_seg, v_seg, idx_tok, out, lse);
    if (st == HGA_OK) st = check_bwd_outputs(p, dout, dq, dk_seg, dv_seg);
    if (st != HGA_OK) return st;
    if (p->n_hist_chunks > 16384) return HGA_ERR_UNSUPPORTED;
    const size_t ub = hga::route_union_bytes(*p);
    if (!workspace || !aligned16(workspace) || workspace_bytes < ub + delta_bytes(*p)) return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    const hga::UnionView u = hga::route_union_view(*p, workspace);
    float *delta = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + ub);
    st = hga::launch_route_union(*p, idx_tok, u, status, stream);
    if (st == HGA_OK) st = hga::launch_bwd_delta(*p, out, dout, delta, stream);
    if (st != HGA_OK) return st;
    const hga::FwdRoutes rt{u.list, u.cap, 0, u.count, u.mask};
    return hga::launch_attn_bwd_tc_routes(*p, q, k_hist, v_hist, k_seg, v_seg, rt, lse, delta, dout,
                                          static_cast<float *>(dq), static_cast<float *>(dk_seg),
                                          static_cast<float *>(dv_seg), status, stream);
}

size_t hga_attn_decode_workspace_size(const hga_params_t *p, int n_local) {
    if (check_params(p) != HGA_OK || p->seg_len != 1 || n_local < 1) return 0;
    return hga::decode_workspace_bytes(*p, n_local);
}

hga_status_t hga_attn_decode(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                             const void *k_local, const void *v_local, int n_local, const int32_t *idx, void *out,
                             float *lse, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    CallRange range("hga_attn_decode");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (p->seg_len != 1 || p->q_block != 1 || n_local < 1 || p->seg_head_stride < n_local)
        return HGA_ERR_INVALID_ARG;
    if (p->n_q_heads / p->n_kv_heads > 8) return HGA_ERR_UNSUPPORTED;
    if (!q || !k_local || !v_local || !idx || !out || !lse || !workspace) return HGA_ERR_INVALID_ARG;
    if (p->n_hist_chunks > 0 && (!k_hist || !v_hist)) return HGA_ERR_INVALID_ARG;
    for (const void *ptr : {q, k_hist, v_hist, k_local, v_local, (const void *)out, (const void *)workspace})
        if (ptr && !aligned16(ptr)) return HGA_ERR_INVALID_ARG;
    if (workspace_bytes < hga::decode_workspace_bytes(*p, n_local)) return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    return hga::launch_decode(*p, q, k_hist, v_hist, k_local, v_local, n_local, idx, out, lse,
                              static_cast<float *>(workspace), status, stream);
}

size_t hga_tier_scratch_size(const hga_params_t *p, int stage_slots) {
    if (check_params(p) != HGA_OK || stage_slots < 1 || p->hist_head_stride < 1) return 0;
    const size_t bytes = hga::tier_scratch_entries(*p, stage_slots) * sizeof(int32_t);
    return (bytes + 255) & ~(size_t)255;
}

hga_status_t hga_tier_reset(const hga_params_t *p, int stage_slots, int32_t *scratch, cudaStream_t stream) {
    CallRange range("hga_tier_reset");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (stage_slots < 1 || p->hist_head_stride < 1 || !scratch) return HGA_ERR_INVALID_ARG;
    return hga::launch_tier_reset(*p, stage_slots, scratch, stream);
}

namespace {

// Argument checks shared by hga_fetch_tiered and hga_attn_fwd_tiered.  A
// fetch of `blocks` query blocks may need every routed tile of those blocks,
// and the tiles of the lag - 1 waves before it stay protected, so the cache
// must hold lag times that -- or every routable tile, after which nothing is
// ever evicted.
hga_status_t check_tiered(const hga_params_t *p, const void *host_k, const void *host_v, const int32_t *idx,
                          const void *stage_k, const void *stage_v, int stage_slots, const int32_t *scratch,
                          const int32_t *idx_remapped, int blocks, int lag) {
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (p->q_block != 64) return HGA_ERR_UNSUPPORTED;  // one-token segments go through hga_attn_decode
    if (p->hist_head_stride < 1 || p->hist_head_stride < (long long)p->n_hist_chunks * p->chunk)
        return HGA_ERR_INVALID_ARG;
    if (!host_k || !host_v || !idx || !stage_k || !stage_v || !scratch || !idx_remapped || stage_slots < 1)
        return HGA_ERR_INVALID_ARG;
    for (const void *ptr : {host_k, host_v, stage_k, stage_v})
        if (!aligned16(ptr)) return HGA_ERR_INVALID_ARG;
    const int keff = p->topk < p->n_hist_chunks ? p->topk : p->n_hist_chunks;
    const long long worst = (long long)lag * blocks * p->batch * p->n_kv_heads * keff;
    const long long distinct = (long long)p->batch * p->n_kv_heads * p->n_hist_chunks;
    if ((worst < distinct ? worst : distinct) > stage_slots) {
        hga::record_error("tiered: stage_slots below lag times the tiles one wave can route (or every routable tile)");
        return HGA_ERR_INVALID_ARG;
    }
    return HGA_OK;
}

}  // namespace

hga_status_t hga_fetch_tiered(const hga_params_t *p, const void *host_k, const void *host_v, const int32_t *idx,
                              int qblock_begin, int qblock_end, void *stage_k, void *stage_v, int stage_slots,
                              int32_t *scratch, int32_t *idx_remapped, int32_t *n_fetched, cudaStream_t copy_stream,
                              cudaEvent_t done) {
    CallRange range("hga_fetch_tiered");
    if (!p) return HGA_ERR_INVALID_ARG;
    const int nqb = p->q_block > 0 ? p->seg_len / p->q_block : 0;
    if (qblock_begin < 0 || qblock_end <= qblock_begin || qblock_end > nqb) return HGA_ERR_INVALID_ARG;
    hga_status_t st = check_tiered(p, host_k, host_v, idx, stage_k, stage_v, stage_slots, scratch, idx_remapped,
                                   qblock_end - qblock_begin, 2);
    if (st != HGA_OK) return st;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    st = hga::launch_fetch_tiered(*p, host_k, host_v, idx, qblock_begin, qblock_end, stage_k, stage_v, stage_slots,
                                  2, scratch, idx_remapped, n_fetched, status, copy_stream);
    if (st != HGA_OK) return st;
    if (done) return hga::record_cuda(cudaEventRecord(done, copy_stream));
    return HGA_OK;
}

hga_status_t hga_tier_offload(const hga_params_t *p, const void *k_seg, const void *v_seg, void *host_k,
                              void *host_v, long long dst_token, cudaStream_t stream) {
    CallRange range("hga_tier_offload");
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (!k_seg || !v_seg || !host_k || !host_v || dst_token < 0 || p->hist_head_stride < 1 ||
        dst_token + p->seg_len > p->hist_head_stride)
        return HGA_ERR_INVALID_ARG;
    for (void *hp : {host_k, host_v}) {
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, hp) != cudaSuccess || at.type != cudaMemoryTypeHost) {
            cudaGetLastError();
            hga::record_error("hga_tier_offload: host_k / host_v must be page-locked host memory");
            return HGA_ERR_INVALID_ARG;
        }
    }
    const size_t esize = p->dtype == HGA_BF16 ? 2 : 4;
    const size_t row = (size_t)p->head_dim * esize;
    const size_t width = (size_t)p->seg_len * row;
    const size_t rows = (size_t)p->batch * p->n_kv_heads;
    const size_t spitch = (size_t)p->seg_head_stride * row, dpitch = (size_t)p->hist_head_stride * row;
    for (int kv = 0; kv < 2; ++kv) {
        const void *src = kv ? v_seg : k_seg;
        uint8_t *dst = static_cast<uint8_t *>(kv ? host_v : host_k) + (size_t)dst_token * row;
        const cudaError_t e = cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, rows, cudaMemcpyDeviceToHost, stream);
        if (e != cudaSuccess) return hga::record_cuda(e);
    }
    return HGA_OK;
}

hga_status_t hga_attn_fwd_tiered(const hga_params_t *p, const void *q, const void *host_k, const void *host_v,
                                 const void *k_seg, const void *v_seg, const void *prev_k_seg,
                                 const void *prev_v_seg, const int32_t *idx, void *out, float *lse,
                                 void *stage_k, void *stage_v, int stage_slots, int32_t *scratch,
                                 int32_t *idx_remapped, int wave_blocks, int flags, int32_t *n_fetched,
                                 cudaStream_t stream, cudaStream_t copy_stream, hga_tier_sched_t *sched) {
    CallRange range("hga_attn_fwd_tiered");
    if (!p || wave_blocks < 1 || !sched || (flags & ~(HGA_TIER_RESET | HGA_TIER_CHAIN))) return HGA_ERR_INVALID_ARG;
    const int lag = sched->lag;
    if (lag < 2 || lag > HGA_TIER_MAX_LAG || sched->wave < 0 || !sched->start || !sched->fetched)
        return HGA_ERR_INVALID_ARG;
    for (int i = 0; i < lag; ++i)
        if (!sched->consumed[i]) return HGA_ERR_INVALID_ARG;
    const int nqb = p->q_block > 0 ? p->seg_len / p->q_block : 0;
    const int qb0 = (p->qblock_begin == 0 && p->qblock_end == 0) ? 0 : p->qblock_begin;
    const int qb1 = (p->qblock_begin == 0 && p->qblock_end == 0) ? nqb : p->qblock_end;
    hga_status_t st = check_tiered(p, host_k, host_v, idx, stage_k, stage_v, stage_slots, scratch, idx_remapped,
                                   wave_blocks, lag);
    if (st != HGA_OK) return st;
    if (!q || !k_seg || !v_seg || !out || !lse) return HGA_ERR_INVALID_ARG;
    if ((prev_k_seg == nullptr) != (prev_v_seg == nullptr)) return HGA_ERR_INVALID_ARG;
    if (prev_k_seg && (p->n_hist_chunks < p->seg_len / p->chunk || !aligned16(prev_k_seg) || !aligned16(prev_v_seg)))
        return HGA_ERR_INVALID_ARG;
    hga_params_t pa = *p;  // attention over the staging cache: route indices are slots
    pa.hist_head_stride = 0;
    pa.n_hist_chunks = stage_slots;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    const bool reset = (flags & HGA_TIER_RESET) != 0;
    cudaError_t e = cudaSuccess;
    if (reset || !(flags & HGA_TIER_CHAIN) || sched->wave == 0) {
        // the copy stream starts after everything already on the compute stream
        // (the route that wrote idx, the attention of earlier calls over the cache)
        e = cudaEventRecord(sched->start, stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(copy_stream, sched->start, 0);
        if (e != cudaSuccess) return hga::record_cuda(e);
    }
    if (reset) {
        st = hga::launch_tier_reset(*p, stage_slots, scratch, copy_stream);
        if (st != HGA_OK) return st;
        sched->wave = 0;
    }
    if (p->n_hist_chunks == 0) {
        // nothing routable: plain attention over the segment, after whatever the copy
        // stream holds (the caller may have written idx or the inputs there); it reads
        // idx itself, so the copy stream's later work waits for it
        if ((e = cudaEventRecord(sched->fetched, copy_stream)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(stream, sched->fetched, 0)) != cudaSuccess)
            return hga::record_cuda(e);
        st = hga_attn_fwd(p, q, stage_k, stage_v, k_seg, v_seg, idx, out, lse, stream);
        if (st != HGA_OK) return st;
        if ((e = cudaEventRecord(sched->start, stream)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(copy_stream, sched->start, 0)) != cudaSuccess)
            return hga::record_cuda(e);
        return HGA_OK;
    }
    for (int b0 = qb0; b0 < qb1; b0 += wave_blocks) {
        const int b1 = b0 + wave_blocks < qb1 ? b0 + wave_blocks : qb1;
        const long long h = sched->wave;
        cudaEvent_t consumed = sched->consumed[h % lag];
        // the fetch of wave h may evict the slots wave h - lag read: wait for that attention
        if (h >= lag && (e = cudaStreamWaitEvent(copy_stream, consumed, 0)) != cudaSuccess)
            return hga::record_cuda(e);
        st = hga::launch_fetch_tiered(*p, host_k, host_v, idx, b0, b1, stage_k, stage_v, stage_slots, lag, scratch,
                                      idx_remapped, n_fetched ? n_fetched + (b0 - qb0) / wave_blocks : nullptr,
                                      status, copy_stream, prev_k_seg, prev_v_seg);
        if (st != HGA_OK) return st;
        if ((e = cudaEventRecord(sched->fetched, copy_stream)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(stream, sched->fetched, 0)) != cudaSuccess)
            return hga::record_cuda(e);
        pa.qblock_begin = b0;
        pa.qblock_end = b1;
        st = hga_attn_fwd(&pa, q, stage_k, stage_v, k_seg, v_seg, idx_remapped, out, lse, stream);
        if (st != HGA_OK) return st;
        if ((e = cudaEventRecord(consumed, stream)) != cudaSuccess) return hga::record_cuda(e);
        sched->wave = h + 1;
    }
    return HGA_OK;
}

hga_status_t hga_segment_fwd_tiered(const hga_params_t *p, const void *q, const void *k_seg, const void *v_seg,
                                    const void *prev_k_seg, const void *prev_v_seg, float *summ,
                                    int summ_cap_chunks, int32_t *idx, void *host_k, void *host_v,
                                    void *out, float *lse, void *stage_k, void *stage_v, int stage_slots,
                                    int32_t *scratch, int32_t *idx_remapped, int wave_blocks, int flags,
                                    int32_t *n_fetched, cudaStream_t stream, cudaStream_t copy_stream,
                                    cudaStream_t route_stream, cudaStream_t offload_stream, hga_tier_sched_t *sched) {
    CallRange range("hga_segment_fwd_tiered");
    if (!p || !sched || (flags & ~HGA_TIER_RESET)) return HGA_ERR_INVALID_ARG;
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (!sched->inputs || !sched->offloaded[0] || !sched->offloaded[1] || !sched->routed || !sched->idx_free[0] ||
        !sched->idx_free[1] || !sched->start || sched->segment < 0)
        return HGA_ERR_INVALID_ARG;
    if (p->seg_len % p->chunk != 0) return HGA_ERR_INVALID_ARG;
    const int seg_chunks = p->seg_len / p->chunk;
    const long long T = (long long)p->n_hist_chunks * p->chunk;
    if ((long long)p->n_hist_chunks + seg_chunks > summ_cap_chunks || T + p->seg_len > p->hist_head_stride)
        return HGA_ERR_INVALID_ARG;
    if (!summ || !aligned16(summ) || !k_seg || !aligned16(k_seg)) return HGA_ERR_INVALID_ARG;
    const bool reset = (flags & HGA_TIER_RESET) != 0;
    cudaError_t e = cudaSuccess;
    if (reset) {  // the evaluation starts: the side streams after whatever came before it
        if ((e = cudaEventRecord(sched->start, stream)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(copy_stream, sched->start, 0)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(route_stream, sched->start, 0)) != cudaSuccess)
            return hga::record_cuda(e);
        sched->segment = 0;
    }
    const long long seg = sched->segment;
    // this segment's fetches read host rows the previous segment offloaded, or with
    // prev_k_seg (whose chunks come from device memory) the one before; waited for
    // here, before the offload below re-records the event of the ring
    const long long need = seg - (prev_k_seg ? 2 : 1);
    if (need >= 0 && (e = cudaStreamWaitEvent(copy_stream, sched->offloaded[need & 1], 0)) != cudaSuccess)
        return hga::record_cuda(e);
    // detach into the host tier once the segment's K/V are there
    if ((e = cudaEventRecord(sched->inputs, route_stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(offload_stream, sched->inputs, 0)) != cudaSuccess)
        return hga::record_cuda(e);
    st = hga_tier_offload(p, k_seg, v_seg, host_k, host_v, T, offload_stream);
    if (st != HGA_OK) return st;
    if ((e = cudaEventRecord(sched->offloaded[seg & 1], offload_stream)) != cudaSuccess) return hga::record_cuda(e);
    // the route; its idx buffer was last read by the fetches of segment seg - 2
    if (seg >= 2 && (e = cudaStreamWaitEvent(route_stream, sched->idx_free[seg & 1], 0)) != cudaSuccess)
        return hga::record_cuda(e);
    st = hga_route(p, q, summ, summ_cap_chunks, idx, route_stream);
    if (st != HGA_OK) return st;
    // this segment's fetches: after its route
    if ((e = cudaEventRecord(sched->routed, route_stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(copy_stream, sched->routed, 0)) != cudaSuccess)
        return hga::record_cuda(e);
    st = hga_attn_fwd_tiered(p, q, host_k, host_v, k_seg, v_seg, prev_k_seg, prev_v_seg, idx, out, lse, stage_k,
                             stage_v, stage_slots, scratch, idx_remapped, wave_blocks,
                             reset ? HGA_TIER_RESET : HGA_TIER_CHAIN, n_fetched, stream, copy_stream, sched);
    if (st != HGA_OK) return st;
    if ((e = cudaEventRecord(sched->idx_free[seg & 1], copy_stream)) != cudaSuccess) return hga::record_cuda(e);
    // detach: the segment's chunks become routable for the next segment
    st = hga::launch_summaries(k_seg, p->seg_head_stride, p->batch * p->n_kv_heads, p->head_dim, p->chunk,
                               p->n_hist_chunks, seg_chunks, p->dtype, summ, summ_cap_chunks, route_stream,
                               p->n_hist_chunks);
    if (st != HGA_OK) return st;
    sched->segment = seg + 1;
    return HGA_OK;
}

hga_status_t hga_segment_fwd(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                             const void *k_seg, const void *v_seg, float *summ, int summ_cap_chunks, int32_t *idx,
                             void *out, float *lse, int flags, cudaStream_t stream, cudaStream_t route_stream,
                             hga_tier_sched_t *sched) {
    CallRange range("hga_segment_fwd");
    if (!p || !sched || (flags & ~HGA_TIER_RESET)) return HGA_ERR_INVALID_ARG;
    hga_status_t st = check_params(p);
    if (st != HGA_OK) return st;
    if (!sched->start || !sched->routed || !sched->idx_free[0] || !sched->idx_free[1] || sched->segment < 0)
        return HGA_ERR_INVALID_ARG;
    if (p->seg_len % p->chunk != 0) return HGA_ERR_INVALID_ARG;
    const int seg_chunks = p->seg_len / p->chunk;
    if ((long long)p->n_hist_chunks + seg_chunks > summ_cap_chunks) return HGA_ERR_INVALID_ARG;
    if (!summ || !aligned16(summ) || !k_seg || !aligned16(k_seg)) return HGA_ERR_INVALID_ARG;
    cudaError_t e = cudaSuccess;
    if (flags & HGA_TIER_RESET) {  // the evaluation starts: the route stream after whatever came before it
        if ((e = cudaEventRecord(sched->start, stream)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(route_stream, sched->start, 0)) != cudaSuccess)
            return hga::record_cuda(e);
        sched->segment = 0;
    }
    const long long seg = sched->segment;
    // the route; its idx buffer was last read by the attention of segment seg - 2
    if (seg >= 2 && (e = cudaStreamWaitEvent(route_stream, sched->idx_free[seg & 1], 0)) != cudaSuccess)
        return hga::record_cuda(e);
    st = hga_route(p, q, summ, summ_cap_chunks, idx, route_stream);
    if (st != HGA_OK) return st;
    if ((e = cudaEventRecord(sched->routed, route_stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(stream, sched->routed, 0)) != cudaSuccess)
        return hga::record_cuda(e);
    st = hga_attn_fwd(p, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, stream);
    if (st != HGA_OK) return st;
    if ((e = cudaEventRecord(sched->idx_free[seg & 1], stream)) != cudaSuccess) return hga::record_cuda(e);
    // detach: the segment's chunks become routable for the next segment
    st = hga::launch_summaries(k_seg, p->seg_head_stride, p->batch * p->n_kv_heads, p->head_dim, p->chunk,
                               p->n_hist_chunks, seg_chunks, p->dtype, summ, summ_cap_chunks, route_stream,
                               p->n_hist_chunks);
    if (st != HGA_OK) return st;
    sched->segment = seg + 1;
    return HGA_OK;
}

hga_status_t hga_selftest_wait_timeout(long long wait_cycles, cudaStream_t stream) {
    CallRange range("hga_selftest_wait_timeout");
    if (wait_cycles < 1000 || wait_cycles > (1ll << 32)) return HGA_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    return hga::launch_selftest_wait_timeout(wait_cycles, status, stream);
}

hga_status_t hga_get_device_status(cudaStream_t stream, unsigned int *bits) {
    unsigned *status = status_ptr();
    if (!status) return hga::record_cuda(cudaErrorInvalidDevice);
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return hga::record_cuda(e);
    unsigned v = 0;
    e = cudaMemcpy(&v, status, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return hga::record_cuda(e);
    const unsigned zero = 0;
    e = cudaMemcpy(status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return hga::record_cuda(e);
    if (bits) *bits = v;
    if (v & HGA_DEV_TIMEOUT) return HGA_ERR_TIMEOUT;
    if (v) return HGA_ERR_DEVICE_CHECK;
    return HGA_OK;
}

}  // extern "C"
