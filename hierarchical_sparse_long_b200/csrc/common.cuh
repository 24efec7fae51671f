// Shared device helpers of the HGA CUDA library (sm_100a).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hga.h"

namespace hga {

// Device status word bits (mirrors HGA_DEV_* in hga.h).
constexpr unsigned kDevBadIndex = HGA_DEV_BAD_INDEX;
constexpr unsigned kDevTimeout = HGA_DEV_TIMEOUT;
constexpr unsigned kDevStageFull = HGA_DEV_STAGE_FULL;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Loads VEC = 16 / sizeof(T) consecutive elements (one 16-byte vector) as fp32.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void load(const float *p, float *out) {
        float4 v = *reinterpret_cast<const float4 *>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float *out) {
        uint4 v = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

}  // namespace hga

// Host-side launchers (one translation unit each); all validate nothing --
// the C ABI layer has already checked every argument.
namespace hga {
// k_first_chunk: the chunk index of k's first row (0: k is the start of each slice)
hga_status_t launch_summaries(const void *k, long long head_stride, int bh, int head_dim, int chunk,
                              int first_chunk, int n_chunks, hga_dtype_t dtype, float *summ, int cap,
                              cudaStream_t stream, int k_first_chunk = 0);
hga_status_t launch_route(const hga_params_t &p, const void *q, const float *summ, int cap, int32_t *idx,
                          unsigned *status, cudaStream_t stream);
// Group-stage routes (groups of `group` tokens in the chosen chunks): gidx [B][Hkv][S/q_block][topg].
// slot_idx (may be null): the chunk routes remapped to staging slots of gsumm (one
// shared slice of staged group summaries, chunk / group rows per slot).
hga_status_t launch_route_groups(const hga_params_t &p, const void *q, const float *gsumm, long long cap,
                                 const int32_t *idx, int group, int topg, int32_t *gidx, cudaStream_t stream,
                                 const int32_t *slot_idx = nullptr);
// One fetch of the group summaries of every block's routed chunks into a staging
// cache (hga_route_groups_tiered); p.hist_head_stride = group summaries per (b, g) * group.
hga_status_t launch_fetch_group_summaries(const hga_params_t &p, const float *host_gsumm, int group,
                                          const int32_t *idx, float *stage, int stage_slots, int32_t *scratch,
                                          int32_t *idx_remapped, int32_t *n_fetched, unsigned *status,
                                          cudaStream_t stream);
// Strictly causal routes, one per token: idx [B][Hkv][S][topk].
hga_status_t launch_route_causal(const hga_params_t &p, const void *q, const float *summ, int cap, int32_t *idx,
                          unsigned *status, cudaStream_t stream);
hga_status_t launch_attn_fwd_simt(const hga_params_t &p, const void *q, const void *k_hist,
                                  const void *v_hist, const void *k_seg, const void *v_seg,
                                  const int32_t *idx, void *out, float *lse, unsigned *status,
                                  cudaStream_t stream);
hga_status_t launch_attn_bwd_simt(const hga_params_t &p, const void *q, const void *k_hist,
                                  const void *v_hist, const void *k_seg, const void *v_seg,
                                  const int32_t *idx, const void *out, const float *lse, const void *dout,
                                  void *dq, void *dk_seg, void *dv_seg, float *delta, unsigned *status,
                                  cudaStream_t stream);
hga_status_t launch_bwd_delta(const hga_params_t &p, const void *out, const void *dout, float *delta,
                              cudaStream_t stream);
bool attn_bwd_tc_supported(const hga_params_t &p);
hga_status_t launch_attn_bwd_tc(const hga_params_t &p, const void *q, const void *k_hist, const void *v_hist,
                                const void *k_seg, const void *v_seg, const int32_t *idx, const float *lse,
                                const float *delta, const void *dout, float *dq, float *dk, float *dv,
                                unsigned *status, cudaStream_t stream);
// bf16, head_dim 128, chunk 64, 64-query blocks: the shapes the tcgen05 kernels serve.
bool attn_fwd_tc_shape(const hga_params_t &p);
// attn_fwd_tc_shape and the TMA encoder is available and every row coordinate fits 32 bits.
bool attn_fwd_tc_supported(const hga_params_t &p);
// Routes that fill the history tiles of the tcgen05 attention kernels:
//   chunk routes   list = idx [.][per_block = topk] chunk ids, gs = 0, no masks;
//   group routes   list = gidx [.][per_block = topg] group ids of gs tokens;
//   token-masked   list = the union of a block's per-token routes [.][per_block]
//                  (ascending chunk ids), ucount entries valid per block, and
//                  umask[.][per_block]: bit i set when token i of the block
//                  routes to that chunk.
struct FwdRoutes {
    const int32_t *list;
    int per_block;
    int gs;
    const int32_t *ucount;
    const unsigned long long *umask;
};
hga_status_t launch_attn_fwd_tc_routes(const hga_params_t &p, const void *q, const void *k_hist, const void *v_hist,
                                       const void *k_seg, const void *v_seg, const FwdRoutes &rt, void *out,
                                       float *lse, unsigned *status, cudaStream_t stream);
// Per-block unions of per-token routes (route_union.cu): ulist / umask [.][cap],
// count [.] over the (b, g, block) triples, in a caller workspace.
struct UnionView {
    int cap;
    int32_t *count;
    int32_t *list;
    unsigned long long *mask;
};
int route_union_cap(const hga_params_t &p);
size_t route_union_bytes(const hga_params_t &p);
UnionView route_union_view(const hga_params_t &p, void *ws);
hga_status_t launch_route_union(const hga_params_t &p, const int32_t *idx_tok, const UnionView &v, unsigned *status,
                                cudaStream_t stream);
hga_status_t launch_attn_bwd_tc_routes(const hga_params_t &p, const void *q, const void *k_hist, const void *v_hist,
                                       const void *k_seg, const void *v_seg, const FwdRoutes &rt, const float *lse,
                                       const float *delta, const void *dout, float *dq, float *dk, float *dv,
                                       unsigned *status, cudaStream_t stream);
// The tcgen05 forward as a programmatic dependent of the route kernel launched
// just before it on the same stream (causal segment tiles first; the route is
// waited for before the history tiles).
hga_status_t launch_attn_fwd_tc_after_route(const hga_params_t &p, const void *q, const void *k_hist,
                                            const void *v_hist, const void *k_seg, const void *v_seg,
                                            const int32_t *idx, void *out, float *lse, unsigned *status,
                                            cudaStream_t stream);
hga_status_t launch_attn_fwd_tc(const hga_params_t &p, const void *q, const void *k_hist,
                                const void *v_hist, const void *k_seg, const void *v_seg,
                                const int32_t *idx, void *out, float *lse, unsigned *status,
                                cudaStream_t stream);
size_t decode_workspace_bytes(const hga_params_t &p, int n_local);
hga_status_t launch_decode(const hga_params_t &p, const void *q, const void *kh, const void *vh, const void *kl,
                           const void *vl, int n_local, const int32_t *idx, void *out, float *lse, float *ws,
                           unsigned *status, cudaStream_t stream);
// Tiered staging cache (tiered.cu): scratch entries, reset, and one fetch wave.
long long tier_tile_cap(const hga_params_t &p);
size_t tier_scratch_entries(const hga_params_t &p, int stage_slots);
hga_status_t launch_tier_reset(const hga_params_t &p, int stage_slots, int32_t *scratch, cudaStream_t stream);
hga_status_t launch_fetch_tiered(const hga_params_t &p, const void *host_k, const void *host_v,
                                 const int32_t *idx, int qb0, int qb1, void *stage_k, void *stage_v,
                                 int stage_slots, int lag, int32_t *scratch, int32_t *idx_remapped,
                                 int32_t *n_fetched, unsigned *status, cudaStream_t stream,
                                 const void *prev_k = nullptr, const void *prev_v = nullptr);
hga_status_t launch_selftest_wait_timeout(long long wait_cycles, unsigned *status, cudaStream_t stream);
hga_status_t record_cuda(cudaError_t e);
void record_error(const char *msg);

// Host helpers shared by the launchers (host.cu).
bool tma_encoder_available();
// 2-D TMA map over `rows` rows of 128 bf16 values (256 B), boxes of 64 values
// x box_rows rows, 128-byte swizzle; maps are cached per thread by
// (base, rows, box_rows).
bool tma_rows_map(CUtensorMap *map, const void *base, unsigned long long rows, unsigned box_rows = 64);
// 3-D TMA map over `groups` groups of `rows` rows of D (64 or 128) bf16 values,
// group g starting group_stride_rows rows after group g - 1; boxes of 64 values
// x 64 rows x 1 group, 128-byte swizzle; rows past `rows` read as zeros.
bool tma_group_rows_map(CUtensorMap *map, const void *base, int D, unsigned long long rows,
                        unsigned long long groups, unsigned long long group_stride_rows);
// cudaFuncAttributeMaxDynamicSharedMemorySize, set once per kernel and device.
cudaError_t set_max_dynamic_smem(const void *kernel, int bytes);
// Streaming multiprocessors of the current device (148 when it cannot be queried).
int sm_count();
}  // namespace hga
