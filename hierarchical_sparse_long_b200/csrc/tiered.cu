// Tiered history: bring only the routed chunks' exact K/V from page-locked
// host memory into a device staging buffer.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.2
// (tiered memory: detached history K/V in host RAM/NVMe; the GPU holds the
// active segment, the routed exact K/V and the chunk summaries, so device
// memory grows as O(S) + O(routing budget)) and the author abstract (HGA
// loads a bounded set of exact historical tokens for each query block).
//
// Four kernels on the copy stream, for the query blocks [qb0, qb1):
//   mark   : flag every (b, g, chunk) the blocks route to;
//   scan   : number the flagged tiles -> slot_map[(b*Hkv+g)*Nc + j] = slot or -1,
//            slot_src[slot] = (b*Hkv+g)*Nc + j, n_fetched;
//   copy   : an SM copy of each needed 64 x D K and V tile straight from the
//            mapped host pages into the staging slots (16-byte loads, many in
//            flight, so the host link rather than the SMs is the bound);
//   remap  : idx_remapped = slot of each routed chunk (-1 stays -1).
// The chunk order inside each block's route list is unchanged, so attention
// over the staging buffer runs the same arithmetic in the same order as
// attention over resident history.
#include "common.cuh"

namespace hga {

namespace {

__global__ void tier_mark_kernel(const int32_t *__restrict__ idx, int n_bg, int nqb, int topk, int qb0, int qb1,
                                 int n_chunks, int32_t *__restrict__ slot_map, unsigned *status) {
    const long long per_bg = (long long)(qb1 - qb0) * topk;
    const long long total = per_bg * n_bg;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int bg = (int)(e / per_bg);
        const long long r = e % per_bg;
        const int m = qb0 + (int)(r / topk), a = (int)(r % topk);
        const int j = idx[((long long)bg * nqb + m) * topk + a];
        if (j >= 0 && j < n_chunks) slot_map[(long long)bg * n_chunks + j] = 1;
        else if (j != -1) atomicOr(status, kDevBadIndex);
    }
}

// Single-CTA exclusive scan over the flags (entries are 0 / 1).
__global__ void __launch_bounds__(1024) tier_scan_kernel(int32_t *__restrict__ slot_map, long long n,
                                                         int32_t *__restrict__ slot_src, int32_t *__restrict__ n_out) {
    __shared__ int warp_sums[32];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (long long base = 0; base < n; base += 1024) {
        const long long e = base + tid;
        const int f = (e < n) ? (slot_map[e] != 0) : 0;
        int x = f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, off);
                if (lane >= off) w += y;
            }
            warp_sums[lane] = w;
        }
        __syncthreads();
        const int excl = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x - f;
        if (e < n) {
            slot_map[e] = f ? excl : -1;
            if (f) slot_src[excl] = (int32_t)e;
        }
        __syncthreads();
        if (tid == 1023) carry = excl + f;
        __syncthreads();
    }
    if (tid == 0 && n_out) *n_out = carry;
}

template <int ROW_BYTES>
__global__ void __launch_bounds__(256) tier_copy_kernel(const uint4 *__restrict__ host_k, const uint4 *__restrict__ host_v,
                                                        long long head_stride_bytes, int n_chunks, int chunk,
                                                        const int32_t *__restrict__ slot_src,
                                                        const int32_t *__restrict__ n_fetched, uint4 *__restrict__ stage_k,
                                                        uint4 *__restrict__ stage_v) {
    constexpr int V_PER_ROW = ROW_BYTES / 16;
    const int n = *n_fetched;
    const int tile_vecs = chunk * V_PER_ROW;
    for (int slot = blockIdx.x; slot < n; slot += gridDim.x) {
        const int src = slot_src[slot];
        const int bg = src / n_chunks, j = src % n_chunks;
        const long long off = ((long long)bg * head_stride_bytes + (long long)j * chunk * ROW_BYTES) / 16;
        const uint4 *sk = host_k + off, *sv = host_v + off;
        uint4 *dk = stage_k + (long long)slot * tile_vecs, *dv = stage_v + (long long)slot * tile_vecs;
        // issue every load of this thread before the stores (tile = 2 x chunk*ROW_BYTES)
        constexpr int MAXV = 8;
        uint4 bk[MAXV], bv[MAXV];
        int cnt = 0;
        for (int e = threadIdx.x; e < tile_vecs && cnt < MAXV; e += blockDim.x, ++cnt) {
            bk[cnt] = sk[e];
            bv[cnt] = sv[e];
        }
        cnt = 0;
        for (int e = threadIdx.x; e < tile_vecs && cnt < MAXV; e += blockDim.x, ++cnt) {
            dk[e] = bk[cnt];
            dv[e] = bv[cnt];
        }
        for (int e = threadIdx.x + MAXV * blockDim.x; e < tile_vecs; e += blockDim.x) {
            dk[e] = sk[e];
            dv[e] = sv[e];
        }
    }
}

__global__ void tier_remap_kernel(const int32_t *__restrict__ idx, int n_bg, int nqb, int topk, int qb0, int qb1,
                                  int n_chunks, const int32_t *__restrict__ slot_map, int32_t *__restrict__ out) {
    const long long per_bg = (long long)(qb1 - qb0) * topk;
    const long long total = per_bg * n_bg;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int bg = (int)(e / per_bg);
        const long long r = e % per_bg;
        const int m = qb0 + (int)(r / topk), a = (int)(r % topk);
        const long long at = ((long long)bg * nqb + m) * topk + a;
        const int j = idx[at];
        out[at] = (j >= 0 && j < n_chunks) ? slot_map[(long long)bg * n_chunks + j] : -1;
    }
}

}  // namespace

hga_status_t launch_fetch_tiered(const hga_params_t &p, const void *host_k, const void *host_v,
                                 const int32_t *idx, int qb0, int qb1, void *stage_k, void *stage_v,
                                 int stage_slots, int32_t *slot_map, int32_t *idx_remapped, int32_t *n_fetched,
                                 unsigned *status, cudaStream_t stream) {
    const int n_bg = p.batch * p.n_kv_heads;
    const int nqb = p.seg_len / p.q_block;
    const long long n_map = (long long)n_bg * p.n_hist_chunks;
    int32_t *slot_src = slot_map + n_map;  // stage_slots entries after the map
    void *dk = nullptr, *dv = nullptr;
    cudaError_t e = cudaHostGetDevicePointer(&dk, const_cast<void *>(host_k), 0);
    if (e != cudaSuccess) { cudaGetLastError(); return HGA_ERR_INVALID_ARG; }
    e = cudaHostGetDevicePointer(&dv, const_cast<void *>(host_v), 0);
    if (e != cudaSuccess) { cudaGetLastError(); return HGA_ERR_INVALID_ARG; }
    if (n_map > 0) {
        e = cudaMemsetAsync(slot_map, 0, sizeof(int32_t) * n_map, stream);
        if (e != cudaSuccess) return record_cuda(e);
    }
    const long long marks = (long long)n_bg * (qb1 - qb0) * p.topk;
    const unsigned g1 = (unsigned)((marks + 255) / 256 > 1184 ? 1184 : (marks + 255) / 256);
    if (marks > 0 && n_map > 0)
        tier_mark_kernel<<<g1, 256, 0, stream>>>(idx, n_bg, nqb, p.topk, qb0, qb1, p.n_hist_chunks, slot_map, status);
    // n_fetched doubles as the copy kernel's tile count; keep a device copy even when the caller passes none
    int32_t *count = n_fetched ? n_fetched : slot_src + stage_slots;
    tier_scan_kernel<<<1, 1024, 0, stream>>>(slot_map, n_map, slot_src, count);
    const int esize = p.dtype == HGA_BF16 ? 2 : 4;
    const long long head_stride_bytes = p.hist_head_stride * p.head_dim * esize;
    const int row_bytes = p.head_dim * esize;
    const unsigned g3 = 148;
    if (row_bytes == 128)
        tier_copy_kernel<128><<<g3, 256, 0, stream>>>((const uint4 *)dk, (const uint4 *)dv, head_stride_bytes,
                                                      p.n_hist_chunks, p.chunk, slot_src, count, (uint4 *)stage_k,
                                                      (uint4 *)stage_v);
    else if (row_bytes == 256)
        tier_copy_kernel<256><<<g3, 256, 0, stream>>>((const uint4 *)dk, (const uint4 *)dv, head_stride_bytes,
                                                      p.n_hist_chunks, p.chunk, slot_src, count, (uint4 *)stage_k,
                                                      (uint4 *)stage_v);
    else
        tier_copy_kernel<512><<<g3, 256, 0, stream>>>((const uint4 *)dk, (const uint4 *)dv, head_stride_bytes,
                                                      p.n_hist_chunks, p.chunk, slot_src, count, (uint4 *)stage_k,
                                                      (uint4 *)stage_v);
    if (marks > 0)
        tier_remap_kernel<<<g1, 256, 0, stream>>>(idx, n_bg, nqb, p.topk, qb0, qb1, p.n_hist_chunks, slot_map,
                                                  idx_remapped);
    return record_cuda(cudaGetLastError());
}

}  // namespace hga
