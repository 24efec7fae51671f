// Tiered history: bring only the routed chunks' exact K/V from page-locked
// host memory into a device staging cache, and attend over it.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.2
// (tiered memory: detached history K/V in host RAM/NVMe; the GPU holds the
// active segment, the routed exact K/V and the chunk summaries, so device
// memory grows as O(S) + O(routing budget)) and the author abstract (HGA
// loads a bounded set of exact historical tokens for each query block).
//
// The staging buffer is a cache of `slots` chunk tiles (64 x D keys and the
// same values) shared by every (batch, kv head).  Its bookkeeping lives in a
// caller-owned int32 scratch and persists from call to call:
//   tile_slot[t]  slot holding tile t = (b*Hkv + g)*tile_cap + j, or -1
//   tile_mark[t]  last wave that routed to tile t (de-duplicates a wave)
//   slot_tile[s]  tile held by slot s, or -1
//   slot_wave[s]  last wave whose attention reads slot s
//   new_tile[], new_slot[]  this wave's fetch list
//   ctl           wave counter, allocation cursor, fetch count
// A fetch of query blocks [qb0, qb1) is one wave w, three kernels on the copy
// stream:
//   plan   (one CTA): the wave's distinct tiles; cached ones are re-stamped
//          with w, the others get free slots -- slots whose last reader is
//          wave w-lag or older, taken round-robin from a cursor, evicting their
//          old tile -- and form the fetch list;
//   copy   : an SM copy of each listed K and V tile straight from the mapped
//          host pages into its slot (16-byte loads, many in flight, so the
//          host link rather than the SMs is the bound; CTAs small enough to
//          share an SM with an attention CTA) -- or, for the chunks of the
//          segment that detached last, from its K/V still in device memory
//          (the same bytes the host history received), so a chunk crosses
//          the host link only when it is older than that;
//   remap  : idx_remapped = slot of each routed chunk (-1 stays -1).
// The caller guarantees that the attention of wave w-lag has finished before
// the fetch of wave w starts (hga_attn_fwd_tiered orders its two streams so);
// the attention of waves w-lag+1 .. w-1 may still run, and their slots are
// never evicted.  lag is 2 for the single fetches (hga_fetch_tiered, the
// group-summary cache).
// The chunk order inside each block's route list is unchanged, so attention
// over the staging cache runs the same arithmetic in the same order as
// attention over resident history.
#include "common.cuh"

namespace hga {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kFreeWave = -(1 << 30);  // slot_wave of an empty slot: free for every wave and lag

struct TierScratch {
    int32_t *tile_slot, *tile_mark, *slot_tile, *slot_wave, *new_tile, *new_slot, *ctl;
};

// Chunks [j0, j0 + nj) of every (b, g) read from device memory instead of the
// host (k == nullptr: none); slice bg starts bg * head_stride_bytes in.
struct DevSource {
    const uint4 *k, *v;
    long long head_stride_bytes, j0, nj;
    __device__ bool holds(long long j) const { return k != nullptr && j >= j0 && j < j0 + nj; }
};

TierScratch tier_layout(int32_t *base, long long n_tiles, int slots) {
    TierScratch s;
    s.tile_slot = base;
    s.tile_mark = s.tile_slot + n_tiles;
    s.slot_tile = s.tile_mark + n_tiles;
    s.slot_wave = s.slot_tile + slots;
    s.new_tile = s.slot_wave + slots;
    s.new_slot = s.new_tile + slots;
    s.ctl = s.new_slot + slots;  // [0] last wave, [1] cursor, [2] tiles fetched by the last wave
    return s;
}

__global__ void tier_reset_kernel(TierScratch s, long long n_tiles, int slots) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n_tiles; e += stride) {
        s.tile_slot[e] = -1;
        s.tile_mark[e] = -1;
    }
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < slots; e += stride) {
        s.slot_tile[e] = -1;
        s.slot_wave[e] = kFreeWave;
    }
    if (blockIdx.x == 0 && threadIdx.x < 4) s.ctl[threadIdx.x] = 0;
}

// Block-wide exclusive scan of one flag per thread; returns the prefix and
// writes the total to *total (every thread sees it after the call).
__device__ int block_scan(int f, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = f;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int v = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += y;
        }
        warp_sums[lane] = v;
        if (lane == 31) *total = v;
    }
    __syncthreads();
    const int excl = (warp > 0 ? warp_sums[warp - 1] : 0) + x - f;
    __syncthreads();  // warp_sums is reused by the next call
    return excl;
}

__global__ void __launch_bounds__(kPlanThreads) tier_plan_kernel(const int32_t *__restrict__ idx, int n_bg, int nqb,
                                                                 int topk, int qb0, int qb1, int n_chunks,
                                                                 long long tile_cap, int slots, int lag,
                                                                 TierScratch s, DevSource dev, int32_t *n_fetched,
                                                                 unsigned *status) {
    __shared__ int warp_sums[32];
    __shared__ int n_new, n_host, total, taken_sh, cursor_sh;
    const int tid = threadIdx.x;
    const int w = s.ctl[0] + 1;
    if (tid == 0) {
        n_new = 0;
        n_host = 0;
    }
    __syncthreads();
    // 1. the wave's distinct tiles: cached ones are stamped with w, the others listed
    const long long per_bg = (long long)(qb1 - qb0) * topk;
    const long long total_e = per_bg * n_bg;
    for (long long e = tid; e < total_e; e += kPlanThreads) {
        const int bg = (int)(e / per_bg);
        const long long r = e % per_bg;
        const int m = qb0 + (int)(r / topk), a = (int)(r % topk);
        const int j = idx[((long long)bg * nqb + m) * topk + a];
        if (j < 0 || j >= n_chunks) {
            if (j != -1) atomicOr(status, kDevBadIndex);
            continue;
        }
        const long long t = (long long)bg * tile_cap + j;
        if (atomicExch(&s.tile_mark[t], w) == w) continue;  // listed already by this wave
        const int slot = s.tile_slot[t];
        if (slot >= 0) {
            s.slot_wave[slot] = w;
        } else {
            const int p = atomicAdd(&n_new, 1);
            if (p < slots) s.new_tile[p] = (int32_t)t;
            if (!dev.holds(j)) atomicAdd(&n_host, 1);
        }
    }
    __syncthreads();
    const int need = n_new < slots ? n_new : slots;
    // 2. free slots (last reader wave <= w - lag) round-robin from the cursor
    if (tid == 0) {
        taken_sh = 0;
        cursor_sh = s.ctl[1];
    }
    __syncthreads();
    const int cursor = cursor_sh;
    int last = -1;
    for (int base = 0; base < slots; base += kPlanThreads) {
        if (taken_sh >= need) break;  // uniform: read after the barrier that ends the previous round
        const int off = base + tid;
        const int sl = off < slots ? (cursor + off) % slots : 0;
        const int f = (off < slots && s.slot_wave[sl] <= w - lag) ? 1 : 0;
        const int rank = taken_sh + block_scan(f, warp_sums, &total);
        if (f && rank < need) {
            const int t_new = s.new_tile[rank];
            const int t_old = s.slot_tile[sl];
            if (t_old >= 0) s.tile_slot[t_old] = -1;
            s.slot_tile[sl] = t_new;
            s.tile_slot[t_new] = sl;
            s.slot_wave[sl] = w;
            s.new_slot[rank] = sl;
            if (rank == need - 1) last = off;
        }
        __syncthreads();
        if (tid == 0) taken_sh += total;
        if (last >= 0) cursor_sh = (cursor + last + 1) % slots;
        __syncthreads();
    }
    if (tid == 0) {
        const int got = taken_sh < need ? taken_sh : need;
        if (got < n_new) atomicOr(status, kDevStageFull);  // unfetched tiles stay -1 after the remap
        s.ctl[0] = w;
        s.ctl[1] = cursor_sh;
        s.ctl[2] = got;
        if (n_fetched) *n_fetched = got < n_host ? got : n_host;  // the tiles that cross the host link
    }
}

// 128 threads and at most 64 registers a thread: small enough to share an SM with
// an attention CTA (which leaves neither the registers nor the threads of a
// larger copy CTA free), so a wave's fetch overlaps the previous wave's attention.
constexpr int kCopyThreads = 128;

template <int ROW_BYTES>
__global__ void __launch_bounds__(kCopyThreads, 8)
    tier_copy_kernel(const uint4 *__restrict__ host_k, const uint4 *__restrict__ host_v, long long head_stride_bytes,
                     long long tile_cap, int chunk, TierScratch s, DevSource dev, uint4 *__restrict__ stage_k,
                     uint4 *__restrict__ stage_v) {
    constexpr int V_PER_ROW = ROW_BYTES / 16;
    constexpr int PER = 4;  // vectors of K and of V a thread holds in flight
    const int n = s.ctl[2];
    const int tile_vecs = chunk * V_PER_ROW;
    for (int k = blockIdx.x; k < n; k += gridDim.x) {
        const long long t = s.new_tile[k];
        const int slot = s.new_slot[k];
        const long long bg = t / tile_cap, j = t % tile_cap;
        // host_v / stage_v are null when one tensor is staged (group summaries)
        const bool two = host_v != nullptr;
        const uint4 *sk, *sv;
        if (dev.holds(j)) {
            const long long off = (bg * dev.head_stride_bytes + (j - dev.j0) * chunk * ROW_BYTES) / 16;
            sk = dev.k + off;
            sv = two ? dev.v + off : nullptr;
        } else {
            const long long off = (bg * head_stride_bytes + j * chunk * ROW_BYTES) / 16;
            sk = host_k + off;
            sv = two ? host_v + off : nullptr;
        }
        uint4 *dk = stage_k + (long long)slot * tile_vecs, *dv = two ? stage_v + (long long)slot * tile_vecs : nullptr;
        // every load of a round is issued before its stores
        for (int e0 = threadIdx.x; e0 < tile_vecs; e0 += PER * kCopyThreads) {
            uint4 bk[PER], bv[PER];
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int e = e0 + u * kCopyThreads;
                if (e < tile_vecs) {
                    bk[u] = sk[e];
                    if (two) bv[u] = sv[e];
                }
            }
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int e = e0 + u * kCopyThreads;
                if (e < tile_vecs) {
                    dk[e] = bk[u];
                    if (two) dv[e] = bv[u];
                }
            }
        }
    }
}

__global__ void tier_remap_kernel(const int32_t *__restrict__ idx, int n_bg, int nqb, int topk, int qb0, int qb1,
                                  int n_chunks, long long tile_cap, const int32_t *__restrict__ tile_slot,
                                  int32_t *__restrict__ out) {
    const long long per_bg = (long long)(qb1 - qb0) * topk;
    const long long total = per_bg * n_bg;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int bg = (int)(e / per_bg);
        const long long r = e % per_bg;
        const int m = qb0 + (int)(r / topk), a = (int)(r % topk);
        const long long at = ((long long)bg * nqb + m) * topk + a;
        const int j = idx[at];
        out[at] = (j >= 0 && j < n_chunks) ? tile_slot[(long long)bg * tile_cap + j] : -1;
    }
}

}  // namespace

long long tier_tile_cap(const hga_params_t &p) { return p.hist_head_stride / p.chunk; }

size_t tier_scratch_entries(const hga_params_t &p, int stage_slots) {
    const long long n_tiles = (long long)p.batch * p.n_kv_heads * tier_tile_cap(p);
    return (size_t)(2 * n_tiles + 4ll * stage_slots + 4);
}

hga_status_t launch_tier_reset(const hga_params_t &p, int stage_slots, int32_t *scratch, cudaStream_t stream) {
    const long long n_tiles = (long long)p.batch * p.n_kv_heads * tier_tile_cap(p);
    const TierScratch s = tier_layout(scratch, n_tiles, stage_slots);
    const long long n = n_tiles > stage_slots ? n_tiles : stage_slots;
    const unsigned grid = (unsigned)((n + 255) / 256 > 1184 ? 1184 : (n + 255) / 256 + 1);
    tier_reset_kernel<<<grid, 256, 0, stream>>>(s, n_tiles, stage_slots);
    return record_cuda(cudaGetLastError());
}

namespace {

// One fetch wave of tiles of tile_rows rows of row_bytes bytes (K and V of a
// chunk, or one chunk's group summaries when host_v is null), tile j of (b, g)
// starting at row j * tile_rows of a slice of head_stride_rows rows.
hga_status_t fetch_wave(const hga_params_t &p, const void *host_k, const void *host_v, int tile_rows, int row_bytes,
                        long long head_stride_rows, long long tile_cap, const int32_t *idx, int qb0, int qb1,
                        void *stage_k, void *stage_v, int stage_slots, int lag, int32_t *scratch,
                        int32_t *idx_remapped, int32_t *n_fetched, unsigned *status, cudaStream_t stream,
                        const DevSource &dev) {
    const int n_bg = p.batch * p.n_kv_heads;
    const int nqb = p.seg_len / p.q_block;
    const TierScratch s = tier_layout(scratch, (long long)n_bg * tile_cap, stage_slots);
    void *dk = nullptr, *dv = nullptr;
    cudaError_t e = cudaHostGetDevicePointer(&dk, const_cast<void *>(host_k), 0);
    if (e == cudaSuccess && host_v) e = cudaHostGetDevicePointer(&dv, const_cast<void *>(host_v), 0);
    if (e != cudaSuccess) {
        cudaGetLastError();
        record_error("tiered fetch: the host history is not page-locked (mapped) host memory");
        return HGA_ERR_INVALID_ARG;
    }
    tier_plan_kernel<<<1, kPlanThreads, 0, stream>>>(idx, n_bg, nqb, p.topk, qb0, qb1, p.n_hist_chunks, tile_cap,
                                                     stage_slots, lag, s, dev, n_fetched, status);
    const long long head_stride_bytes = head_stride_rows * row_bytes;
    const unsigned g3 = (unsigned)(2 * sm_count());
    const uint4 *hk = static_cast<const uint4 *>(dk), *hv = static_cast<const uint4 *>(dv);
    uint4 *sk = static_cast<uint4 *>(stage_k), *sv = static_cast<uint4 *>(stage_v);
    if (row_bytes == 128)
        tier_copy_kernel<128><<<g3, kCopyThreads, 0, stream>>>(hk, hv, head_stride_bytes, tile_cap, tile_rows, s, dev,
                                                               sk, sv);
    else if (row_bytes == 256)
        tier_copy_kernel<256><<<g3, kCopyThreads, 0, stream>>>(hk, hv, head_stride_bytes, tile_cap, tile_rows, s, dev,
                                                               sk, sv);
    else
        tier_copy_kernel<512><<<g3, kCopyThreads, 0, stream>>>(hk, hv, head_stride_bytes, tile_cap, tile_rows, s, dev,
                                                               sk, sv);
    const long long marks = (long long)n_bg * (qb1 - qb0) * p.topk;
    const unsigned g1 = (unsigned)((marks + 255) / 256 > 1184 ? 1184 : (marks + 255) / 256);
    if (marks > 0)
        tier_remap_kernel<<<g1, 256, 0, stream>>>(idx, n_bg, nqb, p.topk, qb0, qb1, p.n_hist_chunks, tile_cap,
                                                  s.tile_slot, idx_remapped);
    return record_cuda(cudaGetLastError());
}

}  // namespace

hga_status_t launch_fetch_tiered(const hga_params_t &p, const void *host_k, const void *host_v,
                                 const int32_t *idx, int qb0, int qb1, void *stage_k, void *stage_v,
                                 int stage_slots, int lag, int32_t *scratch, int32_t *idx_remapped,
                                 int32_t *n_fetched, unsigned *status, cudaStream_t stream, const void *prev_k,
                                 const void *prev_v) {
    const int esize = p.dtype == HGA_BF16 ? 2 : 4;
    DevSource dev{nullptr, nullptr, 0, 0, 0};
    if (prev_k && prev_v) {  // the segment before this one: chunks [Nc - S / chunk, Nc)
        dev.k = static_cast<const uint4 *>(prev_k);
        dev.v = static_cast<const uint4 *>(prev_v);
        dev.head_stride_bytes = p.seg_head_stride * p.head_dim * esize;
        dev.nj = p.seg_len / p.chunk;
        dev.j0 = p.n_hist_chunks - dev.nj;
    }
    return fetch_wave(p, host_k, host_v, p.chunk, p.head_dim * esize, p.hist_head_stride, tier_tile_cap(p), idx, qb0,
                      qb1, stage_k, stage_v, stage_slots, lag, scratch, idx_remapped, n_fetched, status, stream, dev);
}

hga_status_t launch_fetch_group_summaries(const hga_params_t &p, const float *host_gsumm, int group,
                                          const int32_t *idx, float *stage, int stage_slots, int32_t *scratch,
                                          int32_t *idx_remapped, int32_t *n_fetched, unsigned *status,
                                          cudaStream_t stream) {
    // a tile = the chunk / group fp32 summaries of one chunk's groups; the slice of
    // (b, g) holds hist_head_stride / group of them
    const int gpc = p.chunk / group;
    const long long rows = p.hist_head_stride / group;
    return fetch_wave(p, host_gsumm, nullptr, gpc, p.head_dim * 4, rows, tier_tile_cap(p), idx, 0,
                      p.seg_len / p.q_block, stage, nullptr, stage_slots, 2, scratch, idx_remapped, n_fetched,
                      status, stream, DevSource{nullptr, nullptr, 0, 0, 0});
}

}  // namespace hga
