// Union of per-token routes per query block, for attention over strictly
// causal routes.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary, limits
// section: sharing one route among a block's tokens lets a token's route
// depend on later tokens; the strictly causal variant routes every token by
// its own prefix of the block (hga_route_causal).  The tensor-core attention
// keeps 64-query blocks, so a block attends the union of its tokens' routed
// chunks, and each chunk carries a 64-bit mask of the tokens that routed to
// it: a token whose bit is clear sees that chunk as masked.
//
// One 256-thread CTA per (b, g, block m):
//   1. a bitmap over the Nc history chunks marks every routed chunk (the
//      64 tokens x k entries; -1 is padding, other out-of-range ids are
//      skipped and flagged);
//   2. a scan of the bitmap's popcounts ranks the marked chunks in ascending
//      order: ulist[rank] = chunk;
//   3. every entry ORs its token's bit into the mask of its chunk's rank;
//   ucount = the number of marked chunks (<= min(64 k, Nc) = ucap).
#include "common.cuh"

namespace hga {

namespace {

constexpr int kUnionThreads = 256;

__global__ void __launch_bounds__(kUnionThreads) route_union_kernel(const int32_t *__restrict__ idx, int seg_len,
                                                                    int topk, int n_chunks, int ucap,
                                                                    int32_t *__restrict__ ulist,
                                                                    unsigned long long *__restrict__ umask,
                                                                    int32_t *__restrict__ ucount, unsigned *status) {
    extern __shared__ uint8_t smem_raw[];
    const int n_words = (n_chunks + 31) / 32;
    unsigned long long *mask = reinterpret_cast<unsigned long long *>(smem_raw);  // [ucap]
    uint32_t *bits = reinterpret_cast<uint32_t *>(mask + ucap);                   // [n_words]
    int *prefix = reinterpret_cast<int *>(bits + n_words);                         // [n_words]
    __shared__ int warp_tot[kUnionThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nqb = seg_len / 64;
    const long long bgm = blockIdx.x;  // (b * Hkv + g) * nqb + m
    const long long bg = bgm / nqb;
    const int m = (int)(bgm % nqb);
    const int32_t *tok = idx + (bg * seg_len + (long long)m * 64) * topk;  // [64][k]

    for (int w = tid; w < n_words; w += kUnionThreads) bits[w] = 0u;
    for (int u = tid; u < ucap; u += kUnionThreads) mask[u] = 0ull;
    __syncthreads();
    for (int e = tid; e < 64 * topk; e += kUnionThreads) {
        const int j = tok[e];
        if (j >= 0 && j < n_chunks) atomicOr(&bits[j >> 5], 1u << (j & 31));
        else if (j != -1) atomicOr(status, kDevBadIndex);
    }
    __syncthreads();
    // exclusive scan of the words' popcounts, each thread owning a contiguous run of words
    const int per = (n_words + kUnionThreads - 1) / kUnionThreads;
    const int w0 = tid * per, w1 = min(w0 + per, n_words);
    int own = 0;
    for (int w = w0; w < w1; ++w) own += __popc(bits[w]);
    int x = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    int before = 0;
    for (int v = 0; v < warp; ++v) before += warp_tot[v];
    int run = before + x - own;
    for (int w = w0; w < w1; ++w) {
        prefix[w] = run;
        uint32_t b = bits[w];
        int r = run;
        while (b) {
            const int bit = __ffs(b) - 1;
            if (r < ucap) ulist[bgm * ucap + r] = w * 32 + bit;
            ++r;
            b &= b - 1;
        }
        run = r;
    }
    __syncthreads();
    int total = 0;
    for (int v = 0; v < kUnionThreads / 32; ++v) total += warp_tot[v];
    for (int e = tid; e < 64 * topk; e += kUnionThreads) {
        const int j = tok[e];
        if (j < 0 || j >= n_chunks) continue;
        const int rank = prefix[j >> 5] + __popc(bits[j >> 5] & ((1u << (j & 31)) - 1u));
        if (rank < ucap) atomicOr(&mask[rank], 1ull << (e / topk));
    }
    __syncthreads();
    const int cnt = min(total, ucap);
    for (int u = tid; u < cnt; u += kUnionThreads) umask[bgm * ucap + u] = mask[u];
    for (int u = cnt + tid; u < ucap; u += kUnionThreads) {
        ulist[bgm * ucap + u] = -1;
        umask[bgm * ucap + u] = 0ull;
    }
    if (tid == 0) ucount[bgm] = cnt;
}

}  // namespace

int route_union_cap(const hga_params_t &p) {
    const long long cap = 64ll * p.topk;
    return (int)(cap < p.n_hist_chunks ? cap : (p.n_hist_chunks > 0 ? p.n_hist_chunks : 1));
}

size_t route_union_bytes(const hga_params_t &p) {
    const long long blocks = (long long)p.batch * p.n_kv_heads * (p.seg_len / 64);
    const long long cap = route_union_cap(p);
    auto up = [](long long b) { return (b + 255) & ~255ll; };
    return (size_t)(up(blocks * 4) + up(blocks * cap * 4) + up(blocks * cap * 8));
}

UnionView route_union_view(const hga_params_t &p, void *ws) {
    const long long blocks = (long long)p.batch * p.n_kv_heads * (p.seg_len / 64);
    const long long cap = route_union_cap(p);
    auto up = [](long long b) { return (b + 255) & ~255ll; };
    uint8_t *base = static_cast<uint8_t *>(ws);
    UnionView v;
    v.cap = (int)cap;
    v.count = reinterpret_cast<int32_t *>(base);
    v.list = reinterpret_cast<int32_t *>(base + up(blocks * 4));
    v.mask = reinterpret_cast<unsigned long long *>(base + up(blocks * 4) + up(blocks * cap * 4));
    return v;
}

hga_status_t launch_route_union(const hga_params_t &p, const int32_t *idx_tok, const UnionView &v, unsigned *status,
                                cudaStream_t stream) {
    const unsigned blocks = (unsigned)((long long)p.batch * p.n_kv_heads * (p.seg_len / 64));
    if (blocks == 0) return HGA_OK;
    const int n_words = (p.n_hist_chunks + 31) / 32;
    const size_t smem = (size_t)v.cap * 8 + (size_t)n_words * 8;
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(route_union_kernel), (int)smem);
    if (e != cudaSuccess) return record_cuda(e);
    route_union_kernel<<<blocks, kUnionThreads, smem, stream>>>(idx_tok, p.seg_len, p.topk, p.n_hist_chunks, v.cap,
                                                                v.list, v.mask, v.count, status);
    return record_cuda(cudaGetLastError());
}

}  // namespace hga
