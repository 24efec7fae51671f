// Query-block routing: score every closed history chunk against the query
// block's summary and keep the top-k chunks.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.1:
// the current query block scores the resident chunk summaries to select the
// most relevant history chunks; the router has no learned weights and carries
// no gradient.  Readings fixed here: the block summary is the fp32 mean of
// the block's queries over the G heads of a KV group, the score is
// fp32 dot / sqrt(D), and the k best chunks are taken by (score descending,
// chunk index ascending) and listed in ascending chunk order.
//
// One CTA per (batch, kv head, query block).  The CTA reads its G*q_block
// query rows once with 16-byte coalesced loads (the kernel's HBM traffic),
// scores the L2-resident summaries with one thread per chunk (fp32 FFMA, no
// tensor cores, so every score is an fp32 dot product in a fixed order),
// then finds the k-th largest score by a 4-pass 8-bit radix select on the
// order-preserving score bits and collects the chunks above it plus the
// lowest-index chunks tied with it.
#include "common.cuh"

namespace hga {

// Order-preserving 32-bit image of an fp32 score (larger score -> larger
// value; -0 and +0 map to the same value).
__device__ __forceinline__ uint32_t ordered_bits(float s) {
    uint32_t u = __float_as_uint(s);
    if (s == 0.0f) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T, int D>
__global__ void __launch_bounds__(256) route_kernel(const T *__restrict__ q, const float *__restrict__ summ,
                                                    int cap, int32_t *__restrict__ idx, int n_q_heads,
                                                    int n_kv_heads, int seg_len, int q_block, int n_chunks,
                                                    int topk, float inv_sqrt_d) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int LPR = D / VEC;
    constexpr int NSLOT = 256 / LPR;
    extern __shared__ uint32_t ord[];  // n_chunks ordered score images
    __shared__ float part[NSLOT][D + 1];
    __shared__ float qbar[D];
    __shared__ int hist[256];
    __shared__ int chosen[64];
    __shared__ int n_chosen;
    __shared__ uint32_t sel_prefix;
    __shared__ int sel_remaining;
    __shared__ int warp_ties[8];
    __shared__ int ties_before;

    const int nqb = seg_len / q_block;
    const int m = blockIdx.x % nqb;
    const int bg = blockIdx.x / nqb;  // b * Hkv + g
    const int b = bg / n_kv_heads, g = bg % n_kv_heads;
    const int G = n_q_heads / n_kv_heads;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // 1. block summary: mean over G heads x q_block rows, fixed order; every
    //    thread keeps 8 independent 16-byte loads in flight
    {
        const int col = (tid % LPR) * VEC, slot = tid / LPR;
        float acc[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
        const int rows = G * q_block;
        int r = slot;
        for (; r + 7 * NSLOT < rows; r += 8 * NSLOT) {
            float v[8][VEC];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int rr = r + u * NSLOT;
                const int h = g * G + rr / q_block, i = m * q_block + rr % q_block;
                Vec16<T>::load(q + (((long long)b * n_q_heads + h) * seg_len + i) * D + col, v[u]);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[e] += v[u][e];
        }
        for (; r < rows; r += NSLOT) {
            const int h = g * G + r / q_block, i = m * q_block + r % q_block;
            float v[VEC];
            Vec16<T>::load(q + (((long long)b * n_q_heads + h) * seg_len + i) * D + col, v);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] += v[e];
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) part[slot][col + e] = acc[e];
    }
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
        for (int sl = 0; sl < NSLOT; ++sl) s += part[sl][tid];
        qbar[tid] = s / (float)(G * q_block);
    }
    if (tid == 0) n_chosen = 0;
    __syncthreads();

    // 2. scores; one thread per chunk, four interleaved partial dot products
    //    over d (mod 4) summed in a fixed order
    const float *sb = summ + (long long)bg * cap * D;
    for (int j = tid; j < n_chunks; j += 256) {
        const float4 *row = reinterpret_cast<const float4 *>(sb + (long long)j * D);
        float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll 8
        for (int e = 0; e < D / 4; ++e) {
            const float4 v = row[e];
            d0 = fmaf(qbar[4 * e + 0], v.x, d0);
            d1 = fmaf(qbar[4 * e + 1], v.y, d1);
            d2 = fmaf(qbar[4 * e + 2], v.z, d2);
            d3 = fmaf(qbar[4 * e + 3], v.w, d3);
        }
        ord[j] = ordered_bits(((d0 + d1) + (d2 + d3)) * inv_sqrt_d);
    }
    __syncthreads();

    int32_t *out = idx + ((long long)bg * nqb + m) * topk;
    const int keff = topk < n_chunks ? topk : n_chunks;
    if (keff == n_chunks) {
        // every chunk is routed
        for (int a = tid; a < topk; a += 256) out[a] = a < n_chunks ? a : -1;
        return;
    }

    // 3. radix select (4 passes of 8 bits, most significant first) of the
    //    keff-th largest score image: sel_prefix ends as that value and
    //    sel_remaining as how many chunks equal to it are taken
    if (tid == 0) {
        sel_prefix = 0u;
        sel_remaining = keff;
    }
    uint32_t mask = 0u;
    for (int shift = 24; shift >= 0; shift -= 8) {
        hist[tid] = 0;
        __syncthreads();
        const uint32_t prefix = sel_prefix;
        for (int base = 0; base < n_chunks; base += 256) {  // warp-uniform trip count
            const int j = base + tid;
            const uint32_t v = j < n_chunks ? ord[j] : 0u;
            const bool in = j < n_chunks && (v & mask) == prefix;
            const int bin = (int)((v >> shift) & 255u);
            // one shared atomic per distinct bin of the warp
            const unsigned act = __ballot_sync(0xffffffffu, in);
            if (in) {
                const unsigned peers = __match_any_sync(act, bin);
                if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[bin], __popc(peers));
            }
        }
        __syncthreads();
        if (warp == 0) {
            // bins from the top: find the bin holding the remaining-th largest
            int rem = sel_remaining;
            int above = 0;  // count in bins above the current 32-bin group
            for (int grp = 7; grp >= 0; --grp) {
                const int c = hist[grp * 32 + lane];
                // inclusive suffix sum within the group (higher bins first)
                int suf = c;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_down_sync(0xffffffffu, suf, off);
                    if (lane + off < 32) suf += y;
                }
                const int total = __shfl_sync(0xffffffffu, suf, 0);
                if (above + total >= rem) {
                    // the bin is the highest lane whose suffix (>= itself) reaches rem
                    const unsigned hit = __ballot_sync(0xffffffffu, above + suf >= rem);
                    const int bl = 31 - __clz(hit);
                    const int above_bin = above + __shfl_sync(0xffffffffu, suf, bl) -
                                          __shfl_sync(0xffffffffu, c, bl);
                    if (lane == 0) {
                        sel_prefix = prefix | ((uint32_t)(grp * 32 + bl) << shift);
                        sel_remaining = rem - above_bin;
                    }
                    break;
                }
                above += total;
            }
        }
        mask |= 255u << shift;
        __syncthreads();
    }
    const uint32_t thr = sel_prefix;
    const int take_ties = sel_remaining;

    // 4. collect: every chunk above the threshold, then the lowest-index
    //    take_ties chunks equal to it (ties go to the lower chunk index)
    for (int j = tid; j < n_chunks; j += 256)
        if (ord[j] > thr) chosen[atomicAdd(&n_chosen, 1)] = j;
    if (tid == 0) ties_before = 0;
    __syncthreads();
    for (int base = 0; base < n_chunks; base += 256) {
        const int j = base + tid;
        const bool tie = j < n_chunks && ord[j] == thr;
        const unsigned bal = __ballot_sync(0xffffffffu, tie);
        if (lane == 0) warp_ties[warp] = __popc(bal);
        __syncthreads();
        int rank = ties_before + __popc(bal & ((1u << lane) - 1u));
        for (int w = 0; w < warp; ++w) rank += warp_ties[w];
        if (tie && rank < take_ties) chosen[keff - take_ties + rank] = j;
        __syncthreads();
        if (tid == 0)
            for (int w = 0; w < 8; ++w) ties_before += warp_ties[w];
        __syncthreads();
        if (ties_before >= take_ties) break;
    }
    __syncthreads();

    // 5. the keff chosen chunks in ascending order, then -1 padding
    if (tid < keff) {
        const int me = chosen[tid];
        int rank = 0;
        for (int a = 0; a < keff; ++a) rank += chosen[a] < me;
        out[rank] = me;
    } else if (tid < topk) {
        out[tid] = -1;
    }
}

template <typename T, int D>
static hga_status_t launch_t(const hga_params_t &p, const void *q, const float *summ, int cap, int32_t *idx,
                             cudaStream_t stream) {
    const size_t smem = sizeof(uint32_t) * (p.n_hist_chunks > 0 ? p.n_hist_chunks : 1);
    auto kern = route_kernel<T, D>;
    if (smem > 32 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return record_cuda(e);
    }
    const int nqb = p.seg_len / p.q_block;
    const unsigned grid = (unsigned)(p.batch * p.n_kv_heads * nqb);
    const float inv_sqrt_d = (float)(1.0 / __builtin_sqrt((double)p.head_dim));
    kern<<<grid, 256, smem, stream>>>(static_cast<const T *>(q), summ, cap, idx, p.n_q_heads, p.n_kv_heads,
                                       p.seg_len, p.q_block, p.n_hist_chunks, p.topk, inv_sqrt_d);
    return record_cuda(cudaGetLastError());
}

hga_status_t launch_route(const hga_params_t &p, const void *q, const float *summ, int cap, int32_t *idx,
                          cudaStream_t stream) {
    if (p.dtype == HGA_BF16)
        return p.head_dim == 128 ? launch_t<__nv_bfloat16, 128>(p, q, summ, cap, idx, stream)
                                 : launch_t<__nv_bfloat16, 64>(p, q, summ, cap, idx, stream);
    return p.head_dim == 128 ? launch_t<float, 128>(p, q, summ, cap, idx, stream)
                             : launch_t<float, 64>(p, q, summ, cap, idx, stream);
}

}  // namespace hga
