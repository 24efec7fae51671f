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
// then ranks 64-bit keys (order-preserving score bits, inverted chunk index)
// with a shared-memory bitonic sort.
#include "common.cuh"

namespace hga {

__device__ __forceinline__ unsigned long long rank_key(float s, int j) {
    uint32_t u = __float_as_uint(s);
    if (s == 0.0f) u = 0u;  // -0 and +0 are the same score
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)ord << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)j);
}

template <typename T, int D>
__global__ void __launch_bounds__(256) route_kernel(const T *__restrict__ q, const float *__restrict__ summ,
                                                    int cap, int32_t *__restrict__ idx, int n_q_heads,
                                                    int n_kv_heads, int seg_len, int q_block, int n_chunks,
                                                    int topk, int npow2, float inv_sqrt_d) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int LPR = D / VEC;
    constexpr int NSLOT = 256 / LPR;
    extern __shared__ unsigned long long keys[];  // npow2 entries
    __shared__ float part[NSLOT][D + 1];
    __shared__ float qbar[D];
    __shared__ int chosen[64];

    const int nqb = seg_len / q_block;
    const int m = blockIdx.x % nqb;
    const int bg = blockIdx.x / nqb;  // b * Hkv + g
    const int b = bg / n_kv_heads, g = bg % n_kv_heads;
    const int G = n_q_heads / n_kv_heads;
    const int tid = threadIdx.x;

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
    __syncthreads();

    // 2. scores -> rank keys; one thread per chunk, four interleaved partial
    //    dot products over d (mod 4) summed in a fixed order
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
        const float dot = (d0 + d1) + (d2 + d3);
        keys[j] = rank_key(dot * inv_sqrt_d, j);
    }
    for (int j = n_chunks + tid; j < npow2; j += 256) keys[j] = 0ull;  // below every real key
    __syncthreads();

    // 3. bitonic sort, descending
    for (int size = 2; size <= npow2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < npow2 / 2; t += 256) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool desc = ((lo & size) == 0);
                const unsigned long long a = keys[lo], c = keys[hi];
                if ((a < c) == desc) { keys[lo] = c; keys[hi] = a; }
            }
            __syncthreads();
        }
    }

    // 4. the k_eff best, emitted in ascending chunk order, then -1 padding
    const int keff = topk < n_chunks ? topk : n_chunks;
    if (tid < keff) chosen[tid] = (int)(0xFFFFFFFFu - (uint32_t)(keys[tid] & 0xFFFFFFFFull));
    __syncthreads();
    int32_t *out = idx + ((long long)bg * nqb + m) * topk;
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
    int npow2 = 1;
    while (npow2 < p.n_hist_chunks) npow2 <<= 1;
    const size_t smem = sizeof(unsigned long long) * npow2;
    auto kern = route_kernel<T, D>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return record_cuda(e);
    }
    const int nqb = p.seg_len / p.q_block;
    const unsigned grid = (unsigned)(p.batch * p.n_kv_heads * nqb);
    const float inv_sqrt_d = (float)(1.0 / __builtin_sqrt((double)p.head_dim));
    kern<<<grid, 256, smem, stream>>>(static_cast<const T *>(q), summ, cap, idx, p.n_q_heads, p.n_kv_heads,
                                       p.seg_len, p.q_block, p.n_hist_chunks, p.topk, npow2, inv_sqrt_d);
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
