// Chunk summaries: the mean of each 64-token chunk's keys, per KV head.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.1:
// one compact summary vector per closed chunk stays resident in GPU memory
// and grows with the context (author abstract).  The summary is read here as
// the mean of the chunk's keys.
//
// HBM-bound: every key byte is read once with 16-byte coalesced loads and
// D*4 bytes are written per chunk.  One 256-thread CTA reduces one chunk:
// each thread owns 16 bytes of a row and a fixed set of rows (all its loads
// are in flight together), and the row slots are then summed through shared
// memory in a fixed order, so summaries built in one pass and summaries
// appended segment by segment are bit-identical.
#include "common.cuh"

namespace hga {

template <typename T, int D>
__global__ void __launch_bounds__(256) summaries_kernel(const T *__restrict__ k, long long head_stride,
                                                        int n_slices, int chunk, int first_chunk,
                                                        int n_chunks, int k_first_chunk,
                                                        float *__restrict__ summ, int cap) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int LPR = D / VEC;     // threads per row
    constexpr int NSLOT = 256 / LPR; // row slots
    static_assert(LPR >= 1 && LPR <= 256 && 256 % LPR == 0, "unsupported head_dim");
    __shared__ float part[NSLOT][D + 1];
    const int tid = threadIdx.x;
    const int slice = (int)(blockIdx.x / n_chunks);
    const int j = first_chunk + (int)(blockIdx.x % n_chunks);
    const int col = (tid % LPR) * VEC;
    const int rslot = tid / LPR;
    const T *base = k + ((long long)slice * head_stride + (long long)(j - k_first_chunk) * chunk) * D + col;

    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    int r = rslot;
    for (; r + 3 * NSLOT < chunk; r += 4 * NSLOT) {
        float v[4][VEC];
#pragma unroll
        for (int u = 0; u < 4; ++u) Vec16<T>::load(base + (long long)(r + u * NSLOT) * D, v[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] += v[u][e];
    }
    for (; r < chunk; r += NSLOT) {
        float v[VEC];
        Vec16<T>::load(base + (long long)r * D, v);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += v[e];
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) part[rslot][col + e] = acc[e];
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
#pragma unroll
        for (int sl = 0; sl < NSLOT; ++sl) s += part[sl][tid];
        summ[((long long)slice * cap + j) * D + tid] = s / (float)chunk;
    }
}

template <typename T, int D>
static hga_status_t launch_t(const void *k, long long head_stride, int bh, int chunk, int first_chunk,
                             int n_chunks, int k_first_chunk, float *summ, int cap, cudaStream_t stream) {
    const long long blocks = (long long)bh * n_chunks;
    summaries_kernel<T, D><<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const T *>(k), head_stride, bh,
                                                                 chunk, first_chunk, n_chunks, k_first_chunk,
                                                                 summ, cap);
    return record_cuda(cudaGetLastError());
}

hga_status_t launch_summaries(const void *k, long long head_stride, int bh, int head_dim, int chunk,
                              int first_chunk, int n_chunks, hga_dtype_t dtype, float *summ, int cap,
                              cudaStream_t stream, int k_first_chunk) {
    if (n_chunks == 0 || bh == 0) return HGA_OK;
    const int k0 = k_first_chunk;
    if (dtype == HGA_BF16) {
        if (head_dim == 128)
            return launch_t<__nv_bfloat16, 128>(k, head_stride, bh, chunk, first_chunk, n_chunks, k0, summ, cap,
                                                stream);
        return launch_t<__nv_bfloat16, 64>(k, head_stride, bh, chunk, first_chunk, n_chunks, k0, summ, cap, stream);
    }
    if (head_dim == 128)
        return launch_t<float, 128>(k, head_stride, bh, chunk, first_chunk, n_chunks, k0, summ, cap, stream);
    return launch_t<float, 64>(k, head_stride, bh, chunk, first_chunk, n_chunks, k0, summ, cap, stream);
}

}  // namespace hga
