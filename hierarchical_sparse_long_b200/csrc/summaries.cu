// Chunk summaries: the mean of each 64-token chunk's keys, per KV head.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.1:
// one compact summary vector per closed chunk stays resident in GPU memory
// and grows with the context (author abstract).  The summary is read here as
// the mean of the chunk's keys.
//
// HBM-bound: every key byte is read once with 16-byte coalesced loads and
// D*4 bytes are written per chunk.  One warp reduces one chunk; each lane
// owns 16 bytes of a row and walks every (32 / lanes_per_row)-th row, so a
// warp instruction reads 512 contiguous bytes.  The reduction order is fixed
// (per-lane sequential, then a fixed butterfly), so summaries built in one
// pass and summaries appended segment by segment are bit-identical.
#include "common.cuh"

namespace hga {

template <typename T, int D>
__global__ void __launch_bounds__(256) summaries_kernel(const T *__restrict__ k, long long head_stride,
                                                        int n_slices, int chunk, int first_chunk,
                                                        int n_chunks, float *__restrict__ summ, int cap) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int LPR = D / VEC;   // lanes per row
    constexpr int RPI = 32 / LPR;  // rows per warp step
    static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "unsupported head_dim");
    const int lane = threadIdx.x & 31;
    const long long task = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (task >= (long long)n_slices * n_chunks) return;
    const int slice = (int)(task / n_chunks);
    const int j = first_chunk + (int)(task % n_chunks);
    const int col = (lane % LPR) * VEC;
    const int rslot = lane / LPR;
    const T *base = k + ((long long)slice * head_stride + (long long)j * chunk) * D + col;

    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    int r = rslot;
    // 8 loads in flight per lane
    for (; r + 7 * RPI < chunk; r += 8 * RPI) {
        float v[8][VEC];
#pragma unroll
        for (int u = 0; u < 8; ++u) Vec16<T>::load(base + (long long)(r + u * RPI) * D, v[u]);
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] += v[u][e];
    }
    for (; r < chunk; r += RPI) {
        float v[VEC];
        Vec16<T>::load(base + (long long)r * D, v);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += v[e];
    }
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    if (rslot == 0) {
        float *dst = summ + ((long long)slice * cap + j) * D + col;
        const float n = (float)chunk;
#pragma unroll
        for (int e = 0; e < VEC; e += 4) {
            float4 o = make_float4(acc[e] / n, acc[e + 1] / n, acc[e + 2] / n, acc[e + 3] / n);
            *reinterpret_cast<float4 *>(dst + e) = o;
        }
    }
}

template <typename T, int D>
static hga_status_t launch_t(const void *k, long long head_stride, int bh, int chunk, int first_chunk,
                             int n_chunks, float *summ, int cap, cudaStream_t stream) {
    const long long tasks = (long long)bh * n_chunks;
    const int warps_per_block = 8;
    const long long blocks = (tasks + warps_per_block - 1) / warps_per_block;
    summaries_kernel<T, D><<<(unsigned)blocks, 32 * warps_per_block, 0, stream>>>(
        static_cast<const T *>(k), head_stride, bh, chunk, first_chunk, n_chunks, summ, cap);
    return record_cuda(cudaGetLastError());
}

hga_status_t launch_summaries(const void *k, long long head_stride, int bh, int head_dim, int chunk,
                              int first_chunk, int n_chunks, hga_dtype_t dtype, float *summ, int cap,
                              cudaStream_t stream) {
    if (n_chunks == 0 || bh == 0) return HGA_OK;
    if (dtype == HGA_BF16) {
        if (head_dim == 128)
            return launch_t<__nv_bfloat16, 128>(k, head_stride, bh, chunk, first_chunk, n_chunks, summ, cap, stream);
        return launch_t<__nv_bfloat16, 64>(k, head_stride, bh, chunk, first_chunk, n_chunks, summ, cap, stream);
    }
    if (head_dim == 128)
        return launch_t<float, 128>(k, head_stride, bh, chunk, first_chunk, n_chunks, summ, cap, stream);
    return launch_t<float, 64>(k, head_stride, bh, chunk, first_chunk, n_chunks, summ, cap, stream);
}

}  // namespace hga
