// Exact-token HGA attention on CUDA cores (fp32 arithmetic): forward and
// backward.  This is the path for fp32 inputs (where tensor-core TF32 would
// not hold fp32 accuracy) and for shapes the tcgen05 kernels do not cover.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.1
// (exact K/V of the routed chunks attended next to a local window; routing
// without gradient, gather and attention differentiable) and section 2.2
// (segment-wise backward: history detached, only the active segment gets
// K/V gradients).
//
// Key tiles are 64 tokens: one routed history chunk, or one 64-token tile of
// the active segment (tiles 0..m for query block m, the last one masked
// causally).  A CTA holds 64 query rows; each of its 256 threads owns a
// 4 x 4 patch of every 64 x 64 score tile (rows 4*rg.., columns cg + 16*c).
#include "common.cuh"

namespace hga {

namespace {

constexpr int TILE = 64;
constexpr int NT = 256;

// Copies a 64 x D tile (row stride D in global) into shared fp32 rows of stride LD.
template <typename T, int D, int LD>
__device__ __forceinline__ void load_tile(float *dst, const T *src, int tid) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int PER_ROW = D / VEC;
    for (int e = tid; e < TILE * PER_ROW; e += NT) {
        const int r = e / PER_ROW, c = (e % PER_ROW) * VEC;
        float v[VEC];
        Vec16<T>::load(src + (long long)r * D + c, v);
#pragma unroll
        for (int u = 0; u < VEC; ++u) dst[r * LD + c + u] = v[u];
    }
}

// Builds the list of key tiles of query block m: the valid routed chunks
// (indices outside [-1, Nc) are flagged and skipped) then local tiles 0..m.
__device__ __forceinline__ int route_list(const int32_t *sel, int topk, int n_chunks, int *list,
                                          unsigned *status, bool report) {
    int n = 0;
    for (int a = 0; a < topk; ++a) {
        const int j = sel[a];
        if (j >= 0 && j < n_chunks) list[n++] = j;
        else if (j != -1 && report) atomicOr(status, kDevBadIndex);
    }
    return n;
}

}  // namespace

// ---------------------------------------------------------------- forward
template <typename T, int D>
__global__ void __launch_bounds__(NT) fwd_simt_kernel(hga_params_t p, const T *__restrict__ q,
                                                      const T *__restrict__ k_hist, const T *__restrict__ v_hist,
                                                      const T *__restrict__ k_seg, const T *__restrict__ v_seg,
                                                      const int32_t *__restrict__ idx, T *__restrict__ out,
                                                      float *__restrict__ lse, unsigned *status, int qb0, int n_blocks) {
    constexpr int LD = D + 1;
    constexpr int DPT = D / 16;  // output columns per thread
    extern __shared__ float sm[];
    float *Qs = sm;                 // [64][LD]
    float *Ks = Qs + TILE * LD;     // [64][LD]
    float *Vs = Ks + TILE * LD;     // [64][LD]
    float *Ps = Vs + TILE * LD;     // [64][65]
    __shared__ int tiles[64];
    __shared__ int s_nhist;

    const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
    const int G = p.n_q_heads / p.n_kv_heads;
    const int nqb = p.seg_len / p.q_block;
    // longest-first: later query blocks have more local tiles
    const int blk = blockIdx.x;
    const int m = qb0 + n_blocks - 1 - blk / (p.batch * p.n_q_heads);
    const int bh = blk % (p.batch * p.n_q_heads);
    const int b = bh / p.n_q_heads, h = bh % p.n_q_heads, g = h / G;
    const int bg = b * p.n_kv_heads + g;
    const float scale = rsqrtf((float)D);

    const T *qbase = q + ((long long)bh * p.seg_len + (long long)m * TILE) * D;
    load_tile<T, D, LD>(Qs, qbase, tid);
    if (tid == 0)
        s_nhist = route_list(idx + ((long long)bg * nqb + m) * p.topk, p.topk, p.n_hist_chunks, tiles, status,
                             (h % G) == 0);
    __syncthreads();
    const int n_hist = s_nhist;
    const int n_tiles = n_hist + m + 1;

    float mrow[4], lrow[4], o[4][DPT];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        mrow[r] = -INFINITY;
        lrow[r] = 0.f;
#pragma unroll
        for (int c = 0; c < DPT; ++c) o[r][c] = 0.f;
    }

    for (int t = 0; t < n_tiles; ++t) {
        const bool hist = t < n_hist;
        const int lt = t - n_hist;
        const T *kt = hist ? k_hist + ((long long)bg * p.hist_head_stride + (long long)tiles[t] * TILE) * D
                           : k_seg + ((long long)bg * p.seg_head_stride + (long long)lt * TILE) * D;
        const T *vt = hist ? v_hist + ((long long)bg * p.hist_head_stride + (long long)tiles[t] * TILE) * D
                           : v_seg + ((long long)bg * p.seg_head_stride + (long long)lt * TILE) * D;
        __syncthreads();  // previous tile fully consumed
        load_tile<T, D, LD>(Ks, kt, tid);
        load_tile<T, D, LD>(Vs, vt, tid);
        __syncthreads();

        float s[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[r][c] = 0.f;
        for (int d = 0; d < D; ++d) {
            float qa[4], kb[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) qa[r] = Qs[(rg * 4 + r) * LD + d];
#pragma unroll
            for (int c = 0; c < 4; ++c) kb[c] = Ks[(cg + 16 * c) * LD + d];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) s[r][c] = fmaf(qa[r], kb[c], s[r][c]);
        }
        const bool diag = !hist && lt == m;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v = s[r][c] * scale;
                if (diag && (cg + 16 * c) > (rg * 4 + r)) v = -INFINITY;
                s[r][c] = v;
                mx = fmaxf(mx, v);
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mnew = fmaxf(mrow[r], mx);
            const float alpha = expf(mrow[r] - mnew);  // exp(-inf) = 0 on the first tile
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float pv = expf(s[r][c] - mnew);
                s[r][c] = pv;
                sum += pv;
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            lrow[r] = lrow[r] * alpha + sum;
            mrow[r] = mnew;
#pragma unroll
            for (int c = 0; c < DPT; ++c) o[r][c] *= alpha;
#pragma unroll
            for (int c = 0; c < 4; ++c) Ps[(rg * 4 + r) * 65 + cg + 16 * c] = s[r][c];
        }
        __syncthreads();
        for (int kk = 0; kk < TILE; ++kk) {
            float pr[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) pr[r] = Ps[(rg * 4 + r) * 65 + kk];
#pragma unroll
            for (int c = 0; c < DPT; ++c) {
                const float v = Vs[kk * LD + cg + 16 * c];
#pragma unroll
                for (int r = 0; r < 4; ++r) o[r][c] = fmaf(pr[r], v, o[r][c]);
            }
        }
    }

#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = m * TILE + rg * 4 + r;
        const long long row = (long long)bh * p.seg_len + i;
        const float inv = 1.f / lrow[r];
#pragma unroll
        for (int c = 0; c < DPT; ++c) out[row * D + cg + 16 * c] = from_f32<T>(o[r][c] * inv);
        if (cg == 0) lse[row] = mrow[r] + logf(lrow[r]);
    }
}

// ---------------------------------------------------------------- backward
// delta_i = sum_d dO_i,d * O_i,d.  TPR threads per row, each one 16-byte
// vector of O and of dO (8 bf16 or 4 fp32), DELTA_ROWS rows per thread with
// every load in flight; the TPR partial dots are added by a fixed shuffle tree.
constexpr int kDeltaThreads = 256;
constexpr int kDeltaRows = 4;
template <typename T, int D>
__global__ void __launch_bounds__(kDeltaThreads) bwd_delta_kernel(const T *__restrict__ out,
                                                                   const T *__restrict__ dout,
                                                                   float *__restrict__ delta, long long rows) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int TPR = D / VEC;                 // 8 .. 32
    constexpr int RPP = kDeltaThreads / TPR;     // rows per pass of the block
    const int sub = threadIdx.x % TPR, rl = threadIdx.x / TPR;
    const long long base = (long long)blockIdx.x * RPP * kDeltaRows + rl;
    float o[kDeltaRows][VEC], g[kDeltaRows][VEC];
#pragma unroll
    for (int u = 0; u < kDeltaRows; ++u) {
        const long long row = base + (long long)u * RPP;
        if (row < rows) {
            Vec16<T>::load(out + row * D + sub * VEC, o[u]);
            Vec16<T>::load(dout + row * D + sub * VEC, g[u]);
        } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) o[u][e] = g[u][e] = 0.f;
        }
    }
#pragma unroll
    for (int u = 0; u < kDeltaRows; ++u) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) s = fmaf(o[u][e], g[u][e], s);
#pragma unroll
        for (int off = TPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        const long long row = base + (long long)u * RPP;
        if (sub == 0 && row < rows) delta[row] = s;
    }
}

// dQ: query-major over the block's history and local tiles.
template <typename T, int D>
__global__ void __launch_bounds__(NT) bwd_dq_simt_kernel(hga_params_t p, const T *__restrict__ q,
                                                         const T *__restrict__ k_hist, const T *__restrict__ v_hist,
                                                         const T *__restrict__ k_seg, const T *__restrict__ v_seg,
                                                         const int32_t *__restrict__ idx, const float *__restrict__ lse,
                                                         const float *__restrict__ delta, const T *__restrict__ dout,
                                                         float *__restrict__ dq, unsigned *status) {
    constexpr int LD = D + 1;
    constexpr int DPT = D / 16;
    extern __shared__ float sm[];
    float *Qs = sm, *dOs = Qs + TILE * LD, *Ks = dOs + TILE * LD, *Vs = Ks + TILE * LD;
    float *dSs = Vs + TILE * LD;  // [64][65]
    __shared__ int tiles[64];
    __shared__ int s_nhist;

    const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
    const int G = p.n_q_heads / p.n_kv_heads;
    const int nqb = p.seg_len / p.q_block;
    const int m = nqb - 1 - blockIdx.x / (p.batch * p.n_q_heads);
    const int bh = blockIdx.x % (p.batch * p.n_q_heads);
    const int b = bh / p.n_q_heads, h = bh % p.n_q_heads, g = h / G;
    const int bg = b * p.n_kv_heads + g;
    const float scale = rsqrtf((float)D);
    const long long row0 = (long long)bh * p.seg_len + (long long)m * TILE;

    load_tile<T, D, LD>(Qs, q + row0 * D, tid);
    load_tile<T, D, LD>(dOs, dout + row0 * D, tid);
    if (tid == 0)
        s_nhist = route_list(idx + ((long long)bg * nqb + m) * p.topk, p.topk, p.n_hist_chunks, tiles, status,
                             false);
    __syncthreads();
    const int n_hist = s_nhist;
    const int n_tiles = n_hist + m + 1;
    float lr[4], dr[4], acc[4][DPT];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        lr[r] = lse[row0 + rg * 4 + r];
        dr[r] = delta[row0 + rg * 4 + r];
#pragma unroll
        for (int c = 0; c < DPT; ++c) acc[r][c] = 0.f;
    }
    for (int t = 0; t < n_tiles; ++t) {
        const bool hist = t < n_hist;
        const int lt = t - n_hist;
        const long long off = hist ? ((long long)bg * p.hist_head_stride + (long long)tiles[t] * TILE) * D
                                   : ((long long)bg * p.seg_head_stride + (long long)lt * TILE) * D;
        __syncthreads();
        load_tile<T, D, LD>(Ks, (hist ? k_hist : k_seg) + off, tid);
        load_tile<T, D, LD>(Vs, (hist ? v_hist : v_seg) + off, tid);
        __syncthreads();
        float s[4][4], dp[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[r][c] = dp[r][c] = 0.f;
        for (int d = 0; d < D; ++d) {
            float qa[4], ga[4], kb[4], vb[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) { qa[r] = Qs[(rg * 4 + r) * LD + d]; ga[r] = dOs[(rg * 4 + r) * LD + d]; }
#pragma unroll
            for (int c = 0; c < 4; ++c) { kb[c] = Ks[(cg + 16 * c) * LD + d]; vb[c] = Vs[(cg + 16 * c) * LD + d]; }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    s[r][c] = fmaf(qa[r], kb[c], s[r][c]);
                    dp[r][c] = fmaf(ga[r], vb[c], dp[r][c]);
                }
        }
        const bool diag = !hist && lt == m;
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float pv = expf(s[r][c] * scale - lr[r]);
                if (diag && (cg + 16 * c) > (rg * 4 + r)) pv = 0.f;
                dSs[(rg * 4 + r) * 65 + cg + 16 * c] = pv * (dp[r][c] - dr[r]);
            }
        __syncthreads();
        for (int kk = 0; kk < TILE; ++kk) {
            float a[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = dSs[(rg * 4 + r) * 65 + kk];
#pragma unroll
            for (int c = 0; c < DPT; ++c) {
                const float kv = Ks[kk * LD + cg + 16 * c];
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[r][c] = fmaf(a[r], kv, acc[r][c]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < DPT; ++c) dq[(row0 + rg * 4 + r) * D + cg + 16 * c] = acc[r][c] * scale;
}

// dK/dV of the active segment: key-major, summing over the later query
// blocks and the G heads of the group in a fixed order (no atomics).
template <typename T, int D>
__global__ void __launch_bounds__(NT) bwd_dkdv_simt_kernel(hga_params_t p, const T *__restrict__ q,
                                                           const T *__restrict__ k_seg, const T *__restrict__ v_seg,
                                                           const float *__restrict__ lse, const float *__restrict__ delta,
                                                           const T *__restrict__ dout, float *__restrict__ dk,
                                                           float *__restrict__ dv) {
    constexpr int LD = D + 1;
    constexpr int DPT = D / 16;
    extern __shared__ float sm[];
    float *Ks = sm, *Vs = Ks + TILE * LD, *Qs = Vs + TILE * LD, *dOs = Qs + TILE * LD;
    float *Ps = dOs + TILE * LD, *dSs = Ps + TILE * 65;
    __shared__ float lq[TILE], dq_[TILE];

    const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
    const int G = p.n_q_heads / p.n_kv_heads;
    const int nqb = p.seg_len / p.q_block;
    // longest-first: early key tiles are seen by more query blocks
    const int n = blockIdx.x / (p.batch * p.n_kv_heads);
    const int bg = blockIdx.x % (p.batch * p.n_kv_heads);
    const int b = bg / p.n_kv_heads, g = bg % p.n_kv_heads;
    const float scale = rsqrtf((float)D);
    const long long kv_off = ((long long)bg * p.seg_head_stride + (long long)n * TILE) * D;
    load_tile<T, D, LD>(Ks, k_seg + kv_off, tid);
    load_tile<T, D, LD>(Vs, v_seg + kv_off, tid);
    float akk[4][DPT], avv[4][DPT];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < DPT; ++c) akk[r][c] = avv[r][c] = 0.f;

    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        for (int m = n; m < nqb; ++m) {
            const long long row0 = ((long long)(b * p.n_q_heads + h)) * p.seg_len + (long long)m * TILE;
            __syncthreads();
            load_tile<T, D, LD>(Qs, q + row0 * D, tid);
            load_tile<T, D, LD>(dOs, dout + row0 * D, tid);
            if (tid < TILE) { lq[tid] = lse[row0 + tid]; dq_[tid] = delta[row0 + tid]; }
            __syncthreads();
            // S^T[key][query] and dP^T[key][query]; thread: keys 4*rg+r, queries cg+16c
            float s[4][4], dp[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) s[r][c] = dp[r][c] = 0.f;
            for (int d = 0; d < D; ++d) {
                float ka[4], va[4], qb_[4], gb[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) { ka[r] = Ks[(rg * 4 + r) * LD + d]; va[r] = Vs[(rg * 4 + r) * LD + d]; }
#pragma unroll
                for (int c = 0; c < 4; ++c) { qb_[c] = Qs[(cg + 16 * c) * LD + d]; gb[c] = dOs[(cg + 16 * c) * LD + d]; }
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        s[r][c] = fmaf(ka[r], qb_[c], s[r][c]);
                        dp[r][c] = fmaf(va[r], gb[c], dp[r][c]);
                    }
            }
            const bool diag = (m == n);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int qi = cg + 16 * c, ki = rg * 4 + r;
                    float pv = expf(s[r][c] * scale - lq[qi]);
                    if (diag && qi < ki) pv = 0.f;
                    Ps[ki * 65 + qi] = pv;
                    dSs[ki * 65 + qi] = pv * (dp[r][c] - dq_[qi]);
                }
            __syncthreads();
            for (int qq = 0; qq < TILE; ++qq) {
                float pa[4], sa[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) { pa[r] = Ps[(rg * 4 + r) * 65 + qq]; sa[r] = dSs[(rg * 4 + r) * 65 + qq]; }
#pragma unroll
                for (int c = 0; c < DPT; ++c) {
                    const float gv = dOs[qq * LD + cg + 16 * c], qv = Qs[qq * LD + cg + 16 * c];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        avv[r][c] = fmaf(pa[r], gv, avv[r][c]);
                        akk[r][c] = fmaf(sa[r], qv, akk[r][c]);
                    }
                }
            }
        }
    }
    const long long out0 = ((long long)bg * p.seg_len + (long long)n * TILE) * D;
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < DPT; ++c) {
            dk[out0 + (rg * 4 + r) * D + cg + 16 * c] = akk[r][c] * scale;
            dv[out0 + (rg * 4 + r) * D + cg + 16 * c] = avv[r][c];
        }
}

// ---------------------------------------------------------------- launchers
template <typename T, int D>
static hga_status_t fwd_t(const hga_params_t &p, const void *q, const void *kh, const void *vh, const void *ks,
                          const void *vs, const int32_t *idx, void *out, float *lse, unsigned *status,
                          cudaStream_t stream) {
    const size_t smem = sizeof(float) * (3 * TILE * (D + 1) + TILE * 65);
    auto kern = fwd_simt_kernel<T, D>;
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), (int)smem);
    if (e != cudaSuccess) return record_cuda(e);
    const int nqb = p.seg_len / p.q_block;
    const int qb0 = p.qblock_end > 0 ? p.qblock_begin : 0;
    const int qb1 = p.qblock_end > 0 ? p.qblock_end : nqb;
    const unsigned grid = (unsigned)((qb1 - qb0) * p.batch * p.n_q_heads);
    if (grid == 0) return HGA_OK;
    kern<<<grid, NT, smem, stream>>>(p, (const T *)q, (const T *)kh, (const T *)vh, (const T *)ks, (const T *)vs,
                                     idx, (T *)out, lse, status, qb0, qb1 - qb0);
    return record_cuda(cudaGetLastError());
}

template <typename T, int D>
static hga_status_t bwd_t(const hga_params_t &p, const void *q, const void *kh, const void *vh, const void *ks,
                          const void *vs, const int32_t *idx, const void *out, const float *lse, const void *dout,
                          void *dq, void *dk, void *dv, float *delta, unsigned *status, cudaStream_t stream) {
    hga_status_t st = launch_bwd_delta(p, out, dout, delta, stream);
    if (st != HGA_OK) return st;
    cudaError_t e = cudaSuccess;
    const int nqb = p.seg_len / p.q_block;
    {
        const size_t smem = sizeof(float) * (4 * TILE * (D + 1) + TILE * 65);
        auto kern = bwd_dq_simt_kernel<T, D>;
        e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), (int)smem);
        if (e != cudaSuccess) return record_cuda(e);
        kern<<<(unsigned)(nqb * p.batch * p.n_q_heads), NT, smem, stream>>>(
            p, (const T *)q, (const T *)kh, (const T *)vh, (const T *)ks, (const T *)vs, idx, lse, delta,
            (const T *)dout, (float *)dq, status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return record_cuda(e);
    }
    {
        const size_t smem = sizeof(float) * (4 * TILE * (D + 1) + 2 * TILE * 65);
        auto kern = bwd_dkdv_simt_kernel<T, D>;
        e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), (int)smem);
        if (e != cudaSuccess) return record_cuda(e);
        kern<<<(unsigned)(nqb * p.batch * p.n_kv_heads), NT, smem, stream>>>(
            p, (const T *)q, (const T *)ks, (const T *)vs, lse, delta, (const T *)dout, (float *)dk, (float *)dv);
        e = cudaGetLastError();
    }
    return record_cuda(e);
}

hga_status_t launch_bwd_delta(const hga_params_t &p, const void *out, const void *dout, float *delta,
                              cudaStream_t stream) {
    const long long rows = (long long)p.batch * p.n_q_heads * p.seg_len;
    const int tpr = p.head_dim / (p.dtype == HGA_BF16 ? 8 : 4);
    const long long per_block = (long long)(kDeltaThreads / tpr) * kDeltaRows;
    const unsigned grid = (unsigned)((rows + per_block - 1) / per_block);
    if (p.dtype == HGA_BF16) {
        if (p.head_dim == 128)
            bwd_delta_kernel<__nv_bfloat16, 128><<<grid, kDeltaThreads, 0, stream>>>(
                (const __nv_bfloat16 *)out, (const __nv_bfloat16 *)dout, delta, rows);
        else
            bwd_delta_kernel<__nv_bfloat16, 64><<<grid, kDeltaThreads, 0, stream>>>(
                (const __nv_bfloat16 *)out, (const __nv_bfloat16 *)dout, delta, rows);
    } else {
        if (p.head_dim == 128)
            bwd_delta_kernel<float, 128><<<grid, kDeltaThreads, 0, stream>>>((const float *)out, (const float *)dout, delta,
                                                                   rows);
        else
            bwd_delta_kernel<float, 64><<<grid, kDeltaThreads, 0, stream>>>((const float *)out, (const float *)dout, delta,
                                                                  rows);
    }
    return record_cuda(cudaGetLastError());
}

hga_status_t launch_attn_fwd_simt(const hga_params_t &p, const void *q, const void *kh, const void *vh,
                                  const void *ks, const void *vs, const int32_t *idx, void *out, float *lse,
                                  unsigned *status, cudaStream_t stream) {
    if (p.dtype == HGA_BF16)
        return p.head_dim == 128 ? fwd_t<__nv_bfloat16, 128>(p, q, kh, vh, ks, vs, idx, out, lse, status, stream)
                                 : fwd_t<__nv_bfloat16, 64>(p, q, kh, vh, ks, vs, idx, out, lse, status, stream);
    return p.head_dim == 128 ? fwd_t<float, 128>(p, q, kh, vh, ks, vs, idx, out, lse, status, stream)
                             : fwd_t<float, 64>(p, q, kh, vh, ks, vs, idx, out, lse, status, stream);
}

hga_status_t launch_attn_bwd_simt(const hga_params_t &p, const void *q, const void *kh, const void *vh,
                                  const void *ks, const void *vs, const int32_t *idx, const void *out,
                                  const float *lse, const void *dout, void *dq, void *dk, void *dv, float *delta,
                                  unsigned *status, cudaStream_t stream) {
    if (p.dtype == HGA_BF16)
        return p.head_dim == 128
                   ? bwd_t<__nv_bfloat16, 128>(p, q, kh, vh, ks, vs, idx, out, lse, dout, dq, dk, dv, delta, status, stream)
                   : bwd_t<__nv_bfloat16, 64>(p, q, kh, vh, ks, vs, idx, out, lse, dout, dq, dk, dv, delta, status, stream);
    return p.head_dim == 128
               ? bwd_t<float, 128>(p, q, kh, vh, ks, vs, idx, out, lse, dout, dq, dk, dv, delta, status, stream)
               : bwd_t<float, 64>(p, q, kh, vh, ks, vs, idx, out, lse, dout, dq, dk, dv, delta, status, stream);
}

}  // namespace hga
