// Single-query HGA decode: one new token per sequence attends, with exact
// softmax, the tokens of its routed history chunks and the local window of
// not-yet-detached tokens it closes.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.1
// (routed exact chunks next to a local window) applied to generation: the
// route of the token comes from hga_route over a one-token segment
// (seg_len = q_block = 1), so its block summary is the mean of its G query
// heads.
//
// With G query rows per KV head there is no matrix shape for the tensor
// cores; the step is bound by HBM (each attended chunk's K and V are read
// once for the G heads).  Split-K over 64-token units:
//   decode_partial  one CTA per (batch, kv head, split) takes units
//                   split, split + n_split, ... of the list [routed chunks,
//                   then the local window in 64-token pieces]; per unit the
//                   K rows give the G x 64 scores (two threads per key row,
//                   16-byte loads), an online softmax in the log2 domain
//                   updates (m, l) per head, and one thread per dimension
//                   accumulates o += p V (coalesced V rows); the CTA writes
//                   its (m, l, o) per head to the workspace.
//   decode_combine  one CTA per (batch, q head) merges the splits in order:
//                   O = sum_s 2^(m_s - M) o_s / L, LSE = (M + log2 L) ln 2.
#include "common.cuh"

namespace hga {

namespace {

constexpr int CHK = 64;      // tokens per unit (one chunk)
constexpr int kDecThreads = 2 * CHK;  // two threads per key row; one per dimension (D <= 128) for P V
constexpr int MAXG = 8;      // query heads per KV head supported here
constexpr int kSplitTarget = 1184;  // aim for about 8 CTAs per SM over the whole grid

struct DecArgs {
    const void *q;
    const void *kh;
    const void *vh;
    const void *kl;
    const void *vl;
    const int32_t *idx;
    void *out;
    float *lse;
    float *ws;
    unsigned *status;
    long long hist_stride, local_stride;
    int batch, n_q_heads, n_kv_heads, topk, n_hist_chunks, n_local, n_split;
    float scale_log2;  // log2(e) / sqrt(D)
};

template <typename T> __device__ __forceinline__ float ld1(const T *p) { return to_f32(*p); }

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads) decode_partial(const DecArgs a) {
    constexpr int NT = kDecThreads;
    static_assert(D <= NT, "one thread per dimension in the P V phase");
    constexpr int VEC = Vec16<T>::N;   // elements per 16-byte load
    constexpr int HALF = D / 2;        // dimensions per thread in the score phase
    __shared__ float qs[MAXG][D];      // queries, pre-scaled by log2(e)/sqrt(D)
    __shared__ float ps[MAXG][CHK];    // scores, then p, of the current unit
    __shared__ __align__(16) T vs[CHK][D];  // V rows of the current unit
    __shared__ float m_s[MAXG], l_s[MAXG], c_s[MAXG];
    __shared__ int units[64 + 1];      // valid routed chunks of this (b, g)
    __shared__ int n_routed;

    const int tid = threadIdx.x;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int split = (int)blockIdx.x % a.n_split;
    const int bg = (int)blockIdx.x / a.n_split;
    const int b = bg / a.n_kv_heads, g = bg % a.n_kv_heads;

    for (int e = tid; e < G * D; e += NT) {
        const int hh = e / D, d = e % D;
        qs[hh][d] = ld1(static_cast<const T *>(a.q) + ((long long)(b * a.n_q_heads + g * G + hh)) * D + d) *
                    a.scale_log2;
    }
    if (tid < MAXG) {
        m_s[tid] = -INFINITY;
        l_s[tid] = 0.f;
    }
    if (tid == 0) {
        // the routed chunks of the token; -1 is padding, anything else out of range is skipped
        const int32_t *sel = a.idx + (long long)bg * a.topk;
        int n = 0;
        for (int i = 0; i < a.topk; ++i) {
            const int j = sel[i];
            if (j >= 0 && j < a.n_hist_chunks) units[n++] = j;
            else if (j != -1 && split == 0) atomicOr(a.status, kDevBadIndex);
        }
        n_routed = n;
    }
    __syncthreads();
    const int n_units = n_routed + (a.n_local + CHK - 1) / CHK;
    float o[MAXG];
#pragma unroll
    for (int hh = 0; hh < MAXG; ++hh) o[hh] = 0.f;

    const int key = tid >> 1, part = tid & 1;  // score phase: key row of the unit, half of D
    for (int u = split; u < n_units; u += a.n_split) {
        const bool hist = u < n_routed;
        const T *kbase, *vbase;
        int ntok;
        if (hist) {
            const long long row0 = (long long)bg * a.hist_stride + (long long)units[u] * CHK;
            kbase = static_cast<const T *>(a.kh) + row0 * D;
            vbase = static_cast<const T *>(a.vh) + row0 * D;
            ntok = CHK;
        } else {
            const int t0 = (u - n_routed) * CHK;
            const long long row0 = (long long)bg * a.local_stride + t0;
            kbase = static_cast<const T *>(a.kl) + row0 * D;
            vbase = static_cast<const T *>(a.vl) + row0 * D;
            ntok = min(CHK, a.n_local - t0);
        }
        // K and V rows of the unit (two threads per row, 16-byte loads, all in flight
        // together); V goes to shared memory for the P V phase; scores
        // s[h][key] = q_h . k_key in log2 units
        {
            float kv[HALF];
            // V: 16-byte pieces in row-major order, consecutive threads on consecutive
            // pieces (coalesced reads, conflict-free shared-memory writes)
            constexpr int VPR = D / VEC;  // 16-byte pieces per row
            uint4 vraw[CHK * VPR / NT];
#pragma unroll
            for (int v = 0; v < CHK * VPR / NT; ++v) {
                const int piece = tid + v * NT, r = piece / VPR, c = piece % VPR;
                if (r < ntok) vraw[v] = *reinterpret_cast<const uint4 *>(vbase + (long long)r * D + c * VEC);
            }
            if (key < ntok) {
#pragma unroll
                for (int v = 0; v < HALF / VEC; ++v)
                    Vec16<T>::load(kbase + (long long)key * D + part * HALF + v * VEC, kv + v * VEC);
            } else {
#pragma unroll
                for (int e = 0; e < HALF; ++e) kv[e] = 0.f;
            }
#pragma unroll
            for (int hh = 0; hh < MAXG; ++hh) {
                if (hh < G) {
                    float acc = 0.f;
#pragma unroll
                    for (int e = 0; e < HALF; ++e) acc = fmaf(qs[hh][part * HALF + e], kv[e], acc);
                    const float other = __shfl_xor_sync(0xffffffffu, acc, 1);
                    const float s = part == 0 ? acc + other : other + acc;
                    if (part == 0) ps[hh][key] = key < ntok ? s : -INFINITY;
                }
            }
#pragma unroll
            for (int v = 0; v < CHK * VPR / NT; ++v) {
                const int piece = tid + v * NT, r = piece / VPR, c = piece % VPR;
                if (r < ntok) *reinterpret_cast<uint4 *>(&vs[r][c * VEC]) = vraw[v];
            }
        }
        __syncthreads();
        // online softmax per head: warp w takes heads w, w + NT/32, ...
        const int warp = tid >> 5, lane = tid & 31;
        for (int hh = warp; hh < G; hh += NT / 32) {
            const float s0 = ps[hh][lane], s1 = ps[hh][lane + 32];
            float mx = fmaxf(s0, s1);
#pragma unroll
            for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_old = m_s[hh];
            const float m_new = fmaxf(m_old, mx);
            const float p0 = exp2f(s0 - m_new), p1 = exp2f(s1 - m_new);
            float sum = p0 + p1;
#pragma unroll
            for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            ps[hh][lane] = p0;
            ps[hh][lane + 32] = p1;
            __syncwarp();
            if (lane == 0) {
                const float corr = exp2f(m_old - m_new);  // 0 while m_old is -inf
                c_s[hh] = corr;
                l_s[hh] = l_s[hh] * corr + sum;
                m_s[hh] = m_new;
            }
        }
        __syncthreads();
        // o[h][d] = o[h][d] * corr + sum_t p[h][t] V[t][d]: one thread per dimension
        if (tid < D) {
#pragma unroll
            for (int hh = 0; hh < MAXG; ++hh)
                if (hh < G) o[hh] *= c_s[hh];
            for (int t = 0; t < ntok; ++t) {
                const float v = to_f32(vs[t][tid]);
#pragma unroll
                for (int hh = 0; hh < MAXG; ++hh)
                    if (hh < G) o[hh] = fmaf(ps[hh][t], v, o[hh]);
            }
        }
        __syncthreads();
    }
    // this split's (m, l, o) per head
    float *w = a.ws + ((long long)bg * a.n_split + split) * G * (D + 2);
    if (tid < D) {
#pragma unroll
        for (int hh = 0; hh < MAXG; ++hh)
            if (hh < G) w[hh * (D + 2) + 2 + tid] = o[hh];
    }
    if (tid < G) {
        w[tid * (D + 2) + 0] = m_s[tid];
        w[tid * (D + 2) + 1] = l_s[tid];
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(D) decode_combine(const DecArgs a) {
    const int bh = blockIdx.x;
    const int b = bh / a.n_q_heads, h = bh % a.n_q_heads;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int g = h / G, hh = h % G;
    const int bg = b * a.n_kv_heads + g;
    const float *w = a.ws + (long long)bg * a.n_split * G * (D + 2) + hh * (D + 2);
    const long long sstride = (long long)G * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < a.n_split; ++s) M = fmaxf(M, w[s * sstride]);
    float L = 0.f, acc = 0.f;
    for (int s = 0; s < a.n_split; ++s) {
        const float ms = w[s * sstride];
        const float f = ms == -INFINITY ? 0.f : exp2f(ms - M);  // a split without units adds nothing
        L = fmaf(w[s * sstride + 1], f, L);
        acc = fmaf(w[s * sstride + 2 + threadIdx.x], f, acc);
    }
    static_cast<T *>(a.out)[(long long)bh * D + threadIdx.x] = from_f32<T>(acc / L);
    if (threadIdx.x == 0) a.lse[bh] = (M + log2f(L)) * 0.69314718055994530942f;
}

int decode_splits(const hga_params_t &p, int n_local) {
    const int units = (p.topk < p.n_hist_chunks ? p.topk : p.n_hist_chunks) + (n_local + CHK - 1) / CHK;
    const long long bg = (long long)p.batch * p.n_kv_heads;
    long long s = (kSplitTarget + bg - 1) / bg;
    if (s > units) s = units;
    return s < 1 ? 1 : (int)s;
}

template <typename T, int D>
hga_status_t launch_t(const DecArgs &a, cudaStream_t stream) {
    const unsigned bg = (unsigned)(a.batch * a.n_kv_heads);
    decode_partial<T, D><<<bg * a.n_split, kDecThreads, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e);
    decode_combine<T, D><<<(unsigned)(a.batch * a.n_q_heads), D, 0, stream>>>(a);
    return record_cuda(cudaGetLastError());
}

}  // namespace

size_t decode_workspace_bytes(const hga_params_t &p, int n_local) {
    const int G = p.n_q_heads / p.n_kv_heads;
    const size_t floats = (size_t)p.batch * p.n_kv_heads * decode_splits(p, n_local) * G * (p.head_dim + 2);
    return (floats * sizeof(float) + 255) & ~(size_t)255;
}

hga_status_t launch_decode(const hga_params_t &p, const void *q, const void *kh, const void *vh, const void *kl,
                           const void *vl, int n_local, const int32_t *idx, void *out, float *lse, float *ws,
                           unsigned *status, cudaStream_t stream) {
    DecArgs a;
    a.q = q;
    a.kh = kh;
    a.vh = vh;
    a.kl = kl;
    a.vl = vl;
    a.idx = idx;
    a.out = out;
    a.lse = lse;
    a.ws = ws;
    a.status = status;
    a.hist_stride = p.hist_head_stride;
    a.local_stride = p.seg_head_stride;
    a.batch = p.batch;
    a.n_q_heads = p.n_q_heads;
    a.n_kv_heads = p.n_kv_heads;
    a.topk = p.topk;
    a.n_hist_chunks = p.n_hist_chunks;
    a.n_local = n_local;
    a.n_split = decode_splits(p, n_local);
    a.scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)p.head_dim));
    if (p.dtype == HGA_BF16)
        return p.head_dim == 128 ? launch_t<__nv_bfloat16, 128>(a, stream) : launch_t<__nv_bfloat16, 64>(a, stream);
    return p.head_dim == 128 ? launch_t<float, 128>(a, stream) : launch_t<float, 64>(a, stream);
}

}  // namespace hga
