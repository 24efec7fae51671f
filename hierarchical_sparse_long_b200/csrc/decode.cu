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
// The step is bound by HBM: each attended chunk's K and V are read once for
// the G <= 8 query heads of its KV head.  Split-K over 64-token units:
//   decode_partial  one CTA per (batch, kv head, split) takes units
//                   split, split + n_split, ... of the list [routed chunks,
//                   then the local window in 64-token pieces].  A producer
//                   warp streams each unit's K and V rows into a ring of
//                   shared-memory stages; four consumer warps own 16 keys of
//                   every unit each and keep their own online softmax (m, l)
//                   and o = sum p V per head in registers, so the unit loop
//                   has no CTA-wide barrier.  Every consumer warp writes its
//                   (m, l, o) per head to the workspace as one partial.
//                   bf16: TMA tiles (128-byte swizzle) and warp-level bf16
//                   MMAs with the heads as the 16-row M side (rows >= G are
//                   zero): S = Q K^T and O += P V, P passed from the score
//                   fragments to the product operand in registers.  fp32:
//                   bulk copies and fp32 FMAs.
//   decode_combine  one CTA per (batch, q head) merges the partials in
//                   order: O = sum_s 2^(m_s - M) o_s / L,
//                   LSE = (M + log2 L) ln 2.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace hga {

namespace {

constexpr int CHK = 64;                      // tokens per unit (one chunk)
constexpr int kCW = 4;                       // consumer warps
constexpr int KPW = CHK / kCW;               // keys of every unit one consumer warp owns
constexpr int kDecThreads = 32 * (kCW + 1);  // consumers + one producer warp
constexpr int MAXG = 8;                      // query heads per KV head supported here
constexpr int kMaxRouted = 64;               // topk limit of the parameter check
constexpr int kRingBudget = 96 * 1024;       // stage bytes per CTA: two CTAs per SM
constexpr int kCtasPerSm = 2;

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
    int n_part;        // partials per (b, g): n_split * kCW
    float scale_log2;  // log2(e) / sqrt(D)
};

template <typename T, int D> struct DecGeom {
    static constexpr int kUnitBytes = CHK * D * static_cast<int>(sizeof(T));  // K (or V) rows of a unit
    static constexpr int kStageBytes = 2 * kUnitBytes;
    static constexpr int kFit = kRingBudget / kStageBytes;
    static constexpr int kStages = kFit < 2 ? 2 : (kFit > 4 ? 4 : kFit);
    static constexpr int kPsOff = kStages * kStageBytes;
    static constexpr int kBarOff = kPsOff + kCW * MAXG * KPW * 4;
    static constexpr int kSmem = kBarOff + 2 * kStages * 8;
};

// N consecutive elements at p (N * sizeof(T) = 4, 8 or 16 bytes, aligned) as floats.
template <typename T, int N> __device__ __forceinline__ void ld_vec(const T *p, float (&o)[N]) {
    constexpr int B = N * static_cast<int>(sizeof(T));
    static_assert(B == 4 || B == 8 || B == 16, "vector width");
    uint32_t w[B / 4];
    if constexpr (B == 16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (B == 8) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        w[0] = v.x; w[1] = v.y;
    } else {
        w[0] = *reinterpret_cast<const uint32_t *>(p);
    }
#pragma unroll
    for (int i = 0; i < B / 4; ++i) {
        if constexpr (sizeof(T) == 4) {
            o[i] = __uint_as_float(w[i]);
        } else {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

// Waits, with fresh bounds, for the bulk copies of units [from, to) after an abort.
template <int S> __device__ void drain_stages(uint64_t *full, int from, int to) {
    for (int i = from; i < to; ++i) {
        const long long t0 = clock64();
        while (!tc::mbar_try_wait(&full[i % S], (i / S) & 1) && clock64() - t0 < (1ll << 31)) {
        }
    }
}

// GP: G rounded up to a power of two (head slots >= G carry zero queries).
template <typename T, int D, int GP>
__global__ void __launch_bounds__(kDecThreads, 1) decode_partial(const DecArgs a) {
    using Geo = DecGeom<T, D>;
    constexpr int S = Geo::kStages;
    extern __shared__ __align__(128) uint8_t smem[];
    float *ps_all = reinterpret_cast<float *>(smem + Geo::kPsOff);  // [kCW][GP][KPW]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Geo::kBarOff);
    uint64_t *empty = full + S;
    __shared__ int units[kMaxRouted];  // valid routed chunks of this (b, g)
    __shared__ int n_routed, issued_s, abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int split = (int)blockIdx.x % a.n_split;
    const int bg = (int)blockIdx.x / a.n_split;
    const int b = bg / a.n_kv_heads, g = bg % a.n_kv_heads;

    if (tid == 0) {
        abort_flag = 0;
        issued_s = 0;
        // the routed chunks of the token; -1 is padding, anything else out of range is skipped
        const int32_t *sel = a.idx + (long long)bg * a.topk;
        int n = 0;
        for (int i = 0; i < a.topk; ++i) {
            const int j = sel[i];
            if (j >= 0 && j < a.n_hist_chunks) units[n++] = j;
            else if (j != -1 && split == 0) atomicOr(a.status, kDevBadIndex);
        }
        n_routed = n;
        for (int st = 0; st < S; ++st) {
            tc::mbar_init(&full[st], 1);
            tc::mbar_init(&empty[st], kCW);
        }
        tc::fence_mbar_init();
    }
    __syncthreads();
    const int nr = n_routed;
    const int n_units = nr + (a.n_local + CHK - 1) / CHK;
    const int my_units = n_units > split ? (n_units - split + a.n_split - 1) / a.n_split : 0;

    // the rows of unit i of this CTA: base pointers and token count
    auto unit_src = [&](int i, const T *&kb, const T *&vb) {
        const int u = split + i * a.n_split;
        if (u < nr) {
            const long long row0 = (long long)bg * a.hist_stride + (long long)units[u] * CHK;
            kb = static_cast<const T *>(a.kh) + row0 * D;
            vb = static_cast<const T *>(a.vh) + row0 * D;
            return CHK;
        }
        const int t0 = (u - nr) * CHK;
        const long long row0 = (long long)bg * a.local_stride + t0;
        kb = static_cast<const T *>(a.kl) + row0 * D;
        vb = static_cast<const T *>(a.vl) + row0 * D;
        return min(CHK, a.n_local - t0);
    };

    if (warp == kCW) {
        // producer: one lane issues the bulk copies of unit i into stage i % S once
        // the consumers have released the unit that held it before
        if (lane == 0) {
            int i = 0;
            for (; i < my_units; ++i) {
                const int st = i % S;
                if (i >= S) {
                    if (!tc::mbar_wait(&empty[st], ((i / S) - 1) & 1, &abort_flag, a.status)) break;
                    tc::fence_proxy_async();
                }
                const T *kb, *vb;
                const int ntok = unit_src(i, kb, vb);
                const uint32_t bytes = static_cast<uint32_t>(ntok * D * sizeof(T));
                uint8_t *dst = smem + st * Geo::kStageBytes;
                tc::mbar_arrive_expect_tx(&full[st], 2 * bytes);
                tc::bulk_load(dst, kb, bytes, &full[st]);
                tc::bulk_load(dst + Geo::kUnitBytes, vb, bytes, &full[st]);
            }
            issued_s = i;
        }
    } else {
        constexpr int LOGGP = GP == 8 ? 3 : GP == 4 ? 2 : GP == 2 ? 1 : 0;
        // score phase: 16 lanes per key row, two rows per warp instruction; lane
        // s16 holds pieces s16, s16 + 16, ... of PB bytes of the row
        constexpr int RB = D * static_cast<int>(sizeof(T));
        constexpr int PB = RB >= 256 ? 16 : 8;
        constexpr int NP = RB / (16 * PB);
        constexpr int EPP = PB / static_cast<int>(sizeof(T));
        // P V phase: lane owns dimensions lane * DPL .. lane * DPL + DPL - 1
        constexpr int DPL = D / 32;
        const int half = lane >> 4, s16 = lane & 15;
        const int my_h = s16 >> (4 - LOGGP);
        const bool writer = (s16 & ((1 << (4 - LOGGP)) - 1)) == 0;

        float qreg[GP][NP * EPP];  // queries pre-scaled by log2(e)/sqrt(D)
        {
            const T *qb = static_cast<const T *>(a.q) + ((long long)b * a.n_q_heads + (long long)g * G) * D;
#pragma unroll
            for (int h = 0; h < GP; ++h)
#pragma unroll
                for (int u = 0; u < NP; ++u)
#pragma unroll
                    for (int e = 0; e < EPP; ++e)
                        qreg[h][u * EPP + e] =
                            h < G ? to_f32(qb[(long long)h * D + (s16 + 16 * u) * EPP + e]) * a.scale_log2 : 0.f;
        }
        float m_run[GP], l_run[GP], acc[GP][DPL];
#pragma unroll
        for (int h = 0; h < GP; ++h) {
            m_run[h] = -INFINITY;
            l_run[h] = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
        }
        float *ps = ps_all + warp * GP * KPW;  // [GP][KPW] of this warp
        const int kw0 = warp * KPW;

        for (int i = 0; i < my_units; ++i) {
            const int st = i % S;
            bool ok = tc::mbar_wait(&full[st], (i / S) & 1, &abort_flag, a.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            const T *kb, *vb;
            const int ntok = unit_src(i, kb, vb);
            const int nk = min(KPW, max(0, ntok - kw0));  // valid keys of this warp (warp-uniform)
            const T *Ks = reinterpret_cast<const T *>(smem + st * Geo::kStageBytes);
            const T *Vs = reinterpret_cast<const T *>(smem + st * Geo::kStageBytes + Geo::kUnitBytes);

            // scores s[h][key] = q_h . k_key (log2 units); keys past ntok get -inf
#pragma unroll 2
            for (int pr = 0; pr < KPW / 2; ++pr) {
                const int kl = 2 * pr + half;
                float x[NP * EPP];
                if (kl < nk) {
#pragma unroll
                    for (int u = 0; u < NP; ++u) {
                        float t[EPP];
                        ld_vec<T, EPP>(Ks + (kw0 + kl) * D + (s16 + 16 * u) * EPP, t);
#pragma unroll
                        for (int e = 0; e < EPP; ++e) x[u * EPP + e] = t[e];
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < NP * EPP; ++e) x[e] = 0.f;
                }
                float v[GP];
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < NP * EPP; ++e) s = fmaf(qreg[h][e], x[e], s);
                    v[h] = s;
                }
                // fold the 16 lanes of the row (xor 8, 4, 2, 1): while several heads
                // remain, each step halves them between lane pairs
#pragma unroll
                for (int stp = 0; stp < 4; ++stp) {
                    const int o = 8 >> stp;
                    const int w = GP >> stp;
                    if (w > 1) {
                        const bool up = (s16 & o) != 0;
#pragma unroll
                        for (int e = 0; e < w / 2; ++e) {
                            const float send = up ? v[e] : v[e + w / 2];
                            const float keep = up ? v[e + w / 2] : v[e];
                            v[e] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                        }
                    } else {
                        v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
                    }
                }
                if (writer) ps[my_h * KPW + kl] = kl < nk ? v[0] : -INFINITY;
            }
            __syncwarp();

            // online softmax of the warp's keys: entry e = lane + 32 r is (head e / KPW,
            // key e % KPW); segments of KPW lanes reduce, the per-head results go to all lanes
            float corr[GP];
            {
                constexpr int HPR = 32 / KPW;  // heads per 32 entries
                constexpr int NR = (GP * KPW + 31) / 32;
                const int seg = lane / KPW;
                float sv[NR], tmax[GP], tsum[GP], m_new[GP];
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const int e = lane + 32 * r;
                    sv[r] = e < GP * KPW ? ps[e] : -INFINITY;
                    float mx = sv[r];
#pragma unroll
                    for (int o = KPW / 2; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
#pragma unroll
                    for (int hb = 0; hb < HPR; ++hb)
                        if (HPR * r + hb < GP) tmax[HPR * r + hb] = __shfl_sync(0xffffffffu, mx, KPW * hb);
                }
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    m_new[h] = fmaxf(m_run[h], tmax[h]);
                    corr[h] = m_new[h] == -INFINITY ? 1.f : exp2f(m_run[h] - m_new[h]);  // 0 while m_run is -inf
                }
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const int e = lane + 32 * r;
                    float mh = m_new[0];
#pragma unroll
                    for (int hb = 0; hb < HPR; ++hb)
                        if (HPR * r + hb < GP && seg == hb) mh = m_new[HPR * r + hb];
                    const float p = sv[r] == -INFINITY ? 0.f : exp2f(sv[r] - mh);
                    if (e < GP * KPW) ps[e] = p;
                    float sm = p;
#pragma unroll
                    for (int o = KPW / 2; o; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
#pragma unroll
                    for (int hb = 0; hb < HPR; ++hb)
                        if (HPR * r + hb < GP) tsum[HPR * r + hb] = __shfl_sync(0xffffffffu, sm, KPW * hb);
                }
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    l_run[h] = fmaf(l_run[h], corr[h], tsum[h]);
                    m_run[h] = m_new[h];
                }
            }
            __syncwarp();

            // o[h] = o[h] * corr[h] + sum_key p[h][key] V[key]
#pragma unroll
            for (int h = 0; h < GP; ++h)
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc[h][e] *= corr[h];
#pragma unroll
            for (int k4 = 0; k4 < KPW; k4 += 4) {
                if (k4 >= nk) break;
                float4 p4[GP];
#pragma unroll
                for (int h = 0; h < GP; ++h) p4[h] = *reinterpret_cast<const float4 *>(ps + h * KPW + k4);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if (k4 + kk < nk) {
                        float vv[DPL];
                        ld_vec<T, DPL>(Vs + (kw0 + k4 + kk) * D + lane * DPL, vv);
#pragma unroll
                        for (int h = 0; h < GP; ++h) {
                            const float p = kk == 0 ? p4[h].x : kk == 1 ? p4[h].y : kk == 2 ? p4[h].z : p4[h].w;
#pragma unroll
                            for (int e = 0; e < DPL; ++e) acc[h][e] = fmaf(p, vv[e], acc[h][e]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&empty[st]);  // stage free for the producer
        }

        // this warp's partial (m, l, o) per head
        float *w = a.ws + ((long long)bg * a.n_part + (long long)split * kCW + warp) * G * (D + 2);
#pragma unroll
        for (int h = 0; h < GP; ++h) {
            if (h < G) {
#pragma unroll
                for (int e = 0; e < DPL; ++e) w[h * (D + 2) + 2 + lane * DPL + e] = acc[h][e];
                if (lane == 0) {
                    w[h * (D + 2) + 0] = m_run[h];
                    w[h * (D + 2) + 1] = l_run[h];
                }
            }
        }
    }
    __syncthreads();
    // copies still in flight after an abort land before the CTA's shared memory is released
    if (tid == 0 && abort_flag) drain_stages<S>(full, issued_s > S ? issued_s - S : 0, issued_s);
}

// bf16 tiles of 64 rows in 128-byte swizzle atoms (64 values of a row per atom).
template <int D> struct TcGeom {
    static constexpr int kAtoms = D / 64;
    static constexpr int kAtomBytes = CHK * 128;
    static constexpr int kUnitBytes = kAtoms * kAtomBytes;  // K (or V) rows of a unit
    static constexpr int kStageBytes = 2 * kUnitBytes;
    static constexpr int kFit = kRingBudget / kStageBytes;
    static constexpr int kStages = kFit < 2 ? 2 : (kFit > 4 ? 4 : kFit);
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kSmem = 1024 + kBarOff + 2 * kStages * 8;  // + slack for 1024-byte alignment
};

// Shared-memory address of 16-byte chunk c of row r of a tile (128-byte swizzle:
// the chunk index is XORed with the row index mod 8 inside each atom).
__device__ __forceinline__ uint32_t sw128(uint32_t tile, int r, int c) {
    return tile + (c >> 3) * (CHK * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_partial_tc(const __grid_constant__ CUtensorMap mkh, const __grid_constant__ CUtensorMap mvh,
                      const __grid_constant__ CUtensorMap mkl, const __grid_constant__ CUtensorMap mvl,
                      const DecArgs a) {
    using Geo = TcGeom<D>;
    constexpr int S = Geo::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the swizzle pattern follows address bits 4-9: stages start on 1024-byte boundaries
    uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Geo::kBarOff);
    uint64_t *empty = full + S;
    __shared__ int units[kMaxRouted];
    __shared__ int n_routed, issued_s, abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int split = (int)blockIdx.x % a.n_split;
    const int bg = (int)blockIdx.x / a.n_split;
    const int b = bg / a.n_kv_heads, gkv = bg % a.n_kv_heads;

    if (tid == 0) {
        abort_flag = 0;
        issued_s = 0;
        const int32_t *sel = a.idx + (long long)bg * a.topk;
        int n = 0;
        for (int i = 0; i < a.topk; ++i) {
            const int j = sel[i];
            if (j >= 0 && j < a.n_hist_chunks) units[n++] = j;
            else if (j != -1 && split == 0) atomicOr(a.status, kDevBadIndex);
        }
        n_routed = n;
        for (int st = 0; st < S; ++st) {
            tc::mbar_init(&full[st], 1);
            tc::mbar_init(&empty[st], kCW);
        }
        tc::fence_mbar_init();
    }
    __syncthreads();
    const int nr = n_routed;
    const int n_units = nr + (a.n_local + CHK - 1) / CHK;
    const int my_units = n_units > split ? (n_units - split + a.n_split - 1) / a.n_split : 0;

    if (warp == kCW) {
        // producer: K and V tiles of unit i into stage i % S (rows of the local window
        // past n_local arrive as zeros)
        if (lane == 0) {
            int i = 0;
            for (; i < my_units; ++i) {
                const int st = i % S;
                if (i >= S) {
                    if (!tc::mbar_wait(&empty[st], ((i / S) - 1) & 1, &abort_flag, a.status)) break;
                    tc::fence_proxy_async();
                }
                const int u = split + i * a.n_split;
                const bool hist = u < nr;
                const CUtensorMap *mk = hist ? &mkh : &mkl;
                const CUtensorMap *mv = hist ? &mvh : &mvl;
                const int y = hist ? units[u] * CHK : (u - nr) * CHK;
                uint8_t *dst = smem + st * Geo::kStageBytes;
                tc::mbar_arrive_expect_tx(&full[st], Geo::kStageBytes);
#pragma unroll
                for (int at = 0; at < Geo::kAtoms; ++at) {
                    tc::tma_load_3d(dst + at * Geo::kAtomBytes, mk, 64 * at, y, bg, &full[st]);
                    tc::tma_load_3d(dst + Geo::kUnitBytes + at * Geo::kAtomBytes, mv, 64 * at, y, bg, &full[st]);
                }
            }
            issued_s = i;
        }
    } else {
        // fragment coordinates: row g (a head) and column pair 2 t4, 2 t4 + 1
        const int g = lane >> 2, t4 = lane & 3;
        // ldmatrix: this lane addresses row rr of matrix mi
        const int mi = lane >> 3, rr = lane & 7;
        // Q rows as A fragments (raw bf16; rows 8..15 and heads >= G are zero)
        uint32_t qa[D / 16][2];
        {
            const __nv_bfloat16 *qb =
                static_cast<const __nv_bfloat16 *>(a.q) + ((long long)b * a.n_q_heads + (long long)gkv * G + g) * D;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qa[ks][0] = g < G ? *reinterpret_cast<const uint32_t *>(qb + 16 * ks + 2 * t4) : 0u;
                qa[ks][1] = g < G ? *reinterpret_cast<const uint32_t *>(qb + 16 * ks + 8 + 2 * t4) : 0u;
            }
        }
        float m_run = -INFINITY, l_run = 0.f;  // head g; l_run sums this lane's keys only
        float o[D / 8][4];                     // O of head g: dims 8 nt + 2 t4, +1 in [0], [1]
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        const uint32_t sbase = tc::smem_u32(smem);
        const int kw0 = warp * KPW;

        for (int i = 0; i < my_units; ++i) {
            const int st = i % S;
            bool ok = tc::mbar_wait(&full[st], (i / S) & 1, &abort_flag, a.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int u = split + i * a.n_split;
            const int ntok = u < nr ? CHK : min(CHK, a.n_local - (u - nr) * CHK);
            const int nk = min(KPW, max(0, ntok - kw0));  // valid keys of this warp
            const uint32_t ktile = sbase + st * Geo::kStageBytes;
            const uint32_t vtile = ktile + Geo::kUnitBytes;

            // S = Q K^T for the warp's keys kw0 .. kw0 + 15 (two 8-key column tiles);
            // matrices: keys 0-7 / 8-15 (mi >> 1) x dims 16 ks + 0-7 / 8-15 (mi & 1)
            float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const int krow = kw0 + ((mi >> 1) << 3) + rr;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t b0, b1, b2, b3;
                tc::ldsm_x4(sw128(ktile, krow, 2 * ks + (mi & 1)), b0, b1, b2, b3);
                const uint32_t af[4] = {qa[ks][0], 0u, qa[ks][1], 0u};
                tc::mma_16816(sacc[0], af, b0, b1);
                tc::mma_16816(sacc[1], af, b2, b3);
            }

            // online softmax of head g over the warp's 16 keys (a quad holds them all):
            // x[e] is key 2 t4 + (e & 1) + 8 (e >> 1), in log2 units
            float x[4] = {sacc[0][0], sacc[0][1], sacc[1][0], sacc[1][1]};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = 2 * t4 + (e & 1) + 8 * (e >> 1);
                x[e] = key < nk ? x[e] * a.scale_log2 : -INFINITY;
            }
            float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
            const float m_new = fmaxf(m_run, mt);
            const float corr = m_new == -INFINITY ? 1.f : exp2f(m_run - m_new);  // 0 while m_run is -inf
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) p[e] = x[e] == -INFINITY ? 0.f : exp2f(x[e] - m_new);
            l_run = fmaf(l_run, corr, (p[0] + p[1]) + (p[2] + p[3]));
            m_run = m_new;
            if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
                for (int nt = 0; nt < D / 8; ++nt) {
                    o[nt][0] *= corr;
                    o[nt][1] *= corr;
                }
            }

            // O += P V: P (bf16) is the A fragment; V tiles through transposing
            // ldmatrix: matrices keys 0-7 / 8-15 (mi & 1) x dims 16 dp + 0-7 / 8-15 (mi >> 1)
            const uint32_t pa[4] = {tc::pack_bf16(p[0], p[1]), 0u, tc::pack_bf16(p[2], p[3]), 0u};
            const int vrow = kw0 + ((mi & 1) << 3) + rr;
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t v0, v1, v2, v3;
                tc::ldsm_x4_t(sw128(vtile, vrow, 2 * dp + (mi >> 1)), v0, v1, v2, v3);
                tc::mma_16816(o[2 * dp], pa, v0, v1);
                tc::mma_16816(o[2 * dp + 1], pa, v2, v3);
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&empty[st]);  // stage free for the producer
        }

        // this warp's partial (m, l, o) of head g
        float l = l_run + __shfl_xor_sync(0xffffffffu, l_run, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (g < G) {
            float *w = a.ws + (((long long)bg * a.n_part + (long long)split * kCW + warp) * G + g) * (D + 2);
            if (t4 == 0) {
                w[0] = m_run;
                w[1] = l;
            }
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
                w[2 + 8 * nt + 2 * t4] = o[nt][0];
                w[2 + 8 * nt + 2 * t4 + 1] = o[nt][1];
            }
        }
    }
    __syncthreads();
    // copies still in flight after an abort land before the CTA's shared memory is released
    if (tid == 0 && abort_flag) drain_stages<S>(full, issued_s > S ? issued_s - S : 0, issued_s);
}

template <typename T, int D>
__global__ void __launch_bounds__(D) decode_combine(const DecArgs a) {
    const int bh = blockIdx.x;
    const int b = bh / a.n_q_heads, h = bh % a.n_q_heads;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int g = h / G, hh = h % G;
    const int bg = b * a.n_kv_heads + g;
    const float *w = a.ws + (long long)bg * a.n_part * G * (D + 2) + hh * (D + 2);
    const long long sstride = (long long)G * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < a.n_part; ++s) M = fmaxf(M, w[s * sstride]);
    float L = 0.f, acc = 0.f;
    for (int s = 0; s < a.n_part; ++s) {
        const float ms = w[s * sstride];
        const float f = ms == -INFINITY ? 0.f : exp2f(ms - M);  // a partial without keys adds nothing
        L = fmaf(w[s * sstride + 1], f, L);
        acc = fmaf(w[s * sstride + 2 + threadIdx.x], f, acc);
    }
    static_cast<T *>(a.out)[(long long)bh * D + threadIdx.x] = from_f32<T>(acc / L);
    if (threadIdx.x == 0) a.lse[bh] = (M + log2f(L)) * 0.69314718055994530942f;
}

// Splits per (b, g): as many as keep the whole grid resident at kCtasPerSm CTAs
// per SM, at most one per unit.
int decode_splits(const hga_params_t &p, int n_local) {
    const int units = (p.topk < p.n_hist_chunks ? p.topk : p.n_hist_chunks) + (n_local + CHK - 1) / CHK;
    const long long bg = (long long)p.batch * p.n_kv_heads;
    long long s = (long long)kCtasPerSm * sm_count() / bg;
    if (s > units) s = units;
    return s < 1 ? 1 : (int)s;
}

template <typename T, int D, int GP>
hga_status_t launch_gp(const DecArgs &a, cudaStream_t stream) {
    using Geo = DecGeom<T, D>;
    auto kern = decode_partial<T, D, GP>;
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), Geo::kSmem);
    if (e != cudaSuccess) return record_cuda(e);
    const unsigned bg = (unsigned)(a.batch * a.n_kv_heads);
    kern<<<bg * a.n_split, kDecThreads, Geo::kSmem, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e);
    decode_combine<T, D><<<(unsigned)(a.batch * a.n_q_heads), D, 0, stream>>>(a);
    return record_cuda(cudaGetLastError());
}

template <typename T, int D>
hga_status_t launch_t(const DecArgs &a, cudaStream_t stream) {
    const int G = a.n_q_heads / a.n_kv_heads;
    if (G <= 1) return launch_gp<T, D, 1>(a, stream);
    if (G <= 2) return launch_gp<T, D, 2>(a, stream);
    if (G <= 4) return launch_gp<T, D, 4>(a, stream);
    return launch_gp<T, D, 8>(a, stream);
}

template <int D>
hga_status_t launch_tc(const DecArgs &a, cudaStream_t stream) {
    using Geo = TcGeom<D>;
    const unsigned long long groups = (unsigned long long)a.batch * a.n_kv_heads;
    CUtensorMap mkh, mvh, mkl, mvl;
    bool ok = tma_group_rows_map(&mkl, a.kl, D, a.n_local, groups, a.local_stride) &&
              tma_group_rows_map(&mvl, a.vl, D, a.n_local, groups, a.local_stride);
    if (a.n_hist_chunks > 0) {
        ok = ok && tma_group_rows_map(&mkh, a.kh, D, (unsigned long long)a.n_hist_chunks * CHK, groups, a.hist_stride) &&
             tma_group_rows_map(&mvh, a.vh, D, (unsigned long long)a.n_hist_chunks * CHK, groups, a.hist_stride);
    } else {  // no routed units: the history maps are never read
        mkh = mkl;
        mvh = mvl;
    }
    if (!ok) {
        record_error("hga_attn_decode: TMA tensor map encoding failed");
        return HGA_ERR_UNSUPPORTED;
    }
    auto kern = decode_partial_tc<D>;
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), Geo::kSmem);
    if (e != cudaSuccess) return record_cuda(e);
    kern<<<(unsigned)groups * a.n_split, kDecThreads, Geo::kSmem, stream>>>(mkh, mvh, mkl, mvl, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e);
    decode_combine<__nv_bfloat16, D><<<(unsigned)(a.batch * a.n_q_heads), D, 0, stream>>>(a);
    return record_cuda(cudaGetLastError());
}

}  // namespace

size_t decode_workspace_bytes(const hga_params_t &p, int n_local) {
    const int G = p.n_q_heads / p.n_kv_heads;
    const size_t floats = (size_t)p.batch * p.n_kv_heads * decode_splits(p, n_local) * kCW * G * (p.head_dim + 2);
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
    a.n_part = a.n_split * kCW;
    a.scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)p.head_dim));
    if (p.dtype == HGA_BF16) return p.head_dim == 128 ? launch_tc<128>(a, stream) : launch_tc<64>(a, stream);
    return p.head_dim == 128 ? launch_t<float, 128>(a, stream) : launch_t<float, 64>(a, stream);
}

}  // namespace hga
