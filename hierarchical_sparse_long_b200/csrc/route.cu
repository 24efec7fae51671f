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
// One CTA per (batch, kv head, query block); CL consecutive query blocks of
// one (batch, kv head) form a thread-block cluster.
//   1. Summary tiles start streaming at once by bulk copies into a shared-
//      memory ring (4 slots; 8 when the grid is under one CTA per SM, so the
//      next round is in flight while one is scored), while every thread loads
//      its share of the block's G x q_block query rows straight into
//      registers (16-byte loads, all in flight together) and the CTA sums
//      them in a fixed order: the block summary qbar (fp32).
//   2. The cluster's CL summaries are exchanged through distributed shared
//      memory; each CTA scores its 1/CL slice of the chunks against all CL
//      of them, so every chunk summary crosses L2 -> SM once per cluster.
//      16 lanes share one chunk row (coalesced reads), fp32 FFMA only (no
//      tensor cores), and the lane partials fold by shuffles in a fixed
//      tree, so every score is a deterministic fp32 dot product.
//   3. Each CTA gathers its own query block's full score row from the
//      cluster and selects with all its threads: a lower bound of the k-th
//      best score from the per-thread maxima, the few chunks at or above it,
//      and their exact ranks by (score, then the lower chunk index).
// A segment of one query block (a decode token) has no neighbours to share
// its cluster with; there the CL CTAs of a cluster split that block's chunk
// list (SPLIT): each scores only its slice for the one summary, and rank 0
// gathers the row and selects.
#include <algorithm>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace hga {
namespace {

constexpr int kThreads = 256;
constexpr int kRound = 4;        // summary tiles scored per round (contiguous in the ring)
constexpr int kCandCap = 1024;   // candidate list of the selecting warp
constexpr int kMaxSmem = 227 * 1024 - 1024;
constexpr unsigned kFull = 0xffffffffu;

// Byte offsets of the dynamic shared-memory regions (host computed).
struct RouteLayout {
    int ring, part, qown, qall, sc, row, tmax, key, cj, hist, misc, bar, total;
};

struct RouteArgs {
    const void *q;
    const float *summ;
    int32_t *idx;
    unsigned *status;
    long long cap;  // summary rows per (b, g)
    int n_q_heads, n_kv_heads, seg_len, q_block, n, topk;  // q_block: 64, or 1 for a decode token
    int sink;  // chunks 0 .. sink-1 are always routed (attention-sink window)
    int ns;  // chunks per cluster rank (multiple of 4)
    int slots;  // ring slots: kRound, or 2 * kRound (the next round in flight while one is scored)
    float inv_sqrt_d;
    RouteLayout L;
};

constexpr int kTileBytes = 16 * 1024;  // one ring slot: a tile of summary rows
constexpr int kWarps = kThreads / 32;

int round4(int x) { return (x + 3) & ~3; }

RouteLayout route_layout(int D, int esize, int cl, int ns, int n, int slots, int rows) {
    RouteLayout L{};
    int off = 0;
    auto take = [&](int bytes) {
        const int at = off;
        off += (bytes + 15) & ~15;
        return at;
    };
    L.ring = take(slots * kTileBytes);
    L.part = take((kThreads / (D * esize / 16)) * D * 4);
    L.qown = take(D * 4);
    L.qall = take(cl * D * 4);
    L.sc = take(rows * ns * 4);
    L.row = take(cl > 1 ? round4(n) * 4 : 0);
    L.tmax = take(kThreads * 4);
    L.key = take(kCandCap * 8);
    L.cj = take(kCandCap * 4);
    L.hist = take(256 * 4);
    L.misc = take(16 * 4);
    L.bar = take(slots * 8);
    L.total = off;
    return L;
}

// Order-preserving 32-bit image of an fp32 score (larger score -> larger
// value; -0 and +0 map to the same value).
__device__ __forceinline__ uint32_t ordered_bits(float s) {
    uint32_t u = __float_as_uint(s);
    if (s == 0.0f) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 64-bit selection key: score image, then the lower chunk index first.
__device__ __forceinline__ uint64_t sel_key(uint32_t ord, int j) {
    return (static_cast<uint64_t>(ord) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(j));
}

// acc[e] += element e of one 16-byte unit (8 bf16 or 4 fp32).
template <typename T> __device__ __forceinline__ void add_unit(const uint4 &w, float *acc);
template <> __device__ __forceinline__ void add_unit<float>(const uint4 &w, float *acc) {
    acc[0] += __uint_as_float(w.x);
    acc[1] += __uint_as_float(w.y);
    acc[2] += __uint_as_float(w.z);
    acc[3] += __uint_as_float(w.w);
}
template <> __device__ __forceinline__ void add_unit<__nv_bfloat16>(const uint4 &w, float *acc) {
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(v[i] << 16);
        acc[2 * i + 1] += __uint_as_float(v[i] & 0xFFFF0000u);
    }
}

// One warp, the whole row: the k (< n) best chunks of row[0, n) by (score
// image descending, chunk index ascending), written to out[0, k) in ascending
// chunk order.  Radix select (4 passes of 8 bits, most significant first) of
// the k-th largest image, then every chunk above it and the lowest-index
// chunks equal to it.  Used when the candidate list of select_cta overflows.
__device__ void select_warp_radix(const uint32_t *row, int n, int k, int32_t *out, int *hist, int lane) {
    const unsigned lt = (1u << lane) - 1u;
    uint32_t prefix = 0u, mask = 0u;
    int rem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        for (int base = 0; base < n; base += 32) {
            const int p = base + lane;
            const uint32_t v = p < n ? row[p] : 0u;
            const bool in = p < n && (v & mask) == prefix;
            const int bin = static_cast<int>((v >> shift) & 255u);
            const unsigned act = __ballot_sync(kFull, in);
            if (act) {
                // one shared atomic when every active lane hits the same bin
                const int leader = __ffs(act) - 1;
                const int b0 = __shfl_sync(kFull, bin, leader);
                if (__ballot_sync(kFull, in && bin != b0) == 0) {
                    if (lane == leader) atomicAdd(&hist[b0], __popc(act));
                } else if (in) {
                    atomicAdd(&hist[bin], 1);
                }
            }
        }
        __syncwarp();
        // lane l holds bins 8l .. 8l+7; scan from the top bin down
        int cnt[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            cnt[e] = hist[8 * lane + e];
            tot += cnt[e];
        }
        int suf = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_down_sync(kFull, suf, o);
            if (lane + o < 32) suf += y;
        }
        int above = suf - tot, fbin = -1, frem = 0;
#pragma unroll
        for (int e = 7; e >= 0; --e) {
            if (fbin < 0 && above < rem && above + cnt[e] >= rem) {
                fbin = 8 * lane + e;
                frem = rem - above;
            }
            above += cnt[e];
        }
        const unsigned fb = __ballot_sync(kFull, fbin >= 0);
        const int src = fb ? __ffs(fb) - 1 : 0;
        fbin = __shfl_sync(kFull, fbin, src);
        frem = __shfl_sync(kFull, frem, src);
        if (fbin < 0) {  // unreachable: the bins count every chunk matching the prefix
            fbin = 0;
            frem = rem;
        }
        prefix |= static_cast<uint32_t>(fbin) << shift;
        mask |= 255u << shift;
        rem = frem;
        __syncwarp();
    }
    int written = 0, ties = 0;
    for (int base = 0; base < n && written < k; base += 32) {
        const int p = base + lane;
        const uint32_t v = p < n ? row[p] : 0u;
        const bool tie = p < n && v == prefix;
        const unsigned tb = __ballot_sync(kFull, tie);
        const bool take = p < n && (v > prefix || (tie && ties + __popc(tb & lt) < rem));
        const unsigned kb = __ballot_sync(kFull, take);
        if (take) out[written + __popc(kb & lt)] = p;
        written += __popc(kb);
        ties += __popc(tb);
    }
}

struct SelScratch {
    uint32_t *tmax;  // [kThreads] per-thread maxima; 16-byte aligned (read as uint4)
    uint64_t *key;   // [kCandCap] candidate keys
    int *cj;         // [kCandCap] chosen candidates' chunk index, else INT_MAX
    int *hist;       // [256] (whole-row fallback)
    int *misc;       // [16]: candidate count, per-warp minima
};

// The whole CTA: the k (< n) best chunks of row[0, n) by (score image
// descending, chunk index ascending), written to out[0, k) ascending.
//   bound: thr = k-th largest of the kThreads per-thread maxima (thread t
//          takes chunks t, t + kThreads, ...); they are distinct chunks, so
//          at least k chunks have an image >= thr and so do all k best;
//   candidates: the chunks with image >= thr (warp-aggregated append);
//   rank of each candidate among the candidates by its 64-bit key (image,
//   then the lower chunk index); the k of rank < k are the answer and each
//   lands at the count of chosen candidates with a lower chunk index.
__device__ void select_cta(const uint32_t *row, int n, int k, int32_t *out, const SelScratch &s, int tid) {
    const int lane = tid & 31, warp = tid >> 5;
    const unsigned lt = (1u << lane) - 1u;
    uint32_t mx = 0u;  // 0 is below every real score image
    for (int j = tid; j < n; j += kThreads) mx = max(mx, row[j]);
    s.tmax[tid] = mx;
    if (tid == 0) s.misc[0] = 0;
    __syncthreads();
    int gp[4] = {0, 0, 0, 0};  // independent partial counts (short dependency chains)
#pragma unroll 4
    for (int u = 0; u < kThreads; u += 16) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const uint4 v = *reinterpret_cast<const uint4 *>(s.tmax + u + 4 * h);
            gp[h] += (v.x > mx) + (v.y > mx) + (v.z > mx) + (v.w > mx);
        }
    }
    const int greater = (gp[0] + gp[1]) + (gp[2] + gp[3]);
    uint32_t thr = greater < k ? mx : 0xFFFFFFFFu;
#pragma unroll
    for (int o = 16; o; o >>= 1) thr = min(thr, __shfl_xor_sync(kFull, thr, o));
    if (lane == 0) s.misc[8 + warp] = static_cast<int>(thr);
    __syncthreads();
    thr = static_cast<uint32_t>(s.misc[8]);
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) thr = min(thr, static_cast<uint32_t>(s.misc[8 + w]));

    for (int base = 0; base < n; base += kThreads) {  // warp-uniform trip count
        const int j = base + tid;
        const bool in = j < n && row[j] >= thr;
        const unsigned bal = __ballot_sync(kFull, in);
        int wbase = 0;
        if (lane == 0 && bal) wbase = atomicAdd(&s.misc[0], __popc(bal));
        wbase = __shfl_sync(kFull, wbase, 0);
        const int pos = wbase + __popc(bal & lt);
        if (in && pos < kCandCap) s.key[pos] = sel_key(row[j], j);
    }
    __syncthreads();
    const int C = s.misc[0];
    if (C > kCandCap) {  // too many chunks at the bound: radix select on the whole row
        if (warp == 0) select_warp_radix(row, n, k, out, s.hist, lane);
        return;
    }
    for (int c = tid; c < C; c += kThreads) {
        const uint64_t kc = s.key[c];
        int r = 0;
        for (int u = 0; u < C; ++u) r += s.key[u] > kc;
        s.cj[c] = r < k ? static_cast<int>(~static_cast<uint32_t>(kc)) : 0x7FFFFFFF;
    }
    __syncthreads();
    for (int c = tid; c < C; c += kThreads) {
        const int j = s.cj[c];
        if (j != 0x7FFFFFFF) {
            int pos = 0;
            for (int u = 0; u < C; ++u) pos += s.cj[u] < j;
            out[pos] = j;
        }
    }
}

// Waits, with a fresh bound, for bulk copies still in flight after an abort.
__device__ void drain_ring(uint64_t *bar, int from, int to, int slots) {
    for (int i = from; i < to; ++i) {
        const long long t0 = clock64();
        while (!tc::mbar_try_wait(&bar[i % slots], (i / slots) & 1) && clock64() - t0 < (1ll << 31)) {
        }
    }
}

template <typename T, int D, int CL, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 2) route_kernel(const RouteArgs a) {
    // a forward launched as a programmatic dependent may start as soon as every
    // CTA of this grid is running (it waits for this grid before reading idx)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int R = SPLIT ? 1 : CL;  // query blocks scored by this CTA
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int abort_flag;
    const RouteLayout &L = a.L;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nqb = a.seg_len / a.q_block;
    const int m = SPLIT ? 0 : (int)blockIdx.x % nqb;
    const int bg = SPLIT ? (int)blockIdx.x / CL : (int)blockIdx.x / nqb;
    const int b = bg / a.n_kv_heads, g = bg % a.n_kv_heads;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int n = a.n;
    int32_t *out = a.idx + ((long long)bg * nqb + m) * a.topk;
    if (n <= a.topk) {  // every chunk is routed (the same branch for the whole grid)
        for (int t = tid; t < a.topk; t += kThreads) out[t] = t < n ? t : -1;
        return;
    }

    const int rank = CL > 1 ? static_cast<int>(tc::cluster_ctarank()) : 0;  // m % CL, or the slice (SPLIT)
    const int c_begin = rank * a.ns;
    const int n_slice = max(0, min(n, c_begin + a.ns) - c_begin);
    constexpr int TCN = kTileBytes / (D * 4);  // chunks per summary tile
    const int ntiles = (n_slice + TCN - 1) / TCN;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.bar);
    const float *sbase = a.summ + ((long long)bg * a.cap + c_begin) * D;

    auto issue = [&](int t) {
        const int slot = t % a.slots;
        const uint32_t bytes = static_cast<uint32_t>(min(TCN, n_slice - t * TCN) * D * 4);
        tc::mbar_arrive_expect_tx(&bar[slot], bytes);
        tc::bulk_load(smem + L.ring + slot * kTileBytes, sbase + (long long)t * TCN * D, bytes, &bar[slot]);
    };

    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < a.slots; ++s) tc::mbar_init(&bar[s], 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    int issued = 0;  // thread 0's count of issued tiles
    if (tid == 0)
        for (; issued < min(a.slots, ntiles); ++issued) issue(issued);

    // 1. block summary.  Thread (rs, cu) sums the 16-byte column unit cu of
    //    rows rs, rs + NRS, ... of the G x q_block rows (head-major), in order;
    //    the NRS row slots are then added in order.
    constexpr int VEC = Vec16<T>::N;  // elements per 16-byte unit
    constexpr int UPR = D / VEC;      // units per row
    constexpr int NRS = kThreads / UPR;
    constexpr int BATCH = 16;         // loads in flight per thread
    {
        const int cu = tid % UPR, rs = tid / UPR;
        const T *qbase = static_cast<const T *>(a.q) +
                         (((long long)b * a.n_q_heads + (long long)g * G) * a.seg_len + (long long)m * a.q_block) * D +
                         cu * VEC;
        const int rows = G * a.q_block;
        float acc[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
        for (int r0 = rs; r0 < rows; r0 += BATCH * NRS) {
            uint4 raw[BATCH];
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int r = r0 + u * NRS;
                if (r < rows) {
                    const int hh = r / a.q_block, i = r - hh * a.q_block;
                    raw[u] = *reinterpret_cast<const uint4 *>(qbase + ((long long)hh * a.seg_len + i) * D);
                } else {
                    raw[u] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int u = 0; u < BATCH; ++u) add_unit<T>(raw[u], acc);
        }
        float *part = reinterpret_cast<float *>(smem + L.part);
#pragma unroll
        for (int e = 0; e < VEC; ++e) part[rs * D + cu * VEC + e] = acc[e];
    }
    __syncthreads();
    float *qown = reinterpret_cast<float *>(smem + L.qown);
    if (tid < D) {
        const float *part = reinterpret_cast<const float *>(smem + L.part);
        float s = 0.f;
        for (int sl = 0; sl < NRS; ++sl) s += part[sl * D + tid];
        qown[tid] = s / static_cast<float>(G * a.q_block);
    }

    // 2. the cluster's CL block summaries, then this rank's slice of scores
    const float *qall = qown;
    if constexpr (CL > 1 && !SPLIT) {
        tc::cluster_arrive();
        tc::cluster_wait();
        float *qa = reinterpret_cast<float *>(smem + L.qall);
        constexpr int V4 = D / 4;
        for (int t = tid; t < CL * V4; t += kThreads) {
            const int r = t / V4, o = t % V4;
            *reinterpret_cast<uint4 *>(qa + r * D + 4 * o) =
                tc::ld_dsmem_v4(tc::mapa_shared(tc::smem_u32(qown + 4 * o), static_cast<uint32_t>(r)));
        }
        qall = qa;
    }
    __syncthreads();

    constexpr int NV = D / 64;  // float4 per lane per chunk row
    constexpr int LOGR = R == 8 ? 3 : R == 4 ? 2 : R == 2 ? 1 : 0;
    const int half = lane >> 4, s16 = lane & 15;
    float4 qr[R][NV];
#pragma unroll
    for (int mb = 0; mb < R; ++mb)
#pragma unroll
        for (int u = 0; u < NV; ++u) qr[mb][u] = *reinterpret_cast<const float4 *>(qall + mb * D + 4 * s16 + 64 * u);
    uint32_t *sc = reinterpret_cast<uint32_t *>(smem + L.sc);  // [R][ns] score images of the slice
    const int my_mb = s16 >> (4 - LOGR);
    const bool writer = (s16 & ((1 << (4 - LOGR)) - 1)) == 0;
    bool ok = true;
    int done = 0;  // tiles this thread waited for successfully
    // rounds of up to kRound tiles: the round's chunks sit contiguously in the
    // ring, every warp takes chunk pairs warp, warp + kWarps, ... of the round;
    // with more slots the next rounds' copies are in flight meanwhile
    constexpr int UNR = R >= 8 ? 1 : R >= 2 ? 2 : 4;  // chunk pairs in flight per warp
    for (int t0 = 0; t0 < ntiles; t0 += kRound) {
        const int t1 = min(ntiles, t0 + kRound);
        for (int t = t0; t < t1; ++t) {
            ok = ok && tc::mbar_wait(&bar[t % a.slots], (t / a.slots) & 1, &abort_flag, a.status);
            done += ok;
        }
        if (ok) {
            const float *chunks = reinterpret_cast<const float *>(smem + L.ring + (t0 % a.slots) * kTileBytes);
            const int rows = min((t1 - t0) * TCN, n_slice - t0 * TCN);
            const int npairs = (rows + 1) >> 1;
            for (int pr0 = warp; pr0 < npairs; pr0 += UNR * kWarps) {  // warp-uniform
                float v[UNR][R];
#pragma unroll
                for (int q = 0; q < UNR; ++q) {
                    const int cl = 2 * (pr0 + q * kWarps) + half;
                    const bool valid = cl < rows;
                    float4 x[NV];
#pragma unroll
                    for (int u = 0; u < NV; ++u)
                        x[u] = valid ? *reinterpret_cast<const float4 *>(chunks + cl * D + 4 * s16 + 64 * u)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int mb = 0; mb < R; ++mb) {
                        float acc = 0.f;
#pragma unroll
                        for (int u = 0; u < NV; ++u) {
                            acc = fmaf(qr[mb][u].x, x[u].x, acc);
                            acc = fmaf(qr[mb][u].y, x[u].y, acc);
                            acc = fmaf(qr[mb][u].z, x[u].z, acc);
                            acc = fmaf(qr[mb][u].w, x[u].w, acc);
                        }
                        v[q][mb] = acc;
                    }
                }
                // fold the 16 lanes of each chunk (xor 8, 4, 2, 1): while several
                // query blocks remain, each step halves them between lane pairs
#pragma unroll
                for (int st = 0; st < 4; ++st) {
                    const int o = 8 >> st;
                    const int w = R >> st;
#pragma unroll
                    for (int q = 0; q < UNR; ++q) {
                        if (w > 1) {
                            const bool up = (s16 & o) != 0;
#pragma unroll
                            for (int e = 0; e < w / 2; ++e) {
                                const float send = up ? v[q][e] : v[q][e + w / 2];
                                const float keep = up ? v[q][e + w / 2] : v[q][e];
                                v[q][e] = keep + __shfl_xor_sync(kFull, send, o);
                            }
                        } else {
                            v[q][0] += __shfl_xor_sync(kFull, v[q][0], o);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < UNR; ++q) {
                    const int cl = 2 * (pr0 + q * kWarps) + half;
                    if (cl < rows && writer)
                        sc[my_mb * a.ns + t0 * TCN + cl] = ordered_bits(v[q][0] * a.inv_sqrt_d);
                }
            }
        }
        __syncthreads();
        if (tid == 0 && issued < ntiles && !abort_flag) {
            tc::fence_proxy_async();
            for (; issued < min(ntiles, t1 + a.slots); ++issued) issue(issued);
        }
    }

    // 3. this query block's full score row, then the CTA selects (SPLIT: rank 0
    //    gathers the one block's row and selects)
    const bool selector = !SPLIT || rank == 0;
    uint32_t *row = sc;
    if constexpr (CL > 1) {
        tc::cluster_arrive();
        tc::cluster_wait();
        uint32_t *rw = reinterpret_cast<uint32_t *>(smem + L.row);
        const int n4 = a.ns / 4;
        const int my_row = SPLIT ? 0 : rank;  // this block's row in every peer's score slices
        if (selector) {
            for (int t = tid; t < CL * n4; t += kThreads) {
                const int r = t / n4, o = t % n4;
                const int j = r * a.ns + 4 * o;
                if (j < n)
                    *reinterpret_cast<uint4 *>(rw + j) = tc::ld_dsmem_v4(
                        tc::mapa_shared(tc::smem_u32(sc + my_row * a.ns + 4 * o), static_cast<uint32_t>(r)));
            }
        }
        tc::cluster_arrive();  // done reading the peers' shared memory
        row = rw;
    }
    __syncthreads();
    if (a.sink > 0 && selector) {
        // the sink chunks outrank every score (the largest image; ties among them
        // go to the lower index, so they are listed first)
        for (int j = tid; j < a.sink && j < n; j += kThreads) row[j] = 0xFFFFFFFFu;
    }
    __syncthreads();
    if (!abort_flag && selector) {
        SelScratch ss;
        ss.tmax = reinterpret_cast<uint32_t *>(smem + L.tmax);
        ss.key = reinterpret_cast<uint64_t *>(smem + L.key);
        ss.cj = reinterpret_cast<int *>(smem + L.cj);
        ss.hist = reinterpret_cast<int *>(smem + L.hist);
        ss.misc = reinterpret_cast<int *>(smem + L.misc);
        select_cta(row, n, a.topk, out, ss, tid);
    }
    if (tid == 0 && abort_flag) drain_ring(bar, done, issued, a.slots);
    if constexpr (CL > 1) tc::cluster_wait();  // peers may still read this CTA's slice
}

template <typename T, int D, int CL, bool SPLIT>
cudaError_t launch_cl(const RouteArgs &a, unsigned grid, cudaStream_t stream) {
    auto kern = route_kernel<T, D, CL, SPLIT>;
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), a.L.total);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(a.L.total);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = CL > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename T, int D>
cudaError_t launch_t(const RouteArgs &a, int cl, bool split, unsigned grid, cudaStream_t stream) {
    if (split) {
        switch (cl) {
        case 8: return launch_cl<T, D, 8, true>(a, grid, stream);
        case 4: return launch_cl<T, D, 4, true>(a, grid, stream);
        default: return launch_cl<T, D, 2, true>(a, grid, stream);
        }
    }
    switch (cl) {
    case 8: return launch_cl<T, D, 8, false>(a, grid, stream);
    case 4: return launch_cl<T, D, 4, false>(a, grid, stream);
    case 2: return launch_cl<T, D, 2, false>(a, grid, stream);
    default: return launch_cl<T, D, 1, false>(a, grid, stream);
    }
}

// ---------------------------------------------------------------------------
// Strictly causal routing (the technical summary's limits section proposes a
// strictly causal variant of the block-shared route): token i of block m
// routes by the mean over the G heads of the block's queries start .. i, so no
// later query can change its route.  One CTA per (b, g, m):
//   1. the block's G-head row sums (all threads, independent loads), then one
//      thread per dimension turns them into prefix means in row order;
//   2. passes of TP tokens (TP x Nc score images fit in shared memory): every
//      32-row summary tile is loaded once per pass and scored against the
//      pass's TP prefix summaries (thread = one chunk row x TP/8 tokens; fp32
//      FFMA in a fixed order, like route_kernel);
//   3. each warp selects its tokens' top-k with the sink chunks stamped first.
constexpr int kCTile = 32;  // summary rows per tile

struct CausalLayout {
    int qpre, tile, sc, hist, total, tp;
};

CausalLayout causal_layout(int D, int q_block, int n) {
    CausalLayout L{};
    const int n4 = n > 4 ? round4(n) : 4;
    L.qpre = 0;
    L.tile = L.qpre + q_block * D * 4;
    L.hist = L.tile + kCTile * (D + 4) * 4;
    L.sc = L.hist + kWarps * 256 * 4;
    const int room = kMaxSmem - L.sc;
    int tp = room / (n4 * 4);
    tp = tp >= q_block ? q_block : (tp / kWarps) * kWarps;
    L.tp = tp;
    L.total = L.sc + (tp > 0 ? tp : kWarps) * n4 * 4;
    return L;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1) route_causal_kernel(const RouteArgs a, int tp, CausalLayout L) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int QB = a.q_block, nqb = a.seg_len / QB;
    const int m = (int)blockIdx.x % nqb, bg = (int)blockIdx.x / nqb;
    const int b = bg / a.n_kv_heads, g = bg % a.n_kv_heads;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int n = a.n, n4 = n > 4 ? (n + 3) & ~3 : 4;  // score row stride, as in causal_layout
    constexpr int DP = D + 4;  // padded tile row (conflict-free 16-byte reads across rows)
    float *qpre = reinterpret_cast<float *>(smem + L.qpre);
    float *tile = reinterpret_cast<float *>(smem + L.tile);
    uint32_t *sc = reinterpret_cast<uint32_t *>(smem + L.sc);
    int *hist = reinterpret_cast<int *>(smem + L.hist);
    int32_t *out = a.idx + ((long long)bg * a.seg_len + (long long)m * QB) * a.topk;
    if (n <= a.topk) {  // every chunk is routed for every token (the same branch for the whole grid)
        for (int e = tid; e < QB * a.topk; e += kThreads) {
            const int t = e % a.topk;
            out[e] = t < n ? t : -1;
        }
        return;
    }

    // 1. prefix summaries
    const T *qb = static_cast<const T *>(a.q) +
                  (((long long)b * a.n_q_heads + (long long)g * G) * a.seg_len + (long long)m * QB) * D;
    for (int e = tid; e < QB * D; e += kThreads) {
        const int r = e / D, d = e % D;
        float rs = 0.f;
        for (int hh = 0; hh < G; ++hh) rs += to_f32(qb[((long long)hh * a.seg_len + r) * D + d]);
        qpre[e] = rs;
    }
    __syncthreads();
    for (int d = tid; d < D; d += kThreads) {
        float run = 0.f;
        for (int r = 0; r < QB; ++r) {
            run += qpre[r * D + d];
            qpre[r * D + d] = run / static_cast<float>(G * (r + 1));
        }
    }
    __syncthreads();

    const float *sbase = a.summ + (long long)bg * a.cap * D;
    const int jj = tid % kCTile, tg = tid / kCTile;  // chunk row of the tile, token group
    for (int t0 = 0; t0 < QB; t0 += tp) {
        const int ntp = min(tp, QB - t0);
        // 2. scores of tokens t0 .. t0 + ntp - 1, tile by tile
        for (int j0 = 0; j0 < n; j0 += kCTile) {
            const int rows = min(kCTile, n - j0);
            __syncthreads();  // the previous tile is consumed
            for (int e = tid; e < rows * (D / 4); e += kThreads) {
                const int r = e / (D / 4), c = e % (D / 4);
                *reinterpret_cast<float4 *>(tile + r * DP + 4 * c) =
                    *reinterpret_cast<const float4 *>(sbase + (long long)(j0 + r) * D + 4 * c);
            }
            __syncthreads();
            if (jj < rows) {
                const float4 *sv = reinterpret_cast<const float4 *>(tile + jj * DP);
                for (int tk = tg; tk < ntp; tk += kThreads / kCTile) {  // warp-uniform
                    const float4 *qv = reinterpret_cast<const float4 *>(qpre + (t0 + tk) * D);
                    float acc = 0.f;
#pragma unroll 8
                    for (int u = 0; u < D / 4; ++u) {
                        const float4 x = qv[u], y = sv[u];
                        acc = fmaf(x.x, y.x, acc);
                        acc = fmaf(x.y, y.y, acc);
                        acc = fmaf(x.z, y.z, acc);
                        acc = fmaf(x.w, y.w, acc);
                    }
                    sc[tk * n4 + j0 + jj] = ordered_bits(acc * a.inv_sqrt_d);
                }
            }
        }
        __syncthreads();
        // 3. one warp per token: sink chunks first, then the radix select over the row
        for (int tk = warp; tk < ntp; tk += kWarps) {
            uint32_t *row = sc + tk * n4;
            for (int j = lane; j < a.sink && j < n; j += 32) row[j] = 0xFFFFFFFFu;
            __syncwarp();
            select_warp_radix(row, n, a.topk, out + (long long)(t0 + tk) * a.topk, hist + warp * 256, lane);
            __syncwarp();
        }
        __syncthreads();  // the score rows are reused by the next pass
    }
}

// ---------------------------------------------------------------------------
// Group-level second stage (technical summary section 2.1, group selection):
// the groups of `gs` tokens inside a block's chosen chunks are scored against
// the same block summary with their group summaries (mean of the group's
// keys) and the topg best are kept, by (score descending, group index
// ascending), listed ascending and -1 padded.  One CTA per (b, g, m).
constexpr int kMaxCand = 64 * 8;  // k <= 64 chosen chunks x up to 8 groups each

struct GroupArgs {
    const void *q;
    const float *gsumm;
    const int32_t *idx;
    // staged group summaries: when set, chunk j = idx[.][a] has its groups at rows
    // slot_idx[.][a] * gpc .. of one shared slice (cap = 0); ids and order still follow idx
    const int32_t *slot_idx;
    int32_t *gidx;
    long long cap;  // group-summary rows per (b, g)
    int n_q_heads, n_kv_heads, seg_len, q_block, n, topk, gpc, topg;
    float inv_sqrt_d;
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1) route_groups_kernel(const GroupArgs a) {
    constexpr int NRS = kThreads / D;  // row slots of the block-summary sum
    __shared__ float part[NRS][D];
    __shared__ __align__(16) float qbar[D];
    __shared__ uint32_t row[kMaxCand];
    __shared__ int chunks[64], rows[64], sel[kMaxCand], n_chunks;
    __shared__ __align__(16) uint32_t s_tmax[kThreads];  // select_cta reads it as 16-byte vectors
    __shared__ uint64_t s_key[kCandCap];
    __shared__ int s_cj[kCandCap], s_hist[256], s_misc[16];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nqb = a.seg_len / a.q_block;
    const int m = (int)blockIdx.x % nqb, bg = (int)blockIdx.x / nqb;
    const int b = bg / a.n_kv_heads, g = bg % a.n_kv_heads;
    const int G = a.n_q_heads / a.n_kv_heads;
    int32_t *out = a.gidx + ((long long)bg * nqb + m) * a.topg;

    // block summary: thread (rs, d) sums rows rs, rs + NRS, ... of the G x q_block
    // rows (head-major) in order, then the NRS partials are added in order
    {
        const int d = tid % D, rs = tid / D;
        const T *qb = static_cast<const T *>(a.q) +
                      (((long long)b * a.n_q_heads + (long long)g * G) * a.seg_len + (long long)m * a.q_block) * D + d;
        float acc = 0.f;
        for (int r = rs; r < G * a.q_block; r += NRS) {
            const int hh = r / a.q_block, i = r - hh * a.q_block;
            acc += to_f32(qb[((long long)hh * a.seg_len + i) * D]);
        }
        part[rs][d] = acc;
    }
    if (tid == 0) {  // the block's chosen chunks, ascending (insertion sort of <= 64 ids)
        const int32_t *selc = a.idx + ((long long)bg * nqb + m) * a.topk;
        const int32_t *slc = a.slot_idx ? a.slot_idx + ((long long)bg * nqb + m) * a.topk : nullptr;
        int nv = 0;
        for (int t = 0; t < a.topk; ++t) {
            const int j = selc[t];
            if (j < 0 || j >= a.n) continue;
            if (slc && slc[t] < 0) continue;  // not staged
            const int row = slc ? slc[t] : j;  // first summary row of the chunk's groups / gpc
            int p = nv++;
            while (p > 0 && chunks[p - 1] > j) {
                chunks[p] = chunks[p - 1];
                rows[p] = rows[p - 1];
                --p;
            }
            chunks[p] = j;
            rows[p] = row;
        }
        n_chunks = nv;
    }
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
        for (int r = 0; r < NRS; ++r) s += part[r][tid];
        qbar[tid] = s / static_cast<float>(G * a.q_block);
    }
    __syncthreads();

    // scores of the candidate groups: one warp per candidate, D / 32 values per lane
    const int ncand = n_chunks * a.gpc;
    const float *gbase = a.gsumm + (a.slot_idx ? 0ll : (long long)bg * a.cap * D);
    constexpr int VPL = D / 32;
    float qv[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) qv[e] = qbar[lane * VPL + e];
    for (int c = warp; c < ncand; c += kWarps) {
        const int grow = rows[c / a.gpc] * a.gpc + c % a.gpc;  // summary row (slot-based when staged)
        const float *gr = gbase + (long long)grow * D + lane * VPL;
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < VPL; ++e) acc = fmaf(qv[e], gr[e], acc);
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
        if (lane == 0) row[c] = ordered_bits(acc * a.inv_sqrt_d);
    }
    __syncthreads();

    if (a.topg >= ncand) {  // every candidate is kept
        for (int t = tid; t < a.topg; t += kThreads)
            out[t] = t < ncand ? chunks[t / a.gpc] * a.gpc + t % a.gpc : -1;
        return;
    }
    SelScratch ss;
    ss.tmax = s_tmax;
    ss.key = s_key;
    ss.cj = s_cj;
    ss.hist = s_hist;
    ss.misc = s_misc;
    select_cta(row, ncand, a.topg, sel, ss, tid);  // positions, ascending
    __syncthreads();
    for (int t = tid; t < a.topg; t += kThreads) out[t] = chunks[sel[t] / a.gpc] * a.gpc + sel[t] % a.gpc;
}

}  // namespace

hga_status_t launch_route(const hga_params_t &p, const void *q, const float *summ, int cap, int32_t *idx,
                          unsigned *status, cudaStream_t stream) {
    const int n = p.n_hist_chunks, D = p.head_dim;
    const int nqb = p.seg_len / p.q_block;
    const int esize = p.dtype == HGA_BF16 ? 2 : 4;
    // cluster size: the smallest that lets one CTA's slice of the chunk list
    // fit one round of bulk copies, else the largest
    const int ring_chunks = kRound * (kTileBytes / (D * 4));
    // a grid of less than one CTA per SM keeps two rounds in flight (two CTAs
    // per SM overlap each other's copies otherwise) when that layout fits; more
    // slots do not help: one SM's bulk copies stream at about 40 GB/s however
    // many are in flight
    const bool small_grid = (long long)p.batch * p.n_kv_heads * nqb < sm_count();
    int cl = 1, slots = kRound;
    RouteLayout L{};
    for (int sl : {2 * kRound, kRound}) {
        if (sl > kRound && !small_grid) continue;
        slots = sl;
        cl = 1;
        L = route_layout(D, esize, 1, round4(n), n, sl, 1);
        if (n > p.topk) {
            for (int c : {1, 2, 4, 8}) {
                if (nqb % c) continue;
                const RouteLayout Lc =
                    route_layout(D, esize, c, c > 1 ? round4((n + c - 1) / c) : round4(n), n, sl, c);
                if (Lc.total > kMaxSmem) continue;
                cl = c;
                L = Lc;
                if ((n + c - 1) / c <= ring_chunks) break;
            }
        }
        if (L.total <= kMaxSmem) break;
    }
    // one query block per (b, g) and more chunks than one round: a cluster of the
    // largest size that keeps the grid within one CTA per SM splits the chunk
    // list (rank 0 selects)
    bool split = false;
    if (nqb == 1 && n > p.topk && n > ring_chunks) {
        const long long groups = (long long)p.batch * p.n_kv_heads;
        const int sms = sm_count();
        int c_best = 1;
        for (int c : {2, 4, 8})
            if (groups * c <= sms && (n + c - 1) / c >= ring_chunks / 2) c_best = c;
        if (c_best > 1) {
            const int sl = 2 * kRound;
            const RouteLayout Lc = route_layout(D, esize, c_best, round4((n + c_best - 1) / c_best), n, sl, 1);
            if (Lc.total <= kMaxSmem) {
                split = true;
                cl = c_best;
                slots = sl;
                L = Lc;
            }
        }
    }
    if (L.total > kMaxSmem) {
        record_error("hga_route: shared-memory layout exceeds the per-CTA limit");
        return HGA_ERR_UNSUPPORTED;
    }
    RouteArgs a{};
    a.q = q;
    a.summ = summ;
    a.idx = idx;
    a.status = status;
    a.cap = cap;
    a.n_q_heads = p.n_q_heads;
    a.n_kv_heads = p.n_kv_heads;
    a.seg_len = p.seg_len;
    a.n = n;
    a.topk = p.topk;
    a.q_block = p.q_block;
    a.sink = p.sink_chunks;
    a.ns = cl > 1 ? round4((n + cl - 1) / cl) : round4(n);
    a.slots = slots;
    a.inv_sqrt_d = static_cast<float>(1.0 / __builtin_sqrt(static_cast<double>(D)));
    a.L = L;
    const unsigned grid = static_cast<unsigned>(p.batch * p.n_kv_heads * (split ? cl : nqb));
    cudaError_t e;
    if (p.dtype == HGA_BF16)
        e = D == 128 ? launch_t<__nv_bfloat16, 128>(a, cl, split, grid, stream)
                     : launch_t<__nv_bfloat16, 64>(a, cl, split, grid, stream);
    else
        e = D == 128 ? launch_t<float, 128>(a, cl, split, grid, stream) : launch_t<float, 64>(a, cl, split, grid, stream);
    if (e == cudaSuccess) e = cudaGetLastError();
    return record_cuda(e);
}

hga_status_t launch_route_causal(const hga_params_t &p, const void *q, const float *summ, int cap, int32_t *idx,
                                 unsigned *status, cudaStream_t stream) {
    const int n = p.n_hist_chunks, D = p.head_dim;
    // one-token blocks: the block route is already per token
    if (p.q_block == 1) return launch_route(p, q, summ, cap, idx, status, stream);
    const CausalLayout L = causal_layout(D, p.q_block, n);
    if (L.tp < 1 || L.total > kMaxSmem) {
        record_error("hga_route_causal: shared-memory layout exceeds the per-CTA limit");
        return HGA_ERR_UNSUPPORTED;
    }
    RouteArgs a{};
    a.q = q;
    a.summ = summ;
    a.idx = idx;
    a.status = status;
    a.cap = cap;
    a.n_q_heads = p.n_q_heads;
    a.n_kv_heads = p.n_kv_heads;
    a.seg_len = p.seg_len;
    a.q_block = p.q_block;
    a.n = n;
    a.topk = p.topk;
    a.sink = p.sink_chunks;
    a.inv_sqrt_d = static_cast<float>(1.0 / __builtin_sqrt(static_cast<double>(D)));
    const unsigned grid = static_cast<unsigned>(p.batch * p.n_kv_heads * (p.seg_len / p.q_block));
    cudaError_t e;
    auto go = [&](auto kern) {
        cudaError_t err = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), L.total);
        if (err != cudaSuccess) return err;
        kern<<<grid, kThreads, L.total, stream>>>(a, L.tp, L);
        return cudaGetLastError();
    };
    if (p.dtype == HGA_BF16)
        e = D == 128 ? go(route_causal_kernel<__nv_bfloat16, 128>) : go(route_causal_kernel<__nv_bfloat16, 64>);
    else
        e = D == 128 ? go(route_causal_kernel<float, 128>) : go(route_causal_kernel<float, 64>);
    return record_cuda(e);
}

hga_status_t launch_route_groups(const hga_params_t &p, const void *q, const float *gsumm, long long cap,
                                 const int32_t *idx, int group, int topg, int32_t *gidx, cudaStream_t stream,
                                 const int32_t *slot_idx) {
    GroupArgs a{};
    a.q = q;
    a.gsumm = gsumm;
    a.idx = idx;
    a.slot_idx = slot_idx;
    a.gidx = gidx;
    a.cap = cap;
    a.n_q_heads = p.n_q_heads;
    a.n_kv_heads = p.n_kv_heads;
    a.seg_len = p.seg_len;
    a.q_block = p.q_block;
    a.n = p.n_hist_chunks;
    a.topk = p.topk;
    a.gpc = p.chunk / group;
    a.topg = topg;
    a.inv_sqrt_d = static_cast<float>(1.0 / __builtin_sqrt(static_cast<double>(p.head_dim)));
    const unsigned grid = static_cast<unsigned>(p.batch * p.n_kv_heads * (p.seg_len / p.q_block));
    if (p.dtype == HGA_BF16) {
        if (p.head_dim == 128) route_groups_kernel<__nv_bfloat16, 128><<<grid, kThreads, 0, stream>>>(a);
        else route_groups_kernel<__nv_bfloat16, 64><<<grid, kThreads, 0, stream>>>(a);
    } else {
        if (p.head_dim == 128) route_groups_kernel<float, 128><<<grid, kThreads, 0, stream>>>(a);
        else route_groups_kernel<float, 64><<<grid, kThreads, 0, stream>>>(a);
    }
    return record_cuda(cudaGetLastError());
}

}  // namespace hga
