// Exact-token HGA attention forward on the 5th-generation tensor cores
// (tcgen05 / TMEM / TMA), bf16 inputs, fp32 accumulation, head_dim 128.
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.1
// (exact K/V of the routed chunks attended with a local window; summaries
// route only) and the author abstract (a bounded set of exact historical
// tokens per query block).
//
// One CTA per (batch, kv head, query block, head sub-group).  The query heads
// of a KV group share every K/V tile, so a CTA holds HC of them (HC = 4 when
// G % 4 == 0, else 2 when G is even, else 1) as NH M=128 halves of 64-row
// head pairs: each 64-token key tile (a routed history chunk, then the active
// segment's causal tiles 0..m) is read once for HC heads, which lifts a
// history tile from 64 to 256 flop/byte at HC = 4.  G / HC CTAs share one KV
// group (its tiles then come from L2).  With HC = 1 the second 64 rows of the
// M=128 half repeat the head's rows and are not written back.
//
// Warp roles (NH = 2: 416 threads):
//   warp 0      TMA producer: Q once, then K and V of every tile, each into
//               its own 4-stage ring (routed chunk j -> TMA row coordinate
//               (b*Hkv+g)*stride + 64 j); a K stage is released as soon as
//               QK^T of its tile completes, a V stage after PV.
//   warps 1, 3  QK issuers, one thread per M half (warp 1 also owns TMEM):
//               S_h = Q_h K^T   (M128 N64 K128, K-major A and B, SW128), into
//               one of two S buffers once PV two tiles back has read the P
//               stored there.
//   warps 2, 4  PV issuers, one thread per M half:
//               O_h += P_h V    (M128 N128 K64, P from TMEM, V MN-major),
//               issued as soon as the softmax has written P.  The four issue
//               streams run in separate warps, each converged with one lane
//               elected per MMA.
//   warps 5+4h.. softmax of half h: one TMEM lane (= query row) per thread
//               (a warp reads the lane quadrant of its warp index % 4, so any
//               four consecutive warps cover the half's 128 rows); online
//               softmax in the log2 domain, O rescaled in TMEM when the row max
//               grows by more than 2^8, P written as bf16 pairs into the tile's
//               S buffer, where the PV issue reads it.  (Two threads per row,
//               each with half of a tile's columns and a max exchange through
//               shared memory, measured 7% slower on B200: the per-thread
//               softmax chain is not what bounds a tile.)
// TMEM (512 columns): O_h at 128h, S_h double-buffered at 256 + 128h + 64b.
// Every wait is bounded; a timeout sets HGA_DEV_TIMEOUT and the CTA unwinds.
//
// Three kinds of routes fill the history tiles (template MODE):
//   kChunk   a block's routed 64-token chunks, one tile each (hga_attn_fwd);
//   kGroup   a block's routed groups of gs = 8, 16 or 32 tokens (the group
//            stage of the technical summary, section 2.1), packed 64 / gs to a
//            tile, one TMA box of gs rows per group -- each box lands as whole
//            128-byte swizzle atoms, so the MMA descriptors are unchanged; the
//            unfilled slots of a block's last tile repeat a loaded group and
//            their columns are masked;
//   kMasked  the union of the per-token routes of a block's 64 tokens (the
//            strictly causal variant of the technical summary's limits
//            section), one tile per chunk of the union with a 64-bit mask of
//            the block's tokens that route to it: rows whose bit is clear
//            see the whole tile as masked.
//
// SEGF (chunk routes, hga_route_attn_fwd): the kernel is launched as a
// programmatic dependent of the route kernel and takes the causal segment
// tiles 0..m first -- they need no route -- so it runs while the route grid
// finishes; the producer waits for the route grid (griddepcontrol.wait) only
// before the first history tile, builds the tile list and publishes it to the
// other roles through an mbarrier.  Everything else it reads was written
// before the route kernel started.
#include <cudaTypedefs.h>

#include "tc_issue.cuh"
#include "tc_ptx.cuh"

namespace hga {

namespace {

constexpr int D = 128;
constexpr int TILE = 64;
constexpr int NSTAGE = 4;
constexpr float kRescaleLog2 = 8.f;  // lazy-rescale threshold on the running max (log2 units)
constexpr uint32_t Q_HALF_BYTES = 128 * D * 2;   // 32 KiB: [2 col halves][128 rows][128 B]
constexpr uint32_t KV_TILE_BYTES = TILE * D * 2; // 16 KiB: [2 col halves][64 rows][128 B]
constexpr uint32_t IDESC_QK = tc::idesc_bf16(128, TILE, false, false);
constexpr uint32_t IDESC_PV = tc::idesc_bf16(128, D, false, true);
constexpr int kChunk = 0, kGroup = 1, kMasked = 2;
constexpr int kMaxGroups = 512;  // routed groups per block (k <= 64 chunks x 8 groups)

template <int NH>
struct Smem {
    static constexpr uint32_t Q = 0;
    static constexpr uint32_t K = Q + NH * Q_HALF_BYTES;      // K ring
    static constexpr uint32_t V = K + NSTAGE * KV_TILE_BYTES; // V ring
    static constexpr uint32_t GLIST = V + NSTAGE * KV_TILE_BYTES;  // routed group ids (kGroup)
    static constexpr uint32_t BAR = GLIST + kMaxGroups * 4;
    static constexpr uint32_t TOTAL = BAR + 1024;  // barriers, tile list, flags
    static constexpr uint32_t ALLOC = TOTAL + 1024; // + alignment slack
};

// D[tmem] (+)= A[tmem] * B[smem] for one K=16 step of kind::f16 (A read from TMEM).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct Bars {
    uint64_t q_full;
    uint64_t k_full[NSTAGE];
    uint64_t k_empty[NSTAGE];  // released once QK^T of the tile completes (both halves)
    uint64_t v_full[NSTAGE];
    uint64_t v_empty[NSTAGE];  // released once PV of the tile completes (both halves)
    uint64_t s_full[2][2];  // [half][S/P buffer]: S of the buffer's tile in TMEM
    uint64_t p_full[2][2];  // [half][S/P buffer]: P of the buffer's tile written to TMEM
    uint64_t o_done[2][2];  // [half][S/P buffer]: PV of the buffer's tile completed
    uint64_t drain[4];      // one per issuing thread (abort path)
    uint64_t route_ready;   // SEGF: the history tile list is built
    uint32_t tmem_base;
    int abort;
    int n_hist;
    int issued_k;  // K / V tiles the producer issued
    int issued_v;
    int sm0_tiles;  // tiles whose softmax half 0 has finished (scheduling hint)
    int n_groups;   // kGroup: routed groups of this block
    int tiles[64];
};

static_assert(sizeof(Bars) <= 1024, "barrier block must fit its region");

struct FwdArgs {
    int batch, n_q_heads, n_kv_heads, seg_len, topk, n_hist_chunks;
    // kGroup: tokens per group; kMasked: routes per block in idx (the union capacity),
    // their count and the per-route token masks
    int gs;
    const int32_t *ucount;
    const unsigned long long *umask;
    int n_sub, hc;  // CTAs per KV group, query heads per CTA (4, 2 or 1)
    long long hist_stride, seg_stride;
    int qb0, n_blocks;
    const int32_t *idx;
    __nv_bfloat16 *out;
    float *lse;
    unsigned *status;
    float scale_log2;  // log2(e) / sqrt(D)
};

// Five control warps (producer, QK0, PV0, QK1, PV1) and 4 NH softmax warps.
// With NH = 2 the 416 threads launch at up to 152 registers each.
// Bounded wait until the shared counter reaches `target` (same contract as mbar_wait).
__device__ __forceinline__ bool wait_count(int *counter, int target, volatile int *abort, unsigned *status) {
    volatile int *c = counter;
    if (*c >= target) return true;
    const long long t0 = clock64();
    while (*c < target) {
        if (*abort) return false;
        if (clock64() - t0 > (1ll << 31)) {
            *abort = 1;
            atomicOr(status, kDevTimeout);
            return false;
        }
    }
    return true;
}

constexpr int kCtrlWarps = 5;

template <int NH, int MODE, bool SEGF>
__global__ void __launch_bounds__(32 * kCtrlWarps + 128 * NH, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kh,
                       const __grid_constant__ CUtensorMap tm_vh, const __grid_constant__ CUtensorMap tm_ks,
                       const __grid_constant__ CUtensorMap tm_vs, const FwdArgs a) {
    using L = Smem<NH>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bars = reinterpret_cast<Bars *>(smem + L::BAR);
    const uint32_t sbase = tc::smem_u32(smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nqb = a.seg_len / TILE;
    const int n_units = a.batch * a.n_kv_heads * a.n_sub;
    const int m = a.qb0 + a.n_blocks - 1 - (int)blockIdx.x / n_units;  // longest (latest) blocks first
    const int unit = (int)blockIdx.x % n_units;
    const int bg = unit / a.n_sub;
    const int b = bg / a.n_kv_heads, g = bg % a.n_kv_heads;
    // first query head of this CTA: the KV group's heads g*G .., HC per CTA
    const int h0 = g * (a.n_q_heads / a.n_kv_heads) + (unit % a.n_sub) * a.hc;

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->q_full, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            tc::mbar_init(&bars->k_full[s], 1);
            tc::mbar_init(&bars->k_empty[s], NH);
            tc::mbar_init(&bars->v_full[s], 1);
            tc::mbar_init(&bars->v_empty[s], NH);
        }
        for (int h = 0; h < 2; ++h)
            for (int bb = 0; bb < 2; ++bb) {
                tc::mbar_init(&bars->s_full[h][bb], 1);
                tc::mbar_init(&bars->p_full[h][bb], 4);  // every softmax warp of the half
                tc::mbar_init(&bars->o_done[h][bb], 1);
            }
        for (int d = 0; d < 4; ++d) tc::mbar_init(&bars->drain[d], 1);
        tc::mbar_init(&bars->route_ready, 1);
        bars->issued_k = 0;
        bars->issued_v = 0;
        bars->sm0_tiles = 0;
        bars->abort = 0;
        tc::fence_mbar_init();
    }
    int *glist = reinterpret_cast<int *>(smem + L::GLIST);
    const long long bgm = (long long)bg * nqb + m;
    // routed history chunks of this block; -1 is padding, anything else out of range is skipped
    auto build_chunk_list = [&]() -> int {
        const int32_t *sel = a.idx + bgm * a.topk;
        int n = 0;
        for (int i = 0; i < a.topk; ++i) {
            const int j = sel[i];
            if (j >= 0 && j < a.n_hist_chunks) bars->tiles[n++] = j;
            else if (j != -1) atomicOr(a.status, kDevBadIndex);
        }
        return n;
    };
    if (SEGF && warp == 2 && lane == 0) bars->n_hist = 0;  // published by the producer once routed
    if (!SEGF && warp == 2 && lane == 0) {
        const int32_t *sel = a.idx + bgm * a.topk;
        int n = 0;
        if constexpr (MODE == kChunk) {
            n = build_chunk_list();
        } else if constexpr (MODE == kGroup) {
            const int n_groups = a.n_hist_chunks * (TILE / a.gs);
            int ng = 0;
            for (int i = 0; i < a.topk && ng < kMaxGroups; ++i) {
                const int u = sel[i];
                if (u >= 0 && u < n_groups) glist[ng++] = u;
                else if (u != -1) atomicOr(a.status, kDevBadIndex);
            }
            bars->n_groups = ng;
            n = (ng * a.gs + TILE - 1) / TILE;
        } else {
            // the union list was validated when it was built
            const int cnt = a.ucount[bgm];
            n = cnt < 0 ? 0 : (cnt > a.topk ? a.topk : cnt);
        }
        bars->n_hist = n;
    }
    if (warp == 1) tc::tmem_alloc<512>(&bars->tmem_base);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort = &bars->abort;
    // Tile order: history tiles then segment tiles 0..m, or (SEGF) segment tiles
    // then history tiles, whose count is known once the route is (resolve_tiles).
    int n_hist = SEGF ? 0 : bars->n_hist;
    int n_tiles = SEGF ? m + 2 : n_hist + m + 1;  // SEGF: provisional until tile m + 1
    const int first_seg = SEGF ? 0 : n_hist;        // first segment tile (fixed once resolved)
    // SEGF: at tile m + 1 every role waits for the producer's tile list
    auto resolve_tiles = [&](int j) -> bool {
        if (!SEGF || j != m + 1) return true;
        if (!tc::mbar_wait(&bars->route_ready, 0, abort, a.status)) return false;
        n_hist = *reinterpret_cast<volatile int *>(&bars->n_hist);
        n_tiles = m + 1 + n_hist;
        return true;
    };

    if (warp < kCtrlWarps) {
    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producer
            tc::tma_prefetch_desc(&tm_q);
            tc::tma_prefetch_desc(&tm_kh);
            tc::tma_prefetch_desc(&tm_ks);
            tc::tma_prefetch_desc(&tm_vh);
            tc::tma_prefetch_desc(&tm_vs);
            tc::mbar_arrive_expect_tx(&bars->q_full, NH * Q_HALF_BYTES);
            for (int hh = 0; hh < 2 * NH; ++hh) {
                const int qrow = (b * a.n_q_heads + h0 + (a.hc == 1 ? 0 : hh)) * a.seg_len + m * TILE;
                uint8_t *dst = smem + L::Q + (hh >> 1) * Q_HALF_BYTES + (hh & 1) * (64 * 128);
                tc::tma_load_2d(dst, &tm_q, 0, qrow, &bars->q_full);
                tc::tma_load_2d(dst + 128 * 128, &tm_q, 64, qrow, &bars->q_full);
            }
            // K(j), then V(j): a K stage frees once QK^T(j - NSTAGE) completes, a V
            // stage once PV(j - NSTAGE) does; routed chunk j is row (b*Hkv+g)*stride + 64 j
            // a tile as TMA boxes: one 64-row box per column half, or (kGroup history
            // tiles) 64 / gs boxes of gs rows per column half, group slot u at row u*gs
            const int n_groups = MODE == kGroup ? bars->n_groups : 0;
            auto load_tile = [&](uint8_t *dst, const CUtensorMap *mh, const CUtensorMap *ms, int jt, uint64_t *bar) {
                // segment tile jt - first_seg (SEGF: jt <= m), else history tile j
                const bool seg = SEGF ? jt <= m : jt >= n_hist;
                const int j = SEGF ? jt - m - 1 : jt;
                if (seg) {
                    const int row = (int)((long long)bg * a.seg_stride + (long long)(jt - first_seg) * TILE);
                    tc::tma_load_2d(dst, ms, 0, row, bar);
                    tc::tma_load_2d(dst + 64 * 128, ms, 64, row, bar);
                } else if constexpr (MODE == kGroup) {
                    const int gpt = TILE / a.gs;
                    for (int u = 0; u < gpt; ++u) {
                        const int at = j * gpt + u;
                        const int grp = glist[at < n_groups ? at : j * gpt];  // unfilled slots repeat a group
                        const int row = (int)((long long)bg * a.hist_stride + (long long)grp * a.gs);
                        tc::tma_load_2d(dst + u * a.gs * 128, mh, 0, row, bar);
                        tc::tma_load_2d(dst + 64 * 128 + u * a.gs * 128, mh, 64, row, bar);
                    }
                } else {
                    const int chunk = MODE == kChunk ? bars->tiles[j] : a.idx[bgm * a.topk + j];
                    const int row = (int)((long long)bg * a.hist_stride + (long long)chunk * TILE);
                    tc::tma_load_2d(dst, mh, 0, row, bar);
                    tc::tma_load_2d(dst + 64 * 128, mh, 64, row, bar);
                }
            };
            int nk = 0, nv = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % NSTAGE, u = j / NSTAGE;
                if (SEGF && j == m + 1) {
                    // the route grid has finished and its writes are visible after this
                    asm volatile("griddepcontrol.wait;" ::: "memory");
                    n_hist = build_chunk_list();
                    bars->n_hist = n_hist;
                    n_tiles = m + 1 + n_hist;
                    tc::mbar_arrive(&bars->route_ready);
                    if (j >= n_tiles) break;
                }
                if (j >= NSTAGE && !tc::mbar_wait(&bars->k_empty[s], (u - 1) & 1, abort, a.status)) break;
                tc::mbar_arrive_expect_tx(&bars->k_full[s], KV_TILE_BYTES);
                load_tile(smem + L::K + s * KV_TILE_BYTES, &tm_kh, &tm_ks, j, &bars->k_full[s]);
                nk = j + 1;
                if (j >= NSTAGE && !tc::mbar_wait(&bars->v_empty[s], (u - 1) & 1, abort, a.status)) break;
                tc::mbar_arrive_expect_tx(&bars->v_full[s], KV_TILE_BYTES);
                load_tile(smem + L::V + s * KV_TILE_BYTES, &tm_vh, &tm_vs, j, &bars->v_full[s]);
                nv = j + 1;
            }
            bars->issued_k = nk;
            bars->issued_v = nv;
        }
    } else if (warp < kCtrlWarps) {
        // ------------------------------------------------------------ UMMA issuers
        const int h = (warp - 1) >> 1;      // M half
        const bool qk = (warp & 1) != 0;    // warps 1, 3: QK^T; warps 2, 4: PV
        if (warp <= 4 && h < NH) {
            // The whole warp runs the loop (waits included) and elects one lane per MMA.
            // Descriptors are built once; a K-step, stage or buffer offset is added
            // to the start-address field (addresses stay below 2^18, so no carry).
            bool ok = true;
            if (qk) {
                const uint64_t q_desc = tc::desc_sw128(sbase + L::Q + h * Q_HALF_BYTES, 16, 1024);
                const uint64_t k_desc = tc::desc_sw128(sbase + L::K, 16, 1024);
                ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->q_full, 0, abort, a.status));
                for (int j = 0; ok && j < n_tiles; ++j) {
                    const int s = j % NSTAGE, bb = j & 1;
                    if (!__all_sync(0xffffffffu, resolve_tiles(j))) break;
                    if (j >= n_tiles) break;
                    if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->k_full[s], (j / NSTAGE) & 1, abort, a.status)))
                        break;
                    // S buffer bb is free once PV(j-2), which read P(j-2) from it, has completed
                    if (j >= 2 && !__all_sync(0xffffffffu, tc::mbar_wait(&bars->o_done[h][bb], ((j >> 1) - 1) & 1,
                                                                         abort, a.status)))
                        break;
                    // half 1 runs half a tile behind half 0: its S(j) lands while half 0
                    // is in the exp phase of tile j, so the two softmax groups take
                    // turns on the MUFU instead of stalling on it together
                    if (h == 1 && j >= 1 && !__all_sync(0xffffffffu, wait_count(&bars->sm0_tiles, j, abort, a.status)))
                        break;
                    tc::fence_after_sync();
                    const uint64_t kd = k_desc + (uint64_t)((s * KV_TILE_BYTES) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = ((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4;
                        const uint32_t qoff = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
                        if (tc::elect_one())
                            tc::mma_f16(tmem + 256 + 128 * h + 64 * bb, q_desc + qoff, kd + koff, IDESC_QK,
                                        kk > 0 ? 1u : 0u);
                        __syncwarp();
                    }
                    if (tc::elect_one()) {
                        tc::mma_commit(&bars->s_full[h][bb]);
                        tc::mma_commit(&bars->k_empty[s]);  // one arrival per half
                    }
                    __syncwarp();
                }
            } else {
                const uint64_t v_desc = tc::desc_sw128(sbase + L::V, 8192, 1024);
                const uint32_t o_tmem = tmem + 128 * h;
                for (int t = 0; t < n_tiles; ++t) {
                    const int s = t % NSTAGE, pb = t & 1;
                    if (!__all_sync(0xffffffffu, resolve_tiles(t))) break;
                    if (t >= n_tiles) break;
                    if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->v_full[s], (t / NSTAGE) & 1, abort, a.status) &&
                                                     tc::mbar_wait(&bars->p_full[h][pb], (t >> 1) & 1, abort,
                                                                   a.status)))
                        break;
                    tc::fence_after_sync();
                    const uint64_t vd = v_desc + (uint64_t)((s * KV_TILE_BYTES) >> 4);
                    // P(t) as bf16 pairs in the first 32 columns of S buffer pb: 8 columns per K step
                    const uint32_t pa = tmem + 256 + 128 * h + 64 * pb;
#pragma unroll
                    for (int kk = 0; kk < TILE / 16; ++kk) {
                        if (tc::elect_one())
                            mma_f16_ts(o_tmem, pa + 8 * kk, vd + (kk * 2048 >> 4), IDESC_PV,
                                       (t > 0 || kk > 0) ? 1u : 0u);
                        __syncwarp();
                    }
                    if (tc::elect_one()) {
                        tc::mma_commit(&bars->o_done[h][pb]);
                        tc::mma_commit(&bars->v_empty[s]);  // one arrival per half
                    }
                    __syncwarp();
                }
            }
        }
    }
    } else {
        // -------------------------------------------------------------- softmax / epilogue
        const int h = (warp - kCtrlWarps) >> 2;  // M half
        const int quad = warp & 3;               // TMEM lane quadrant this warp may access
        const int r = quad * 32 + lane;          // row within the half = TMEM lane
        const int hh = 2 * h + (r >> 6);         // head within the group
        const int i = r & 63;                    // query row within the block
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const uint32_t o_addr = tmem + lane_addr + 128 * h;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        // kGroup: valid columns of the last history tile; kMasked: this row's bit of the
        // next tile's token mask (read one tile ahead)
        const int last_cols = MODE == kGroup ? bars->n_groups * a.gs - (n_hist - 1) * TILE : TILE;
        unsigned long long mask_next = 0ull;
        if (MODE == kMasked && n_hist > 0) mask_next = a.umask[bgm * a.topk];
        for (int j = 0; j < n_tiles; ++j) {
            const int bb = j & 1;
            if (!__all_sync(0xffffffffu, resolve_tiles(j))) {
                ok = false;
                break;
            }
            if (j >= n_tiles) break;
            bool row_off = false;  // kMasked: the whole tile is masked for this row
            if constexpr (MODE == kMasked) {
                if (j < n_hist) {
                    row_off = ((mask_next >> i) & 1ull) == 0ull;
                    if (j + 1 < n_hist) mask_next = a.umask[bgm * a.topk + j + 1];
                }
            }
            // tcgen05.ld/st below are warp-collective: keep every decision warp-uniform
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->s_full[h][bb], (j >> 1) & 1, abort, a.status))) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            uint32_t sr[64];
            {
                uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
                uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
                const uint32_t s_addr = tmem + lane_addr + 256 + 128 * h + 64 * bb;
                tc::tmem_ld32(s_addr, lo);
                tc::tmem_ld32(s_addr + 32, hi);
                tc::tmem_wait_ld();
            }
            float x[64];
            const bool diag = (j == (SEGF ? m : n_tiles - 1));  // the local tile of this block (warp-uniform)
#pragma unroll
            for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(sr[c]);
            if (diag) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c > i) x[c] = -INFINITY;
            }
            if constexpr (MODE == kGroup) {
                if (j == n_hist - 1 && last_cols < TILE) {  // repeated groups past the routed ones
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c >= last_cols) x[c] = -INFINITY;
                }
            }
            if constexpr (MODE == kMasked) {
                if (row_off) {
#pragma unroll
                    for (int c = 0; c < 64; ++c) x[c] = -INFINITY;
                }
            }
            // row max of the raw scores (the scale is positive), 8 independent chains
            float mpart[8];
#pragma unroll
            for (int c = 0; c < 64; ++c) mpart[c & 7] = (c < 8) ? x[c] : fmaxf(mpart[c & 7], x[c]);
            const float mx = fmaxf(fmaxf(fmaxf(mpart[0], mpart[1]), fmaxf(mpart[2], mpart[3])),
                                   fmaxf(fmaxf(mpart[4], mpart[5]), fmaxf(mpart[6], mpart[7]))) *
                             a.scale_log2;
            // Lazy rescaling: the reference max only moves when the row max grows by
            // more than kRescaleLog2, so P stays <= 2^kRescaleLog2 and O is rescaled
            // in TMEM only on those (rare) tiles.
            const bool grow = mx > m_run + kRescaleLog2;
            const float m_use = grow ? mx : m_run;
            const float alpha = grow ? tc::ex2(m_run - m_use) : 1.f;
            // a row with no unmasked key yet keeps m = -inf; its p must come out 0, not NaN
            const float m_sub = m_use == -INFINITY ? 0.f : m_use;
            float spart[8];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                // p = 2^(s * log2(e)/sqrt(D) - m)
                x[c] = tc::ex2(fmaf(x[c], a.scale_log2, -m_sub));
                spart[c & 7] = (c < 8) ? x[c] : spart[c & 7] + x[c];
            }
            const float sum = ((spart[0] + spart[1]) + (spart[2] + spart[3])) +
                              ((spart[4] + spart[5]) + (spart[6] + spart[7]));
            l_run = l_run * alpha + sum;
            const int pb = j & 1;
            // a rescale needs O complete up to tile j-1 (PV(j-1) done) before PV(j) adds to it;
            // rows that keep their reference max have alpha == 1, an exact no-op
            if (j >= 1 && __any_sync(0xffffffffu, grow)) {
                if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->o_done[h][pb ^ 1], ((j - 1) >> 1) & 1, abort,
                                                            a.status))) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tc::tmem_ld32(o_addr + c0, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tc::tmem_st32(o_addr + c0, o);
                }
                tc::tmem_wait_st();
            }
            m_run = m_use;
            // P as bf16 pairs over the first 32 columns of this tile's S buffer (already
            // read into registers); PV reads it from there as its A operand
            {
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) pk[c] = tc::pack_bf16(x[2 * c], x[2 * c + 1]);
                tc::tmem_st32(tmem + lane_addr + 256 + 128 * h + 64 * pb, pk);
                tc::tmem_wait_st();
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->p_full[h][pb]);
            if (NH == 2 && warp == kCtrlWarps && lane == 0) *reinterpret_cast<volatile int *>(&bars->sm0_tiles) = j + 1;
        }
        if (ok && __all_sync(0xffffffffu, tc::mbar_wait(&bars->o_done[h][(n_tiles - 1) & 1],
                                                        ((n_tiles - 1) >> 1) & 1, abort, a.status))) {
            tc::fence_after_sync();
            const bool write = hh < a.hc;  // rows 64..127 repeat the head when HC = 1
            const long long row = ((long long)(b * a.n_q_heads + h0 + (write ? hh : 0))) * a.seg_len + m * TILE + i;
            __nv_bfloat16 *orow = a.out + row * D;
            const float inv_l = 1.f / l_run;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                tc::tmem_ld32(o_addr + c0, o);
                tc::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; c += 8) {
                    if (!write) break;
                    uint4 v;
                    v.x = tc::pack_bf16(__uint_as_float(o[c + 0]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
                    v.y = tc::pack_bf16(__uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
                    v.z = tc::pack_bf16(__uint_as_float(o[c + 4]) * inv_l, __uint_as_float(o[c + 5]) * inv_l);
                    v.w = tc::pack_bf16(__uint_as_float(o[c + 6]) * inv_l, __uint_as_float(o[c + 7]) * inv_l);
                    *reinterpret_cast<uint4 *>(orow + c0 + c) = v;
                }
            }
            if (write) a.lse[row] = (m_run + __log2f(l_run)) * 0.69314718055994530942f;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (*abort) {
        // a wait gave up: let the copies and UMMAs still in flight finish before
        // shared memory and TMEM are released
        int never = 0;
        if (warp == 0 && lane == 0) {
            for (int pass = 0; pass < 2; ++pass) {
                const int issued = pass == 0 ? bars->issued_k : bars->issued_v;
                uint64_t *full = pass == 0 ? bars->k_full : bars->v_full;
                for (int j = issued - NSTAGE < 0 ? 0 : issued - NSTAGE; j < issued; ++j)
                    tc::mbar_wait(&full[j % NSTAGE], (j / NSTAGE) & 1, &never, a.status, 1ll << 28);
            }
            tc::mbar_wait(&bars->q_full, 0, &never, a.status, 1ll << 28);
        }
        if (warp >= 1 && warp <= 4 && ((warp - 1) >> 1) < NH) {
            // the lane that issued this warp's MMAs commits and waits for them
            if (tc::elect_one()) {
                tc::mma_commit(&bars->drain[warp - 1]);
                tc::mbar_wait(&bars->drain[warp - 1], 0, &never, a.status, 1ll << 28);
            }
        }
        __syncwarp();
        tc::fence_after_sync();
    }
    if (warp == 1) {
        __syncwarp();
        tc::tmem_dealloc<512>(tmem);
    }
}

// ------------------------------------------------------------------ host side
bool make_map(CUtensorMap *map, const void *base, unsigned long long rows) {
    return tma_rows_map(map, base, rows);
}

template <int NH, int MODE, bool SEGF>
hga_status_t launch_nh(const hga_params_t &p, const void *q, const void *kh, const void *vh, const void *ks,
                       const void *vs, const FwdRoutes &rt, void *out, float *lse, unsigned *status,
                       cudaStream_t stream) {
    CUtensorMap mq, mkh, mvh, mks, mvs;
    const long long n_bg = (long long)p.batch * p.n_kv_heads;
    const unsigned long long q_rows = (unsigned long long)p.batch * p.n_q_heads * p.seg_len;
    const long long hist_rows =
        p.hist_head_stride > 0 ? (n_bg - 1) * p.hist_head_stride + (long long)p.n_hist_chunks * p.chunk
                               : (long long)p.n_hist_chunks * p.chunk;
    const unsigned long long seg_rows = (unsigned long long)((n_bg - 1) * p.seg_head_stride + p.seg_len);
    if (!make_map(&mq, q, q_rows) || !make_map(&mks, ks, seg_rows) || !make_map(&mvs, vs, seg_rows))
        return HGA_ERR_INVALID_ARG;
    if (hist_rows > 0) {
        // group routes read boxes of gs rows, one per routed group
        const unsigned box = MODE == kGroup ? (unsigned)rt.gs : 64u;
        if (!tma_rows_map(&mkh, kh, (unsigned long long)hist_rows, box) ||
            !tma_rows_map(&mvh, vh, (unsigned long long)hist_rows, box))
            return HGA_ERR_INVALID_ARG;
    } else {
        mkh = mks;  // never read: no routable history
        mvh = mvs;
    }
    const int nqb = p.seg_len / p.q_block;
    FwdArgs a;
    const int G = p.n_q_heads / p.n_kv_heads;
    a.hc = NH == 2 ? 4 : (G % 2 == 0 ? 2 : 1);
    a.n_sub = G / a.hc;
    a.batch = p.batch;
    a.n_q_heads = p.n_q_heads;
    a.n_kv_heads = p.n_kv_heads;
    a.seg_len = p.seg_len;
    a.topk = rt.per_block;
    a.n_hist_chunks = p.n_hist_chunks;
    a.gs = rt.gs;
    a.ucount = rt.ucount;
    a.umask = rt.umask;
    a.hist_stride = p.hist_head_stride;
    a.seg_stride = p.seg_head_stride;
    a.qb0 = p.qblock_end > 0 ? p.qblock_begin : 0;
    a.n_blocks = (p.qblock_end > 0 ? p.qblock_end : nqb) - a.qb0;
    a.idx = rt.list;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.status = status;
    a.scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)D));
    const size_t smem = Smem<NH>::ALLOC;
    auto kern = attn_fwd_tc_kernel<NH, MODE, SEGF>;
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), (int)smem);
    if (e != cudaSuccess) return record_cuda(e);
    const unsigned grid = (unsigned)(a.n_blocks * n_bg * a.n_sub);
    if (grid == 0) return HGA_OK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 * kCtrlWarps + 128 * NH);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    // SEGF: a programmatic dependent of the route kernel launched just before it
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = SEGF ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, mq, mkh, mvh, mks, mvs, a);
    if (e == cudaSuccess) e = cudaGetLastError();
    return record_cuda(e);
}

template <int MODE, bool SEGF = false>
hga_status_t launch_mode(const hga_params_t &p, const void *q, const void *kh, const void *vh, const void *ks,
                         const void *vs, const FwdRoutes &rt, void *out, float *lse, unsigned *status,
                         cudaStream_t stream) {
    const int G = p.n_q_heads / p.n_kv_heads;
    if (G % 4 == 0) return launch_nh<2, MODE, SEGF>(p, q, kh, vh, ks, vs, rt, out, lse, status, stream);
    return launch_nh<1, MODE, SEGF>(p, q, kh, vh, ks, vs, rt, out, lse, status, stream);
}

}  // namespace

bool attn_fwd_tc_shape(const hga_params_t &p) {
    return p.dtype == HGA_BF16 && p.head_dim == 128 && p.chunk == 64 && p.q_block == 64;
}

bool attn_fwd_tc_supported(const hga_params_t &p) {
    if (!attn_fwd_tc_shape(p)) return false;
    // TMA row coordinates are 32-bit
    const long long n_bg = (long long)p.batch * p.n_kv_heads;
    if (n_bg * (p.hist_head_stride > p.seg_head_stride ? p.hist_head_stride : p.seg_head_stride) >= (1ll << 31))
        return false;
    if ((long long)p.batch * p.n_q_heads * p.seg_len >= (1ll << 31)) return false;
    return tma_encoder_available();
}

hga_status_t launch_attn_fwd_tc(const hga_params_t &p, const void *q, const void *kh, const void *vh,
                                const void *ks, const void *vs, const int32_t *idx, void *out, float *lse,
                                unsigned *status, cudaStream_t stream) {
    FwdRoutes rt{idx, p.topk, 0, nullptr, nullptr};
    return launch_mode<kChunk>(p, q, kh, vh, ks, vs, rt, out, lse, status, stream);
}

hga_status_t launch_attn_fwd_tc_after_route(const hga_params_t &p, const void *q, const void *kh, const void *vh,
                                            const void *ks, const void *vs, const int32_t *idx, void *out,
                                            float *lse, unsigned *status, cudaStream_t stream) {
    FwdRoutes rt{idx, p.topk, 0, nullptr, nullptr};
    return launch_mode<kChunk, true>(p, q, kh, vh, ks, vs, rt, out, lse, status, stream);
}

hga_status_t launch_attn_fwd_tc_routes(const hga_params_t &p, const void *q, const void *kh, const void *vh,
                                       const void *ks, const void *vs, const FwdRoutes &rt, void *out, float *lse,
                                       unsigned *status, cudaStream_t stream) {
    if (rt.gs > 0) return launch_mode<kGroup>(p, q, kh, vh, ks, vs, rt, out, lse, status, stream);
    if (rt.umask) return launch_mode<kMasked>(p, q, kh, vh, ks, vs, rt, out, lse, status, stream);
    return launch_mode<kChunk>(p, q, kh, vh, ks, vs, rt, out, lse, status, stream);
}

}  // namespace hga
