// Backward of the exact-token HGA attention on tcgen05 tensor cores (bf16
// inputs, fp32 accumulation in TMEM, head_dim 128).
//
// "Long-Context Fine-Tuning with Limited VRAM", technical summary sections
// 2.1 (routing without gradient; gather and attention differentiable) and 2.2
// (segment-wise backward: history K/V detached at the segment boundary).
// With P = softmax row of query i (recomputed from the forward's LSE) and
// delta_i = rowsum(dO * O):
//   dS = P * (dO V^T - delta)
//   dQ = dS K / sqrt(D)                      over routed history and segment keys
//   dK_seg = dS^T Q / sqrt(D), dV_seg = P^T dO   over segment keys only
//
// Two block types in one launch of 384-thread blocks, no atomics (results are
// deterministic):
//   dQ blocks  : query-major, one CTA per M=128 tile of query rows: HC heads of the
//                group (4, 2 or 1, as in the forward) x 128 / HC rows of one query
//                block (two CTAs per block when HC = 4);
//                Q and dO copied once into TMEM; per key tile: S = Q K^T and
//                dP = dO V^T (M128 N64 K128, A from TMEM) into one of two TMEM
//                buffers, the dS rows in bf16 into one of two shared-memory buffers,
//                dQ += dS K (M128 N128 K64); warp 0 loads, warps 1, 2 and 3 issue S,
//                dP and dQ, warps 4-11 take half a row each (32 key columns).
//   dK/dV blocks: key-major over the active segment, one CTA per (batch, kv
//                head, 128 segment keys); for every later 64-query tile of
//                every head of the group: S^T = K Q^T and dP^T = V dO^T
//                (M128 N64 K128) into one of two TMEM buffers, P^T and dS^T in
//                bf16 written back into that buffer, dV += P^T dO and dK += dS^T Q
//                (M128 N128 K64, A from TMEM); warp 0 loads, warps 1 and 2 issue
//                S^T and dP^T, warp 3 dV and dK, warps 4-11 take half a key row
//                each (32 query columns).
// Each MMA-issuing warp runs its loop converged and elects one lane per MMA and for
// the commits that track them; warp 1 owns TMEM.
// Every wait is bounded and every warp-collective TMEM access is made from a
// converged warp with warp-uniform decisions.
//
// The dQ blocks take the same three kinds of routes as the forward (template
// MODE): whole routed chunks, routed groups of gs tokens (gs-row TMA boxes,
// the unfilled slots of the last tile repeating a loaded group with their
// columns masked), or the union of per-token routes with a token mask per
// chunk.  A masked key gets P = 0, so it adds nothing to dQ.
#include <cudaTypedefs.h>

#include "tc_issue.cuh"
#include "tc_ptx.cuh"

namespace hga {

namespace {

constexpr int D = 128;
constexpr int TILE = 64;
constexpr uint32_t HALF_BYTES = 128 * D * 2;    // 32 KiB: [2 col halves][128 rows][128 B]
constexpr uint32_t TILE_BYTES = TILE * D * 2;   // 16 KiB: [2 col halves][64 rows][128 B]
constexpr uint32_t ROWS128_K64 = 128 * TILE * 2; // 16 KiB: [128 rows][128 B] bf16, K = 64
constexpr uint32_t IDESC_N64 = tc::idesc_bf16(128, TILE, false, false);
constexpr uint32_t IDESC_N128_BMN = tc::idesc_bf16(128, D, false, true);
constexpr int kChunk = 0, kGroup = 1, kMasked = 2;

struct BwdArgs {
    int batch, n_q_heads, n_kv_heads, seg_len, topk, n_hist_chunks;
    int gs;                           // kGroup: tokens per group
    const int32_t *ucount;            // kMasked: valid routes per block
    const unsigned long long *umask;  // kMasked: token mask per route
    int n_sub, hc;  // dQ CTAs per KV group, query heads per dQ CTA (4, 2 or 1)
    int rph;        // query rows per head in a dQ CTA (32 when hc = 4, else 64)
    long long hist_stride, seg_stride;
    const int32_t *idx;
    const float *lse;
    const float *delta;
    float *dq;
    float *dk;
    float *dv;
    unsigned *status;
    float scale_log2;  // log2(e) / sqrt(D)
    float scale;       // 1 / sqrt(D)
};

// D[tmem] (+)= A[tmem] * B[smem] for one K=16 step of kind::f16 (A read from TMEM:
// lane = row, 8 columns of bf16 pairs per K step).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// ============================================================ dQ kernel
// A dQ CTA holds one M=128 tile of query rows: HC heads x RPH rows of one query block
// (4 x 32, two CTAs per block, when HC = 4; 2 x 64 when HC = 2; 64 rows repeated when
// HC = 1).  Q and dO are copied once into TMEM, so S_j = Q K_j^T and dP_j = dO V_j^T
// (M128 N64 K128, each from its own issuing warp) read only K_j / V_j from shared memory
// (an MMA with both operands there re-reads 4 KiB of A for every 2 KiB of B, and shared-
// memory operand bandwidth bounds the tile); they land in one of two TMEM buffers, dS_j
// goes in bf16 into one of two shared-memory buffers, dQ += dS_j K_j (M128 N128 K64, a
// third issuing warp).  Two warps per row (32 key columns each) form dS.
struct DqSmem {
    static constexpr int NSTAGE = 4;
    static constexpr uint32_t Q = 0;                                // [2 col halves][128 rows][128 B]
    static constexpr uint32_t DO = Q + HALF_BYTES;
    static constexpr uint32_t KV = DO + HALF_BYTES;                 // per stage: K tile, V tile
    static constexpr uint32_t DS = KV + NSTAGE * 2 * TILE_BYTES;    // 2 x [128 rows][128 B]
    static constexpr uint32_t BAR = DS + 2 * ROWS128_K64;
    static constexpr uint32_t ALLOC = BAR + 1024 + 1024;
};

struct DqBars {
    uint64_t q_full;
    uint64_t kv_full[DqSmem::NSTAGE];
    uint64_t kv_empty[DqSmem::NSTAGE];  // dP issuer (V read) + dQ issuer (K read)
    uint64_t qt_full;                   // Q and dO copied into TMEM (8 row warps)
    uint64_t sdp_full[2];               // S issuer + dP issuer
    uint64_t sdp_free[2];               // 8 row warps have read S, dP
    uint64_t ds_full[2];                // 8 row warps have stored dS
    uint64_t ds_free[2];                // dQ += dS K of that buffer done
    uint64_t drain[3];
    uint32_t tmem_base;
    int abort;
    int n_hist;
    int n_groups;  // kGroup: valid routed groups of the block
    int issued;
    int tiles[64];
};

static_assert(sizeof(DqBars) <= 1024, "dQ barrier block must fit its region");
static_assert(DqSmem::ALLOC <= 227 * 1024, "dQ shared memory must fit one block's 227 KiB");

// TMEM columns of a dQ CTA: dQ accumulator [0, 128); S/dP buffer b (b < 2) at
// 128 + 128 b (S in its first 64 columns, dP in the next 64); Q as bf16 pairs at
// [384, 448), dO at [448, 512).
template <int MODE>
__device__ __forceinline__ void dq_body(const int blk, uint8_t *smem_raw, const CUtensorMap &tm_qd,
                                        const CUtensorMap &tm_dod, const CUtensorMap &tm_kh, const CUtensorMap &tm_vh,
                                        const CUtensorMap &tm_ks, const CUtensorMap &tm_vs, const BwdArgs &a) {
    using L = DqSmem;
    constexpr int NST = L::NSTAGE;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DqBars *bars = reinterpret_cast<DqBars *>(smem + L::BAR);
    const uint32_t sbase = tc::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nqb = a.seg_len / TILE;
    const int n_slices = TILE / a.rph;
    const int n_units = a.batch * a.n_kv_heads * a.n_sub * n_slices;
    const int m = nqb - 1 - blk / n_units;  // longest blocks first
    int rem = blk % n_units;
    const int slice = rem % n_slices;
    rem /= n_slices;
    const int bg = rem / a.n_sub;
    const int b = bg / a.n_kv_heads, g = bg % a.n_kv_heads;
    const int h0 = g * (a.n_q_heads / a.n_kv_heads) + (rem % a.n_sub) * a.hc;  // first query head of the CTA
    const int row0 = m * TILE + slice * a.rph;                                // first query row of the slice

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->q_full, 1);
        for (int s = 0; s < NST; ++s) {
            tc::mbar_init(&bars->kv_full[s], 1);
            tc::mbar_init(&bars->kv_empty[s], 2);
        }
        tc::mbar_init(&bars->qt_full, 8);
        for (int bb = 0; bb < 2; ++bb) {
            tc::mbar_init(&bars->sdp_full[bb], 2);
            tc::mbar_init(&bars->sdp_free[bb], 8);
        }
        for (int bb = 0; bb < 2; ++bb) {
            tc::mbar_init(&bars->ds_full[bb], 8);
            tc::mbar_init(&bars->ds_free[bb], 1);
        }
        for (int d = 0; d < 3; ++d) tc::mbar_init(&bars->drain[d], 1);
        bars->abort = 0;
        bars->issued = 0;
        tc::fence_mbar_init();
    }
    const long long bgm = (long long)bg * nqb + m;
    if (warp == 2 && lane == 0) {
        const int32_t *sel = a.idx + bgm * a.topk;
        int n = 0;
        if constexpr (MODE == kChunk) {
            for (int i = 0; i < a.topk; ++i) {
                const int j = sel[i];
                if (j >= 0 && j < a.n_hist_chunks) bars->tiles[n++] = j;
            }
        } else if constexpr (MODE == kGroup) {
            const int n_all = a.n_hist_chunks * (TILE / a.gs);
            int ng = 0;
            for (int i = 0; i < a.topk; ++i) ng += (sel[i] >= 0 && sel[i] < n_all) ? 1 : 0;
            bars->n_groups = ng;
            n = (ng * a.gs + TILE - 1) / TILE;
        } else {
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
    const int n_hist = bars->n_hist;
    const int n_tiles = n_hist + m + 1;
    volatile int *abort = &bars->abort;

    if (warp == 0) {
        if (lane == 0) {
            // Q and dO: TMEM lane r holds head r / RPH (repeating head 0 when HC = 1), row row0 + r % RPH
            tc::mbar_arrive_expect_tx(&bars->q_full, 2 * HALF_BYTES);
            for (int hh = 0; hh < 128 / a.rph; ++hh) {
                const int qrow = (b * a.n_q_heads + h0 + (hh < a.hc ? hh : 0)) * a.seg_len + row0;
                const uint32_t off = hh * a.rph * 128;
                tc::tma_load_2d(smem + L::Q + off, &tm_qd, 0, qrow, &bars->q_full);
                tc::tma_load_2d(smem + L::Q + off + 128 * 128, &tm_qd, 64, qrow, &bars->q_full);
                tc::tma_load_2d(smem + L::DO + off, &tm_dod, 0, qrow, &bars->q_full);
                tc::tma_load_2d(smem + L::DO + off + 128 * 128, &tm_dod, 64, qrow, &bars->q_full);
            }
            int issued = 0;
            // kGroup: the routed groups in list order (invalid entries skipped), 64 / gs per tile
            const int32_t *gsel = a.idx + bgm * a.topk;
            const int n_all = MODE == kGroup ? a.n_hist_chunks * (TILE / a.gs) : 0;
            const int n_groups = MODE == kGroup ? bars->n_groups : 0;
            int gcur = 0, gtaken = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % NST, u = j / NST;
                if (j >= NST && !tc::mbar_wait(&bars->kv_empty[s], (u - 1) & 1, abort, a.status)) break;
                uint8_t *kdst = smem + L::KV + s * 2 * TILE_BYTES;
                uint8_t *vdst = kdst + TILE_BYTES;
                tc::mbar_arrive_expect_tx(&bars->kv_full[s], 2 * TILE_BYTES);
                if (j < n_hist && MODE == kGroup) {
                    const int gpt = TILE / a.gs;
                    int first = 0;
                    for (int v = 0; v < gpt; ++v) {
                        int grp = first;  // unfilled slots repeat the tile's first group
                        if (gtaken < n_groups) {
                            while (!(gsel[gcur] >= 0 && gsel[gcur] < n_all)) ++gcur;
                            grp = gsel[gcur++];
                            ++gtaken;
                        }
                        if (v == 0) first = grp;
                        const int row = (int)((long long)bg * a.hist_stride + (long long)grp * a.gs);
                        tc::tma_load_2d(kdst + v * a.gs * 128, &tm_kh, 0, row, &bars->kv_full[s]);
                        tc::tma_load_2d(kdst + 64 * 128 + v * a.gs * 128, &tm_kh, 64, row, &bars->kv_full[s]);
                        tc::tma_load_2d(vdst + v * a.gs * 128, &tm_vh, 0, row, &bars->kv_full[s]);
                        tc::tma_load_2d(vdst + 64 * 128 + v * a.gs * 128, &tm_vh, 64, row, &bars->kv_full[s]);
                    }
                } else {
                    const bool hist = j < n_hist;
                    const CUtensorMap *mk = hist ? &tm_kh : &tm_ks;
                    const CUtensorMap *mv = hist ? &tm_vh : &tm_vs;
                    int chunk = 0;
                    if (hist) chunk = MODE == kChunk ? bars->tiles[j] : a.idx[bgm * a.topk + j];
                    const int row = hist ? (int)((long long)bg * a.hist_stride + (long long)chunk * TILE)
                                         : (int)((long long)bg * a.seg_stride + (long long)(j - n_hist) * TILE);
                    tc::tma_load_2d(kdst, mk, 0, row, &bars->kv_full[s]);
                    tc::tma_load_2d(kdst + 64 * 128, mk, 64, row, &bars->kv_full[s]);
                    tc::tma_load_2d(vdst, mv, 0, row, &bars->kv_full[s]);
                    tc::tma_load_2d(vdst + 64 * 128, mv, 64, row, &bars->kv_full[s]);
                }
                ++issued;
            }
            bars->issued = issued;
        }
    } else if (warp == 1 || warp == 2) {
        // warp 1: S_j = Q K_j^T; warp 2: dP_j = dO V_j^T (and the V half of the stage's release)
        const bool is_s = warp == 1;
        const uint32_t a_tmem = tmem + (is_s ? 384u : 448u);  // Q or dO as bf16 pairs, 8 columns per K step
        const uint64_t kv_desc = tc::desc_sw128(sbase + L::KV + (is_s ? 0u : TILE_BYTES), 16, 1024);
        bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->qt_full, 0, abort, a.status));
        for (int j = 0; ok && j < n_tiles; ++j) {
            const int s = j % NST, sb = j & 1;
            ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->kv_full[s], (j / NST) & 1, abort, a.status) &&
                                             (j < 2 || tc::mbar_wait(&bars->sdp_free[sb], ((j >> 1) - 1) & 1, abort,
                                                                     a.status)));
            if (!ok) break;
            tc::fence_after_sync();
            const uint64_t kd = kv_desc + (uint64_t)((s * 2 * TILE_BYTES) >> 4);
            const uint32_t d = tmem + 128 + 128 * sb + (is_s ? 0u : 64u);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t boff = ((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4;
                if (tc::elect_one()) mma_f16_ts(d, a_tmem + 8 * kk, kd + boff, IDESC_N64, kk > 0 ? 1u : 0u);
                __syncwarp();
            }
            if (tc::elect_one()) {
                tc::mma_commit(&bars->sdp_full[sb]);
                if (!is_s) tc::mma_commit(&bars->kv_empty[s]);
            }
            __syncwarp();
        }
    } else if (warp == 3) {
        // dQ += dS_j K_j (K MN-major), then the K half of the stage's release
        const uint64_t kmn_desc = tc::desc_sw128(sbase + L::KV, 8192, 1024);
        const uint64_t ds_desc = tc::desc_sw128(sbase + L::DS, 16, 1024);
        for (int j = 0; j < n_tiles; ++j) {
            const int s = j % NST, bb = j & 1;
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->ds_full[bb], (j >> 1) & 1, abort, a.status))) break;
            tc::fence_after_sync();
            const uint64_t kd = kmn_desc + (uint64_t)((s * 2 * TILE_BYTES) >> 4);
            const uint64_t dd = ds_desc + (uint64_t)((bb * ROWS128_K64) >> 4);
#pragma unroll
            for (int kk = 0; kk < TILE / 16; ++kk) {
                if (tc::elect_one())
                    tc::mma_f16(tmem, dd + (kk * 32 >> 4), kd + (kk * 2048 >> 4), IDESC_N128_BMN,
                                (j > 0 || kk > 0) ? 1u : 0u);
                __syncwarp();
            }
            if (tc::elect_one()) {
                tc::mma_commit(&bars->ds_free[bb]);
                tc::mma_commit(&bars->kv_empty[s]);
            }
            __syncwarp();
        }
    } else if (warp >= 4) {
        const int quad = warp & 3;
        const int part = (warp - 4) >> 2;  // key columns 32 part .. 32 part + 31 of each tile
        const int r = quad * 32 + lane;
        const int hh = r / a.rph;
        const int i = slice * a.rph + r % a.rph;  // row within the query block
        const bool write = hh < a.hc;             // rows 64..127 repeat the head when HC = 1
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const long long row = ((long long)(b * a.n_q_heads + h0 + (write ? hh : 0))) * a.seg_len + m * TILE + i;
        const float lse2 = a.lse[row] * 1.4426950408889634f;
        const float dlt = a.delta[row];
        const uint32_t ds_row = sbase + L::DS + (r >> 3) * 1024 + (r & 7) * 128;
        bool ok = true;
        // Q (part 0) or dO (part 1) row r from its 128-byte-swizzled shared-memory tile into
        // TMEM lane r as 64 columns of bf16 pairs
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->q_full, 0, abort, a.status))) {
            ok = false;
        } else {
            const uint8_t *src = smem + (part ? L::DO : L::Q) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(src + hf * 16384 + ((c ^ (r & 7)) << 4));
                    v[4 * c] = w.x;
                    v[4 * c + 1] = w.y;
                    v[4 * c + 2] = w.z;
                    v[4 * c + 3] = w.w;
                }
                tc::tmem_st32(tmem + lane_addr + (part ? 448u : 384u) + 32 * hf, v);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->qt_full);
        }
        // kGroup: valid columns of the last history tile; kMasked: the row's token bit of
        // the next tile's mask (read one tile ahead)
        const int last_cols = MODE == kGroup ? bars->n_groups * a.gs - (n_hist - 1) * TILE : TILE;
        unsigned long long mask_next = 0ull;
        if (MODE == kMasked && n_hist > 0) mask_next = a.umask[bgm * a.topk];
        for (int j = 0; ok && j < n_tiles; ++j) {
            const int bb = j & 1, sb = j & 1;
            // columns >= ncols of this tile are masked for this row
            int ncols = TILE;
            if constexpr (MODE == kGroup) {
                if (j == n_hist - 1) ncols = last_cols;
            }
            if constexpr (MODE == kMasked) {
                if (j < n_hist) {
                    if (((mask_next >> i) & 1ull) == 0ull) ncols = 0;
                    if (j + 1 < n_hist) mask_next = a.umask[bgm * a.topk + j + 1];
                }
            }
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->sdp_full[sb], (j >> 1) & 1, abort, a.status))) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const bool diag = (j == n_tiles - 1);
            uint32_t pk[16];
            {
                uint32_t sv[32], dpv[32];
                const uint32_t s_addr = tmem + lane_addr + 128 + 128 * sb + 32 * part;
                tc::tmem_ld32(s_addr, sv);
                tc::tmem_ld32(s_addr + 64, dpv);
                tc::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const int c0 = 32 * part + c;
                    float p0 = tc::ex2(__uint_as_float(sv[c]) * a.scale_log2 - lse2);
                    float p1 = tc::ex2(__uint_as_float(sv[c + 1]) * a.scale_log2 - lse2);
                    if ((diag && c0 > i) || c0 >= ncols) p0 = 0.f;
                    if ((diag && c0 + 1 > i) || c0 + 1 >= ncols) p1 = 0.f;
                    pk[c / 2] = tc::pack_bf16(p0 * (__uint_as_float(dpv[c]) - dlt),
                                              p1 * (__uint_as_float(dpv[c + 1]) - dlt));
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->sdp_free[sb]);
            // dS buffer bb is free once dQ += dS K of tile j - 2 has read it
            if (j >= 2 &&
                !__all_sync(0xffffffffu, tc::mbar_wait(&bars->ds_free[bb], ((j >> 1) - 1) & 1, abort, a.status))) {
                ok = false;
                break;
            }
            // this warp's 64 bytes of the row: 16-byte chunks 4 part .. 4 part + 3 (128-byte swizzle)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
                tc::st_shared_v4(ds_row + bb * ROWS128_K64 + (((4 * part + cc) ^ (r & 7)) << 4), pk[4 * cc],
                                 pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->ds_full[bb]);
        }
        const int jl = n_tiles - 1;
        if (ok && __all_sync(0xffffffffu, tc::mbar_wait(&bars->ds_free[jl & 1], (jl >> 1) & 1, abort, a.status))) {
            tc::fence_after_sync();
            float *out = a.dq + row * D;
#pragma unroll 1
            for (int c0 = 64 * part; c0 < 64 * part + 64; c0 += 32) {
                uint32_t o[32];
                tc::tmem_ld32(tmem + lane_addr + c0, o);
                tc::tmem_wait_ld();
                if (!write) continue;
#pragma unroll
                for (int c = 0; c < 32; c += 4)
                    *reinterpret_cast<float4 *>(out + c0 + c) =
                        make_float4(__uint_as_float(o[c]) * a.scale, __uint_as_float(o[c + 1]) * a.scale,
                                    __uint_as_float(o[c + 2]) * a.scale, __uint_as_float(o[c + 3]) * a.scale);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (*abort) {
        int never = 0;
        if (warp == 0 && lane == 0) {
            const int issued = bars->issued;
            for (int j = issued - NST < 0 ? 0 : issued - NST; j < issued; ++j)
                tc::mbar_wait(&bars->kv_full[j % NST], (j / NST) & 1, &never, a.status, 1ll << 28);
            tc::mbar_wait(&bars->q_full, 0, &never, a.status, 1ll << 28);
        }
        if (warp >= 1 && warp <= 3) {
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

// ============================================================ dK/dV kernel
// A dK/dV CTA holds 128 segment keys (TMEM lanes) and walks the (head, later query
// tile) steps of its KV group.  Per step t: S^T = K Q_t^T (warp 1) and dP^T = V dO_t^T
// (warp 2) into one of two TMEM buffers; two warps per key row (warps 4-7: query columns
// 0..31, warps 8-11: 32..63) write P^T and dS^T as bf16 pairs back into the same buffer,
// each over the first half of the S^T / dP^T columns it has read, and warp 3 issues
// dV += P^T dO_t and dK += dS^T Q_t with A read from TMEM.  So the next step's S^T /
// dP^T run while the softmax works on this one.
struct DkvSmem {
    static constexpr int NSTAGE = 4;
    static constexpr uint32_t K = 0;                          // 128 keys, K-major
    static constexpr uint32_t V = K + HALF_BYTES;
    static constexpr uint32_t RING = V + HALF_BYTES;          // per stage: Q tile, dO tile
    static constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr uint32_t ROWT = RING + NSTAGE * STAGE_BYTES;  // per stage: lse[64], delta[64]
    static constexpr uint32_t BAR = ROWT + NSTAGE * 512;
    static constexpr uint32_t ALLOC = BAR + 1024 + 1024;
};

struct DkvBars {
    uint64_t kv_full;
    uint64_t ring_full[DkvSmem::NSTAGE];
    uint64_t ring_empty[DkvSmem::NSTAGE];  // dV / dK of the step done (the last readers of Q_t, dO_t)
    uint64_t sdp_full[2];                  // S^T issuer + dP^T issuer
    uint64_t pds_full[2];                  // 8 row warps have stored P^T, dS^T
    uint64_t buf_free[2];                  // dV / dK of that buffer done
    uint64_t drain[3];
    uint32_t tmem_base;
    int abort;
    int issued;
};

// 32 lanes x 16 consecutive 32-bit columns from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

static_assert(sizeof(DkvBars) <= 1024, "dK/dV barrier block must fit its region");
static_assert(DkvSmem::ALLOC <= 227 * 1024, "dK/dV shared memory must fit one block's 227 KiB");

// TMEM columns of a dK/dV CTA: dV [0, 128), dK [128, 256), step buffer b at 256 + 128 b:
// S^T in its first 64 columns, dP^T in the next 64; P^T of query columns 0..31 / 32..63
// lands in columns 0..15 / 32..47 of the buffer, dS^T in 64..79 / 96..111.
__device__ __forceinline__ void dkdv_body(const int blk, uint8_t *smem_raw, const CUtensorMap &tm_q,
                                          const CUtensorMap &tm_do, const CUtensorMap &tm_ks,
                                          const CUtensorMap &tm_vs, const BwdArgs &a) {
    using L = DkvSmem;
    constexpr int NST = L::NSTAGE;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DkvBars *bars = reinterpret_cast<DkvBars *>(smem + L::BAR);
    const uint32_t sbase = tc::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int nqb = a.seg_len / TILE;
    const int n_bg = a.batch * a.n_kv_heads;
    const int n = blk / n_bg;  // 128-key tile, earliest (most work) first
    const int bg = blk % n_bg;
    const int b = bg / a.n_kv_heads, g = bg % a.n_kv_heads;
    const int key0 = 128 * n;
    const int m0 = key0 / TILE;
    const int n_steps = G * (nqb - m0);  // (head, query tile) pairs, head-major

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->kv_full, 1);
        for (int s = 0; s < NST; ++s) {
            tc::mbar_init(&bars->ring_full[s], 1);
            tc::mbar_init(&bars->ring_empty[s], 1);
        }
        for (int bb = 0; bb < 2; ++bb) {
            tc::mbar_init(&bars->sdp_full[bb], 2);
            tc::mbar_init(&bars->pds_full[bb], 8);
            tc::mbar_init(&bars->buf_free[bb], 1);
        }
        for (int d = 0; d < 3; ++d) tc::mbar_init(&bars->drain[d], 1);
        bars->abort = 0;
        bars->issued = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc<512>(&bars->tmem_base);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort = &bars->abort;

    if (warp == 0) {
        if (lane == 0) {
            // the CTA's 128 keys and values (rows past the segment read as zero or are never written back)
            const int krow = (int)((long long)bg * a.seg_stride + key0);
            tc::mbar_arrive_expect_tx(&bars->kv_full, 2 * HALF_BYTES);
            for (int part = 0; part < 2; ++part) {
                const uint32_t off = part * (64 * 128);
                tc::tma_load_2d(smem + L::K + off, &tm_ks, 0, krow + 64 * part, &bars->kv_full);
                tc::tma_load_2d(smem + L::K + off + 128 * 128, &tm_ks, 64, krow + 64 * part, &bars->kv_full);
                tc::tma_load_2d(smem + L::V + off, &tm_vs, 0, krow + 64 * part, &bars->kv_full);
                tc::tma_load_2d(smem + L::V + off + 128 * 128, &tm_vs, 64, krow + 64 * part, &bars->kv_full);
            }
            int issued = 0;
            for (int t = 0; t < n_steps; ++t) {
                const int s = t % NST, u = t / NST;
                if (t >= NST && !tc::mbar_wait(&bars->ring_empty[s], (u - 1) & 1, abort, a.status)) break;
                const int hh = t / (nqb - m0), mq = m0 + t % (nqb - m0);
                const long long qrow = ((long long)(b * a.n_q_heads + g * G + hh)) * a.seg_len + (long long)mq * TILE;
                uint8_t *qdst = smem + L::RING + s * L::STAGE_BYTES;
                uint8_t *gdst = qdst + TILE_BYTES;
                tc::mbar_arrive_expect_tx(&bars->ring_full[s], 2 * TILE_BYTES + 512);
                tc::tma_load_2d(qdst, &tm_q, 0, (int)qrow, &bars->ring_full[s]);
                tc::tma_load_2d(qdst + 64 * 128, &tm_q, 64, (int)qrow, &bars->ring_full[s]);
                tc::tma_load_2d(gdst, &tm_do, 0, (int)qrow, &bars->ring_full[s]);
                tc::tma_load_2d(gdst + 64 * 128, &tm_do, 64, (int)qrow, &bars->ring_full[s]);
                tc::bulk_load(smem + L::ROWT + s * 512, a.lse + qrow, 256, &bars->ring_full[s]);
                tc::bulk_load(smem + L::ROWT + s * 512 + 256, a.delta + qrow, 256, &bars->ring_full[s]);
                ++issued;
            }
            bars->issued = issued;
        }
    } else if (warp == 1 || warp == 2) {
        // warp 1: S^T = K Q_t^T; warp 2: dP^T = V dO_t^T
        const bool is_s = warp == 1;
        const uint64_t a_desc = tc::desc_sw128(sbase + (is_s ? L::K : L::V), 16, 1024);
        const uint64_t ring_desc = tc::desc_sw128(sbase + L::RING + (is_s ? 0u : TILE_BYTES), 16, 1024);
        bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->kv_full, 0, abort, a.status));
        for (int t = 0; ok && t < n_steps; ++t) {
            const int s = t % NST, bb = t & 1;
            ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->ring_full[s], (t / NST) & 1, abort, a.status) &&
                                             (t < 2 || tc::mbar_wait(&bars->buf_free[bb], ((t >> 1) - 1) & 1, abort,
                                                                     a.status)));
            if (!ok) break;
            tc::fence_after_sync();
            const uint64_t bd = ring_desc + (uint64_t)((s * L::STAGE_BYTES) >> 4);
            const uint32_t d = tmem + 256 + 128 * bb + (is_s ? 0u : 64u);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t aoff = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
                const uint32_t boff = ((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4;
                if (tc::elect_one()) tc::mma_f16(d, a_desc + aoff, bd + boff, IDESC_N64, kk > 0 ? 1u : 0u);
                __syncwarp();
            }
            if (tc::elect_one()) tc::mma_commit(&bars->sdp_full[bb]);
            __syncwarp();
        }
    } else if (warp == 3) {
        // dV += P^T dO_t and dK += dS^T Q_t (A from TMEM, B MN-major in the ring stage)
        const uint64_t ring_mn_desc = tc::desc_sw128(sbase + L::RING, 8192, 1024);
        for (int t = 0; t < n_steps; ++t) {
            const int s = t % NST, bb = t & 1;
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->pds_full[bb], (t >> 1) & 1, abort, a.status))) break;
            tc::fence_after_sync();
            const uint64_t qd = ring_mn_desc + (uint64_t)((s * L::STAGE_BYTES) >> 4);
            const uint64_t gd = qd + (uint64_t)(TILE_BYTES >> 4);
            // P^T (dS^T) of query columns 0..31 at columns 0..15 (64..79), of 32..63 at 32..47 (96..111)
            const uint32_t pa = tmem + 256 + 128 * bb;
#pragma unroll
            for (int kk = 0; kk < TILE / 16; ++kk) {
                const uint32_t ka = (kk & 1) * 8 + (kk >> 1) * 32;
                if (tc::elect_one())
                    mma_f16_ts(tmem, pa + ka, gd + (kk * 2048 >> 4), IDESC_N128_BMN, (t > 0 || kk > 0) ? 1u : 0u);
                __syncwarp();
            }
#pragma unroll
            for (int kk = 0; kk < TILE / 16; ++kk) {
                const uint32_t ka = (kk & 1) * 8 + (kk >> 1) * 32;
                if (tc::elect_one())
                    mma_f16_ts(tmem + 128, pa + 64 + ka, qd + (kk * 2048 >> 4), IDESC_N128_BMN,
                               (t > 0 || kk > 0) ? 1u : 0u);
                __syncwarp();
            }
            if (tc::elect_one()) {
                tc::mma_commit(&bars->buf_free[bb]);
                tc::mma_commit(&bars->ring_empty[s]);
            }
            __syncwarp();
        }
    } else if (warp >= 4) {
        const int quad = warp & 3;
        const int part = (warp - 4) >> 2;  // query columns 32 part .. 32 part + 31 of each step
        const int r = quad * 32 + lane;  // key row = TMEM lane
        const int key = key0 + r;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        bool ok = true;
        for (int t = 0; t < n_steps; ++t) {
            const int s = t % NST, bb = t & 1;
            const int mq = m0 + t % (nqb - m0);
            // the stage's lse / delta rows (TMA-written) and this step's S^T, dP^T in TMEM
            if (!__all_sync(0xffffffffu,
                            tc::mbar_wait(&bars->ring_full[s], (t / NST) & 1, abort, a.status) &&
                                tc::mbar_wait(&bars->sdp_full[bb], (t >> 1) & 1, abort, a.status))) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const float *lse2 = reinterpret_cast<const float *>(smem + L::ROWT + s * 512);
            const float *dlt = lse2 + 64;
            const int q0 = mq * TILE;  // first query position of the tile
            const uint32_t buf = tmem + lane_addr + 256 + 128 * bb + 32 * part;
            uint32_t ppk[16], dpk[16];
            {
                uint32_t sv[32], dpv[32];
                tc::tmem_ld32(buf, sv);
                tc::tmem_ld32(buf + 64, dpv);
                tc::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const int c0 = 32 * part + c;
                    float p0 = tc::ex2(__uint_as_float(sv[c]) * a.scale_log2 - lse2[c0] * 1.4426950408889634f);
                    float p1 = tc::ex2(__uint_as_float(sv[c + 1]) * a.scale_log2 - lse2[c0 + 1] * 1.4426950408889634f);
                    if (key > q0 + c0) p0 = 0.f;      // causal: the key comes after the query
                    if (key > q0 + c0 + 1) p1 = 0.f;
                    ppk[c / 2] = tc::pack_bf16(p0, p1);
                    dpk[c / 2] = tc::pack_bf16(p0 * (__uint_as_float(dpv[c]) - dlt[c0]),
                                               p1 * (__uint_as_float(dpv[c + 1]) - dlt[c0 + 1]));
                }
            }
            // P^T / dS^T over the first 16 of the 32 S^T / dP^T columns this warp has read
            tmem_st16(buf, ppk);
            tmem_st16(buf + 64, dpk);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->pds_full[bb]);
        }
        const int tl = n_steps - 1;
        const bool done = ok && n_steps > 0 &&
                          __all_sync(0xffffffffu, tc::mbar_wait(&bars->buf_free[tl & 1], (tl >> 1) & 1, abort,
                                                                a.status));
        if (done) {
            tc::fence_after_sync();
            const bool valid = key < a.seg_len;
            const long long orow = (long long)bg * a.seg_len + key;
            {
                const int which = part;  // part 0 writes dV, part 1 dK
                float *out = (which ? a.dk : a.dv) + orow * D;
                const float sc = which ? a.scale : 1.f;
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tc::tmem_ld32(tmem + lane_addr + 128 * which + c0, o);
                    tc::tmem_wait_ld();
                    if (valid) {
#pragma unroll
                        for (int c = 0; c < 32; c += 4)
                            *reinterpret_cast<float4 *>(out + c0 + c) =
                                make_float4(__uint_as_float(o[c]) * sc, __uint_as_float(o[c + 1]) * sc,
                                            __uint_as_float(o[c + 2]) * sc, __uint_as_float(o[c + 3]) * sc);
                    }
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (*abort) {
        int never = 0;
        if (warp == 0 && lane == 0) {
            const int issued = bars->issued;
            for (int t = issued - NST < 0 ? 0 : issued - NST; t < issued; ++t)
                tc::mbar_wait(&bars->ring_full[t % NST], (t / NST) & 1, &never, a.status, 1ll << 28);
            tc::mbar_wait(&bars->kv_full, 0, &never, a.status, 1ll << 28);
        }
        if (warp >= 1 && warp <= 3) {
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

// One launch for both gradient passes: the first n_kv_ctas blocks run the
// key-major dK/dV body (most work first), the rest the query-major dQ body.
// The causal dK/dV blocks are very uneven (the first key tile is seen by
// every later query tile), so the dQ blocks fill the SMs around them.
// tm_q / tm_do have 64-row boxes (dK/dV query tiles), tm_qd / tm_dod boxes of
// RPH rows (a dQ CTA's rows of one head).
template <int MODE>
__global__ void __launch_bounds__(384, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_qd, const __grid_constant__ CUtensorMap tm_dod,
                  const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_vh,
                  const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                  const BwdArgs a, const int n_kv_ctas) {
    extern __shared__ uint8_t smem_raw[];
    if ((int)blockIdx.x < n_kv_ctas)
        dkdv_body((int)blockIdx.x, smem_raw, tm_q, tm_do, tm_ks, tm_vs, a);
    else
        dq_body<MODE>((int)blockIdx.x - n_kv_ctas, smem_raw, tm_qd, tm_dod, tm_kh, tm_vh, tm_ks, tm_vs, a);
}

template <int MODE>
hga_status_t launch_bwd(const hga_params_t &p, const CUtensorMap &mq, const CUtensorMap &mdo, const CUtensorMap &mqd,
                        const CUtensorMap &mdod, const CUtensorMap &mkh, const CUtensorMap &mvh,
                        const CUtensorMap &mks, const CUtensorMap &mvs, const BwdArgs &a, cudaStream_t stream) {
    auto kern = bwd_tc_kernel<MODE>;
    const size_t smem = DqSmem::ALLOC > DkvSmem::ALLOC ? DqSmem::ALLOC : DkvSmem::ALLOC;
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), (int)smem);
    if (e != cudaSuccess) return record_cuda(e);
    const int n_bg = p.batch * p.n_kv_heads;
    const int n_kv_ctas = ((p.seg_len + 127) / 128) * n_bg;
    const unsigned grid = (unsigned)(n_kv_ctas + (p.seg_len / p.q_block) * n_bg * a.n_sub * (TILE / a.rph));
    kern<<<grid, 384, smem, stream>>>(mq, mdo, mqd, mdod, mkh, mvh, mks, mvs, a, n_kv_ctas);
    return record_cuda(cudaGetLastError());
}

}  // namespace

bool attn_bwd_tc_supported(const hga_params_t &p) {
    if (!attn_fwd_tc_shape(p)) return false;
    const long long n_bg = (long long)p.batch * p.n_kv_heads;
    if (n_bg * (p.hist_head_stride > p.seg_head_stride ? p.hist_head_stride : p.seg_head_stride) >= (1ll << 31))
        return false;
    if ((long long)p.batch * p.n_q_heads * p.seg_len >= (1ll << 31)) return false;
    return tma_encoder_available();
}

namespace {

template <int MODE>
hga_status_t launch_bwd_mode(const hga_params_t &p, const void *q, const void *kh, const void *vh, const void *ks,
                             const void *vs, const FwdRoutes &rt, const float *lse, const float *delta,
                             const void *dout, float *dq, float *dk, float *dv, unsigned *status,
                             cudaStream_t stream) {
    CUtensorMap mq, mdo, mqd, mdod, mkh, mvh, mks, mvs;
    const long long n_bg = (long long)p.batch * p.n_kv_heads;
    const unsigned long long q_rows = (unsigned long long)p.batch * p.n_q_heads * p.seg_len;
    const long long hist_rows =
        p.hist_head_stride > 0 ? (n_bg - 1) * p.hist_head_stride + (long long)p.n_hist_chunks * p.chunk
                               : (long long)p.n_hist_chunks * p.chunk;
    const unsigned long long seg_rows = (unsigned long long)((n_bg - 1) * p.seg_head_stride + p.seg_len);
    if (!make_map(&mq, q, q_rows) || !make_map(&mdo, dout, q_rows) || !make_map(&mks, ks, seg_rows) ||
        !make_map(&mvs, vs, seg_rows))
        return HGA_ERR_INVALID_ARG;
    if (hist_rows > 0) {
        const unsigned box = MODE == kGroup ? (unsigned)rt.gs : 64u;  // group routes: one box per group
        if (!tma_rows_map(&mkh, kh, (unsigned long long)hist_rows, box) ||
            !tma_rows_map(&mvh, vh, (unsigned long long)hist_rows, box))
            return HGA_ERR_INVALID_ARG;
    } else {
        mkh = mks;
        mvh = mvs;
    }
    BwdArgs a;
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
    a.idx = rt.list;
    a.lse = lse;
    a.delta = delta;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.status = status;
    a.scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)D));
    a.scale = (float)(1.0 / __builtin_sqrt((double)D));
    const int G = p.n_q_heads / p.n_kv_heads;
    a.hc = G % 4 == 0 ? 4 : (G % 2 == 0 ? 2 : 1);
    a.n_sub = G / a.hc;
    a.rph = a.hc == 4 ? 32 : 64;
    if (a.rph == 64) {
        mqd = mq;
        mdod = mdo;
    } else if (!tma_rows_map(&mqd, q, q_rows, (unsigned)a.rph) || !tma_rows_map(&mdod, dout, q_rows, (unsigned)a.rph)) {
        return HGA_ERR_INVALID_ARG;
    }
    return launch_bwd<MODE>(p, mq, mdo, mqd, mdod, mkh, mvh, mks, mvs, a, stream);
}

}  // namespace

hga_status_t launch_attn_bwd_tc(const hga_params_t &p, const void *q, const void *kh, const void *vh,
                                const void *ks, const void *vs, const int32_t *idx, const float *lse,
                                const float *delta, const void *dout, float *dq, float *dk, float *dv,
                                unsigned *status, cudaStream_t stream) {
    FwdRoutes rt{idx, p.topk, 0, nullptr, nullptr};
    return launch_bwd_mode<kChunk>(p, q, kh, vh, ks, vs, rt, lse, delta, dout, dq, dk, dv, status, stream);
}

hga_status_t launch_attn_bwd_tc_routes(const hga_params_t &p, const void *q, const void *kh, const void *vh,
                                       const void *ks, const void *vs, const FwdRoutes &rt, const float *lse,
                                       const float *delta, const void *dout, float *dq, float *dk, float *dv,
                                       unsigned *status, cudaStream_t stream) {
    if (rt.gs > 0)
        return launch_bwd_mode<kGroup>(p, q, kh, vh, ks, vs, rt, lse, delta, dout, dq, dk, dv, status, stream);
    if (rt.umask)
        return launch_bwd_mode<kMasked>(p, q, kh, vh, ks, vs, rt, lse, delta, dout, dq, dk, dv, status, stream);
    return launch_bwd_mode<kChunk>(p, q, kh, vh, ks, vs, rt, lse, delta, dout, dq, dk, dv, status, stream);
}

}  // namespace hga
