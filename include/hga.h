/*
 * hga.h -- C ABI of the B200 (sm_100a) Hierarchical Global Attention layer.
 *
 * What the layer computes is described in "Long-Context Fine-Tuning with
 * Limited VRAM" (Fedosov, Sazhin, Grinenko, Woernle; the gist.science
 * technical summary, sections 2.1 "Hierarchical Global Attention" and 2.2
 * "Segment-wise backward and tiered storage", and the author abstract):
 * the context is cut into fixed 64-token chunks; a compact summary of every
 * closed chunk stays resident on the GPU; each query block scores those
 * summaries, keeps the best history chunks and attends, with exact softmax,
 * to the exact keys/values of those chunks together with a local window;
 * routing carries no gradient; training runs segment by segment and only the
 * active segment is differentiable; detached history may live in host memory.
 *
 * Readings fixed by this library where the pages leave a step open:
 *   chunk summary       = mean of the chunk's keys, per KV head (fp32);
 *   query-block summary = mean of the block's queries over the G query heads
 *                         of the KV group (q head h reads KV head h / G);
 *   score               = fp32 dot(query-block summary, chunk summary)/sqrt(D);
 *   selection           = the min(k, Nc) best chunks by (score descending,
 *                         chunk index ascending), listed in ascending chunk
 *                         order and padded with -1;
 *   local window        = every active-segment token at or before the query;
 *   attention sink      = with sink_chunks = s, history chunks 0 .. s-1 are
 *                         always chosen, inside the k slots (hga_route);
 *   group stage         = hga_route_groups: the best groups of 8, 16 or 32
 *                         tokens inside the chosen chunks (a second routing
 *                         stage), attended by hga_attn_fwd/bwd_groups;
 *   strictly causal     = hga_route_causal: token i routes by its block's
 *                         queries up to i, attended by hga_attn_fwd/bwd_causal;
 *   decode              = hga_attn_decode: one new token per sequence, routed
 *                         as a one-token block.
 * With chunk routes, query i of the active segment attends exactly
 * min(k, Nc) * chunk + i + 1 tokens.
 *
 * Conventions for every entry point:
 *   - The caller owns all memory.  Device pointers are CUDA device (or
 *     managed) addresses; "host" pointers are page-locked host memory.  The
 *     library allocates and frees nothing.
 *   - Every call is asynchronous on the given stream: it validates its
 *     arguments on the host, enqueues kernels and returns.  Arguments are
 *     checked before anything is launched; a bad argument returns
 *     HGA_ERR_INVALID_ARG (or HGA_ERR_UNSUPPORTED for a valid shape this
 *     build has no kernel for) and enqueues nothing.  HGA_ERR_CUDA reports
 *     a launch failure (the CUDA error string is kept for hga_last_error()).
 *   - Errors found by kernels (an out-of-range route index, a pipeline
 *     wait that ran out of time) are OR-ed into a device status word that
 *     hga_get_device_status() reads back; kernels never trap.
 *   - Tensors are row-major with the head dimension D contiguous.  Token
 *     strides between consecutive (batch, head) slices are given in tokens
 *     so that history and segment K/V may be two views of one buffer.
 */
#ifndef HGA_H
#define HGA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HGA_OK = 0,
    HGA_ERR_INVALID_ARG = -1,
    HGA_ERR_UNSUPPORTED = -2,
    HGA_ERR_CUDA = -3,
    HGA_ERR_DEVICE_CHECK = -4,
    HGA_ERR_TIMEOUT = -5
} hga_status_t;

typedef enum { HGA_BF16 = 0, HGA_FP32 = 1 } hga_dtype_t;

/* Device status bits (hga_get_device_status). */
#define HGA_DEV_BAD_INDEX 1u   /* a route index outside [-1, Nc) was skipped */
#define HGA_DEV_TIMEOUT   2u   /* a pipeline wait gave up; results are invalid */
#define HGA_DEV_STAGE_FULL 4u  /* a tiered fetch found too few free staging slots; the
                                  tiles it could not place were not attended */

/* Shape of one HGA attention layer call.
 *   batch B, n_q_heads Hq, n_kv_heads Hkv (Hq % Hkv == 0, G = Hq / Hkv),
 *   head_dim D (64 or 128), chunk c (64), q_block (64), topk k (1..64),
 *   seg_len S (multiple of q_block and chunk), n_hist_chunks Nc (T = Nc*c
 *   history tokens routable), dtype of q/k/v/out/grads.
 *   hist_head_stride: tokens between (b, g) slices of k_hist / v_hist; 0 is
 *     allowed and means one shared slice (used for a staging buffer whose
 *     route indices were remapped to slots by hga_fetch_tiered).
 *   seg_head_stride: tokens between (b, g) slices of k_seg / v_seg (>= S).
 *   qblock_begin / qblock_end: the range of query blocks hga_attn_fwd
 *     processes; 0 / 0 means every block (0 .. S/q_block).
 *   sink_chunks: attention-sink window (0 .. topk; 0 = none): hga_route
 *     always routes history chunks 0 .. min(sink_chunks, k_eff) - 1 and fills
 *     the remaining slots by score ("Long-Context Fine-Tuning with Limited
 *     VRAM", technical summary section 2.1: fixed sink and local windows next
 *     to the routed chunks; the width is not given there, 1 chunk = 64 tokens
 *     is the reading used by the benchmarks). */
typedef struct {
    int batch;
    int n_q_heads;
    int n_kv_heads;
    int head_dim;
    int chunk;
    int q_block;
    int topk;
    int seg_len;
    int n_hist_chunks;
    hga_dtype_t dtype;
    long long hist_head_stride;
    long long seg_head_stride;
    int qblock_begin;
    int qblock_end;
    int sink_chunks;
} hga_params_t;

/* Chunk summaries (technical summary section 2.1: one compact vector per
 * closed chunk, resident on the GPU; here the mean of the chunk's keys).
 * For every (b, g) and chunk j in [first_chunk, first_chunk + n_chunks):
 *   summ[((b*n_kv_heads + g)*summ_cap_chunks + j)*head_dim + d]
 *     = (1/chunk) * sum_{r<chunk} k[((b*n_kv_heads + g)*head_stride + j*chunk + r)*head_dim + d]
 * accumulated in fp32 in a fixed order, so an incremental append after each
 * detached segment is bit-identical to a full rebuild.
 *   k: device, dtype elements, [B][Hkv][head_stride][D] with token 0 of each
 *      slice being history token 0.   summ: device fp32, capacity
 *      summ_cap_chunks per (b, g) slice; first_chunk + n_chunks <= cap.
 * n_chunks == 0 is a no-op. */
hga_status_t hga_build_summaries(const void *k, long long head_stride, int batch, int n_kv_heads,
                                 int head_dim, int chunk, int first_chunk, int n_chunks,
                                 hga_dtype_t dtype, float *summ, int summ_cap_chunks,
                                 cudaStream_t stream);

/* Routing (technical summary section 2.1: the current query block scores the
 * chunk summaries and keeps the most relevant history chunks; no learned
 * weights, no gradient).  For every (b, g, query block m):
 *   qbar   = fp32 mean over the G heads of group g and the q_block queries of m;
 *   s_j    = fp32 dot(qbar, summ[b][g][j]) / sqrt(D), j < Nc;
 *   idx[((b*Hkv + g)*nqb + m)*k + a], a < k: the min(k, Nc) chunks with the
 *            largest s_j (ties: lower j), ascending, then -1 padding; with
 *            sink_chunks = s the chunks j < min(s, min(k, Nc)) are taken
 *            first and the rest of the slots by score.
 *   q: device [B][Hq][S][D] dtype.  summ: device fp32 with summ_cap_chunks per
 *   (b, g) slice (>= Nc).  idx: device int32 [B][Hkv][S/q_block][k]. */
hga_status_t hga_route(const hga_params_t *p, const void *q, const float *summ, int summ_cap_chunks,
                       int32_t *idx, cudaStream_t stream);

/* Group-level second routing stage (technical summary section 2.1, group
 * selection: the chosen chunks are split into smaller groups, e.g. 8 tokens,
 * and the router keeps the best groups inside the chosen chunks).  For every
 * (b, g, query block m) with its chunk route idx (from hga_route):
 *   candidates = the groups of `group` tokens of every valid chunk in
 *                idx[b][g][m][*] (chunk j holds groups j*c/group .. +c/group-1);
 *   s_u        = fp32 dot(qbar, gsumm[b][g][u]) / sqrt(D), qbar as in hga_route;
 *   gidx[((b*Hkv + g)*nqb + m)*topg + a], a < topg: the topg candidates with the
 *                largest s_u (ties: lower u), ascending, then -1 padding.
 *   gsumm: device fp32 group summaries (the mean of each group's keys, e.g.
 *     hga_build_summaries with chunk = group), gsumm_cap_groups rows per
 *     (b, g) slice (>= Nc * c / group).
 *   group: 8, 16 or 32 tokens.  topg: 1 .. topk * c / group.
 *   gidx: device int32 [B][Hkv][S/q_block][topg]. */
hga_status_t hga_route_groups(const hga_params_t *p, const void *q, const float *gsumm, int gsumm_cap_groups,
                              const int32_t *idx, int group, int topg, int32_t *gidx, cudaStream_t stream);

/* hga_route_groups with the group summaries kept in page-locked host memory
 * and a device cache of them (technical summary section 2.2: group summaries
 * are cached on the GPU and misses are fetched from the host).  For every
 * block's routed chunks, the chunk's chunk/group group summaries (one cache
 * tile) are copied from host_gsumm ([B][Hkv][gsumm_cap_groups][D] fp32) into
 * stage_gsumm ([stage_slots][chunk/group][D] fp32) unless the cache already
 * holds them -- the staging cache, its scratch, eviction rule and device
 * status bits are those of hga_fetch_tiered, one fetch wave per call, all on
 * stream -- and the routes are then computed from the cache: gidx equals
 * hga_route_groups' over the same values, bit for bit.
 *   p->hist_head_stride must be gsumm_cap_groups * group (the history tokens the
 *   group summaries cover; hga_tier_scratch_size / hga_tier_reset with this p
 *   size and empty the cache); idx_remapped (same shape as idx) receives the
 *   routed chunks' cache slots; n_fetched (may be NULL): tiles copied.
 *   stage_slots >= min(2 * (S/q_block) * B * Hkv * min(k, Nc), B * Hkv * Nc). */
hga_status_t hga_route_groups_tiered(const hga_params_t *p, const void *q, const float *host_gsumm,
                                     int gsumm_cap_groups, const int32_t *idx, int group, int topg, int32_t *gidx,
                                     float *stage_gsumm, int stage_slots, int32_t *scratch, int32_t *idx_remapped,
                                     int32_t *n_fetched, cudaStream_t stream);

/* Strictly causal routing (technical summary, limits section: sharing one
 * route among the tokens of a block is a weak causal side channel; a strictly
 * causal variant is proposed as future work).  Every token i of block m
 * routes by qbar_i = fp32 mean over the G heads of group g and the queries
 * m*q_block .. i of its block, with the score, selection, ties and sink rule
 * of hga_route.  The last token of a block routes by the same block mean as
 * hga_route, summed in another fp32 order, so its route equals the block's up
 * to rounding (at near-ties of the k-th score the two may differ).
 *   idx: device int32 [B][Hkv][S][k], one route per token.  Other arguments
 *   as hga_route.  q_block = 1 gives the plain per-token route.
 * HGA_ERR_UNSUPPORTED when one token's score row set does not fit the CTA's
 * shared memory (n_hist_chunks above about 5,000 for D = 128). */
hga_status_t hga_route_causal(const hga_params_t *p, const void *q, const float *summ, int summ_cap_chunks,
                              int32_t *idx, cudaStream_t stream);

/* Exact-token attention forward (technical summary section 2.1; author
 * abstract: a bounded set of exact historical tokens per query block).  For
 * query (b, h, i) of a processed block m = i / q_block, g = h / G:
 *   U = {history tokens of chunks idx[b][g][m][*] >= 0} u {segment tokens t <= i}
 *   z_t = q . k_t / sqrt(D),  out = sum_t softmax(z)_t v_t,  lse = ln sum_t exp(z_t)
 * History chunk j of head (b, g) is rows [j*c, j*c + c) of the slice at
 * k_hist + (b*Hkv + g)*hist_head_stride*D.  Kernels by shape, never by
 * environment: bf16 with head_dim 128 runs on tcgen05 tensor cores with fp32
 * accumulation (P is rounded to bf16 for the P.V product; any GQA group size,
 * packed 4, 2 or 1 query heads per CTA) and returns HGA_ERR_UNSUPPORTED when
 * that kernel cannot run (no TMA tensor-map encoder in the driver, or a row
 * coordinate beyond 32 bits); fp32 inputs run on fp32 CUDA cores (TF32 tensor
 * cores would not meet fp32 accuracy), as does bf16 with head_dim 64.
 *   out: device [B][Hq][S][D] dtype; lse: device fp32 [B][Hq][S].  Rows of
 *   blocks outside [qblock_begin, qblock_end) are not written.
 * Route indices outside [-1, Nc) are skipped and flagged HGA_DEV_BAD_INDEX. */
hga_status_t hga_attn_fwd(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                          const void *k_seg, const void *v_seg, const int32_t *idx, void *out,
                          float *lse, cudaStream_t stream);

/* Exact-token attention over group routes (technical summary section 2.1,
 * group selection: only the exact K/V of the selected groups inside the chosen
 * chunks are attended).  As hga_attn_fwd with the history part of U taken from
 * gidx (hga_route_groups): for query (b, h, i) of block m,
 *   U = {tokens u*group .. u*group + group - 1 of every u in gidx[b][g][m][*] >= 0}
 *       u {segment tokens t <= i}
 * so query i attends (valid groups) * group + i + 1 tokens.
 *   gidx: device int32 [B][Hkv][S/q_block][topg], group ids < Nc * chunk / group
 *   (others than -1 are skipped and flagged HGA_DEV_BAD_INDEX); group: 8, 16 or
 *   32; topg: 1 .. min(topk * chunk / group, 512).  bf16 with head_dim 128 only
 *   (tcgen05; anything else is HGA_ERR_UNSUPPORTED).  Groups are gathered as
 *   group-row TMA boxes, 64 / group of them per 64-key tile. */
hga_status_t hga_attn_fwd_groups(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                                 const void *k_seg, const void *v_seg, const int32_t *gidx, int group, int topg,
                                 void *out, float *lse, cudaStream_t stream);

/* Backward of hga_attn_fwd_groups (routes frozen): dq over the routed groups'
 * and the segment's keys, dk_seg / dv_seg over the segment's keys; outputs and
 * workspace (>= hga_attn_bwd_workspace_size(p) bytes) as hga_attn_bwd. */
hga_status_t hga_attn_bwd_groups(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                                 const void *k_seg, const void *v_seg, const int32_t *gidx, int group, int topg,
                                 const void *out, const float *lse, const void *dout, void *dq, void *dk_seg,
                                 void *dv_seg, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Exact-token attention over strictly causal routes (technical summary,
 * limits section: the proposed strictly causal variant of block routing).
 * idx_tok: device int32 [B][Hkv][S][topk], one route per token (from
 * hga_route_causal).  Query (b, h, i) attends
 *   U_i = {tokens of the chunks idx_tok[b][g][i][*] >= 0} u {segment tokens t <= i},
 * i.e. min(k, Nc) * chunk + i + 1 tokens, equal to hga_attn_fwd with one-token
 * query blocks.  The tcgen05 kernel keeps 64-query blocks: a first kernel
 * builds, per block, the ascending union of its tokens' routed chunks and a
 * 64-bit mask of the tokens routed to each (in workspace); the attention then
 * masks, row by row, the union chunks a token did not route to.
 *   workspace: device, >= hga_attn_causal_workspace_size(p, 0) bytes, 16-byte
 *   aligned (the unions: B*Hkv*(S/64) * (4 + min(64 k, Nc) * 12) bytes).
 *   Nc <= 16384; bf16 with head_dim 128 only (else HGA_ERR_UNSUPPORTED). */
size_t hga_attn_causal_workspace_size(const hga_params_t *p, int backward);
hga_status_t hga_attn_fwd_causal(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                                 const void *k_seg, const void *v_seg, const int32_t *idx_tok, void *out, float *lse,
                                 void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Backward of hga_attn_fwd_causal (routes frozen): outputs as hga_attn_bwd;
 * workspace >= hga_attn_causal_workspace_size(p, 1) bytes (the unions, then
 * the fp32 row terms). */
hga_status_t hga_attn_bwd_causal(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                                 const void *k_seg, const void *v_seg, const int32_t *idx_tok, const void *out,
                                 const float *lse, const void *dout, void *dq, void *dk_seg, void *dv_seg,
                                 void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* hga_route then hga_attn_fwd in one call, overlapped (technical summary
 * section 2.1: the block routes, then attends its routed chunks and its local
 * window).  idx gets the routes exactly as from hga_route.  The attention is
 * launched as a programmatic dependent of the route kernel: it starts while
 * the route grid is still running, takes the causal segment tiles first (they
 * need no route) and waits for the route grid before the routed history
 * tiles.  out / lse agree with hga_route + hga_attn_fwd within rounding (the
 * tiles are summed in another order), not bit for bit.  Arguments and errors
 * as the two calls; fp32 and bf16 head_dim 64 run the two calls in order. */
hga_status_t hga_route_attn_fwd(const hga_params_t *p, const void *q, const float *summ, int summ_cap_chunks,
                                int32_t *idx, const void *k_hist, const void *v_hist, const void *k_seg,
                                const void *v_seg, void *out, float *lse, cudaStream_t stream);

/* Bytes of device workspace hga_attn_bwd needs (fp32 row terms
 * delta = rowsum(dO * O), [B][Hq][S]).  Returns 0 for an invalid p. */
size_t hga_attn_bwd_workspace_size(const hga_params_t *p);

/* Backward of the exact-token attention with routes frozen (technical
 * summary sections 2.1 and 2.2: routing without gradient, gather and
 * attention differentiable, history detached at the segment boundary).
 * With P the softmax row of query (b, h, i) and delta_i = sum_d dO*O:
 *   dS_t = P_t (dO . v_t - delta_i)
 *   dq[b][h][i]      = sum_{t in U} dS_t k_t / sqrt(D)       (history and segment keys)
 *   dk_seg[b][g][t] = sum_{h in g, i >= t} dS_t q_i / sqrt(D) (segment keys only)
 *   dv_seg[b][g][t] = sum_{h in g, i >= t} P_t dO_i           (segment keys only)
 * History K/V get no gradient.  out / lse are the forward's outputs for
 * every block (qblock_begin/end must be 0/0).  dq [B][Hq][S][D], dk_seg and
 * dv_seg [B][Hkv][S][D]: device fp32 for every input dtype, overwritten.  This
 * is a deliberate departure from "gradients in the input dtype": gradients
 * are sums over many rows, and one bf16 rounding of a value >= 8 is already
 * off by up to 0.03, above the 2e-2 bf16 parity tolerance; the price is twice
 * the bytes of a bf16 store.  Kernels by shape as for hga_attn_fwd.  workspace: device, >=
 * hga_attn_bwd_workspace_size(p) bytes, 16-byte aligned. */
hga_status_t hga_attn_bwd(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                          const void *k_seg, const void *v_seg, const int32_t *idx, const void *out,
                          const float *lse, const void *dout, void *dq, void *dk_seg, void *dv_seg,
                          void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* hga_attn_bwd without a caller-supplied workspace.  The source pages have
 * no counterpart to this call; it exists for callers that cannot allocate
 * device memory themselves -- a plugin or serving runtime that owns every
 * byte of device memory through its own pool and only hands the library
 * tensors and a stream, or a hot path that must not call cudaMalloc.  It
 * computes exactly what hga_attn_bwd computes, with the same arguments minus
 * workspace / workspace_bytes, and allocates nothing: the fp32 row terms live
 * in a fixed 4 MiB array inside the library, which every GPU that loads the
 * library keeps until the process exits.
 *   Limit: batch * n_q_heads * seg_len <= 1,048,576 query rows; larger
 *   shapes return HGA_ERR_INVALID_ARG (message in hga_last_error()).
 *   The first call on a device looks up that device's copy of the array
 *   (with the device current); make that first call before any stream
 *   capture.  All calls on a device share the one array: calls that overlap
 *   on the GPU (different streams without ordering between them) race and
 *   must be serialised by the caller.  The array keeps the last call's
 *   contents; nothing in it needs clearing, as every call rewrites the row
 *   terms before reading them. */
hga_status_t hga_attn_bwd_noalloc(const hga_params_t *p, const void *q, const void *k_hist,
                                  const void *v_hist, const void *k_seg, const void *v_seg,
                                  const int32_t *idx, const void *out, const float *lse, const void *dout,
                                  void *dq, void *dk_seg, void *dv_seg, cudaStream_t stream);

/* Single-query decode (generation: one new token per sequence).  The token's
 * route comes from hga_route over a one-token segment (seg_len = q_block = 1:
 * its block summary is the mean of its G query heads); it then attends, with
 * exact softmax, the tokens of its routed history chunks and the n_local
 * tokens of its local window (the not-yet-detached tokens, itself last):
 * technical summary section 2.1, routed exact chunks next to a local window.
 *   p: seg_len = q_block = 1, n_q_heads / n_kv_heads <= 8; seg_head_stride =
 *     tokens between (b, g) slices of k_local / v_local (>= n_local);
 *     hist_head_stride / n_hist_chunks / topk as for hga_attn_fwd.
 *   q: device [B][Hq][1][D] dtype.  k_local, v_local: device [B][Hkv][*][D].
 *   idx: device int32 [B][Hkv][1][k] (from hga_route).
 *   out: device [B][Hq][1][D] dtype.  lse: device fp32 [B][Hq][1] (natural log).
 *   workspace: device, at least hga_attn_decode_workspace_size(p, n_local)
 *     bytes, 16-byte aligned (per-split partial results; nothing in it needs
 *     clearing).  The size depends on the current device's SM count (the
 *     split count fills one wave): query it with that device current.
 * Two kernels on stream (split-K partial attention, then the merge); nothing
 * is allocated.  Out-of-range route indices are skipped and flagged.  bf16
 * reads K/V through TMA tensor maps: HGA_ERR_UNSUPPORTED when they cannot be
 * encoded (no driver entry point). */
size_t hga_attn_decode_workspace_size(const hga_params_t *p, int n_local);
hga_status_t hga_attn_decode(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                             const void *k_local, const void *v_local, int n_local, const int32_t *idx,
                             void *out, float *lse, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Tiered history (technical summary section 2.2: detached K/V live in host
 * RAM, only the routed exact K/V are brought to the GPU; device memory grows
 * with the routing budget, not with the context).
 *
 * The device side is a staging cache of stage_slots chunk tiles (stage_k /
 * stage_v: [stage_slots][chunk][D], dtype) shared by every (b, g), and its
 * bookkeeping in a caller-owned int32 scratch of hga_tier_scratch_size bytes
 * (tile -> slot map, slot -> tile map, the last wave reading each slot, the
 * fetch list, a wave counter and an allocation cursor).  The cache persists
 * from call to call: a tile fetched once is reused by every later wave that
 * routes to it until it is evicted.  Tiles are (b, g, chunk j) of the host
 * history host_k / host_v ([B][Hkv][hist_head_stride][D], page-locked), so the
 * cache stays valid while the history only grows; reset it whenever the host
 * history is replaced (or to start a segment with an empty cache).
 *
 * hga_tier_scratch_size: bytes of scratch for p (hist_head_stride tokens of
 * host history per (b, g)) and stage_slots; 0 for invalid arguments.
 * hga_tier_reset: marks every slot empty (one kernel on stream). */
size_t hga_tier_scratch_size(const hga_params_t *p, int stage_slots);
hga_status_t hga_tier_reset(const hga_params_t *p, int stage_slots, int32_t *scratch, cudaStream_t stream);

/* One fetch wave: for the query blocks [qblock_begin, qblock_end) of idx, the
 * distinct (b, g, chunk) tiles they route to that the cache does not hold are
 * copied (K and V) from page-locked host memory into free slots -- slots whose
 * last reading wave is two or more waves back, taken round-robin, evicting
 * their old tile -- and idx_remapped (same shape as idx, rows of those blocks
 * only) gets each index replaced by its slot.  hga_attn_fwd over the same
 * blocks with k_hist = stage_k, v_hist = stage_v, hist_head_stride = 0,
 * n_hist_chunks = stage_slots and idx = idx_remapped gives output
 * bit-identical to attending the history in device memory.
 *   Ordering contract: the attention of the wave two fetches back must have
 *   completed before this fetch starts (the previous wave's may still run);
 *   hga_attn_fwd_tiered keeps it.
 *   stage_slots >= min(2 * (blocks) * B * Hkv * min(k, Nc), B * Hkv * Nc),
 *     else HGA_ERR_INVALID_ARG (the device flags HGA_DEV_STAGE_FULL if it
 *     still runs out of free slots).
 *   n_fetched (device int32, may be NULL): tiles copied by this wave.
 *   host_k / host_v must be page-locked (mapped) host memory: anything else
 *   returns HGA_ERR_INVALID_ARG before any launch.
 * All work is enqueued on copy_stream; done (may be NULL) is recorded there
 * after the last kernel. */
hga_status_t hga_fetch_tiered(const hga_params_t *p, const void *host_k, const void *host_v,
                              const int32_t *idx, int qblock_begin, int qblock_end, void *stage_k,
                              void *stage_v, int stage_slots, int32_t *scratch, int32_t *idx_remapped,
                              int32_t *n_fetched, cudaStream_t copy_stream, cudaEvent_t done);

/* Detach into the host tier (technical summary section 2.2: the history K/V
 * that leave the active segment live in host memory): copies tokens [0, S) of
 * every (b, g) slice of k_seg / v_seg (device, seg_head_stride tokens apart)
 * to tokens [dst_token, dst_token + S) of host_k / host_v (page-locked,
 * [B][Hkv][hist_head_stride][D]), one 2-D copy each, on stream.  Later fetches
 * of those chunks must be ordered after it (issue them on the same stream, or
 * wait for it).  HGA_ERR_INVALID_ARG for pageable host memory or a range
 * past hist_head_stride. */
hga_status_t hga_tier_offload(const hga_params_t *p, const void *k_seg, const void *v_seg, void *host_k,
                              void *host_v, long long dst_token, cudaStream_t stream);

/* Cross-stream schedule of hga_attn_fwd_tiered, owned by the caller and kept
 * from call to call over one staging cache.  Wave h of the schedule is one
 * fetch (on the copy stream) and the attention that reads it (on the compute
 * stream); the fetch of wave h may evict the slots that wave h - lag read, so
 * it starts only after that attention (consumed[h % lag]) and may overlap the
 * attention of the lag - 1 waves before it.  The cache then holds the tiles of
 * lag waves: stage_slots >= min(lag * wave_blocks * B * Hkv * min(k, Nc),
 * B * Hkv * Nc).
 *   Create the events (cudaEventDisableTiming is enough; inputs, offloaded,
 *   routed and idx_free only for hga_segment_fwd_tiered), set lag (2 ..
 *   HGA_TIER_MAX_LAG), wave = 0 and segment = 0; the library records the
 *   events and advances the counters.  Use one compute stream and one copy
 *   stream for all calls of a schedule, and no other fetch into its cache
 *   (hga_fetch_tiered, hga_route_groups_tiered) between them.  A schedule's
 *   first call (wave 0) is never chained. */
#define HGA_TIER_MAX_LAG 4
typedef struct {
    cudaEvent_t start;                       /* unchained calls: the copy stream after the compute stream */
    cudaEvent_t fetched;                     /* attention of wave h after the fetch of wave h */
    cudaEvent_t consumed[HGA_TIER_MAX_LAG];  /* fetch of wave h after the attention of wave h - lag */
    cudaEvent_t inputs;                      /* hga_segment_fwd_tiered: the offload after the segment's inputs */
    cudaEvent_t offloaded[2];                /* hga_segment_fwd_tiered: fetches after the previous offload */
    cudaEvent_t routed;                      /* hga_segment_fwd_tiered: fetches after the segment's route */
    cudaEvent_t idx_free[2];                 /* hga_segment_fwd_tiered: a route after the last reader of its idx */
    int lag;
    long long wave;                          /* waves issued through the schedule since its cache was emptied */
    long long segment;                       /* segments through hga_segment_fwd_tiered since then */
} hga_tier_sched_t;

/* hga_attn_fwd over host-resident history, overlapping fetch and attention:
 * the blocks [qblock_begin, qblock_end) (0/0: all) are taken in waves of
 * wave_blocks query blocks; the fetch of each wave runs on copy_stream while
 * earlier waves' attention runs on stream, ordered by sched (above).  Output
 * (out, lse) is bit-identical to hga_attn_fwd with the history resident.  On
 * return, stream is ordered after every fetch of the call (with Nc = 0, after
 * all work then on copy_stream, and copy_stream after the attention, which
 * reads idx).
 *   flags: HGA_TIER_RESET empties the cache first (and sets sched->wave = 0).
 *   Without HGA_TIER_CHAIN, and always with HGA_TIER_RESET, the copy stream
 *   first waits for everything already enqueued on stream (the route that
 *   wrote idx, earlier attention over the cache).  With HGA_TIER_CHAIN alone
 *   the call continues the schedule of the previous call (the next segment of
 *   an evaluation): the copy stream does not wait for stream -- the caller
 *   orders it after whatever wrote idx and after the host rows the fetches
 *   read -- so the first fetches overlap the previous call's last attention.
 *   Chained calls need a non-decreasing Nc, and idx_remapped must not be a
 *   buffer that an attention still in flight reads: the fetch of wave h
 *   writes its blocks' rows once wave h - lag is done, so chained calls of n
 *   waves each rotate ceil(lag / n) idx_remapped buffers.
 *   prev_k_seg / prev_v_seg (may be NULL): the K/V of the segment that
 *   detached last, tokens [T - S, T) (T = Nc * chunk), laid out like k_seg /
 *   v_seg and still in device memory until the call's fetches are done; its
 *   chunks are then copied from there instead of across the host link (the
 *   host history holds the same bytes, so the output does not change).
 *   n_fetched (device int32, may be NULL): one count per wave, of the tiles
 *   copied from the host.  Other arguments as hga_fetch_tiered and
 *   hga_attn_fwd.  HGA_ERR_INVALID_ARG for a null event, a lag outside 2 ..
 *   HGA_TIER_MAX_LAG, unknown flags, or prev_k_seg with Nc < S / chunk. */
#define HGA_TIER_RESET 1
#define HGA_TIER_CHAIN 2
hga_status_t hga_attn_fwd_tiered(const hga_params_t *p, const void *q, const void *host_k, const void *host_v,
                                 const void *k_seg, const void *v_seg, const void *prev_k_seg,
                                 const void *prev_v_seg, const int32_t *idx, void *out, float *lse,
                                 void *stage_k, void *stage_v, int stage_slots, int32_t *scratch,
                                 int32_t *idx_remapped, int wave_blocks, int flags, int32_t *n_fetched,
                                 cudaStream_t stream, cudaStream_t copy_stream, hga_tier_sched_t *sched);

/* One segment of an evaluation whose detached history lives in page-locked
 * host memory (technical summary section 2.2, tiered memory; section 2.1 for
 * the route and the exact-token attention; the segment detaches at its end),
 * on four streams, so that a segment's route and fetches run under the
 * attention of the segments before it:
 *   route_stream  : hga_route of the segment into idx, then the detach-time
 *                   append of the segment's S / chunk summaries to chunks
 *                   [Nc, Nc + S / chunk) of summ.
 *   copy_stream   : the fetch waves of hga_attn_fwd_tiered, chained from the
 *                   previous segment, after the segment's route and the
 *                   previous segment's offload -- or, given prev_k_seg /
 *                   prev_v_seg (the previous segment's K/V, which its chunks
 *                   are then copied from), the offload of the one before.
 *   offload_stream: k_seg / v_seg copied to tokens [T, T + S) of host_k /
 *                   host_v (T = Nc * chunk) once the inputs are ready.
 *   stream        : the attention waves, writing out and lse.
 * q, k_seg and v_seg must be ready in route_stream's order (the caller copies
 * them in there, or orders route_stream after their producer).  idx: the
 * segment's route table; the route of segment s + 2 waits until the fetches
 * of segment s have read theirs, so rotate two buffers (a route may then run
 * a segment ahead).  flags: HGA_TIER_RESET for the evaluation's first segment
 * (the side streams first wait for stream; the cache is emptied;
 * sched->wave and sched->segment restart); 0 continues the evaluation.  On
 * return stream is ordered after the segment's fetches; the caller orders
 * stream after route_stream and offload_stream before it reads summ or the
 * host history itself.  idx_remapped as in hga_attn_fwd_tiered (rotate
 * ceil(lag / waves per segment) buffers).  HGA_ERR_INVALID_ARG when
 * summ_cap_chunks < Nc + S / chunk, T + S > hist_head_stride, the host
 * history is not page-locked, or an event of sched is null; other arguments
 * and checks as hga_route, hga_attn_fwd_tiered and hga_tier_offload. */
hga_status_t hga_segment_fwd_tiered(const hga_params_t *p, const void *q, const void *k_seg, const void *v_seg,
                                    const void *prev_k_seg, const void *prev_v_seg, float *summ,
                                    int summ_cap_chunks, int32_t *idx, void *host_k, void *host_v,
                                    void *out, float *lse, void *stage_k, void *stage_v, int stage_slots,
                                    int32_t *scratch, int32_t *idx_remapped, int wave_blocks, int flags,
                                    int32_t *n_fetched, cudaStream_t stream, cudaStream_t copy_stream,
                                    cudaStream_t route_stream, cudaStream_t offload_stream, hga_tier_sched_t *sched);

/* One segment of an evaluation with the history resident in device memory
 * (technical summary section 2.1: route, then exact-token attention; the
 * segment detaches at its end), on two streams, so that a segment's route runs
 * under the attention of the segment before it:
 *   route_stream: hga_route of the segment into idx, then the detach-time
 *                 append of the segment's S / chunk summaries to chunks
 *                 [Nc, Nc + S / chunk) of summ (read from k_seg).
 *   stream      : hga_attn_fwd of the segment, once its route is done.
 * The inputs (q, k_seg, v_seg and the history) must be ready in route_stream's
 * order (the caller copies them in there, or orders route_stream after their
 * producer).  idx: the segment's route table; the route of segment s + 2 waits
 * until the attention of segment s has read its buffer, so rotate two buffers.
 * flags: HGA_TIER_RESET for the evaluation's first segment (route_stream first
 * waits for stream; sched->segment restarts); 0 continues the evaluation.
 * sched: a schedule object as for hga_segment_fwd_tiered, of which this call
 * uses start, routed, idx_free and segment.  On return stream is ordered after
 * the segment's route; the caller orders stream after route_stream before it
 * reads summ itself.  Other arguments and checks as hga_route and hga_attn_fwd;
 * HGA_ERR_INVALID_ARG when summ_cap_chunks < Nc + S / chunk or an event is
 * null. */
hga_status_t hga_segment_fwd(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                             const void *k_seg, const void *v_seg, float *summ, int summ_cap_chunks, int32_t *idx,
                             void *out, float *lse, int flags, cudaStream_t stream, cudaStream_t route_stream,
                             hga_tier_sched_t *sched);

/* Self-test of the bounded waits (the source pages have no counterpart): every
 * pipeline wait in the tensor-core kernels gives up after a cycle limit instead
 * of hanging, sets HGA_DEV_TIMEOUT and lets the kernel end.  This launches one
 * CTA whose only thread waits on an mbarrier nothing ever arrives at, with a
 * limit of wait_cycles (1e3 .. 2^32 SM cycles); afterwards
 * hga_get_device_status() reports HGA_ERR_TIMEOUT and the context stays usable.
 * Returns HGA_ERR_INVALID_ARG for a limit outside that range. */
hga_status_t hga_selftest_wait_timeout(long long wait_cycles, cudaStream_t stream);

/* Reads (after synchronising stream) and clears the device status word of the
 * current device; *bits gets the HGA_DEV_* bits seen since the last call.
 * Returns HGA_ERR_DEVICE_CHECK or HGA_ERR_TIMEOUT when bits are set. */
hga_status_t hga_get_device_status(cudaStream_t stream, unsigned int *bits);

/* Human-readable name of a status code. */
const char *hga_status_string(hga_status_t s);

/* Text of the last CUDA error seen by this thread's calls (or ""). */
const char *hga_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* HGA_H */
