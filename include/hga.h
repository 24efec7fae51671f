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
 *                         stage; the attention entry points read chunk routes);
 *   strictly causal     = hga_route_causal: token i routes by its block's
 *                         queries up to i;
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

/* Strictly causal routing (technical summary, limits section: sharing one
 * route among the tokens of a block is a weak causal side channel; a strictly
 * causal variant is proposed as future work).  Every token i of block m
 * routes by qbar_i = fp32 mean over the G heads of group g and the queries
 * m*q_block .. i of its block, with the score, selection, ties and sink rule
 * of hga_route; the last token of a block gets the block's route.
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
 * k_hist + (b*Hkv + g)*hist_head_stride*D.  bf16 inputs use tcgen05 tensor
 * cores with fp32 accumulation (P is rounded to bf16 for the P.V product);
 * fp32 inputs use fp32 CUDA-core arithmetic.
 *   out: device [B][Hq][S][D] dtype; lse: device fp32 [B][Hq][S].  Rows of
 *   blocks outside [qblock_begin, qblock_end) are not written.
 * Route indices outside [-1, Nc) are skipped and flagged HGA_DEV_BAD_INDEX. */
hga_status_t hga_attn_fwd(const hga_params_t *p, const void *q, const void *k_hist, const void *v_hist,
                          const void *k_seg, const void *v_seg, const int32_t *idx, void *out,
                          float *lse, cudaStream_t stream);

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
 * dv_seg [B][Hkv][S][D]: device fp32 for every input dtype (gradients are
 * sums over many rows; fp32 keeps them within the tolerance a bf16 store
 * would exceed once |grad| >= 8), overwritten.  workspace: device, >=
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
 * RAM, only the routed exact K/V are brought to the GPU).  For the query
 * blocks [qblock_begin, qblock_end) of idx, gathers the distinct (b, g, chunk)
 * tiles they route to, copies only those K and V tiles from page-locked host
 * memory (host_k / host_v: [B][Hkv][hist_head_stride][D], dtype) into the
 * device staging buffers stage_k / stage_v ([stage_slots][chunk][D]) and
 * writes idx_remapped (same shape as idx) with each index replaced by its
 * staging slot.  hga_attn_fwd over the same blocks with k_hist = stage_k,
 * v_hist = stage_v, hist_head_stride = 0 and idx = idx_remapped gives output
 * bit-identical to attending the history in device memory.
 *   slot_map: device int32 scratch of at least B*Hkv*Nc + stage_slots + 1
 *     entries (tile flags / slot numbers, then the slot -> tile list).
 *   n_fetched (device int32, may be NULL): number of tiles fetched.
 * The attention call over the staging buffer passes n_hist_chunks =
 * stage_slots (route indices are now slot numbers).
 * All work is enqueued on copy_stream; when done != NULL it is recorded on
 * copy_stream after the last kernel.  Returns HGA_ERR_INVALID_ARG when the
 * blocks can need more tiles than stage_slots. */
hga_status_t hga_fetch_tiered(const hga_params_t *p, const void *host_k, const void *host_v,
                              const int32_t *idx, int qblock_begin, int qblock_end, void *stage_k,
                              void *stage_v, int stage_slots, int32_t *slot_map, int32_t *idx_remapped,
                              int32_t *n_fetched, cudaStream_t copy_stream, cudaEvent_t done);

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
