/*
 * CPU oracle for the Hierarchical Global Attention (HGA) layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is compiled into a separate shared
 * library that only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg load.  The CUDA library never links, includes or calls it,
 * and it shares no code, header or constant with the CUDA sources.
 *
 * Plain, single-threaded, fp64 C.  Every function follows the method's steps
 * in the order the source pages give them; nothing is blocked, fused or
 * reordered.  Sources (titles and sections of the pages this follows):
 *   [TS2.1]  "Long-Context Fine-Tuning with Limited VRAM", gist.science
 *            technical summary, section 2.1 "Hierarchical Global Attention":
 *            fixed-size chunks (64 tokens), a compact summary per closed
 *            chunk kept resident, the current query block scores the
 *            summaries and keeps the most relevant history chunks next to a
 *            fixed local window; exact K/V of the selected tokens are
 *            attended; summaries are used for routing only; routing carries
 *            no gradient while gather and attention are differentiable.
 *   [TS2.2]  same page, section 2.2 "Segment-wise backward and tiered
 *            storage": loss and backward per segment, history K/V detached
 *            at the segment boundary.
 *   [ABS]    the author abstract (franklineh.com and fugumt.com pages):
 *            only the active segment is differentiable; HGA loads a bounded
 *            set of exact historical tokens for each query block.
 * Where the pages leave a step open the plainest reading is taken:
 *   summary of chunk j = mean of its c keys (per KV head);
 *   query-block summary = mean of the block's q_block queries over the G
 *     query heads of the KV group (q head h uses KV head h / G);
 *   score = dot(query-block summary, chunk summary) / sqrt(D);
 *   selection = the min(k, Nc) best chunks by (score descending, chunk index
 *     ascending), emitted in ascending chunk order, padded with -1;
 *   local window = every active-segment token at or before the query;
 *   sink window (sink_chunks = s): the first s history chunks are always
 *     chosen, inside the k slots;
 *   group stage (group = gs > 0) [TS2.1, group selection]: each chosen chunk
 *     is split into c / gs groups of gs consecutive tokens; group summary =
 *     mean of its gs keys; group score = dot(query-block summary, group
 *     summary) / sqrt(D); the block keeps the topg best groups of its chosen
 *     chunks by (score descending, group index ascending), emitted in
 *     ascending group order and padded with -1, and attends their tokens.
 *
 * Layouts (row-major, D contiguous):
 *   q, dout, out, dq   [B][Hq][S][D]
 *   k_hist, v_hist     [B][Hkv][T][D]   (T = Nc * c)
 *   k_seg, v_seg, dk_seg, dv_seg  [B][Hkv][S][D]
 *   summ               [B][Hkv][Nc][D]
 *   idx                [B][Hkv][S/q_block][k]
 *   lse                [B][Hq][S]   natural log of the softmax denominator
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int batch, n_q_heads, n_kv_heads, head_dim, chunk, q_block, topk, seg_len, n_hist_chunks;
    int sink_chunks; /* attention-sink window: history chunks 0..sink_chunks-1 are always routed */
    int group;       /* group stage: tokens per group (divides chunk); 0 = attend whole chunks */
    int topg;        /* group stage: groups kept per query block */
} oracle_shape_t;

static long long ix4(long long a, long long A1, long long b, long long B1, long long c, long long C1, long long d)
{
    return ((a * A1 + b) * B1 + c) * C1 + d;
}

/* [TS2.1] summary of chunk j: the mean of its c key rows, per KV head.
 * k has tokens [0, n_chunks*c) of each head, head_stride tokens apart. */
int oracle_summaries(const double *k, int batch, int n_kv_heads, long long head_stride, int head_dim,
                     int chunk, int n_chunks, double *summ)
{
    if (!k || !summ || chunk <= 0 || head_dim <= 0) return -1;
    for (int b = 0; b < batch; ++b)
        for (int g = 0; g < n_kv_heads; ++g) {
            const double *kh = k + ((long long)b * n_kv_heads + g) * head_stride * head_dim;
            for (int j = 0; j < n_chunks; ++j)
                for (int d = 0; d < head_dim; ++d) {
                    double s = 0.0;
                    for (int r = 0; r < chunk; ++r) s += kh[((long long)j * chunk + r) * head_dim + d];
                    summ[ix4(b, n_kv_heads, g, n_chunks, j, head_dim, d)] = s / chunk;
                }
        }
    return 0;
}

/* [TS2.1] the query block's summary: mean over the G heads of the group and
 * the q_block queries of block m. */
static void query_block_summary(const oracle_shape_t *p, const double *q, int b, int g, int m, double *qbar)
{
    const int G = p->n_q_heads / p->n_kv_heads, D = p->head_dim, S = p->seg_len;
    for (int d = 0; d < D; ++d) qbar[d] = 0.0;
    for (int hh = 0; hh < G; ++hh) {
        int h = g * G + hh;
        for (int i = m * p->q_block; i < (m + 1) * p->q_block; ++i)
            for (int d = 0; d < D; ++d) qbar[d] += q[ix4(b, p->n_q_heads, h, S, i, D, d)];
    }
    for (int d = 0; d < D; ++d) qbar[d] /= (double)(G * p->q_block);
}

/* Is chunk a ranked before chunk b?  Higher score first; equal scores go to
 * the lower chunk index. */
static int ranks_before(double sa, int a, double sb, int b)
{
    if (sa > sb) return 1;
    if (sa < sb) return 0;
    return a < b;
}

/* The selection step of a route, given the Nc scores s of one routing query:
 * the sink chunks first, then the best remaining chunk until k_eff chunks
 * (and one more, for the gap) are ranked.  out gets the chosen ids in
 * ascending order, -1 padded to K; *gap (if given) the relative distance
 * between the last chunk taken by score and the next one (+inf if none). */
static void select_chunks(const double *s, int Nc, int K, int sink_chunks, int *order, char *taken, int *out,
                          double *gap)
{
    const int keff = K < Nc ? K : Nc;
    memset(taken, 0, Nc > 0 ? Nc : 1);
    const int n_sink = sink_chunks < keff ? (sink_chunks > 0 ? sink_chunks : 0) : keff;
    for (int r = 0; r < n_sink; ++r) {
        order[r] = r;
        taken[r] = 1;
    }
    int n_rank = keff + (Nc > keff ? 1 : 0);
    for (int r = n_sink; r < n_rank; ++r) {
        int best = -1;
        for (int j = 0; j < Nc; ++j)
            if (!taken[j] && (best < 0 || ranks_before(s[j], j, s[best], best))) best = j;
        order[r] = best;
        if (r < keff) taken[best] = 1;
    }
    int w = 0;
    for (int j = 0; j < Nc; ++j)
        if (taken[j]) out[w++] = j;
    for (; w < K; ++w) out[w] = -1;
    if (gap) {
        double g_rel = INFINITY;
        if (Nc > keff && keff > n_sink) {
            double a = s[order[keff - 1]], c = s[order[keff]];
            double den = fabs(a) > fabs(c) ? fabs(a) : fabs(c);
            if (den < 1e-30) den = 1e-30;
            g_rel = (a - c) / den;
        }
        *gap = g_rel;
    }
}

/* [TS2.1] routing: score every closed history chunk against the query-block
 * summary and keep the k best.  idx gets the chosen chunk ids in ascending
 * order, padded with -1 when k > Nc.  gap (optional) gets, per query block,
 * the relative distance between the k-th and (k+1)-th best scores, or
 * +inf when every chunk is taken.  scores (optional) gets all Nc scores.
 * [TS2.1, the fixed sink window] with sink_chunks = s > 0 the first
 * min(s, k_eff) chunks are taken before any score is looked at and the
 * remaining slots go to the best of the other chunks; gap then compares the
 * last chunk taken by score with the next one (+inf if none is). */
int oracle_route(const oracle_shape_t *p, const double *q, const double *summ,
                 int *idx, double *gap, double *scores)
{
    const int B = p->batch, Hkv = p->n_kv_heads, D = p->head_dim, Nc = p->n_hist_chunks, K = p->topk;
    if (p->n_q_heads % Hkv || p->seg_len % p->q_block || K <= 0) return -1;
    const int nqb = p->seg_len / p->q_block;
    double *qbar = (double *)malloc(sizeof(double) * D);
    double *s = (double *)malloc(sizeof(double) * (Nc > 0 ? Nc : 1));
    int *order = (int *)malloc(sizeof(int) * (Nc > 0 ? Nc : 1));
    char *taken = (char *)malloc(Nc > 0 ? Nc : 1);
    if (!qbar || !s || !order || !taken) return -2;
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g)
            for (int m = 0; m < nqb; ++m) {
                query_block_summary(p, q, b, g, m, qbar);
                for (int j = 0; j < Nc; ++j) {
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += qbar[d] * summ[ix4(b, Hkv, g, Nc, j, D, d)];
                    s[j] = dot / sqrt((double)D);
                    if (scores) scores[ix4(b, Hkv, g, nqb, m, Nc, j)] = s[j];
                }
                select_chunks(s, Nc, K, p->sink_chunks, order, taken, idx + ix4(b, Hkv, g, nqb, m, K, 0),
                              gap ? gap + (b * Hkv + g) * nqb + m : NULL);
            }
    free(qbar); free(s); free(order); free(taken);
    return 0;
}

/* [TS5, causal leakage; TS2.1] strictly causal routing: sharing one route
 * among the tokens of a block lets a token's route depend on later tokens;
 * here every token routes by the summary of its block's queries up to and
 * including itself (the mean over the G heads of the group and the queries
 * m*q_block .. i), so nothing after i can change the route of i.  The last
 * token of a block gets the block's route; with q_block = 1 every token
 * routes alone.  idx gets one route per token, [B][Hkv][S][k] (use it with
 * q_block = 1 in the attention); gap, if given, [B][Hkv][S]; the sink rule
 * applies as in oracle_route. */
int oracle_route_causal(const oracle_shape_t *p, const double *q, const double *summ, int *idx, double *gap)
{
    const int B = p->batch, Hq = p->n_q_heads, Hkv = p->n_kv_heads, D = p->head_dim, S = p->seg_len;
    const int Nc = p->n_hist_chunks, K = p->topk;
    if (Hq % Hkv || S % p->q_block || K <= 0) return -1;
    const int G = Hq / Hkv;
    double *qsum = (double *)malloc(sizeof(double) * D);
    double *s = (double *)malloc(sizeof(double) * (Nc > 0 ? Nc : 1));
    int *order = (int *)malloc(sizeof(int) * (Nc > 0 ? Nc : 1));
    char *taken = (char *)malloc(Nc > 0 ? Nc : 1);
    if (!qsum || !s || !order || !taken) return -2;
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g)
            for (int i = 0; i < S; ++i) {
                const int start = (i / p->q_block) * p->q_block;
                /* prefix summary of the block: queries start .. i of the G heads */
                for (int d = 0; d < D; ++d) qsum[d] = 0.0;
                for (int hh = 0; hh < G; ++hh)
                    for (int t = start; t <= i; ++t)
                        for (int d = 0; d < D; ++d) qsum[d] += q[ix4(b, Hq, g * G + hh, S, t, D, d)];
                const double cnt = (double)G * (i - start + 1);
                for (int j = 0; j < Nc; ++j) {
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += (qsum[d] / cnt) * summ[ix4(b, Hkv, g, Nc, j, D, d)];
                    s[j] = dot / sqrt((double)D);
                }
                select_chunks(s, Nc, K, p->sink_chunks, order, taken, idx + ix4(b, Hkv, g, S, i, K, 0),
                              gap ? gap + ((long long)b * Hkv + g) * S + i : NULL);
            }
    free(qsum); free(s); free(order); free(taken);
    return 0;
}

/* [TS2.1, group selection] second routing stage: for each query block, the
 * groups of gs = p->group tokens inside its chosen chunks (idx, from
 * oracle_route) are scored against the same query-block summary with their
 * group summaries gsumm ([B][Hkv][Nc * c / gs][D], the mean of each group's
 * keys), and the topg best (score descending, group index ascending) are
 * kept.  gidx ([B][Hkv][S/q_block][topg]) gets the global group ids
 * (chunk * c / gs + group within the chunk) in ascending order, padded with
 * -1 when the chosen chunks hold fewer than topg groups.  gap (optional) gets
 * the relative distance between the topg-th and (topg+1)-th best group
 * scores, +inf when every candidate group is kept. */
int oracle_route_groups(const oracle_shape_t *p, const double *q, const double *gsumm, const int *idx,
                        int *gidx, double *gap)
{
    const int B = p->batch, Hkv = p->n_kv_heads, D = p->head_dim, Nc = p->n_hist_chunks, K = p->topk;
    const int gs = p->group, KG = p->topg;
    if (p->n_q_heads % Hkv || p->seg_len % p->q_block || K <= 0 || gs <= 0 || p->chunk % gs || KG <= 0)
        return -1;
    const int gpc = p->chunk / gs;  /* groups per chunk */
    const int Ng = Nc * gpc;        /* groups in the history */
    const int nqb = p->seg_len / p->q_block;
    const int ncand_max = K * gpc;
    double *qbar = (double *)malloc(sizeof(double) * D);
    double *s = (double *)malloc(sizeof(double) * ncand_max);
    int *cand = (int *)malloc(sizeof(int) * ncand_max);
    int *order = (int *)malloc(sizeof(int) * (ncand_max + 1));
    char *taken = (char *)malloc(ncand_max);
    if (!qbar || !s || !cand || !order || !taken) return -2;
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g)
            for (int m = 0; m < nqb; ++m) {
                query_block_summary(p, q, b, g, m, qbar);
                /* the candidate groups: every group of every chosen chunk, ascending */
                const int *sel = idx + ix4(b, Hkv, g, nqb, m, K, 0);
                int nc = 0;
                for (int a = 0; a < K; ++a) {
                    const int j = sel[a];
                    if (j < 0 || j >= Nc) continue;
                    for (int u = 0; u < gpc; ++u) cand[nc++] = j * gpc + u;
                }
                for (int c = 0; c < nc; ++c) {
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += qbar[d] * gsumm[ix4(b, Hkv, g, Ng, cand[c], D, d)];
                    s[c] = dot / sqrt((double)D);
                }
                /* plain selection of the best remaining candidate, kg times (and one
                 * more for the gap) */
                const int kg = KG < nc ? KG : nc;
                memset(taken, 0, ncand_max);
                const int n_rank = kg + (nc > kg ? 1 : 0);
                for (int r = 0; r < n_rank; ++r) {
                    int best = -1;
                    for (int c = 0; c < nc; ++c)
                        if (!taken[c] && (best < 0 || ranks_before(s[c], cand[c], s[best], cand[best]))) best = c;
                    order[r] = best;
                    if (r < kg) taken[best] = 1;
                }
                int *out = gidx + ix4(b, Hkv, g, nqb, m, KG, 0);
                int w = 0;
                for (int c = 0; c < nc; ++c) /* candidates are in ascending group order */
                    if (taken[c]) out[w++] = cand[c];
                for (; w < KG; ++w) out[w] = -1;
                if (gap) {
                    double g_rel = INFINITY;
                    if (nc > kg && kg > 0) {
                        double a = s[order[kg - 1]], c2 = s[order[kg]];
                        double den = fabs(a) > fabs(c2) ? fabs(a) : fabs(c2);
                        if (den < 1e-30) den = 1e-30;
                        g_rel = (a - c2) / den;
                    }
                    gap[(b * Hkv + g) * nqb + m] = g_rel;
                }
            }
    free(qbar); free(s); free(cand); free(order); free(taken);
    return 0;
}

/* The key set U_i of query (b, h, i) [TS2.1, ABS]: the tokens of the routed
 * history chunks (with the group stage: of the routed groups) followed by the
 * active-segment tokens 0..i.  Returns the count and fills pointers to each
 * key and value row. */
static int gather_keys(const oracle_shape_t *p, const double *k_hist, const double *v_hist,
                       const double *k_seg, const double *v_seg, const int *idx,
                       int b, int g, int i, const double **kr, const double **vr, int *seg_pos)
{
    const int Hkv = p->n_kv_heads, D = p->head_dim, S = p->seg_len;
    /* routing unit: a chunk, or a group of the group stage */
    const int c = p->group > 0 ? p->group : p->chunk;
    const int K = p->group > 0 ? p->topg : p->topk;
    const int n_units = p->group > 0 ? p->n_hist_chunks * (p->chunk / p->group) : p->n_hist_chunks;
    const int nqb = S / p->q_block, m = i / p->q_block;
    const long long T = (long long)p->n_hist_chunks * p->chunk;
    int n = 0;
    const int *sel = idx + ix4(b, Hkv, g, nqb, m, K, 0);
    for (int a = 0; a < K; ++a) {
        int j = sel[a];
        if (j < 0 || j >= n_units) continue;
        for (int r = 0; r < c; ++r) {
            long long t = (long long)j * c + r;
            kr[n] = k_hist + (((long long)b * Hkv + g) * T + t) * D;
            vr[n] = v_hist + (((long long)b * Hkv + g) * T + t) * D;
            seg_pos[n] = -1;
            ++n;
        }
    }
    for (int t = 0; t <= i; ++t) {
        kr[n] = k_seg + (((long long)b * Hkv + g) * S + t) * D;
        vr[n] = v_seg + (((long long)b * Hkv + g) * S + t) * D;
        seg_pos[n] = t;
        ++n;
    }
    return n;
}

/* Exact softmax attention of one query row over its gathered key set:
 * logits z_t = q.k_t / sqrt(D), P = softmax(z), o = sum_t P_t v_t,
 * lse = log sum_t exp(z_t).  P is returned in prob (length n). */
static double attend_row(const double *qrow, int D, int n, const double **kr, const double **vr,
                         double *prob, double *orow)
{
    double zmax = -INFINITY;
    for (int t = 0; t < n; ++t) {
        double z = 0.0;
        for (int d = 0; d < D; ++d) z += qrow[d] * kr[t][d];
        z /= sqrt((double)D);
        prob[t] = z;
        if (z > zmax) zmax = z;
    }
    double sum = 0.0;
    for (int t = 0; t < n; ++t) { prob[t] = exp(prob[t] - zmax); sum += prob[t]; }
    for (int t = 0; t < n; ++t) prob[t] /= sum;
    for (int d = 0; d < D; ++d) orow[d] = 0.0;
    for (int t = 0; t < n; ++t)
        for (int d = 0; d < D; ++d) orow[d] += prob[t] * vr[t][d];
    return zmax + log(sum);
}

/* [TS2.1] exact-token attention forward, with the routes as an input.
 * rows (optional): a list of n_rows flat query indices (b*Hq + h)*S + i to
 * compute; NULL computes every row.  Rows not computed are left untouched. */
int oracle_attn_fwd(const oracle_shape_t *p, const double *q, const double *k_hist, const double *v_hist,
                    const double *k_seg, const double *v_seg, const int *idx,
                    const long long *rows, long long n_rows, double *out, double *lse)
{
    const int Hq = p->n_q_heads, Hkv = p->n_kv_heads, D = p->head_dim, S = p->seg_len;
    if (Hq % Hkv || S % p->q_block) return -1;
    const int G = Hq / Hkv;
    const long long hist_cap = p->group > 0 ? (long long)p->topg * p->group : (long long)p->topk * p->chunk;
    const long long cap = hist_cap + S;
    const double **kr = (const double **)malloc(sizeof(double *) * cap);
    const double **vr = (const double **)malloc(sizeof(double *) * cap);
    int *pos = (int *)malloc(sizeof(int) * cap);
    double *prob = (double *)malloc(sizeof(double) * cap);
    if (!kr || !vr || !pos || !prob) return -2;
    const long long total = (long long)p->batch * Hq * S;
    const long long count = rows ? n_rows : total;
    for (long long r = 0; r < count; ++r) {
        long long f = rows ? rows[r] : r;
        if (f < 0 || f >= total) continue;
        int i = (int)(f % S), h = (int)((f / S) % Hq), b = (int)(f / ((long long)S * Hq));
        int n = gather_keys(p, k_hist, v_hist, k_seg, v_seg, idx, b, h / G, i, kr, vr, pos);
        double l = attend_row(q + f * D, D, n, kr, vr, prob, out + f * D);
        if (lse) lse[f] = l;
    }
    free(kr); free(vr); free(pos); free(prob);
    return 0;
}

/* [TS2.1, TS2.2, ABS] backward of the exact-token attention with routes
 * frozen: for each query row, with P its softmax row and dO its upstream
 * gradient,
 *   dP_t = dO . v_t,  delta = sum_t P_t dP_t,  dS_t = P_t (dP_t - delta),
 *   dQ   = sum_t dS_t k_t / sqrt(D),
 *   dK_t += dS_t q / sqrt(D),  dV_t += P_t dO   for active-segment keys only.
 * History keys and values receive no gradient (they are detached).
 * q_need / key_need (optional, [B][Hq][S] and [B][Hkv][S] bytes) restrict
 * which dQ rows and which dK/dV rows are produced; NULL means all.  Outputs
 * are overwritten (zeroed first). */
int oracle_attn_bwd(const oracle_shape_t *p, const double *q, const double *k_hist, const double *v_hist,
                    const double *k_seg, const double *v_seg, const int *idx, const double *dout,
                    const unsigned char *q_need, const unsigned char *key_need,
                    double *dq, double *dk_seg, double *dv_seg)
{
    const int B = p->batch, Hq = p->n_q_heads, Hkv = p->n_kv_heads, D = p->head_dim, S = p->seg_len;
    if (Hq % Hkv || S % p->q_block) return -1;
    const int G = Hq / Hkv;
    const long long hist_cap = p->group > 0 ? (long long)p->topg * p->group : (long long)p->topk * p->chunk;
    const long long cap = hist_cap + S;
    const double **kr = (const double **)malloc(sizeof(double *) * cap);
    const double **vr = (const double **)malloc(sizeof(double *) * cap);
    int *pos = (int *)malloc(sizeof(int) * cap);
    double *prob = (double *)malloc(sizeof(double) * cap);
    double *dp = (double *)malloc(sizeof(double) * cap);
    double *orow = (double *)malloc(sizeof(double) * D);
    if (!kr || !vr || !pos || !prob || !dp || !orow) return -2;
    memset(dq, 0, sizeof(double) * (size_t)B * Hq * S * D);
    memset(dk_seg, 0, sizeof(double) * (size_t)B * Hkv * S * D);
    memset(dv_seg, 0, sizeof(double) * (size_t)B * Hkv * S * D);
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            /* earliest active key whose gradient is requested for this group */
            int first_key = S;
            for (int t = 0; t < S; ++t)
                if (!key_need || key_need[((long long)b * Hkv + g) * S + t]) { first_key = t; break; }
            for (int i = 0; i < S; ++i) {
                const long long f = ((long long)b * Hq + h) * S + i;
                const int want_q = !q_need || q_need[f];
                if (!want_q && i < first_key) continue;
                const double *qrow = q + f * D, *gorow = dout + f * D;
                int n = gather_keys(p, k_hist, v_hist, k_seg, v_seg, idx, b, g, i, kr, vr, pos);
                attend_row(qrow, D, n, kr, vr, prob, orow);
                double delta = 0.0;
                for (int t = 0; t < n; ++t) {
                    double s = 0.0;
                    for (int d = 0; d < D; ++d) s += gorow[d] * vr[t][d];
                    dp[t] = s;
                    delta += prob[t] * s;
                }
                for (int t = 0; t < n; ++t) {
                    const double ds = prob[t] * (dp[t] - delta);
                    if (want_q)
                        for (int d = 0; d < D; ++d) dq[f * D + d] += ds * kr[t][d] * inv_sqrt_d;
                    if (pos[t] >= 0) {
                        const long long kf = ((long long)b * Hkv + g) * S + pos[t];
                        if (key_need && !key_need[kf]) continue;
                        for (int d = 0; d < D; ++d) {
                            dk_seg[kf * D + d] += ds * qrow[d] * inv_sqrt_d;
                            dv_seg[kf * D + d] += prob[t] * gorow[d];
                        }
                    }
                }
            }
        }
    free(kr); free(vr); free(pos); free(prob); free(dp); free(orow);
    return 0;
}

/* Dense causal attention over [history | segment]: query i of the segment sits
 * at absolute position T + i and attends every token at or before it.  This is
 * the standard attention HGA replaces [TS2.1]; it is what HGA reduces to when
 * the routing budget covers every history chunk. */
int oracle_dense_causal(const oracle_shape_t *p, const double *q, const double *k_all, const double *v_all,
                        double *out, double *lse)
{
    const int B = p->batch, Hq = p->n_q_heads, Hkv = p->n_kv_heads, D = p->head_dim, S = p->seg_len;
    if (Hq % Hkv) return -1;
    const int G = Hq / Hkv;
    const long long T = (long long)p->n_hist_chunks * p->chunk, L = T + S;
    const double **kr = (const double **)malloc(sizeof(double *) * L);
    const double **vr = (const double **)malloc(sizeof(double *) * L);
    double *prob = (double *)malloc(sizeof(double) * L);
    if (!kr || !vr || !prob) return -2;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h)
            for (int i = 0; i < S; ++i) {
                const long long f = ((long long)b * Hq + h) * S + i;
                const int g = h / G;
                int n = 0;
                for (long long t = 0; t <= T + i; ++t) {
                    kr[n] = k_all + (((long long)b * Hkv + g) * L + t) * D;
                    vr[n] = v_all + (((long long)b * Hkv + g) * L + t) * D;
                    ++n;
                }
                double l = attend_row(q + f * D, D, n, kr, vr, prob, out + f * D);
                if (lse) lse[f] = l;
            }
    free(kr); free(vr); free(prob);
    return 0;
}
