"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

Each test fixes a result by something other than the oracle's own code: a
hand-worked example under tests/golden, a closed form on a constructed input,
a library routine (torch scaled-dot-product attention, torch autograd,
numpy's stable sort) on a case that reduces to it, or central finite
differences.  No GPU is needed.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from inputs import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _shape(B=1, Hq=2, Hkv=1, D=16, c=16, qb=16, k=2, S=64, Nc=4):
    return oracle.shape(B, Hq, Hkv, D, c, qb, k, S, Nc)


def _random_layer(sh, seed=0):
    r = _rng(seed)
    T = sh.n_hist_chunks * sh.chunk
    q = r.standard_normal((sh.batch, sh.n_q_heads, sh.seg_len, sh.head_dim))
    kh = r.standard_normal((sh.batch, sh.n_kv_heads, T, sh.head_dim))
    vh = r.standard_normal((sh.batch, sh.n_kv_heads, T, sh.head_dim))
    ks = r.standard_normal((sh.batch, sh.n_kv_heads, sh.seg_len, sh.head_dim))
    vs = r.standard_normal((sh.batch, sh.n_kv_heads, sh.seg_len, sh.head_dim))
    return q, kh, vh, ks, vs


def _allowed_mask(sh, idx):
    """Boolean [B][Hkv][S][T+S]: which keys query i may see (routed chunks + causal segment)."""
    T = sh.n_hist_chunks * sh.chunk
    S = sh.seg_len
    mask = np.zeros((sh.batch, sh.n_kv_heads, S, T + S), dtype=bool)
    for b in range(sh.batch):
        for g in range(sh.n_kv_heads):
            for i in range(S):
                for j in idx[b, g, i // sh.q_block]:
                    if j >= 0:
                        mask[b, g, i, j * sh.chunk:(j + 1) * sh.chunk] = True
                mask[b, g, i, T:T + i + 1] = True
    return mask


def _sdpa(sh, q, kh, vh, ks, vs, mask):
    """torch's attention (fp64) over [history | segment] with an explicit boolean mask."""
    G = sh.n_q_heads // sh.n_kv_heads
    k_all = torch.from_numpy(np.concatenate([kh, ks], axis=2)).repeat_interleave(G, dim=1)
    v_all = torch.from_numpy(np.concatenate([vh, vs], axis=2)).repeat_interleave(G, dim=1)
    m = torch.from_numpy(mask).repeat_interleave(G, dim=1)
    qt = torch.from_numpy(q)
    out = torch.nn.functional.scaled_dot_product_attention(qt, k_all, v_all, attn_mask=m)
    logits = torch.einsum("bhid,bhtd->bhit", qt, k_all) / math.sqrt(sh.head_dim)
    lse = torch.logsumexp(logits.masked_fill(~m, -math.inf), dim=-1)
    return out.numpy(), lse.numpy()


# ----------------------------------------------------------------- summaries

def test_summaries_golden_hand_example():
    lines = [ln.split("#")[0].strip() for ln in open(os.path.join(GOLDEN, "summaries_tiny.txt"))]
    lines = [ln for ln in lines if ln]
    chunk = int(lines[0].split()[1])
    keys = np.array([[float(x) for x in ln.split(":")[1].split()] for ln in lines if ln.startswith("key")])
    want = np.array([[float(x) for x in ln.split(":")[1].split()] for ln in lines if ln.startswith("summary")])
    got = oracle.summaries(keys[None, None], chunk)[0, 0]
    assert np.array_equal(got, want)


def test_summaries_linear_ramp_closed_form():
    # k[t][d] = t + 1000*d: the mean of chunk j is j*c + (c-1)/2 + 1000*d
    c, nc, D = 64, 7, 5
    t = np.arange(nc * c, dtype=np.float64)
    k = (t[:, None] + 1000.0 * np.arange(D)[None, :])[None, None]
    got = oracle.summaries(k, c)[0, 0]
    want = np.arange(nc)[:, None] * c + (c - 1) / 2 + 1000.0 * np.arange(D)[None, :]
    assert np.allclose(got, want, rtol=0, atol=1e-9)


def test_summaries_heads_are_independent():
    c = 8
    k = np.zeros((2, 3, 4 * c, 2))
    for b in range(2):
        for g in range(3):
            k[b, g] = 10 * b + g
    s = oracle.summaries(k, c)
    for b in range(2):
        for g in range(3):
            assert np.all(s[b, g] == 10 * b + g)


# ----------------------------------------------------------------- routing

def _constructed_route_case(alpha, k, G=2, qb=16, c=16, D=8, S=32):
    """Keys of chunk j all equal alpha_j * u; group queries average to u exactly.

    Then the chunk summary is alpha_j * u and the score of chunk j is
    alpha_j * |u|^2 / sqrt(D) = alpha_j / sqrt(D) for a unit u.
    """
    nc = len(alpha)
    u = np.zeros(D)
    u[3] = 1.0
    kh = np.repeat(np.asarray(alpha, dtype=np.float64)[:, None] * u[None, :], c, axis=0)[None, None]
    q = np.zeros((1, G, S, D))
    q[0, 0] = G * u  # head 0 carries G*u, the other heads 0: the group mean is u only if
    # the mean runs over the G heads (and over the block's rows)
    sh = oracle.shape(1, G, 1, D, c, qb, k, S, nc)
    summ = oracle.summaries(kh, c)
    return sh, oracle.route(sh, q, summ, with_scores=True)


def test_route_constructed_scores_and_selection():
    alpha = [0.5, -2.0, 3.0, 1.25, 7.0, -0.25, 2.5, 0.0]
    k = 3
    sh, (idx, gap, scores) = _constructed_route_case(alpha, k)
    D = sh.head_dim
    assert np.allclose(scores[0, 0, 0], np.array(alpha) / math.sqrt(D), rtol=0, atol=1e-15)
    # numpy's stable argsort on -alpha gives (alpha desc, index asc)
    best = np.sort(np.argsort(-np.array(alpha), kind="stable")[:k])
    for m in range(sh.seg_len // sh.q_block):
        assert list(idx[0, 0, m]) == list(best)
    a_sorted = sorted(alpha, reverse=True)
    want_gap = (a_sorted[k - 1] - a_sorted[k]) / max(abs(a_sorted[k - 1]), abs(a_sorted[k]))
    assert gap[0, 0, 0] == pytest.approx(want_gap, rel=1e-12)


def test_route_mean_over_group_heads():
    # If the query-block summary summed instead of averaging over the G heads,
    # the scores would be scaled by G.
    alpha = [1.0, 2.0, 3.0, 4.0]
    for G in (1, 2, 4):
        sh, (_, _, scores) = _constructed_route_case(alpha, 2, G=G)
        assert np.allclose(scores[0, 0, 0], np.array(alpha) / math.sqrt(sh.head_dim), atol=1e-15)


def test_route_ties_go_to_lower_index():
    alpha = [1.0, 3.0, 3.0, 3.0, 0.0, 3.0]
    _, (idx, gap, _) = _constructed_route_case(alpha, 2)
    assert list(idx[0, 0, 0]) == [1, 2]
    assert gap[0, 0, 0] == 0.0
    # all scores equal -> the first k chunks
    _, (idx, _, _) = _constructed_route_case([0.7] * 6, 4)
    assert list(idx[0, 0, 0]) == [0, 1, 2, 3]


def test_route_budget_above_history_pads():
    alpha = [1.0, -1.0, 0.5]
    _, (idx, gap, _) = _constructed_route_case(alpha, 5)
    assert list(idx[0, 0, 0]) == [0, 1, 2, -1, -1]
    assert np.isinf(gap[0, 0, 0])
    # no history at all: everything is padding
    sh = oracle.shape(1, 2, 1, 8, 16, 16, 3, 32, 0)
    idx, gap, _ = oracle.route(sh, np.ones((1, 2, 32, 8)), np.zeros((1, 1, 0, 8)))
    assert np.all(idx == -1)


def test_route_uses_own_group_and_own_block_only():
    # 2 KV groups of 2 heads, 2 query blocks; chunk j's keys point along e_j.
    D, c, qb, S, nc, G = 8, 16, 16, 32, 6, 2
    kh = np.zeros((1, 2, nc * c, D))
    for g in range(2):
        for j in range(nc):
            kh[0, g, j * c:(j + 1) * c, j] = 1.0
    q = np.zeros((1, 4, S, D))
    q[0, 0, 0:16, 4] = 5.0      # group 0, block 0 -> chunk 4
    q[0, 1, 16:32, 1] = 5.0     # group 0, block 1 -> chunk 1
    q[0, 3, 0:16, 2] = 5.0      # group 1, block 0 -> chunk 2
    q[0, 2, 16:32, 5] = 5.0     # group 1, block 1 -> chunk 5
    sh = oracle.shape(1, 4, 2, D, c, qb, 1, S, nc)
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, c))
    assert idx[0, :, :, 0].tolist() == [[4, 1], [2, 5]]


def test_route_planted_chunk_is_selected():
    # the pages' workloads: a chunk whose offset is aligned with the block's
    # queries must win the routing
    r = _rng(5)
    D, c, qb, S, nc = 32, 64, 64, 128, 12
    kh = r.standard_normal((1, 1, nc * c, D))
    direction = r.standard_normal(D)
    direction /= np.linalg.norm(direction)
    kh[0, 0, 7 * c:8 * c] += 3.0 * direction
    q = r.standard_normal((1, 2, S, D)) + 2.0 * direction
    sh = oracle.shape(1, 2, 1, D, c, qb, 1, S, nc)
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, c))
    assert np.all(idx[..., 0] == 7)


# ----------------------------------------------------------------- attention forward

@pytest.mark.parametrize("Nc,k", [(4, 4), (4, 9), (0, 2)])
def test_full_coverage_equals_dense_causal_attention(Nc, k):
    sh = _shape(Nc=Nc, k=k, Hq=4, Hkv=2)
    q, kh, vh, ks, vs = _random_layer(sh, seed=Nc + k)
    idx = np.tile(np.r_[np.arange(Nc), -np.ones(max(k - Nc, 0))].astype(np.int32)[:k],
                  (1, 2, sh.seg_len // sh.q_block, 1))
    out, lse = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx)
    # torch SDPA with the plain causal mask over [history | segment]
    T, S = Nc * sh.chunk, sh.seg_len
    causal = np.zeros((1, 2, S, T + S), dtype=bool)
    for i in range(S):
        causal[:, :, i, :T + i + 1] = True
    o_ref, lse_ref = _sdpa(sh, q, kh, vh, ks, vs, causal)
    assert np.max(np.abs(out - o_ref)) < 1e-12
    assert np.max(np.abs(lse - lse_ref)) < 1e-12
    # the oracle's dense routine agrees as well
    od, ld = oracle.dense_causal(sh, q, np.concatenate([kh, ks], 2), np.concatenate([vh, vs], 2))
    assert np.max(np.abs(od - o_ref)) < 1e-12 and np.max(np.abs(ld - lse_ref)) < 1e-12


def test_partial_routes_equal_masked_attention():
    sh = _shape(Nc=6, k=2, Hq=4, Hkv=2, S=64)
    q, kh, vh, ks, vs = _random_layer(sh, seed=11)
    r = _rng(3)
    nqb = sh.seg_len // sh.q_block
    idx = np.zeros((1, 2, nqb, 2), dtype=np.int32)
    for g in range(2):
        for m in range(nqb):
            idx[0, g, m] = np.sort(r.choice(6, 2, replace=False))
    idx[0, 1, 2] = [4, -1]  # a padded slot
    out, lse = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx)
    o_ref, lse_ref = _sdpa(sh, q, kh, vh, ks, vs, _allowed_mask(sh, idx))
    assert np.max(np.abs(out - o_ref)) < 1e-12
    assert np.max(np.abs(lse - lse_ref)) < 1e-12


def test_attended_count_golden():
    rows = [ln.split("#")[0].split() for ln in open(os.path.join(GOLDEN, "attended_count.txt"))]
    rows = [list(map(int, r)) for r in rows if r]
    for Nc, k, c, S, i, count in rows:
        sh = oracle.shape(1, 2, 1, 16, c, 64, k, S, Nc)
        T = Nc * c
        q = np.zeros((1, 2, S, 16))
        r = _rng(i)
        kh, vh = r.standard_normal((1, 1, T, 16)), r.standard_normal((1, 1, T, 16))
        ks, vs = r.standard_normal((1, 1, S, 16)), r.standard_normal((1, 1, S, 16))
        summ = oracle.summaries(kh, c) if Nc else np.zeros((1, 1, 0, 16))
        idx, _, _ = oracle.route(sh, q, summ)
        _, lse = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx, rows=[i, S + i])
        assert lse[0, 0, i] == pytest.approx(math.log(count), abs=1e-13)
        assert lse[0, 1, i] == pytest.approx(math.log(count), abs=1e-13)


def test_softmax_rows_sum_to_one():
    sh = _shape(Nc=5, k=3, S=48, qb=16)
    q, kh, vh, ks, vs = _random_layer(sh, seed=2)
    vh[..., 0] = 1.0
    vs[..., 0] = 1.0
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, sh.chunk))
    out, _ = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx)
    assert np.max(np.abs(out[..., 0] - 1.0)) < 1e-14


def test_row_subset_matches_full():
    sh = _shape(Nc=5, k=2, S=48, Hq=4, Hkv=2)
    q, kh, vh, ks, vs = _random_layer(sh, seed=4)
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, sh.chunk))
    full_o, full_l = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx)
    rows = np.array([0, 47, 48 + 13, 3 * 48 + 40])
    o, l = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx, rows=rows)
    fo, fl = full_o.reshape(-1, sh.head_dim), full_l.reshape(-1)
    assert np.array_equal(o.reshape(-1, sh.head_dim)[rows], fo[rows])
    assert np.array_equal(l.reshape(-1)[rows], fl[rows])


# ----------------------------------------------------------------- backward

def _loss(sh, q, kh, vh, ks, vs, idx, dout):
    out, _ = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx)
    return float(np.sum(out * dout))


def test_backward_central_finite_differences():
    sh = _shape(B=1, Hq=4, Hkv=2, D=8, c=16, qb=16, k=2, S=48, Nc=4)
    q, kh, vh, ks, vs = _random_layer(sh, seed=21)
    dout = _rng(22).standard_normal(q.shape)
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, sh.chunk))  # routes frozen below
    dq, dk, dv = oracle.attn_bwd(sh, q, kh, vh, ks, vs, idx, dout)
    h = 1e-6
    r = _rng(23)
    for name, arr, grad in (("q", q, dq), ("k_seg", ks, dk), ("v_seg", vs, dv)):
        for _ in range(12):
            pos = tuple(r.integers(0, n) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[pos] += h
            minus[pos] -= h
            args = {"q": q, "k_seg": ks, "v_seg": vs}
            args_p, args_m = dict(args), dict(args)
            args_p[name], args_m[name] = plus, minus
            fd = (_loss(sh, args_p["q"], kh, vh, args_p["k_seg"], args_p["v_seg"], idx, dout)
                  - _loss(sh, args_m["q"], kh, vh, args_m["k_seg"], args_m["v_seg"], idx, dout)) / (2 * h)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def test_backward_full_coverage_matches_autograd():
    sh = _shape(Hq=4, Hkv=2, D=16, c=16, qb=16, k=3, S=48, Nc=3)
    q, kh, vh, ks, vs = _random_layer(sh, seed=31)
    dout = _rng(32).standard_normal(q.shape)
    idx = np.tile(np.arange(3, dtype=np.int32), (1, 2, 3, 1))
    dq, dk, dv = oracle.attn_bwd(sh, q, kh, vh, ks, vs, idx, dout)
    G, T, S = 2, 48, 48
    qt = torch.from_numpy(q).requires_grad_()
    kst = torch.from_numpy(ks).requires_grad_()
    vst = torch.from_numpy(vs).requires_grad_()
    k_all = torch.cat([torch.from_numpy(kh), kst], 2).repeat_interleave(G, 1)
    v_all = torch.cat([torch.from_numpy(vh), vst], 2).repeat_interleave(G, 1)
    mask = torch.zeros(S, T + S, dtype=torch.bool)
    for i in range(S):
        mask[i, :T + i + 1] = True
    out = torch.nn.functional.scaled_dot_product_attention(qt, k_all, v_all, attn_mask=mask)
    (out * torch.from_numpy(dout)).sum().backward()
    assert np.max(np.abs(dq - qt.grad.numpy())) < 1e-12
    assert np.max(np.abs(dk - kst.grad.numpy())) < 1e-12
    assert np.max(np.abs(dv - vst.grad.numpy())) < 1e-12


def test_backward_row_restriction_matches_full():
    sh = _shape(Hq=4, Hkv=2, D=8, c=16, qb=16, k=2, S=64, Nc=5)
    q, kh, vh, ks, vs = _random_layer(sh, seed=41)
    dout = _rng(42).standard_normal(q.shape)
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, sh.chunk))
    dq, dk, dv = oracle.attn_bwd(sh, q, kh, vh, ks, vs, idx, dout)
    qn = np.zeros(q.shape[:3], dtype=np.uint8)
    qn[0, 1, [3, 60]] = 1
    kn = np.zeros(ks.shape[:3], dtype=np.uint8)
    kn[0, 0, [50, 63]] = 1
    kn[0, 1, 17] = 1
    dq2, dk2, dv2 = oracle.attn_bwd(sh, q, kh, vh, ks, vs, idx, dout, q_need=qn, key_need=kn)
    assert np.array_equal(dq2[qn.astype(bool)], dq[qn.astype(bool)])
    assert np.array_equal(dk2[kn.astype(bool)], dk[kn.astype(bool)])
    assert np.array_equal(dv2[kn.astype(bool)], dv[kn.astype(bool)])


# ----------------------------------------------------------------- generator

def test_generator_slices_agree_and_offsets_have_norm_two():
    w = gen.custom("t", seq_len=512, seg_starts=(256,), dtype="bf16", head_dim=32)
    full = gen.keys(w, 0, 512)
    part = gen.keys(w, 128, 320)
    assert np.array_equal(full[:, :, 128:320], part)
    assert np.array_equal(gen.round_bf16(full), full)
    off = gen.chunk_offsets(w, 0, 8)
    assert np.allclose(np.linalg.norm(off, axis=-1), 2.0)


def test_generator_normal_moments():
    z = gen.normals(gen.stream_key(7, 1), np.arange(200000))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01


def test_torch_generator_matches_numpy_recipe():
    w = gen.custom("t", seq_len=512, seg_starts=(256,), dtype="bf16", head_dim=32, n_q_heads=4, n_kv_heads=2)
    for fn_np, fn_t in ((gen.keys, gen.keys_torch), (gen.values, gen.values_torch),
                        (gen.queries, gen.queries_torch)):
        a = fn_np(w, 128, 384)
        b = fn_t(w, 128, 384, "cpu").float().numpy()
        mismatch = np.mean(a != b)
        assert mismatch < 1e-3 and np.max(np.abs(a - b)) < 1e-2, (fn_np.__name__, mismatch)


# ---------------------------------------------------------------- attention-sink window

def _expected_sink_route(scores, k, sink):
    """The rule written out with numpy: chunks 0..min(sink, k_eff)-1 first, then the
    best of the others by (score descending, chunk index ascending); ascending, -1 padded."""
    nc = scores.shape[-1]
    keff = min(k, nc)
    ns = min(sink, keff)
    rest = np.arange(ns, nc)
    order = rest[np.lexsort((rest, -scores[ns:]))]  # primary: score desc; then index asc
    chosen = sorted(list(range(ns)) + list(order[:keff - ns]))
    return chosen + [-1] * (k - keff)


def test_route_sink_window_rule():
    """The technical summary (section 2.1) puts a fixed sink window next to the routed
    chunks; with sink_chunks = s the first s chunks are routed whatever their score and
    the remaining slots go to the best other chunks."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, D, c, qb, S, nc, k = 2, 4, 2, 16, 16, 16, 48, 13, 5
    q = rng.standard_normal((B, Hq, S, D))
    summ = rng.standard_normal((B, Hkv, nc, D))
    for sink in (0, 1, 2, 5):
        sh = oracle.shape(B, Hq, Hkv, D, c, qb, k, S, nc, sink)
        idx, gap, scores = oracle.route(sh, q, summ, with_scores=True)
        for b in range(B):
            for g in range(Hkv):
                for m in range(S // qb):
                    want = _expected_sink_route(scores[b, g, m], k, sink)
                    assert list(idx[b, g, m]) == want, (sink, b, g, m)
        if sink == k:
            assert np.all(np.isinf(gap))  # no slot is decided by score


def test_route_sink_keeps_a_low_scoring_first_chunk():
    # chunk 0's summary points away from the queries: without a sink it is never routed
    D, c, qb, S, nc, k = 8, 8, 8, 8, 6, 2
    q = np.zeros((1, 2, S, D))
    q[..., 0] = 1.0
    summ = np.zeros((1, 1, nc, D))
    summ[0, 0, :, 0] = [-5.0, 1.0, 2.0, 3.0, 4.0, 0.5]
    idx0, _, _ = oracle.route(oracle.shape(1, 2, 1, D, c, qb, k, S, nc, 0), q, summ)
    idx1, _, _ = oracle.route(oracle.shape(1, 2, 1, D, c, qb, k, S, nc, 1), q, summ)
    assert list(idx0[0, 0, 0]) == [3, 4]
    assert list(idx1[0, 0, 0]) == [0, 4]
    # k >= Nc: every chunk is routed with or without the sink
    idx2, _, _ = oracle.route(oracle.shape(1, 2, 1, D, c, qb, 8, S, nc, 1), q, summ)
    assert list(idx2[0, 0, 0]) == [0, 1, 2, 3, 4, 5, -1, -1]


# ---------------------------------------------------------------- single-query decode

def test_decode_token_equals_masked_attention():
    """A decode token is a one-token query block (q_block = 1): its route uses the mean of
    its G query heads, and its output is exact attention over the routed chunks and the
    local window up to itself (torch, fp64, explicit mask; routes from the oracle)."""
    rng = np.random.default_rng(51)
    B, Hq, Hkv, D, c, L, nc, k = 2, 4, 2, 16, 8, 11, 9, 3
    sh = oracle.shape(B, Hq, Hkv, D, c, 1, k, L, nc)
    q = rng.standard_normal((B, Hq, L, D))
    kh, vh = rng.standard_normal((B, Hkv, nc * c, D)), rng.standard_normal((B, Hkv, nc * c, D))
    ks, vs = rng.standard_normal((B, Hkv, L, D)), rng.standard_normal((B, Hkv, L, D))
    summ = oracle.summaries(kh, c)
    idx, _, scores = oracle.route(sh, q, summ, with_scores=True)
    # the last token's route: top-k of its own block summary's scores (ties -> lower index)
    for b in range(B):
        for g in range(Hkv):
            qbar = q[b, g * 2:(g + 1) * 2, L - 1].mean(axis=0)
            s = summ[b, g] @ qbar / np.sqrt(D)
            assert np.allclose(scores[b, g, L - 1], s, rtol=1e-12, atol=1e-12)
            want = sorted(np.lexsort((np.arange(nc), -s))[:k])
            assert list(idx[b, g, L - 1]) == want
    rows = np.array([(b * Hq + h) * L + L - 1 for b in range(B) for h in range(Hq)])
    out, lse = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx, rows=rows)
    ref_out, ref_lse = _sdpa(sh, q, kh, vh, ks, vs, _allowed_mask(sh, idx))
    assert np.allclose(out[:, :, L - 1], ref_out[:, :, L - 1], atol=1e-12)
    assert np.allclose(lse[:, :, L - 1], ref_lse[:, :, L - 1], atol=1e-12)


# ------------------------------------------------- group-level second-stage routing

def _group_mask(sh, gidx):
    """Boolean [B][Hkv][S][T+S]: routed groups' tokens + the causal segment."""
    T = sh.n_hist_chunks * sh.chunk
    S = sh.seg_len
    mask = np.zeros((sh.batch, sh.n_kv_heads, S, T + S), dtype=bool)
    for b in range(sh.batch):
        for g in range(sh.n_kv_heads):
            for i in range(S):
                for u in gidx[b, g, i // sh.q_block]:
                    if u >= 0:
                        mask[b, g, i, u * sh.group:(u + 1) * sh.group] = True
                mask[b, g, i, T:T + i + 1] = True
    return mask


def test_group_summaries_average_to_the_chunk_summary():
    """A chunk's summary (mean of its c keys) is the mean of its c / gs group summaries
    (means of equal-size parts), and a linear ramp K[t] = t v gives group j the summary
    (gs j + (gs - 1) / 2) v."""
    rng = np.random.default_rng(61)
    k = rng.standard_normal((2, 3, 5 * 64, 16))
    chunk = oracle.summaries(k, 64)
    groups = oracle.summaries(k, 8)
    assert groups.shape == (2, 3, 40, 16)
    assert np.allclose(groups.reshape(2, 3, 5, 8, 16).mean(axis=3), chunk, rtol=1e-13, atol=1e-13)
    v = rng.standard_normal(16)
    ramp = np.arange(128, dtype=np.float64)[None, None, :, None] * v
    g = oracle.summaries(ramp, 8)
    for j in range(16):
        assert np.allclose(g[0, 0, j], (8 * j + 3.5) * v, rtol=1e-14, atol=1e-12)


def test_route_groups_constructed_scores_stay_inside_the_chosen_chunks():
    """Group scores built so the order is known: q-bar = e0 and group summaries whose
    first coordinate is the score times sqrt(D).  The best groups of the chosen chunks
    win (equal scores go to the lower group index); a higher-scoring group of an
    unchosen chunk is never taken."""
    D, c, gs, qb, S, nc = 4, 16, 8, 8, 16, 4
    q = np.zeros((1, 2, S, D))
    q[..., 0] = 1.0
    gsumm = np.zeros((1, 1, nc * c // gs, D))
    # groups 0..7: chunk j holds groups 2j, 2j + 1
    gsumm[0, 0, :, 0] = np.array([1.0, 5.0, 9.0, 2.0, 4.0, 4.0, 3.0, 0.5]) * 2.0
    idx = np.array([[[[0, 2, 3], [1, 2, -1]]]], dtype=np.int32)  # block 0: chunks 0, 2, 3; block 1: 1, 2
    sh = oracle.shape(1, 2, 1, D, c, qb, 3, S, nc, 0, gs, 3)
    gidx, gap = oracle.route_groups(sh, q, gsumm, idx)
    # block 0 candidates: groups 0, 1 (1, 5), 4, 5 (4, 4), 6, 7 (3, 0.5): best 1, then 4 and 5 tie
    assert list(gidx[0, 0, 0]) == [1, 4, 5]
    # block 1 candidates: 2, 3 (9, 2), 4, 5 (4, 4): 2, 4, 5; group 1 of chunk 0 (5) is not a candidate
    assert list(gidx[0, 0, 1]) == [2, 4, 5]
    # the 3rd and 4th best of block 0 are 4 (group 5) and 3 (group 6): gap (4 - 3) / 4
    assert gap[0, 0, 0] == pytest.approx(0.25, rel=1e-14)
    # a tie at the budget edge goes to the lower index: topg = 2 keeps groups 1 and 4
    sh2 = oracle.shape(1, 2, 1, D, c, qb, 3, S, nc, 0, gs, 2)
    gidx2, gap2 = oracle.route_groups(sh2, q, gsumm, idx)
    assert list(gidx2[0, 0, 0]) == [1, 4]
    assert gap2[0, 0, 0] == 0.0
    # topg = 1: the best group alone, gap between the best (5) and the runner-up (4)
    sh1 = oracle.shape(1, 2, 1, D, c, qb, 3, S, nc, 0, gs, 1)
    gidx1, gap1 = oracle.route_groups(sh1, q, gsumm, idx)
    assert list(gidx1[0, 0, 0]) == [1] and list(gidx1[0, 0, 1]) == [2]
    assert gap1[0, 0, 0] == pytest.approx(0.2, rel=1e-14)


def test_route_groups_matches_a_numpy_ranking():
    """Random layers: the group route is the top-topg of the candidate groups by
    (score descending, group index ascending) (numpy lexsort over the candidates)."""
    rng = np.random.default_rng(62)
    B, Hq, Hkv, D, c, gs, qb, S, nc, k, kg = 2, 4, 2, 8, 16, 4, 8, 24, 7, 3, 5
    sh = oracle.shape(B, Hq, Hkv, D, c, qb, k, S, nc, 0, gs, kg)
    q = rng.standard_normal((B, Hq, S, D))
    kh = rng.standard_normal((B, Hkv, nc * c, D))
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, c))
    gsumm = oracle.summaries(kh, gs)
    gidx, _ = oracle.route_groups(sh, q, gsumm, idx)
    G = Hq // Hkv
    for b in range(B):
        for g in range(Hkv):
            for m in range(S // qb):
                qbar = q[b, g * G:(g + 1) * G, m * qb:(m + 1) * qb].mean(axis=(0, 1))
                cand = np.array([j * (c // gs) + u for j in idx[b, g, m] if j >= 0 for u in range(c // gs)])
                s = gsumm[b, g, cand] @ qbar / np.sqrt(D)
                best = cand[np.lexsort((cand, -s))[:kg]]
                assert list(gidx[b, g, m]) == sorted(best.tolist())


def test_route_groups_pads_when_the_budget_exceeds_the_candidates():
    rng = np.random.default_rng(63)
    D, c, gs, qb, S, nc = 8, 16, 8, 16, 16, 3
    sh = oracle.shape(1, 2, 1, D, c, qb, 2, S, nc, 0, gs, 6)  # 2 chunks x 2 groups < 6
    q = rng.standard_normal((1, 2, S, D))
    gsumm = rng.standard_normal((1, 1, nc * 2, D))
    idx = np.array([[[[0, 2]]]], dtype=np.int32)
    gidx, gap = oracle.route_groups(sh, q, gsumm, idx)
    assert list(gidx[0, 0, 0]) == [0, 1, 4, 5, -1, -1]
    assert np.isinf(gap[0, 0, 0])


def test_all_groups_of_the_chosen_chunks_equal_the_chunk_route():
    """topg = k c / gs keeps every group of every chosen chunk: the same tokens in the
    same order, so forward and backward equal the chunk-routed ones bit for bit."""
    sh = _shape(Hq=4, Hkv=2, D=16, c=16, qb=16, k=2, S=48, Nc=5)
    q, kh, vh, ks, vs = _random_layer(sh, seed=64)
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, 16))
    shg = oracle.shape(1, 4, 2, 16, 16, 16, 2, 48, 5, 0, 4, 8)
    gidx, gap = oracle.route_groups(shg, q, oracle.summaries(kh, 4), idx)
    assert np.all(np.isinf(gap))
    for b, g, m in np.ndindex(*idx.shape[:3]):
        assert list(gidx[b, g, m]) == [4 * j + u for j in idx[b, g, m] for u in range(4)]
    out, lse = oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx)
    outg, lseg = oracle.attn_fwd(shg, q, kh, vh, ks, vs, gidx)
    assert np.array_equal(out, outg) and np.array_equal(lse, lseg)
    dout = _rng(65).standard_normal(q.shape)
    grads = oracle.attn_bwd(sh, q, kh, vh, ks, vs, idx, dout)
    gradsg = oracle.attn_bwd(shg, q, kh, vh, ks, vs, gidx, dout)
    for a, bb in zip(grads, gradsg):
        assert np.array_equal(a, bb)


def test_group_routes_equal_masked_attention_and_autograd():
    """Attention over routed groups = torch attention (fp64) over an explicit mask of
    the groups' tokens and the causal segment; the backward = torch autograd of it."""
    sh = _shape(Hq=4, Hkv=2, D=16, c=16, qb=16, k=3, S=48, Nc=6)
    q, kh, vh, ks, vs = _random_layer(sh, seed=66)
    idx, _, _ = oracle.route(sh, q, oracle.summaries(kh, 16))
    shg = oracle.shape(1, 4, 2, 16, 16, 16, 3, 48, 6, 0, 4, 5)
    gidx, _ = oracle.route_groups(shg, q, oracle.summaries(kh, 4), idx)
    mask = _group_mask(shg, gidx)
    out, lse = oracle.attn_fwd(shg, q, kh, vh, ks, vs, gidx)
    o_ref, lse_ref = _sdpa(shg, q, kh, vh, ks, vs, mask)
    assert np.max(np.abs(out - o_ref)) < 1e-12
    assert np.max(np.abs(lse - lse_ref)) < 1e-12
    dout = _rng(67).standard_normal(q.shape)
    dq, dk, dv = oracle.attn_bwd(shg, q, kh, vh, ks, vs, gidx, dout)
    G = 2
    qt = torch.from_numpy(q).requires_grad_()
    kst = torch.from_numpy(ks).requires_grad_()
    vst = torch.from_numpy(vs).requires_grad_()
    k_all = torch.cat([torch.from_numpy(kh), kst], 2).repeat_interleave(G, 1)
    v_all = torch.cat([torch.from_numpy(vh), vst], 2).repeat_interleave(G, 1)
    m = torch.from_numpy(mask).repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, k_all, v_all, attn_mask=m)
    (o * torch.from_numpy(dout)).sum().backward()
    assert np.max(np.abs(dq - qt.grad.numpy())) < 1e-12
    assert np.max(np.abs(dk - kst.grad.numpy())) < 1e-12
    assert np.max(np.abs(dv - vst.grad.numpy())) < 1e-12


def test_group_attended_count():
    """q = 0 makes every logit 0, so LSE = ln(#attended keys) = ln(gs * #routed groups + i + 1)."""
    sh = oracle.shape(1, 2, 1, 8, 16, 8, 2, 24, 4, 0, 4, 3)
    rng = np.random.default_rng(68)
    q = np.zeros((1, 2, 24, 8))
    kh, vh = rng.standard_normal((1, 1, 64, 8)), rng.standard_normal((1, 1, 64, 8))
    ks, vs = rng.standard_normal((1, 1, 24, 8)), rng.standard_normal((1, 1, 24, 8))
    gidx = np.array([[[[0, 5, 9], [2, -1, -1], [-1, -1, -1]]]], dtype=np.int32)
    _, lse = oracle.attn_fwd(sh, q, kh, vh, ks, vs, gidx)
    for i in range(24):
        n_groups = (gidx[0, 0, i // 8] >= 0).sum()
        assert lse[0, 0, i] == pytest.approx(math.log(4 * n_groups + i + 1), rel=1e-14)


# ------------------------------------------------------------ strictly causal routing

def _causal_layer(seed, B=2, Hq=4, Hkv=2, D=8, c=8, qb=8, S=24, nc=9, k=3, sink=0):
    rng = np.random.default_rng(seed)
    sh = oracle.shape(B, Hq, Hkv, D, c, qb, k, S, nc, sink)
    q = rng.standard_normal((B, Hq, S, D))
    kh = rng.standard_normal((B, Hkv, nc * c, D))
    return sh, q, kh, oracle.summaries(kh, c)


def test_causal_route_matches_a_numpy_prefix_ranking():
    """Token i routes by the mean of its block's queries start .. i over the G heads
    (numpy prefix means, lexsort by score then index)."""
    sh, q, _, summ = _causal_layer(71)
    idx, _ = oracle.route_causal(sh, q, summ)
    G = sh.n_q_heads // sh.n_kv_heads
    for b, g, i in np.ndindex(sh.batch, sh.n_kv_heads, sh.seg_len):
        start = (i // sh.q_block) * sh.q_block
        qbar = q[b, g * G:(g + 1) * G, start:i + 1].mean(axis=(0, 1))
        s = summ[b, g] @ qbar / np.sqrt(sh.head_dim)
        want = sorted(np.lexsort((np.arange(sh.n_hist_chunks), -s))[:sh.topk].tolist())
        assert list(idx[b, g, i]) == want


def test_causal_route_of_a_block_end_is_the_block_route():
    """The last token of a block summarises the whole block, so it gets the block's
    route (also with a sink window)."""
    for sink in (0, 1):
        sh, q, _, summ = _causal_layer(72, sink=sink)
        idx_tok, gap_tok = oracle.route_causal(sh, q, summ)
        idx_blk, gap_blk, _ = oracle.route(sh, q, summ)
        for m in range(sh.seg_len // sh.q_block):
            i = m * sh.q_block + sh.q_block - 1
            assert np.array_equal(idx_tok[:, :, i], idx_blk[:, :, m])
            assert np.array_equal(gap_tok[:, :, i], gap_blk[:, :, m])


def test_causal_route_ignores_later_queries():
    """The point of the variant: changing queries after i leaves the routes of tokens
    0..i unchanged, while the block route of i's block changes with them."""
    sh, q, _, summ = _causal_layer(73)
    idx0, _ = oracle.route_causal(sh, q, summ)
    blk0, _, _ = oracle.route(sh, q, summ)
    q2 = q.copy()
    q2[:, :, 11:] = -5.0 * q2[:, :, 11:] + 3.0   # everything after token 10 (block 1 spans 8..15)
    idx1, _ = oracle.route_causal(sh, q2, summ)
    blk1, _, _ = oracle.route(sh, q2, summ)
    assert np.array_equal(idx0[:, :, :11], idx1[:, :, :11])
    assert not np.array_equal(idx0[:, :, 11:], idx1[:, :, 11:])
    assert not np.array_equal(blk0[:, :, 1], blk1[:, :, 1])  # the shared block route leaks


def test_causal_routes_with_one_token_blocks_equal_the_plain_route():
    sh, q, _, summ = _causal_layer(74, qb=1)
    idx_tok, _ = oracle.route_causal(sh, q, summ)
    idx_blk, _, _ = oracle.route(sh, q, summ)
    assert np.array_equal(idx_tok, idx_blk)


def test_attention_with_causal_routes_equals_masked_attention():
    """Per-token routes drive the attention through a one-token-block shape: exact
    attention over each token's own routed chunks and the causal segment (torch, fp64)."""
    sh, q, kh, summ = _causal_layer(75, B=1)
    idx_tok, _ = oracle.route_causal(sh, q, summ)
    rng = np.random.default_rng(76)
    vh = rng.standard_normal(kh.shape)
    ks = rng.standard_normal((1, sh.n_kv_heads, sh.seg_len, sh.head_dim))
    vs = rng.standard_normal((1, sh.n_kv_heads, sh.seg_len, sh.head_dim))
    sh1 = oracle.shape(1, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, sh.chunk, 1, sh.topk, sh.seg_len,
                       sh.n_hist_chunks)
    out, lse = oracle.attn_fwd(sh1, q, kh, vh, ks, vs, idx_tok)
    o_ref, lse_ref = _sdpa(sh1, q, kh, vh, ks, vs, _allowed_mask(sh1, idx_tok))
    assert np.max(np.abs(out - o_ref)) < 1e-12
    assert np.max(np.abs(lse - lse_ref)) < 1e-12
