"""GPU parity of attention over group routes and over strictly causal (per-token)
routes, through the C ABI, against the fp64 oracle.

* Group stage ("Long-Context Fine-Tuning with Limited VRAM", technical summary
  section 2.1, group selection): hga_attn_fwd_groups / hga_attn_bwd_groups attend
  the exact K/V of the routed groups (8, 16 or 32 tokens) plus the causal segment;
  the oracle gathers the same groups (its shape's group / topg fields).
* Strictly causal routing (the limits section's proposed variant):
  hga_attn_fwd_causal / hga_attn_bwd_causal attend each token's own routed chunks
  plus the causal segment; the oracle computes that as attention with one-token
  query blocks over the per-token routes.

Both sides receive the oracle's routes.  Tolerances as everywhere: bf16 max-abs
2e-2 and mean-abs 2e-3.  Cases cover partly filled last tiles (repeated groups
masked), -1 padded group lists, G = 1, 2 and 4, a budget above the history, a
sink window, and full-size 16K layers on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from inputs import gen
from tests import hga_cases as hc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    hc.ensure_built()
    assert torch.cuda.is_available()
    yield
    import hierarchical_sparse_long_b200 as hga
    assert hga.hga_get_device_status() == 0


def _inputs(name, Hq, Hkv, k, S, T, seed, sink=0, backward=True):
    w = gen.custom(name, dtype="bf16", head_dim=128, n_q_heads=Hq, n_kv_heads=Hkv, topk=k, seg_len=S,
                   seq_len=T + S, seg_starts=(T,), seed=seed, sink_chunks=sink, backward=backward)
    return w, hc.segment_arrays(w, 0)


def _oracle_args(arrs):
    T = arrs["T"]
    return (arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T], arrs["k_all"][:, :, T:],
            arrs["v_all"][:, :, T:])


def _rows_of(w, rows):
    return None if rows is None else np.asarray(rows, dtype=np.int64)


def _check_out(w, out, lse, out_o, lse_o, rows, what):
    D = w.head_dim
    if rows is None:
        hc.compare(hc.f32(out), out_o, "bf16", f"{what} out")
        hc.compare(hc.f32(lse), lse_o, "bf16", f"{what} lse")
    else:
        hc.compare(hc.f32(out).reshape(-1, D)[rows], out_o.reshape(-1, D)[rows], "bf16", f"{what} out")
        hc.compare(hc.f32(lse).reshape(-1)[rows], lse_o.reshape(-1)[rows], "bf16", f"{what} lse")


# ---------------------------------------------------------------- group routes

GROUP_CASES = [
    # (name, Hq, Hkv, k, S, T, group, topg, seed, backward)
    ("grp8_partial_tile", 8, 2, 4, 128, 30 * 64, 8, 20, 101, True),     # 160 keys: 2.5 tiles
    ("grp16_padded", 8, 2, 12, 128, 5 * 64, 16, 24, 102, True),        # 20 of 24 groups valid
    ("grp32_g1", 2, 2, 3, 128, 20 * 64, 32, 3, 103, True),             # G = 1, 96 keys
    ("grp8_wide", 4, 1, 64, 64, 80 * 64, 8, 300, 104, False),           # 2,400 keys: 37.5 tiles
    ("grp8_g2", 4, 2, 6, 192, 50 * 64, 8, 13, 105, True),               # G = 2, 104 keys
]


def _group_routes(w, arrs, group, topg):
    T = arrs["T"]
    sh, _, idx_o, _ = hc.oracle_route(w, arrs)
    shg = oracle.shape(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 64, 64, w.topk, w.seg_len, T // 64,
                       w.sink_chunks, group, topg)
    gidx, _ = oracle.route_groups(shg, arrs["q"], oracle.summaries(arrs["k_all"][:, :, :T], group), idx_o)
    return shg, gidx


def _run_groups(w, arrs, group, topg, rows=None, backward=False):
    import hierarchical_sparse_long_b200 as hga
    shg, gidx_o = _group_routes(w, arrs, group, topg)
    g = hc.GpuSegment(w, arrs)
    gidx = torch.from_numpy(gidx_o).cuda()
    out = torch.full_like(g.q, float("nan"))
    lse = torch.full(g.q.shape[:3], float("nan"), device="cuda")
    hga.hga_attn_fwd_groups(g.p, g.q, g.k_all, g.v_all, g.k_seg, g.v_seg, gidx, group, topg, out, lse)
    torch.cuda.synchronize()
    out_o, lse_o = oracle.attn_fwd(shg, *_oracle_args(arrs), gidx_o, rows=rows)
    _check_out(w, out, lse, out_o, lse_o, rows, w.name)
    if backward:
        dq = torch.empty(g.q.shape, device="cuda")
        dk = torch.empty(w.batch, w.n_kv_heads, w.seg_len, w.head_dim, device="cuda")
        dv = torch.empty_like(dk)
        ws = torch.empty(hga.hga_attn_bwd_workspace_size(g.p) // 4 + 1, device="cuda")
        hga.hga_attn_bwd_groups(g.p, g.q, g.k_all, g.v_all, g.k_seg, g.v_seg, gidx, group, topg, out, lse, g.dout,
                                dq, dk, dv, ws)
        torch.cuda.synchronize()
        dq_o, dk_o, dv_o = oracle.attn_bwd(shg, *_oracle_args(arrs), gidx_o, arrs["dout"])
        hc.compare(hc.f32(dq), dq_o, "bf16", f"{w.name} dq")
        hc.compare(hc.f32(dk), dk_o, "bf16", f"{w.name} dk")
        hc.compare(hc.f32(dv), dv_o, "bf16", f"{w.name} dv")
    return gidx_o


@pytest.mark.parametrize("case", GROUP_CASES, ids=[c[0] for c in GROUP_CASES])
def test_group_attention_matches_oracle(case):
    name, Hq, Hkv, k, S, T, group, topg, seed, backward = case
    w, arrs = _inputs(name, Hq, Hkv, k, S, T, seed)
    _run_groups(w, arrs, group, topg, backward=backward)


def test_group_attention_count_invariant():
    # q = 0: every logit is 0, so lse_i = ln(valid groups * group + i + 1) exactly
    import hierarchical_sparse_long_b200 as hga
    w, arrs = _inputs("grp_count", 8, 2, 4, 128, 30 * 64, 106)
    arrs = dict(arrs)
    arrs["q"] = np.zeros_like(arrs["q"])
    for group, topg in ((8, 20), (16, 9), (32, 3)):
        _, gidx_o = _group_routes(w, arrs, group, topg)
        g = hc.GpuSegment(w, arrs)
        out = torch.empty_like(g.q)
        lse = torch.empty(g.q.shape[:3], device="cuda")
        hga.hga_attn_fwd_groups(g.p, g.q, g.k_all, g.v_all, g.k_seg, g.v_seg, torch.from_numpy(gidx_o).cuda(),
                                group, topg, out, lse)
        torch.cuda.synchronize()
        nvalid = (gidx_o >= 0).sum(-1)  # [B][Hkv][nqb]
        G = w.n_q_heads // w.n_kv_heads
        i = np.arange(w.seg_len)
        want = np.log(np.repeat(np.repeat(nvalid, 64, axis=2), G, axis=1) * group + i + 1.0)
        assert np.max(np.abs(hc.f32(lse) - want)) < 1e-5, (group, topg)


def test_group_attention_full_size_16k_sampled():
    w = gen.WORKLOADS["qwen3_16k_fwd"]
    arrs = hc.segment_arrays(w, 0)
    rows = np.unique(np.concatenate([
        np.random.default_rng(9).integers(0, w.n_q_heads * w.seg_len, 160),
        [0, 63, 64, w.seg_len - 1, (w.n_q_heads - 1) * w.seg_len + 5]]))
    _run_groups(w, arrs, 8, 64, rows=rows)


# ---------------------------------------------------------------- strictly causal routes

CAUSAL_CASES = [
    # (name, Hq, Hkv, k, S, T, sink, seed, backward)
    ("causal_attn_g4", 8, 2, 8, 192, 40 * 64, 0, 111, True),
    ("causal_attn_sink", 8, 2, 8, 128, 40 * 64, 2, 112, True),
    ("causal_attn_k_above_nc", 4, 1, 16, 128, 8 * 64, 0, 113, True),
    ("causal_attn_g1", 2, 2, 4, 128, 30 * 64, 0, 114, True),
    ("causal_attn_k32", 4, 1, 32, 64, 300 * 64, 0, 115, False),
]


def _causal_routes(w, arrs):
    T = arrs["T"]
    sh = hc.oracle_shape(w, T)
    idx_tok, gap = oracle.route_causal(sh, arrs["q"], oracle.summaries(arrs["k_all"][:, :, :T], 64)
                                       if T else np.zeros((w.batch, w.n_kv_heads, 0, w.head_dim)))
    sh1 = oracle.shape(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 64, 1, w.topk, w.seg_len, T // 64,
                       w.sink_chunks)
    return sh1, idx_tok


def _run_causal(w, arrs, rows=None, backward=False):
    import hierarchical_sparse_long_b200 as hga
    sh1, idx_o = _causal_routes(w, arrs)
    g = hc.GpuSegment(w, arrs)
    idx = torch.from_numpy(idx_o).cuda()
    out = torch.full_like(g.q, float("nan"))
    lse = torch.full(g.q.shape[:3], float("nan"), device="cuda")
    ws = torch.empty(hga.hga_attn_causal_workspace_size(g.p, backward) // 4 + 4, device="cuda")
    hga.hga_attn_fwd_causal(g.p, g.q, g.k_all, g.v_all, g.k_seg, g.v_seg, idx, out, lse, ws)
    torch.cuda.synchronize()
    out_o, lse_o = oracle.attn_fwd(sh1, *_oracle_args(arrs), idx_o, rows=rows)
    _check_out(w, out, lse, out_o, lse_o, rows, w.name)
    if backward:
        dq = torch.empty(g.q.shape, device="cuda")
        dk = torch.empty(w.batch, w.n_kv_heads, w.seg_len, w.head_dim, device="cuda")
        dv = torch.empty_like(dk)
        hga.hga_attn_bwd_causal(g.p, g.q, g.k_all, g.v_all, g.k_seg, g.v_seg, idx, out, lse, g.dout, dq, dk, dv, ws)
        torch.cuda.synchronize()
        dq_o, dk_o, dv_o = oracle.attn_bwd(sh1, *_oracle_args(arrs), idx_o, arrs["dout"])
        hc.compare(hc.f32(dq), dq_o, "bf16", f"{w.name} dq")
        hc.compare(hc.f32(dk), dk_o, "bf16", f"{w.name} dk")
        hc.compare(hc.f32(dv), dv_o, "bf16", f"{w.name} dv")


@pytest.mark.parametrize("case", CAUSAL_CASES, ids=[c[0] for c in CAUSAL_CASES])
def test_causal_attention_matches_oracle(case):
    name, Hq, Hkv, k, S, T, sink, seed, backward = case
    w, arrs = _inputs(name, Hq, Hkv, k, S, T, seed, sink=sink)
    _run_causal(w, arrs, backward=backward)


def test_causal_attention_gpu_routes_end_to_end():
    """hga_route_causal's own routes into hga_attn_fwd_causal: routes bit-exact with
    the oracle (except near-ties), then the attention on those routes."""
    import hierarchical_sparse_long_b200 as hga
    w, arrs = _inputs("causal_e2e", 8, 2, 8, 128, 40 * 64, 116, backward=False)
    g = hc.GpuSegment(w, arrs)
    summ = g.summaries()
    idx = torch.full((w.batch, w.n_kv_heads, w.seg_len, w.topk), -7, device="cuda", dtype=torch.int32)
    hga.hga_route_causal(g.p, g.q, summ, g.cap, idx)
    sh1, idx_o = _causal_routes(w, arrs)
    T = arrs["T"]
    _, gap = oracle.route_causal(hc.oracle_shape(w, T), arrs["q"], oracle.summaries(arrs["k_all"][:, :, :T], 64))
    torch.cuda.synchronize()
    hard, _ = hc.route_mismatches(hc.f32(idx).astype(np.int32), idx_o, gap)
    assert hard == 0
    out = torch.empty_like(g.q)
    lse = torch.empty(g.q.shape[:3], device="cuda")
    ws = torch.empty(hga.hga_attn_causal_workspace_size(g.p) // 4 + 4, device="cuda")
    hga.hga_attn_fwd_causal(g.p, g.q, g.k_all, g.v_all, g.k_seg, g.v_seg, idx, out, lse, ws)
    torch.cuda.synchronize()
    out_o, lse_o = oracle.attn_fwd(sh1, *_oracle_args(arrs), hc.f32(idx).astype(np.int32))
    _check_out(w, out, lse, out_o, lse_o, None, "causal e2e")


def test_causal_attention_with_block_routes_equals_block_attention():
    """Per-token routes that all equal their block's route make the token-masked
    kernel compute exactly what hga_attn_fwd computes: bit for bit."""
    import hierarchical_sparse_long_b200 as hga
    w, arrs = _inputs("causal_eq_block", 8, 2, 6, 192, 30 * 64, 117, backward=False)
    g = hc.GpuSegment(w, arrs)
    idx_b = g.route(g.summaries())
    out_b, lse_b = g.fwd(idx_b)
    idx_tok = idx_b.repeat_interleave(64, dim=2).contiguous()
    out = torch.empty_like(g.q)
    lse = torch.empty(g.q.shape[:3], device="cuda")
    ws = torch.empty(hga.hga_attn_causal_workspace_size(g.p) // 4 + 4, device="cuda")
    hga.hga_attn_fwd_causal(g.p, g.q, g.k_all, g.v_all, g.k_seg, g.v_seg, idx_tok, out, lse, ws)
    torch.cuda.synchronize()
    assert torch.equal(out, out_b) and torch.equal(lse, lse_b)


def test_causal_attention_full_size_16k_sampled():
    w = gen.WORKLOADS["qwen3_16k_fwd"]
    arrs = hc.segment_arrays(w, 0)
    rows = np.unique(np.concatenate([
        np.random.default_rng(10).integers(0, w.n_q_heads * w.seg_len, 160),
        [0, 1, 63, 64, w.seg_len - 1, (w.n_q_heads - 1) * w.seg_len + 9]]))
    _run_causal(w, arrs, rows=rows)
