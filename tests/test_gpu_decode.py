"""GPU parity of single-query decode (through the C ABI) against the fp64 oracle.

The decode token is the last of an n_local-token local window that follows T
detached history tokens.  The oracle computes it as the last row of a forward
over one-token query blocks (q_block = 1): its route uses the mean of its G
query heads, and it attends its routed chunks plus the whole local window.
Routes must be bit-exact except at oracle near-ties; outputs are compared with
the oracle's routes on both sides (and, where the routes agree, end to end).
"""
import numpy as np
import pytest
import torch

import oracle
from inputs import gen
from tests import hga_cases as hc

pytestmark = pytest.mark.gpu

# (workload recipe, n_local, sink_chunks); seg_len is the local window the inputs are drawn for
CASES = [
    (gen.custom("dec_tiny_fp32", dtype="fp32", head_dim=64, n_q_heads=2, n_kv_heads=1, topk=4, seg_len=37,
                seq_len=1024 + 37, seg_starts=(1024,), seed=61), 37, 0),
    (gen.custom("dec_mid_bf16", dtype="bf16", head_dim=128, n_q_heads=8, n_kv_heads=2, topk=8, seg_len=100,
                seq_len=40 * 64 + 100, seg_starts=(40 * 64,), batch=2, seed=62), 100, 0),
    (gen.custom("dec_self_only", dtype="bf16", head_dim=128, n_q_heads=4, n_kv_heads=1, topk=4, seg_len=1,
                seq_len=640 + 1, seg_starts=(640,), seed=63), 1, 0),
    (gen.custom("dec_k_above_nc", dtype="bf16", head_dim=128, n_q_heads=4, n_kv_heads=1, topk=8, seg_len=20,
                seq_len=192 + 20, seg_starts=(192,), seed=64), 20, 0),
    (gen.custom("dec_sink", dtype="bf16", head_dim=128, n_q_heads=8, n_kv_heads=2, topk=8, seg_len=100,
                seq_len=40 * 64 + 100, seg_starts=(40 * 64,), batch=2, seed=65), 100, 2),
    (gen.custom("dec_g8_fp32", dtype="fp32", head_dim=64, n_q_heads=16, n_kv_heads=2, topk=5, seg_len=70,
                seq_len=30 * 64 + 70, seg_starts=(30 * 64,), seed=66), 70, 0),
    (gen.custom("dec_128k", dtype="bf16", head_dim=128, n_q_heads=8, n_kv_heads=2, topk=32, seg_len=64,
                seq_len=131072, seg_starts=(131072 - 64,), seed=67), 64, 0),
    # bf16 D 64 with 8 heads per KV head; the window ends in a 2-token piece
    (gen.custom("dec_d64_g8_bf16", dtype="bf16", head_dim=64, n_q_heads=16, n_kv_heads=2, topk=6, seg_len=130,
                seq_len=50 * 64 + 130, seg_starts=(50 * 64,), batch=2, seed=69), 130, 0),
    # one query head per KV head
    (gen.custom("dec_g1_bf16", dtype="bf16", head_dim=128, n_q_heads=4, n_kv_heads=4, topk=5, seg_len=33,
                seq_len=20 * 64 + 33, seg_starts=(20 * 64,), seed=70), 33, 0),
    # 300 routable chunks (more than one pass of the route's tile ring) and a sink chunk
    (gen.custom("dec_split_fp32_sink", dtype="fp32", head_dim=64, n_q_heads=4, n_kv_heads=2, topk=6, seg_len=10,
                seq_len=300 * 64 + 10, seg_starts=(300 * 64,), seed=68), 10, 1),
]


@pytest.fixture(scope="module", autouse=True)
def _built():
    hc.ensure_built()
    assert torch.cuda.is_available()
    yield
    import hierarchical_sparse_long_b200 as hga
    assert hga.hga_get_device_status() == 0


def _decode_params(w, T, L, sink):
    import hierarchical_sparse_long_b200 as hga
    return hga.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                      topk=w.topk, seg_len=1, n_hist_chunks=T // w.chunk,
                      dtype=hga.HGA_BF16 if w.dtype == "bf16" else hga.HGA_FP32, hist_head_stride=T + L,
                      seg_head_stride=T + L, chunk=w.chunk, q_block=1, sink_chunks=sink)


@pytest.mark.parametrize("w,L,sink", CASES, ids=[c[0].name for c in CASES])
def test_decode_matches_oracle(w, L, sink):
    import hierarchical_sparse_long_b200 as hga
    T = w.seg_starts[0]
    nc = T // w.chunk
    B, Hq, Hkv, D = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim
    q_loc = gen.queries(w, T, T + L)
    end = -(-(T + L) // w.chunk) * w.chunk  # keys are drawn by whole chunks
    k_all = np.ascontiguousarray(gen.keys(w, 0, end)[:, :, :T + L])
    v_all = np.ascontiguousarray(gen.values(w, 0, end)[:, :, :T + L])

    # oracle: the last row of a forward over one-token query blocks
    sh = oracle.shape(B, Hq, Hkv, D, w.chunk, 1, w.topk, L, nc, sink)
    summ_o = oracle.summaries(k_all[:, :, :T], w.chunk) if nc else np.zeros((B, Hkv, 0, D))
    idx_o, gap, _ = oracle.route(sh, q_loc, summ_o)
    rows = np.array([(b * Hq + h) * L + L - 1 for b in range(B) for h in range(Hq)], dtype=np.int64)
    out_o, lse_o = oracle.attn_fwd(sh, q_loc, k_all[:, :, :T], v_all[:, :, :T], k_all[:, :, T:], v_all[:, :, T:],
                                   idx_o, rows=rows)

    # GPU: route of the token, then decode attention
    kd, vd = hc.to_dev(k_all, w), hc.to_dev(v_all, w)
    summ = torch.zeros(B, Hkv, max(nc, 1), D, device="cuda")
    hga.hga_build_summaries(kd, T + L, B, Hkv, D, w.chunk, 0, nc, summ, max(nc, 1))
    qd = hc.to_dev(q_loc[:, :, L - 1:L], w)
    p = _decode_params(w, T, L, sink)
    idx = torch.full((B, Hkv, 1, w.topk), -7, device="cuda", dtype=torch.int32)
    hga.hga_route(p, qd, summ, max(nc, 1), idx)
    torch.cuda.synchronize()
    idx_g = hc.f32(idx).astype(np.int32)
    hard, exempt = hc.route_mismatches(idx_g, idx_o[:, :, L - 1:L], gap[:, :, L - 1:L])
    assert hard == 0
    print(f"{w.name}: near-tie exemptions {exempt}")

    ws = torch.empty(hga.hga_attn_decode_workspace_size(p, L) // 4 + 1, device="cuda")
    kind = "fp32" if w.dtype == "fp32" else "bf16"
    for route in (torch.from_numpy(np.ascontiguousarray(idx_o[:, :, L - 1:L])).cuda(), idx if exempt == 0 else None):
        if route is None:
            continue
        out = torch.empty(B, Hq, 1, D, device="cuda", dtype=hc.torch_dtype(w))
        lse = torch.empty(B, Hq, 1, device="cuda")
        hga.hga_attn_decode(p, qd, kd, vd, kd[:, :, T:], vd[:, :, T:], L, route, out, lse, ws)
        torch.cuda.synchronize()
        hc.compare(hc.f32(out), out_o[:, :, L - 1:L], kind, f"{w.name} out")
        hc.compare(hc.f32(lse), lse_o[:, :, L - 1:L], "fp32" if w.dtype == "fp32" else "bf16", f"{w.name} lse")


def test_decode_rejects_multi_token_and_bad_windows():
    import hierarchical_sparse_long_b200 as hga
    w = CASES[1][0]
    T, L = w.seg_starts[0], 100
    p = _decode_params(w, T, L, 0)
    t = torch.empty(1 << 16, device="cuda")
    for bad in (dict(seg_len=64, q_block=64), dict(seg_head_stride=50)):
        pb = _decode_params(w, T, L, 0)
        for kk, vv in bad.items():
            setattr(pb, kk, vv)
        with pytest.raises(hga.HGAError):
            hga.hga_attn_decode(pb, t, t, t, t, t, L, t, t, t, t)
    with pytest.raises(hga.HGAError):
        hga.hga_attn_decode(p, t, t, t, t, t, 0, t, t, t, t)
    # one-token blocks are rejected by the multi-token forward
    with pytest.raises(hga.HGAError):
        hga.hga_attn_fwd(p, t, t, t, t, t, t, t, t)
