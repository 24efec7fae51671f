"""GPU parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

Routes must be bit-exact except at oracle near-ties (relative gap of the k-th
and (k+1)-th scores below 1e-5), which are counted and printed.  Attention is
checked with the oracle's routes fed to both sides.  Tolerances: bf16 inputs
max-abs 2e-2 and mean-abs 2e-3, fp32 inputs max-abs 1e-4.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from inputs import gen
from tests import hga_cases as hc

pytestmark = pytest.mark.gpu

W = gen.WORKLOADS
# mid-size bf16 layer: several key tiles per block, ragged route lists (Nc=13)
MID = gen.custom("mid_bf16", n_q_heads=8, n_kv_heads=2, head_dim=128, topk=4, seg_len=256, seq_len=1088,
                 seg_starts=(832,), dtype="bf16", seed=7, backward=True)
EDGE = [
    gen.custom("no_history", topk=4, seg_len=192, seq_len=192, seg_starts=(0,), dtype="bf16", head_dim=128,
               n_q_heads=4, n_kv_heads=1, seed=11, backward=True),
    gen.custom("k_above_nc", topk=9, seg_len=128, seq_len=320, seg_starts=(192,), dtype="bf16", head_dim=128,
               n_q_heads=8, n_kv_heads=2, seed=12, backward=True),
    gen.custom("d64_mha_b2", batch=2, topk=3, seg_len=128, seq_len=768, seg_starts=(640,), dtype="bf16",
               head_dim=64, n_q_heads=2, n_kv_heads=2, seed=13, backward=True),
    gen.custom("fp32_g4", topk=2, seg_len=128, seq_len=512, seg_starts=(384,), dtype="fp32", head_dim=128,
               n_q_heads=8, n_kv_heads=2, seed=14, backward=True),
    gen.custom("one_block", topk=1, seg_len=64, seq_len=192, seg_starts=(128,), dtype="bf16", head_dim=128,
               n_q_heads=4, n_kv_heads=1, seed=15, backward=True),
    # tcgen05 head packing for other GQA groups: G = 1 (rows repeated, half written back),
    # G = 8 (two CTAs of 4 heads per KV group), G = 6 (three CTAs of 2 heads)
    gen.custom("g1_bf16", topk=3, seg_len=128, seq_len=640, seg_starts=(512,), dtype="bf16", head_dim=128,
               n_q_heads=2, n_kv_heads=2, seed=16, backward=True),
    gen.custom("g8_bf16", topk=4, seg_len=128, seq_len=640, seg_starts=(512,), dtype="bf16", head_dim=128,
               n_q_heads=8, n_kv_heads=1, seed=17, backward=True),
    gen.custom("g6_bf16", topk=2, seg_len=192, seq_len=576, seg_starts=(384,), dtype="bf16", head_dim=128,
               n_q_heads=12, n_kv_heads=2, seed=18, backward=True),
]


@pytest.fixture(scope="module", autouse=True)
def _built():
    hc.ensure_built()
    assert torch.cuda.is_available()
    yield
    import hierarchical_sparse_long_b200 as hga
    assert hga.hga_get_device_status() == 0


def _full_fwd_check(w, seg=0):
    arrs = hc.segment_arrays(w, seg)
    g = hc.GpuSegment(w, arrs)
    sh, summ_o, idx_o, gap = hc.oracle_route(w, arrs)
    T = arrs["T"]
    out_o, lse_o = oracle.attn_fwd(sh, arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T],
                                   arrs["k_all"][:, :, T:], arrs["v_all"][:, :, T:], idx_o)
    out, lse = g.fwd(torch.from_numpy(idx_o).cuda())
    torch.cuda.synchronize()
    hc.compare(hc.f32(out), out_o, w.dtype, f"{w.name} out")
    hc.compare(hc.f32(lse), lse_o, "fp32" if w.dtype == "fp32" else "bf16", f"{w.name} lse")
    return g, arrs, sh, idx_o


# ---------------------------------------------------------------- summaries

@pytest.mark.parametrize("name", ["tiny_fp32", "qwen3_16k_fwd"])
def test_summaries_match_oracle(name):
    w = W[name]
    arrs = hc.segment_arrays(w, 0)
    g = hc.GpuSegment(w, arrs)
    s = hc.f32(g.summaries())
    want = oracle.summaries(arrs["k_all"][:, :, :arrs["T"]], w.chunk)
    assert np.max(np.abs(s - want)) < 1e-5


def test_summaries_incremental_equals_full_rebuild():
    import hierarchical_sparse_long_b200 as hga
    w = W["qwen3_16k_fwd"]
    g = hc.GpuSegment(w, hc.segment_arrays(w, 0))
    L = g.T + w.seg_len
    nct = L // w.chunk
    full = torch.zeros(1, 8, nct, 128, device="cuda")
    inc = torch.full_like(full, float("nan"))
    hga.hga_build_summaries(g.k_all, L, 1, 8, 128, 64, 0, nct, full, nct)
    for first in range(0, nct, 32):  # one 2,048-token segment at a time
        hga.hga_build_summaries(g.k_all, L, 1, 8, 128, 64, first, min(32, nct - first), inc, nct)
    torch.cuda.synchronize()
    assert torch.equal(full, inc)


# ---------------------------------------------------------------- routing

@pytest.mark.parametrize("name,seg", [("tiny_fp32", 0), ("qwen3_16k_fwd", 0), ("qwen3_128k_eval", 31),
                                      ("qwen3_128k_eval", 1), ("qwen3_16k_fwd_sink", 0)])
def test_route_matches_oracle(name, seg):
    w = W[name]
    arrs = hc.segment_arrays(w, seg)
    g = hc.GpuSegment(w, arrs)
    idx = hc.f32(g.route(g.summaries())).astype(np.int32)
    _, _, idx_o, gap = hc.oracle_route(w, arrs)
    hard, exempt = hc.route_mismatches(idx, idx_o, gap)
    print(f"{name} seg {seg}: {idx.shape[2]} blocks x {idx.shape[1]} heads, near-tie exemptions {exempt}")
    assert hard == 0


def test_route_edge_cases():
    for w in EDGE:
        arrs = hc.segment_arrays(w, 0)
        g = hc.GpuSegment(w, arrs)
        idx = hc.f32(g.route(g.summaries())).astype(np.int32)
        _, _, idx_o, gap = hc.oracle_route(w, arrs)
        hard, _ = hc.route_mismatches(idx, idx_o, gap)
        assert hard == 0, w.name


# route shapes reaching every selection and cluster path: k > 32 (two keys per
# lane in the bound), and a chunk list split over clusters of 2, 4 and 8 query
# blocks (fp32 and D = 64 included)
ROUTE_SHAPES = [
    gen.custom("k48_n300", topk=48, seg_len=256, seq_len=300 * 64 + 256, seg_starts=(300 * 64,), dtype="bf16",
               head_dim=128, n_q_heads=8, n_kv_heads=2, seed=21),
    gen.custom("k64_n65", topk=64, seg_len=128, seq_len=65 * 64 + 128, seg_starts=(65 * 64,), dtype="bf16",
               head_dim=128, n_q_heads=4, n_kv_heads=1, seed=22),
    gen.custom("cl2_n1100", topk=32, seg_len=128, seq_len=1100 * 64 + 128, seg_starts=(1100 * 64,),
               dtype="bf16", head_dim=128, n_q_heads=8, n_kv_heads=2, seed=23),
    gen.custom("cl4_n600_d64", topk=16, seg_len=256, seq_len=600 * 64 + 256, seg_starts=(600 * 64,),
               dtype="bf16", head_dim=64, n_q_heads=4, n_kv_heads=2, seed=24),
    gen.custom("cl8_n1100_fp32", topk=24, seg_len=512, seq_len=1100 * 64 + 512, seg_starts=(1100 * 64,),
               dtype="fp32", head_dim=128, n_q_heads=4, n_kv_heads=1, seed=25),
    # attention-sink window: 1 chunk, 4 chunks under a cluster of 8, and every slot a sink chunk
    gen.custom("sink1_n300", topk=16, sink_chunks=1, seg_len=256, seq_len=300 * 64 + 256,
               seg_starts=(300 * 64,), dtype="bf16", head_dim=128, n_q_heads=8, n_kv_heads=2, seed=41),
    gen.custom("sink4_cl8_n1100", topk=24, sink_chunks=4, seg_len=512, seq_len=1100 * 64 + 512,
               seg_starts=(1100 * 64,), dtype="bf16", head_dim=128, n_q_heads=4, n_kv_heads=1, seed=42),
    gen.custom("sink_all_d64", topk=3, sink_chunks=3, seg_len=128, seq_len=40 * 64 + 128, seg_starts=(40 * 64,),
               dtype="fp32", head_dim=64, n_q_heads=2, n_kv_heads=2, seed=43),
]


def _route_only(w, q, summ):
    """Route of one segment from host queries and fp32 summaries (device call)."""
    import hierarchical_sparse_long_b200 as hga
    T = w.seg_starts[0]
    nc = T // w.chunk
    idx = torch.full((w.batch, w.n_kv_heads, w.seg_len // w.q_block, w.topk), -7, device="cuda",
                     dtype=torch.int32)
    hga.hga_route(hc.params(w, T), hc.to_dev(q, w), summ, nc, idx)
    torch.cuda.synchronize()
    return hc.f32(idx).astype(np.int32)


@pytest.mark.parametrize("w", ROUTE_SHAPES, ids=[w.name for w in ROUTE_SHAPES])
def test_route_selection_and_cluster_paths(w):
    import hierarchical_sparse_long_b200 as hga
    T, S = w.seg_starts[0], w.seg_len
    q = gen.queries(w, T, T + S)
    k = gen.keys(w, 0, T)
    nc = T // w.chunk
    summ = torch.zeros(w.batch, w.n_kv_heads, nc, w.head_dim, device="cuda")
    hga.hga_build_summaries(hc.to_dev(k, w), T, w.batch, w.n_kv_heads, w.head_dim, w.chunk, 0, nc, summ, nc)
    idx = _route_only(w, q, summ)
    _, _, idx_o, gap = hc.oracle_route(w, dict(T=T, q=q, k_all=k))
    hard, exempt = hc.route_mismatches(idx, idx_o, gap)
    print(f"{w.name}: near-tie exemptions {exempt}")
    assert hard == 0


def test_route_banded_and_equal_scores():
    """Scores banded by chunk index mod 256 leave hundreds of chunks at or
    above the selection's per-thread-maximum bound (several candidates per
    thread); all-equal summaries tie every chunk at the bound, so the
    selection falls back to the whole-row radix select and must route the
    lowest chunk indices."""
    n = 4096
    w = gen.custom("banded", topk=32, seg_len=128, seq_len=n * 64 + 128, seg_starts=(n * 64,),
                   dtype="bf16", head_dim=128, n_q_heads=4, n_kv_heads=1)
    q = np.zeros((1, 4, 128, 128), np.float32)
    q[..., 0] = 1.0  # block summary = e_0, so score_j = summ[j][0] / sqrt(D)
    rng = np.random.default_rng(5)
    summ = np.zeros((1, 1, n, 128), np.float32)
    summ[..., 0] = (np.arange(n) % 256) + rng.permutation(n) / n * 0.5  # distinct, banded
    idx = _route_only(w, q, torch.from_numpy(summ).cuda())
    idx_o, gap, _ = oracle.route(hc.oracle_shape(w, n * 64), q, summ)
    assert np.array_equal(idx, idx_o)
    assert np.all(np.sort(summ[0, 0, idx[0, 0, 0], 0]) == np.sort(summ[0, 0, :, 0])[-32:])

    same = np.broadcast_to(rng.standard_normal(128).astype(np.float32), (1, 1, n, 128)).copy()
    idx = _route_only(w, q, torch.from_numpy(same).cuda())
    assert np.array_equal(idx, np.broadcast_to(np.arange(32, dtype=np.int32), idx.shape))


# ---------------------------------------------------------------- forward

def test_fwd_tiny_fp32_full():
    _full_fwd_check(W["tiny_fp32"])


def test_fwd_mid_bf16_full():
    _full_fwd_check(MID)


@pytest.mark.parametrize("w", EDGE, ids=[w.name for w in EDGE])
def test_fwd_edge_cases(w):
    _full_fwd_check(w)


def _sampled_rows(w, n, seed):
    r = np.random.default_rng(seed)
    S = w.seg_len
    rows = set()
    # first and last rows of blocks, plus random rows, over random heads
    for _ in range(n):
        b = int(r.integers(0, w.batch))
        h = int(r.integers(0, w.n_q_heads))
        i = int(r.integers(0, S))
        rows.add((b * w.n_q_heads + h) * S + i)
    for h in (0, w.n_q_heads - 1):
        for i in (0, 63, 64, S - 1):
            rows.add(h * S + i)
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name,seg,n", [("qwen3_16k_fwd", 0, 384), ("qwen3_128k_eval", 31, 160)])
def test_fwd_full_size_sampled(name, seg, n):
    w = W[name]
    arrs = hc.segment_arrays(w, seg)
    g = hc.GpuSegment(w, arrs)
    sh, _, idx_o, _ = hc.oracle_route(w, arrs)
    T = arrs["T"]
    rows = _sampled_rows(w, n, seed=seg)
    out_o, lse_o = oracle.attn_fwd(sh, arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T],
                                   arrs["k_all"][:, :, T:], arrs["v_all"][:, :, T:], idx_o, rows=rows)
    out, lse = g.fwd(torch.from_numpy(idx_o).cuda())
    D = w.head_dim
    hc.compare(hc.f32(out).reshape(-1, D)[rows], out_o.reshape(-1, D)[rows], "bf16", f"{name} out")
    hc.compare(hc.f32(lse).reshape(-1)[rows], lse_o.reshape(-1)[rows], "bf16", f"{name} lse")


def test_fwd_attended_count_on_gpu():
    # q = 0: every logit is 0 and lse_i = ln(min(k, Nc)*64 + i + 1) exactly
    for w in (MID, EDGE[0], EDGE[1]):
        arrs = dict(hc.segment_arrays(w, 0))
        arrs["q"] = np.zeros_like(arrs["q"])
        g = hc.GpuSegment(w, arrs)
        idx = g.route(g.summaries())
        _, lse = g.fwd(idx)
        keff = min(w.topk, arrs["T"] // 64)
        want = np.log(keff * 64 + np.arange(w.seg_len) + 1.0)
        got = hc.f32(lse)
        assert np.max(np.abs(got - want[None, None, :])) < 1e-5, w.name


def test_fwd_bad_route_index_is_flagged_and_skipped():
    import hierarchical_sparse_long_b200 as hga
    w = MID
    arrs = hc.segment_arrays(w, 0)
    g = hc.GpuSegment(w, arrs)
    sh, _, idx_o, _ = hc.oracle_route(w, arrs)
    bad = idx_o.copy()
    bad[0, 1, 2, 0] = 10_000
    bad[0, 0, 3, 1] = -7
    hga.hga_get_device_status()  # clear
    out, lse = g.fwd(torch.from_numpy(bad).cuda())
    bits = hga.hga_get_device_status()
    assert bits & hga.HGA_DEV_BAD_INDEX
    skipped = bad.copy()
    skipped[(skipped < -1) | (skipped >= sh.n_hist_chunks)] = -1
    T = arrs["T"]
    out_o, _ = oracle.attn_fwd(sh, arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T],
                               arrs["k_all"][:, :, T:], arrs["v_all"][:, :, T:], skipped)
    hc.compare(hc.f32(out), out_o, "bf16", "skipped index")


def test_fwd_summaries_are_not_values():
    # the attention output depends on the routes only, never on summary values
    w = MID
    arrs = hc.segment_arrays(w, 0)
    g = hc.GpuSegment(w, arrs)
    summ = g.summaries()
    idx = g.route(summ)
    out1, _ = g.fwd(idx)
    idx2 = g.route(summ * 3.0)  # positive rescale keeps every ordering
    out2, _ = g.fwd(idx2)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(out1, out2)


# ---------------------------------------------------------------- backward

def _full_bwd_check(w):
    arrs = hc.segment_arrays(w, 0)
    g = hc.GpuSegment(w, arrs)
    sh, _, idx_o, _ = hc.oracle_route(w, arrs)
    T = arrs["T"]
    args = (sh, arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T], arrs["k_all"][:, :, T:],
            arrs["v_all"][:, :, T:], idx_o)
    dq_o, dk_o, dv_o = oracle.attn_bwd(*args, arrs["dout"])
    idx = torch.from_numpy(idx_o).cuda()
    out, lse = g.fwd(idx)
    dq, dk, dv = g.bwd(idx, out, lse)
    torch.cuda.synchronize()
    hc.compare(hc.f32(dq), dq_o, w.dtype, f"{w.name} dq")
    hc.compare(hc.f32(dk), dk_o, w.dtype, f"{w.name} dk")
    hc.compare(hc.f32(dv), dv_o, w.dtype, f"{w.name} dv")


def test_bwd_tiny_fp32_full():
    w = gen.custom("tiny_fp32_bwd", backward=True)
    _full_bwd_check(w)


def test_bwd_mid_bf16_full():
    _full_bwd_check(MID)


@pytest.mark.parametrize("w", EDGE, ids=[w.name for w in EDGE])
def test_bwd_edge_cases(w):
    _full_bwd_check(w)


def test_bwd_full_size_sampled():
    # the 16K training layer's last segment (T = 14,336): sampled dq rows of early,
    # middle and late query blocks, and dk/dv rows of the first 128 active keys of KV
    # head 0 (the dK/dV block every later query tile of the 4 heads reaches: 32 tiles x
    # 4 heads = 128 accumulation steps) and of its last 64 keys
    w = W["qwen3_16k_train"]
    seg = 7
    arrs = hc.segment_arrays(w, seg)
    g = hc.GpuSegment(w, arrs)
    sh, _, idx_o, _ = hc.oracle_route(w, arrs)
    T, S, D = arrs["T"], w.seg_len, w.head_dim
    q_need = np.zeros((1, w.n_q_heads, S), dtype=np.uint8)
    r = np.random.default_rng(3)
    for _ in range(64):
        q_need[0, r.integers(0, w.n_q_heads), r.integers(S - 256, S)] = 1
    for m in (0, 1, 15):  # early blocks: every row of two heads of different groups
        q_need[0, [1, 30], m * 64:(m + 1) * 64] = 1
    key_need = np.zeros((1, w.n_kv_heads, S), dtype=np.uint8)
    key_need[0, 0, :128] = 1
    key_need[0, 0, S - 64:] = 1
    key_need[0, 5, [S - 1, S - 30]] = 1
    dq_o, dk_o, dv_o = oracle.attn_bwd(sh, arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T],
                                       arrs["k_all"][:, :, T:], arrs["v_all"][:, :, T:], idx_o, arrs["dout"],
                                       q_need=q_need, key_need=key_need)
    idx = torch.from_numpy(idx_o).cuda()
    out, lse = g.fwd(idx)
    dq, dk, dv = g.bwd(idx, out, lse)
    qm, km = q_need.astype(bool), key_need.astype(bool)
    hc.compare(hc.f32(dq)[qm], dq_o[qm], "bf16", "dq sampled")
    hc.compare(hc.f32(dk)[km], dk_o[km], "bf16", "dk sampled")
    hc.compare(hc.f32(dv)[km], dv_o[km], "bf16", "dv sampled")


# ---------------------------------------------------------------- segment-wise training (8 segments)

def test_train_segments_route_and_summary_append():
    """8 consecutive 2,048-token segments: summaries appended as each segment
    detaches must equal a rebuild, and every segment's routes match the oracle."""
    import hierarchical_sparse_long_b200 as hga
    w = W["qwen3_16k_train"]
    L = w.seq_len
    k_all = hc.to_dev(gen.keys(w, 0, L), w)
    q_all = hc.to_dev(gen.queries(w, 0, L), w)
    nct = L // 64
    summ = torch.zeros(1, 8, nct, 128, device="cuda")
    total_exempt = 0
    for s, T in enumerate(w.seg_starts):
        p = hc.params(w, T, hist_head_stride=L, seg_head_stride=L)
        q = q_all[:, :, T:T + w.seg_len].contiguous()
        idx = torch.empty(1, 8, w.seg_len // 64, w.topk, device="cuda", dtype=torch.int32)
        hga.hga_route(p, q, summ, nct, idx)
        arrs = dict(T=T, q=hc.f32(q), k_all=hc.f32(k_all[:, :, :T + w.seg_len]))
        _, _, idx_o, gap = hc.oracle_route(w, arrs)
        hard, exempt = hc.route_mismatches(hc.f32(idx).astype(np.int32), idx_o, gap)
        total_exempt += exempt
        assert hard == 0, f"segment {s}"
        # detach: append this segment's 32 chunks
        hga.hga_build_summaries(k_all, L, 1, 8, 128, 64, T // 64, w.seg_len // 64, summ, nct)
    full = torch.zeros_like(summ)
    hga.hga_build_summaries(k_all, L, 1, 8, 128, 64, 0, nct, full, nct)
    torch.cuda.synchronize()
    assert torch.equal(full, summ)
    print(f"near-tie exemptions over 8 segments: {total_exempt}")


# ---------------------------------------------------------------- tiered history

def _tiered_run(w, seg, wave, slots, reps=1):
    """The segment's forward with the history only in pinned host memory, through
    hga_attn_fwd_tiered: the overlapped schedule the benchmark runs (fetch waves on a
    copy stream, attention of the previous wave on the compute stream, the staging
    cache kept across waves, no host synchronisation between waves).  Returns the
    resident forward, the tiered forward of every repetition (the cache is reset before
    the first only), the fetched tiles per repetition, and the tiles routed."""
    import hierarchical_sparse_long_b200 as hga
    arrs = hc.segment_arrays(w, seg)
    g = hc.GpuSegment(w, arrs)
    T, S = arrs["T"], w.seg_len
    idx = g.route(g.summaries())
    out_res, lse_res = g.fwd(idx)
    # history only in pinned host memory
    host_k = g.k_all[:, :, :T].contiguous().cpu().pin_memory()
    host_v = g.v_all[:, :, :T].contiguous().cpu().pin_memory()
    nqb = S // 64
    n_waves = -(-nqb // wave)
    stage_k = torch.empty(slots, 64, w.head_dim, device="cuda", dtype=g.q.dtype)
    stage_v = torch.empty_like(stage_k)
    p = hc.params(w, T, hist_head_stride=T, seg_head_stride=T + S)
    scratch = torch.empty(hga.hga_tier_scratch_size(p, slots) // 4, device="cuda", dtype=torch.int32)
    idx_r = torch.full_like(idx, -5)
    sched = hga.TierSched(lag=2)
    copy = torch.cuda.Stream()
    results, fetched = [], []
    for r in range(reps):
        nf = torch.zeros(n_waves, device="cuda", dtype=torch.int32)
        out = torch.full_like(out_res, float("nan"))
        lse = torch.full_like(lse_res, float("nan"))
        hga.hga_attn_fwd_tiered(p, g.q, host_k, host_v, g.k_seg, g.v_seg, idx, out, lse, stage_k, stage_v, slots,
                                scratch, idx_r, wave, sched, reset_cache=(r == 0), n_fetched=nf, copy_stream=copy)
        results.append((out, lse))
        fetched.append(nf)
    torch.cuda.synchronize()
    i = hc.f32(idx).astype(np.int64)
    routed = {(b, gg, j) for b in range(w.batch) for gg in range(w.n_kv_heads) for j in i[b, gg].ravel() if j >= 0}
    return arrs, idx, (out_res, lse_res), results, [int(f.sum().item()) for f in fetched], len(routed)


def _check_tiered(w, seg, wave, slots, sample_rows=None):
    import hierarchical_sparse_long_b200 as hga
    arrs, idx, (out_res, lse_res), results, fetched, distinct = _tiered_run(w, seg, wave, slots, reps=2)
    for out, lse in results:
        assert torch.equal(out, out_res) and torch.equal(lse, lse_res)
    assert hga.hga_get_device_status() == 0
    # against the oracle as well (the routes the GPU chose, attention in fp64)
    T = arrs["T"]
    sh = hc.oracle_shape(w, T)
    rows = sample_rows
    out_o, lse_o = oracle.attn_fwd(sh, arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T],
                                   arrs["k_all"][:, :, T:], arrs["v_all"][:, :, T:], hc.f32(idx).astype(np.int32),
                                   rows=rows)
    D = w.head_dim
    out, lse = results[0]
    if rows is None:
        hc.compare(hc.f32(out), out_o, w.dtype, "tiered out")
        hc.compare(hc.f32(lse), lse_o, w.dtype, "tiered lse")
    else:
        hc.compare(hc.f32(out).reshape(-1, D)[rows], out_o.reshape(-1, D)[rows], w.dtype, "tiered out")
        hc.compare(hc.f32(lse).reshape(-1)[rows], lse_o.reshape(-1)[rows], w.dtype, "tiered lse")
    return fetched, distinct


def test_tiered_small_cache_evicts_and_matches():
    # 13 history chunks x 2 kv heads; waves of 1 block route 2 x 4 tiles, so 16 slots
    # (twice a wave) force evictions of tiles routed two waves back
    fetched, distinct = _check_tiered(MID, 0, wave=1, slots=16)
    assert fetched[0] >= distinct
    print(f"small cache: fetched {fetched}, distinct {distinct}")


def test_tiered_cache_fetches_each_tile_once():
    # a cache that holds every routable tile: each routed tile crosses the host link
    # once per reset, and a second pass over the same routes fetches nothing
    fetched, distinct = _check_tiered(MID, 0, wave=2, slots=2 * 13)
    assert fetched == [distinct, 0]


def test_tiered_128k_last_segment():
    w = W["qwen3_128k_tiered"]
    nc = w.seg_starts[31] // 64
    slots = w.batch * w.n_kv_heads * nc
    fetched, distinct = _check_tiered(w, 31, wave=8, slots=slots, sample_rows=_sampled_rows(w, 96, seed=5))
    assert fetched == [distinct, 0]
    print(f"tiles fetched for the last 4,096-token segment: {fetched[0]} (distinct routed tiles {distinct})")


# six consecutive 256-token segments of one sequence, for the chained tiered schedule
CHAIN = gen.custom("chain_bf16", n_q_heads=8, n_kv_heads=2, head_dim=128, topk=4, seg_len=256, seq_len=6 * 256,
                   seg_starts=tuple(range(0, 6 * 256, 256)), dtype="bf16", seed=23)


@pytest.mark.parametrize("wave,lag,slots,prev", [(4, 2, 40, False), (1, 4, 32, False), (1, 3, 24, False),
                                                 (2, 2, 32, False), (1, 2, 16, False), (4, 2, 40, True),
                                                 (1, 2, 16, True), (2, 3, 48, True)],
                         ids=["segment_waves_lag2", "block_waves_lag4", "block_waves_lag3", "two_block_waves_lag2",
                              "block_waves_lag2", "segment_waves_lag2_prev", "block_waves_lag2_prev",
                              "two_block_waves_lag3_prev"])
def test_tiered_chained_segments_match_resident(wave, lag, slots, prev):
    _chained_tiered(CHAIN, wave, lag, slots, prev)


# other tile layouts of the staging copy: 128-byte rows (bf16, D = 64; two batches,
# G = 1, the SIMT attention) and 512-byte rows (fp32, D = 128)
CHAIN_LAYOUTS = [
    gen.custom("chain_bf16_d64_b2", batch=2, n_q_heads=2, n_kv_heads=2, head_dim=64, topk=3, seg_len=128,
               seq_len=6 * 128, seg_starts=tuple(range(0, 6 * 128, 128)), dtype="bf16", seed=24),
    gen.custom("chain_fp32_d128", n_q_heads=4, n_kv_heads=2, head_dim=128, topk=3, seg_len=128, seq_len=6 * 128,
               seg_starts=tuple(range(0, 6 * 128, 128)), dtype="fp32", seed=25),
]


@pytest.mark.parametrize("w", CHAIN_LAYOUTS, ids=[w.name for w in CHAIN_LAYOUTS])
@pytest.mark.parametrize("prev", [False, True], ids=["host_only", "prev"])
def test_tiered_chained_other_layouts(w, prev):
    """The chained tiered evaluation with 128- and 512-byte rows, two batches and
    G = 1: bitwise equal to the resident forward, with a cache that evicts."""
    n_bg = w.batch * w.n_kv_heads
    _chained_tiered(w, 1, 2, 2 * n_bg * w.topk, prev)


def _chained_tiered(w, wave, lag, slots, prev):
    """An evaluation of six segments with the history only in pinned host memory,
    through hga_segment_fwd_tiered as the benchmark runs it: each segment's K/V
    offloaded to the host history on one stream, its route and summary append on a
    second, its fetch waves on a third (all three at high priority), its attention
    waves on the compute stream, chained from segment to segment (no host
    synchronisation anywhere), so a segment's route and fetches run under the
    attention of the segments before it.  The host history starts as NaN, so a
    fetch that overtook an offload, or an eviction of a slot still being read, changes
    the output.  Every segment's out and lse equal the resident forward on the same
    routes bit for bit.  Slots: the least the schedule accepts, min(lag x wave x B x
    Hkv x k, B x Hkv x Nc); on the 256-token segments all but the segment-wave cases
    hold fewer than the last segment's 40 routable tiles, so the cache evicts (the
    other layouts' caches evict too).  With prev, each segment's
    fetches copy the previous segment's chunks from its K/V in device memory (and
    wait only for the offload of the segment before that): the outputs are the same
    and fewer tiles cross the host link."""
    import hierarchical_sparse_long_b200 as hga
    L, S, D = w.seq_len, w.seg_len, w.head_dim
    nqb = S // 64
    k_all = hc.to_dev(gen.keys(w, 0, L), w)
    v_all = hc.to_dev(gen.values(w, 0, L), w)
    qs = {T: hc.to_dev(gen.queries(w, T, T + S), w) for T in w.seg_starts}
    nct = L // 64
    # resident reference: routes and forward per segment, history in device memory
    full = torch.zeros(w.batch, w.n_kv_heads, nct, D, device="cuda")
    hga.hga_build_summaries(k_all, L, w.batch, w.n_kv_heads, D, 64, 0, nct, full, nct)
    ref = {}
    for T in w.seg_starts:
        p = hc.params(w, T, hist_head_stride=L, seg_head_stride=L)
        idx = torch.empty(w.batch, w.n_kv_heads, nqb, w.topk, device="cuda", dtype=torch.int32)
        hga.hga_route(p, qs[T], full, nct, idx)
        out = torch.empty_like(qs[T])
        lse = torch.empty(qs[T].shape[:3], device="cuda")
        hga.hga_attn_fwd(p, qs[T], k_all, v_all, k_all[:, :, T:], v_all[:, :, T:], idx, out, lse)
        ref[T] = (out, lse, idx)
    torch.cuda.synchronize()
    # the chained tiered evaluation
    host_k = torch.full((w.batch, w.n_kv_heads, L, D), float("nan"), dtype=k_all.dtype).pin_memory()
    host_v = torch.full_like(host_k, float("nan")).pin_memory()
    summ = torch.zeros_like(full)
    stage_k = torch.empty(slots, 64, D, device="cuda", dtype=k_all.dtype)
    stage_v = torch.empty_like(stage_k)
    p_last = hc.params(w, w.seg_starts[-1], hist_head_stride=L, seg_head_stride=L)
    scratch = torch.empty(hga.hga_tier_scratch_size(p_last, slots) // 4, device="cuda", dtype=torch.int32)
    n_waves = -(-nqb // wave)
    idx_r = [torch.full((w.batch, w.n_kv_heads, nqb, w.topk), -5, device="cuda", dtype=torch.int32)
             for _ in range(-(-lag // n_waves))]
    # stale routes: read before the route that rewrites them, they would be flagged
    idx = [torch.full_like(idx_r[0], 7) for _ in range(2)]
    sched = hga.TierSched(lag=lag)
    compute = torch.cuda.current_stream()
    copy, route_s, off = (torch.cuda.Stream(priority=-1) for _ in range(3))
    nf = torch.zeros(len(w.seg_starts), n_waves, device="cuda", dtype=torch.int32)
    got = {}
    for si, T in enumerate(w.seg_starts):
        p = hc.params(w, T, hist_head_stride=L, seg_head_stride=L)
        out = torch.full_like(qs[T], float("nan"))
        lse = torch.full(qs[T].shape[:3], float("nan"), device="cuda")
        use_prev = prev and si > 0
        hga.hga_segment_fwd_tiered(p, qs[T], k_all[:, :, T:], v_all[:, :, T:], summ, nct, idx[si % 2], host_k,
                                   host_v, out, lse, stage_k, stage_v, slots, scratch, idx_r[si % len(idx_r)], wave,
                                   sched, reset=si == 0, n_fetched=nf[si], copy_stream=copy, route_stream=route_s,
                                   offload_stream=off, prev_k_seg=k_all[:, :, T - S:] if use_prev else None,
                                   prev_v_seg=v_all[:, :, T - S:] if use_prev else None)
        got[T] = (out, lse)
    for st in (copy, route_s, off):
        compute.wait_stream(st)
    torch.cuda.synchronize()
    assert hga.hga_get_device_status() == 0
    for T in w.seg_starts:
        assert torch.equal(got[T][0], ref[T][0]), f"segment at {T}: out"
        assert torch.equal(got[T][1], ref[T][1]), f"segment at {T}: lse"
    assert sched.segment == len(w.seg_starts)
    # the host history holds every segment's K/V
    assert torch.equal(host_k, k_all.cpu()) and torch.equal(host_v, v_all.cpu())
    assert torch.equal(summ, full)
    assert sched.wave == n_waves * (len(w.seg_starts) - 1)  # the first segment has no history: no wave
    fetched = int(nf.sum().item())
    union = {(b, g, int(j)) for T in w.seg_starts for b in range(w.batch) for g in range(w.n_kv_heads)
             for j in ref[T][2][b, g].flatten().tolist() if j >= 0}
    print(f"wave {wave}, lag {lag}, {slots} slots, prev {prev}: fetched from the host {fetched} tiles over "
          f"{len(w.seg_starts)} segments, {len(union)} distinct")
    if not prev:
        assert fetched >= len(union)
        if len(union) > slots:
            assert fetched > slots  # the cache evicted
    elif slots >= w.batch * w.n_kv_heads * ((w.seq_len - S) // 64):
        # a cache that never evicts: a segment's chunks are first routable by the next
        # segment, whose fetches take them from device memory, so only the chunks first
        # routed later than that cross the host link
        assert fetched < len(union)


def test_segment_fwd_pipelined_matches_resident():
    """The same six-segment evaluation with the history resident, through
    hga_segment_fwd on two streams (each segment's route and summary append on a
    high-priority route stream, running under the previous segment's attention, two
    rotating route tables, no host synchronisation): every segment's out and lse equal
    hga_route + hga_attn_fwd on the full summaries bit for bit, and the appended
    summaries equal a rebuild."""
    import hierarchical_sparse_long_b200 as hga
    w = CHAIN
    L, S, D = w.seq_len, w.seg_len, w.head_dim
    nqb = S // 64
    k_all = hc.to_dev(gen.keys(w, 0, L), w)
    v_all = hc.to_dev(gen.values(w, 0, L), w)
    qs = {T: hc.to_dev(gen.queries(w, T, T + S), w) for T in w.seg_starts}
    nct = L // 64
    full = torch.zeros(w.batch, w.n_kv_heads, nct, D, device="cuda")
    hga.hga_build_summaries(k_all, L, w.batch, w.n_kv_heads, D, 64, 0, nct, full, nct)
    ref = {}
    for T in w.seg_starts:
        p = hc.params(w, T, hist_head_stride=L, seg_head_stride=L)
        idx = torch.empty(w.batch, w.n_kv_heads, nqb, w.topk, device="cuda", dtype=torch.int32)
        hga.hga_route(p, qs[T], full, nct, idx)
        out = torch.empty_like(qs[T])
        lse = torch.empty(qs[T].shape[:3], device="cuda")
        hga.hga_attn_fwd(p, qs[T], k_all, v_all, k_all[:, :, T:], v_all[:, :, T:], idx, out, lse)
        ref[T] = (out, lse)
    torch.cuda.synchronize()
    summ = torch.zeros_like(full)
    idx = [torch.full((w.batch, w.n_kv_heads, nqb, w.topk), 7, device="cuda", dtype=torch.int32) for _ in range(2)]
    sched = hga.TierSched(lag=2)
    compute, route_s = torch.cuda.current_stream(), torch.cuda.Stream(priority=-1)
    got = {}
    for rep in range(2):  # a second evaluation restarts the schedule over the same buffers
        summ.zero_()
        for si, T in enumerate(w.seg_starts):
            p = hc.params(w, T, hist_head_stride=L, seg_head_stride=L)
            out = torch.full_like(qs[T], float("nan"))
            lse = torch.full(qs[T].shape[:3], float("nan"), device="cuda")
            hga.hga_segment_fwd(p, qs[T], k_all, v_all, k_all[:, :, T:], v_all[:, :, T:], summ, nct, idx[si % 2],
                                out, lse, sched, reset=si == 0, route_stream=route_s)
            got[(rep, T)] = (out, lse)
        compute.wait_stream(route_s)
    torch.cuda.synchronize()
    assert hga.hga_get_device_status() == 0
    for (rep, T), (out, lse) in got.items():
        assert torch.equal(out, ref[T][0]), f"evaluation {rep}, segment at {T}: out"
        assert torch.equal(lse, ref[T][1]), f"evaluation {rep}, segment at {T}: lse"
    assert torch.equal(summ, full)
    assert sched.segment == len(w.seg_starts)


def test_tiered_rejects_pageable_host_memory_before_any_launch():
    import hierarchical_sparse_long_b200 as hga
    w = MID
    arrs = hc.segment_arrays(w, 0)
    g = hc.GpuSegment(w, arrs)
    T = arrs["T"]
    idx = g.route(g.summaries())
    host_k = g.k_all[:, :, :T].contiguous().cpu()  # pageable: not page-locked
    host_v = g.v_all[:, :, :T].contiguous().cpu().pin_memory()
    slots = 64
    p = hc.params(w, T, hist_head_stride=T, seg_head_stride=T + w.seg_len)
    stage_k = torch.zeros(slots, 64, w.head_dim, device="cuda", dtype=g.q.dtype)
    stage_v = torch.zeros_like(stage_k)
    scratch = torch.full((hga.hga_tier_scratch_size(p, slots) // 4,), 123, device="cuda", dtype=torch.int32)
    idx_r = torch.full_like(idx, -5)
    torch.cuda.synchronize()
    with pytest.raises(hga.HGAError) as err:
        hga.hga_fetch_tiered(p, host_k, host_v, idx, 0, 2, stage_k, stage_v, slots, scratch, idx_r)
    assert err.value.code == -1
    assert b"page-locked" in hga.lib().hga_last_error()
    torch.cuda.synchronize()
    # nothing was enqueued: scratch, staging and the remapped routes are untouched
    assert torch.all(scratch == 123) and torch.all(idx_r == -5) and torch.all(stage_k == 0)
    assert hga.hga_get_device_status() == 0


# ---------------------------------------------------------------- route + attention in one call

@pytest.mark.parametrize("w", [MID, W["tiny_fp32"], *EDGE], ids=[w.name for w in [MID, W["tiny_fp32"], *EDGE]])
def test_route_attn_fwd_matches_route_then_oracle(w):
    """hga_route_attn_fwd writes the same routes as hga_route (bit for bit) and its
    attention, which runs the causal segment tiles before the routed ones and
    overlaps the route, matches the oracle on those routes."""
    import hierarchical_sparse_long_b200 as hga
    arrs = hc.segment_arrays(w, 0)
    g = hc.GpuSegment(w, arrs)
    summ = g.summaries()
    idx_a = g.route(summ)
    idx_b = torch.full_like(idx_a, -9)
    out = torch.full_like(g.q, float("nan"))
    lse = torch.full(g.q.shape[:3], float("nan"), device="cuda")
    hga.hga_route_attn_fwd(g.p, g.q, summ, g.cap, idx_b, g.k_all, g.v_all, g.k_seg, g.v_seg, out, lse)
    torch.cuda.synchronize()
    assert torch.equal(idx_a, idx_b)
    T = arrs["T"]
    sh = hc.oracle_shape(w, T)
    out_o, lse_o = oracle.attn_fwd(sh, arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T],
                                   arrs["k_all"][:, :, T:], arrs["v_all"][:, :, T:], hc.f32(idx_b).astype(np.int32))
    hc.compare(hc.f32(out), out_o, w.dtype, f"{w.name} out")
    hc.compare(hc.f32(lse), lse_o, "fp32" if w.dtype == "fp32" else "bf16", f"{w.name} lse")


@pytest.mark.parametrize("name,seg,n", [("qwen3_16k_fwd", 0, 256), ("qwen3_128k_eval", 31, 128)])
def test_route_attn_fwd_full_size_sampled(name, seg, n):
    import hierarchical_sparse_long_b200 as hga
    w = W[name]
    arrs = hc.segment_arrays(w, seg)
    g = hc.GpuSegment(w, arrs)
    summ = g.summaries()
    idx = torch.empty(w.batch, w.n_kv_heads, w.seg_len // 64, w.topk, device="cuda", dtype=torch.int32)
    out = torch.empty_like(g.q)
    lse = torch.empty(g.q.shape[:3], device="cuda")
    hga.hga_route_attn_fwd(g.p, g.q, summ, g.cap, idx, g.k_all, g.v_all, g.k_seg, g.v_seg, out, lse)
    torch.cuda.synchronize()
    sh, _, idx_o, gap = hc.oracle_route(w, arrs)
    hard, _ = hc.route_mismatches(hc.f32(idx).astype(np.int32), idx_o, gap)
    assert hard == 0
    T = arrs["T"]
    rows = _sampled_rows(w, n, seed=seg + 100)
    out_o, lse_o = oracle.attn_fwd(sh, arrs["q"], arrs["k_all"][:, :, :T], arrs["v_all"][:, :, :T],
                                   arrs["k_all"][:, :, T:], arrs["v_all"][:, :, T:], hc.f32(idx).astype(np.int32),
                                   rows=rows)
    D = w.head_dim
    hc.compare(hc.f32(out).reshape(-1, D)[rows], out_o.reshape(-1, D)[rows], "bf16", f"{name} out")
    hc.compare(hc.f32(lse).reshape(-1)[rows], lse_o.reshape(-1)[rows], "bf16", f"{name} lse")
    assert hga.hga_get_device_status() == 0
