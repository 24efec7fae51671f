"""GPU parity of the group-level second routing stage (hga_route_groups, through the C
ABI) against the oracle: bit-exact group routes except oracle near-ties.

"Long-Context Fine-Tuning with Limited VRAM", technical summary section 2.1 (group
selection): the chosen chunks are split into groups of a few tokens, each group is
scored with its group summary against the same query-block summary, and the best
groups inside the chosen chunks are kept.  Both sides take the oracle's chunk routes
as input, so the test isolates the group stage; group summaries are built on the GPU
by hga_build_summaries with chunk = group and by the oracle in fp64.

Cases: groups of 8, 16 and 32 tokens; topg below the candidate count (selection),
equal to it and above it (every candidate kept, then -1 padding); a budget k above
the history (padded chunk routes, fewer candidates); fp32 and bf16, D = 64 and 128;
and the 16K layer's last segment with groups of 8.
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


CASES = [
    # (name, dtype, D, Hq, Hkv, k, S, T, group, topg, seed)
    ("g8_select", "bf16", 128, 8, 2, 8, 128, 40 * 64, 8, 20, 91),
    ("g16_all_kept", "bf16", 128, 8, 2, 6, 128, 30 * 64, 16, 24, 92),      # topg == 6 chunks x 4 groups
    ("g32_fp32_d64", "fp32", 64, 4, 2, 5, 192, 50 * 64, 32, 3, 93),
    ("g8_k_above_nc_pad", "bf16", 128, 4, 1, 12, 128, 5 * 64, 8, 64, 94),  # 5 chunks -> 40 candidates < 64
    ("g8_k_above_nc_sel", "fp32", 128, 4, 1, 12, 64, 5 * 64, 8, 17, 95),
    ("g8_mha_b2", "bf16", 64, 2, 2, 4, 128, 24 * 64, 8, 9, 96),
    ("g8_k64_wide", "bf16", 128, 4, 1, 64, 64, 80 * 64, 8, 300, 97),        # 512 candidates
]


def _group_route(w, T, group, topg, q, kh, idx_o):
    """(GPU gidx, oracle gidx, oracle gap) for one segment."""
    import hierarchical_sparse_long_b200 as hga
    nc = T // 64
    ng = nc * (64 // group)
    gsumm = torch.zeros(w.batch, w.n_kv_heads, max(ng, 1), w.head_dim, device="cuda")
    if ng:
        hga.hga_build_summaries(hc.to_dev(kh, w), T, w.batch, w.n_kv_heads, w.head_dim, group, 0, ng, gsumm,
                                max(ng, 1))
    nqb = w.seg_len // 64
    gidx = torch.full((w.batch, w.n_kv_heads, nqb, topg), -7, device="cuda", dtype=torch.int32)
    p = hc.params(w, T)
    hga.hga_route_groups(p, hc.to_dev(q, w), gsumm, max(ng, 1), torch.from_numpy(idx_o).cuda(), group, topg, gidx)
    torch.cuda.synchronize()
    sh = oracle.shape(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 64, 64, w.topk, w.seg_len, nc,
                      w.sink_chunks, group, topg)
    gidx_o, gap = oracle.route_groups(sh, q, oracle.summaries(kh, group), idx_o)
    return hc.f32(gidx).astype(np.int32), gidx_o, gap


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_group_route_matches_oracle(case):
    name, dtype, D, Hq, Hkv, k, S, T, group, topg, seed = case
    batch = 2 if name == "g8_mha_b2" else 1
    w = gen.custom(name, batch=batch, dtype=dtype, head_dim=D, n_q_heads=Hq, n_kv_heads=Hkv, topk=k, seg_len=S,
                   seq_len=T + S, seg_starts=(T,), seed=seed)
    q = gen.queries(w, T, T + S)
    kh = gen.keys(w, 0, T)
    _, _, idx_o, _ = hc.oracle_route(w, dict(T=T, q=q, k_all=kh))
    got, want, gap = _group_route(w, T, group, topg, q, kh, idx_o)
    hard, exempt = hc.route_mismatches(got, want, gap)
    print(f"{name}: {got.shape[2]} blocks x {got.shape[1]} heads, near-tie exemptions {exempt}")
    assert hard == 0
    # every kept group lies inside a chosen chunk, and the list is ascending then -1
    gpc = 64 // group
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            for m in range(got.shape[2]):
                row = got[b, g, m]
                valid = row[row >= 0]
                assert np.all(np.diff(valid) > 0)
                assert np.all(row[len(valid):] == -1)
                assert set((valid // gpc).tolist()) <= set(idx_o[b, g, m][idx_o[b, g, m] >= 0].tolist())


def test_group_route_full_size_16k():
    """The 16K layer's last segment (224 history chunks, k = 16): groups of 8, topg = 64
    of the 128 candidate groups per block."""
    w = gen.WORKLOADS["qwen3_16k_fwd"]
    arrs = hc.segment_arrays(w, 0)
    T = arrs["T"]
    _, _, idx_o, _ = hc.oracle_route(w, arrs)
    got, want, gap = _group_route(w, T, 8, 64, arrs["q"], arrs["k_all"][:, :, :T], idx_o)
    hard, exempt = hc.route_mismatches(got, want, gap)
    print(f"16K groups of 8, topg 64: near-tie exemptions {exempt}")
    assert hard == 0


def _tiered_group_route(w, T, group, topg, q, kh, idx_list, slots):
    """hga_route_groups_tiered (group summaries in pinned host memory, a device cache of
    them) against hga_route_groups on the same summaries resident on the device, one
    call per chunk-route table of idx_list (the cache is kept between calls).  Returns
    the tiles fetched by each call and the distinct routed chunks of each table."""
    import hierarchical_sparse_long_b200 as hga
    nc = T // 64
    gpc = 64 // group
    ng = nc * gpc
    gsumm = torch.zeros(w.batch, w.n_kv_heads, ng, w.head_dim, device="cuda")
    hga.hga_build_summaries(hc.to_dev(kh, w), T, w.batch, w.n_kv_heads, w.head_dim, group, 0, ng, gsumm, ng)
    nqb = w.seg_len // 64
    p = hc.params(w, T, hist_head_stride=ng * group)
    qd = hc.to_dev(q, w)
    host = gsumm.cpu().pin_memory()
    stage = torch.empty(slots, gpc, w.head_dim, device="cuda")
    scratch = torch.empty(hga.hga_tier_scratch_size(p, slots) // 4, device="cuda", dtype=torch.int32)
    hga.hga_tier_reset(p, slots, scratch)
    fetched, distinct = [], []
    for idx_o in idx_list:
        idx = torch.from_numpy(np.ascontiguousarray(idx_o)).cuda()
        want = torch.full((w.batch, w.n_kv_heads, nqb, topg), -7, device="cuda", dtype=torch.int32)
        hga.hga_route_groups(p, qd, gsumm, ng, idx, group, topg, want)
        idx_r = torch.full_like(idx, -5)
        got = torch.full_like(want, -9)
        nf = torch.zeros(1, device="cuda", dtype=torch.int32)
        hga.hga_route_groups_tiered(p, qd, host, ng, idx, group, topg, got, stage, slots, scratch, idx_r, nf)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
        fetched.append(int(nf.item()))
        i = np.asarray(idx_o).astype(np.int64)
        distinct.append(len({(b, g, j) for b in range(w.batch) for g in range(w.n_kv_heads)
                             for j in i[b, g].ravel() if j >= 0}))
    assert hga.hga_get_device_status() == 0
    return fetched, distinct


def test_group_route_from_host_cache_equals_resident():
    # a cache holding every routable chunk's groups: each routed chunk's summaries are
    # fetched once, the second call over the same routes fetches nothing
    w = gen.custom("grp_tier", dtype="bf16", head_dim=128, n_q_heads=8, n_kv_heads=2, topk=6, seg_len=192,
                   seq_len=40 * 64 + 192, seg_starts=(40 * 64,), seed=98)
    T = 40 * 64
    q = gen.queries(w, T, T + w.seg_len)
    kh = gen.keys(w, 0, T)
    _, _, idx_o, _ = hc.oracle_route(w, dict(T=T, q=q, k_all=kh))
    fetched, distinct = _tiered_group_route(w, T, 8, 20, q, kh, [idx_o, idx_o], slots=2 * 40)
    assert fetched == [distinct[0], 0]


def test_group_route_from_small_host_cache_evicts():
    # 3 blocks x 2 heads x 6 chunks = at most 36 routed chunks per call, 72 slots (< 80
    # routable): calls over five route tables (four of random chunks) fetch more tiles than the cache
    # holds, so the round-robin eviction reaches the first table's slots, and a last call
    # over the first table fetches some of them back; every call's routes equal the
    # resident ones
    w = gen.custom("grp_tier_small", dtype="fp32", head_dim=64, n_q_heads=4, n_kv_heads=2, topk=6, seg_len=192,
                   seq_len=40 * 64 + 192, seg_starts=(40 * 64,), seed=99)
    T = 40 * 64
    q = gen.queries(w, T, T + w.seg_len)
    kh = gen.keys(w, 0, T)
    _, _, idx_o, _ = hc.oracle_route(w, dict(T=T, q=q, k_all=kh))
    rng = np.random.default_rng(7)
    others = [np.sort(np.stack([[[rng.choice(40, 6, replace=False) for _ in range(3)] for _ in range(2)]]), axis=-1)
              .astype(np.int32) for _ in range(4)]
    fetched, distinct = _tiered_group_route(w, T, 16, 9, q, kh, [idx_o, *others, idx_o], slots=72)
    assert fetched[0] == distinct[0]
    assert sum(fetched[:5]) > 72  # more tiles than slots: the cache evicted
    assert fetched[5] > 0  # the first table's tiles were among them
    print(f"small group-summary cache: fetched {fetched}, distinct {distinct}")
