"""Host-side checks of the C ABI: the library loads without a GPU, exports
every entry point include/hga.h declares, and rejects bad arguments on the
host before touching the device."""
import ctypes
import os
import re

import pytest

import hierarchical_sparse_long_b200 as hga
from hierarchical_sparse_long_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from hierarchical_sparse_long_b200 import build
    build.build()
    return binding.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "hga.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hga_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(binding.EXPORTED)


def test_status_strings(L):
    for code, name in binding.STATUS.items():
        assert L.hga_status_string(code).decode() == name


def _params(**kw):
    base = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, topk=4, seg_len=128, n_hist_chunks=8)
    base.update(kw)
    return hga.Params(**base)


BAD = [
    dict(n_q_heads=3),            # Hq % Hkv
    dict(topk=0),
    dict(topk=65),
    dict(seg_len=100),            # not a multiple of the block
    dict(n_hist_chunks=-1),
    dict(qblock_begin=1, qblock_end=1),
    dict(qblock_begin=0, qblock_end=3),  # 3 > S/64 = 2
    dict(seg_head_stride=64),
    dict(hist_head_stride=100),   # < Nc * c
    dict(sink_chunks=-1),
    dict(sink_chunks=5),          # > topk
]


@pytest.mark.parametrize("kw", BAD)
def test_bad_params_rejected_on_host(L, kw):
    p = _params(**kw).c()
    fake = ctypes.c_void_p(0x1000)
    rc = L.hga_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, None)
    assert rc == -1
    rc = L.hga_route(ctypes.byref(p), fake, fake, 64, fake, None)
    assert rc == -1
    rc = L.hga_route_causal(ctypes.byref(p), fake, fake, 64, fake, None)
    assert rc == -1


def test_group_route_checked_on_host(L):
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)
    p = _params().c()  # Nc 8, k 4
    for group, topg, cap in ((7, 4, 64), (64, 4, 64), (8, 0, 64), (8, 33, 64), (8, 4, 63), (16, 17, 32)):
        assert L.hga_route_groups(ctypes.byref(p), fake, fake, cap, fake, group, topg, fake, None) == -1, (group, topg)
    assert L.hga_route_groups(ctypes.byref(p), odd, fake, 64, fake, 8, 4, fake, None) == -1
    assert L.hga_route_groups(ctypes.byref(p), fake, None, 64, fake, 8, 4, fake, None) == -1
    assert L.hga_route_groups(ctypes.byref(p), fake, fake, 64, fake, 8, 4, None, None) == -1


def test_tiered_group_route_checked_on_host(L):
    fake = ctypes.c_void_p(0x1000)
    # Nc 8, k 4, groups of 8: the group-summary history is 64 groups per (b, g)
    p = _params(hist_head_stride=64 * 8).c()
    args = lambda cap, grp, topg, slots: (ctypes.byref(p), fake, fake, cap, fake, grp, topg, fake, fake, slots, fake,
                                          fake, None, None)
    assert L.hga_route_groups_tiered(*args(64, 7, 4, 16)) == -1       # group size
    assert L.hga_route_groups_tiered(*args(64, 8, 33, 16)) == -1      # topg above k * chunk / group
    assert L.hga_route_groups_tiered(*args(32, 8, 4, 16)) == -1       # capacity below Nc * 8
    assert L.hga_route_groups_tiered(*args(128, 8, 4, 16)) == -1      # hist_head_stride != cap * group
    assert L.hga_route_groups_tiered(*args(64, 8, 4, 15)) == -1       # stage below 2 x 2 blocks x 2 heads x 4
    assert b"stage_slots" in L.hga_last_error()


def test_causal_route_checked_on_host(L):
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)
    p = _params().c()
    assert L.hga_route_causal(ctypes.byref(p), fake, fake, 7, fake, None) == -1   # capacity < Nc
    assert L.hga_route_causal(ctypes.byref(p), odd, fake, 8, fake, None) == -1    # misaligned q
    assert L.hga_route_causal(ctypes.byref(p), fake, None, 8, fake, None) == -1   # no summaries
    assert L.hga_route_causal(ctypes.byref(p), fake, fake, 8, None, None) == -1   # no route table
    big = _params(n_hist_chunks=20000, hist_head_stride=20000 * 64).c()
    assert L.hga_route_causal(ctypes.byref(big), fake, fake, 20000, fake, None) == -2


def test_unsupported_shapes(L):
    fake = ctypes.c_void_p(0x1000)
    for kw in (dict(head_dim=96), dict(chunk=32)):
        p = _params(**kw).c()
        assert L.hga_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, None) == -2
        # the allocation-free backward reports the same status as hga_attn_bwd for a shape it has no kernel for
        args = (ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake)
        assert L.hga_attn_bwd(*args, fake, 1 << 20, None) == -2
        assert L.hga_attn_bwd_noalloc(*args, None) == -2
    bad = _params(topk=0).c()
    args = (ctypes.byref(bad), fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake)
    assert L.hga_attn_bwd_noalloc(*args, None) == -1


def test_null_and_misaligned_pointers(L):
    p = _params().c()
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)
    assert L.hga_attn_fwd(ctypes.byref(p), None, fake, fake, fake, fake, fake, fake, fake, None) == -1
    assert L.hga_attn_fwd(ctypes.byref(p), odd, fake, fake, fake, fake, fake, fake, fake, None) == -1
    assert L.hga_attn_bwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                          fake, 0, None) == -1  # workspace too small
    assert L.hga_build_summaries(fake, 64, 1, 1, 128, 64, 0, 2, 0, fake, 1, None) == -1  # capacity
    assert L.hga_build_summaries(odd, 1024, 1, 1, 128, 64, 0, 2, 0, fake, 4, None) == -1
    assert L.hga_build_summaries(fake, 1024, 1, 1, 128, 64, 0, 0, 0, fake, 4, None) == 0  # no-op


def test_tiered_staging_capacity_checked_on_host(L):
    p = _params(n_hist_chunks=32, hist_head_stride=4096).c()
    fake = ctypes.c_void_p(0x1000)
    # 2 blocks x 2 kv heads x 4 routes = 16 tiles may be needed, and the 16 of the wave
    # before stay protected: 32 slots (fewer than the 64 routable tiles) are required
    rc = L.hga_fetch_tiered(ctypes.byref(p), fake, fake, fake, 0, 2, fake, fake, 31, fake, fake, None, None, None)
    assert rc == -1
    assert b"stage_slots" in L.hga_last_error()
    rc = L.hga_fetch_tiered(ctypes.byref(p), fake, fake, fake, 1, 1, fake, fake, 64, fake, fake, None, None, None)
    assert rc == -1
    rc = L.hga_fetch_tiered(ctypes.byref(p), fake, fake, fake, 0, 2, fake, fake, 64, None, fake, None, None, None)
    assert rc == -1  # no scratch
    # the overlapped schedule: every event set, lag in 2..4, known flags, waves of at
    # least one block, and slots for lag waves
    sc = hga.binding._TierSchedC()
    sc.start = sc.fetched = 0x10
    sc.consumed[0] = sc.consumed[1] = sc.consumed[2] = 0x10
    sc.lag = 2
    # p, q, host_k, host_v, k_seg, v_seg, prev_k_seg, prev_v_seg, idx, out, lse, stage_k, stage_v, slots,
    # scratch, idx_remapped
    args = [ctypes.byref(p), fake, fake, fake, fake, fake, None, None, fake, fake, fake, fake, fake, 64, fake, fake]
    assert L.hga_attn_fwd_tiered(*args, 0, 1, None, None, None, ctypes.byref(sc)) == -1
    assert L.hga_attn_fwd_tiered(*args, 1, 1, None, None, None, None) == -1
    assert L.hga_attn_fwd_tiered(*args, 2, 4, None, None, None, ctypes.byref(sc)) == -1  # unknown flag
    for lag in (1, 5):
        sc.lag = lag
        assert L.hga_attn_fwd_tiered(*args, 2, 1, None, None, None, ctypes.byref(sc)) == -1
    sc.lag = 4  # consumed[3] unset
    assert L.hga_attn_fwd_tiered(*args, 2, 1, None, None, None, ctypes.byref(sc)) == -1
    sc.lag = 2
    sc.fetched = 0
    assert L.hga_attn_fwd_tiered(*args, 2, 1, None, None, None, ctypes.byref(sc)) == -1
    sc.fetched = 0x10
    args[13] = 31  # two waves of 2 blocks need 32 slots
    assert L.hga_attn_fwd_tiered(*args, 2, 1, None, None, None, ctypes.byref(sc)) == -1
    sc.lag = 3
    args[13] = 47  # lag 3: 48 slots (fewer than the 64 routable tiles)
    assert L.hga_attn_fwd_tiered(*args, 2, 1, None, None, None, ctypes.byref(sc)) == -1
    assert b"stage_slots" in L.hga_last_error()
    # the previous segment's K/V come as a pair, and only with a segment's worth of history
    sc.lag = 2
    args[13] = 64
    args[6] = fake
    assert L.hga_attn_fwd_tiered(*args, 2, 1, None, None, None, ctypes.byref(sc)) == -1
    short = _params(n_hist_chunks=1, hist_head_stride=4096).c()  # Nc = 1 < S / chunk = 2
    args[0], args[7] = ctypes.byref(short), fake
    assert L.hga_attn_fwd_tiered(*args, 2, 1, None, None, None, ctypes.byref(sc)) == -1


def test_segment_tiered_checked_on_host(L):
    # one tiered evaluation segment: summaries room for the segment's chunks, the
    # segment inside the host history, the offload events, flags
    p = _params(n_hist_chunks=32, hist_head_stride=4096)
    fake = ctypes.c_void_p(0x1000)
    sc = hga.binding._TierSchedC()
    sc.start = sc.fetched = sc.inputs = 0x10
    sc.consumed[0] = sc.consumed[1] = 0x10
    sc.offloaded[0] = sc.offloaded[1] = 0x10
    sc.routed = sc.idx_free[0] = sc.idx_free[1] = 0x10
    sc.lag = 2
    seg_chunks = p.seg_len // 64

    def call(pp, cap, flags=0, sched=sc):
        return L.hga_segment_fwd_tiered(ctypes.byref(pp.c()), fake, fake, fake, None, None, fake, cap, fake, fake,
                                        fake, fake,
                                        fake, fake, fake, 64, fake, fake, 2, flags, None, None, None, None, None,
                                        ctypes.byref(sched) if sched is not None else None)

    assert call(p, 32 + seg_chunks - 1) == -1  # no room to append the segment's summaries
    assert call(_params(n_hist_chunks=32, hist_head_stride=32 * 64 + p.seg_len - 1), 4096) == -1
    assert call(p, 4096, flags=2) == -1  # only HGA_TIER_RESET is a flag here
    assert call(p, 4096, sched=None) == -1
    sc.offloaded[1] = 0
    assert call(p, 4096) == -1
    sc.offloaded[1] = 0x10
    sc.inputs = 0
    assert call(p, 4096) == -1
    sc.inputs = 0x10
    sc.idx_free[0] = 0
    assert call(p, 4096) == -1


def test_segment_fwd_checked_on_host(L):
    p = _params(n_hist_chunks=32, hist_head_stride=4096)
    fake = ctypes.c_void_p(0x1000)
    sc = hga.binding._TierSchedC()
    sc.start = sc.routed = sc.idx_free[0] = sc.idx_free[1] = 0x10
    sc.lag = 2

    def call(pp, cap, flags=0, sched=sc):
        return L.hga_segment_fwd(ctypes.byref(pp.c()), fake, fake, fake, fake, fake, fake, cap, fake, fake, fake,
                                 flags, None, None, ctypes.byref(sched) if sched is not None else None)

    assert call(p, 32 + p.seg_len // 64 - 1) == -1  # no room to append the segment's summaries
    assert call(p, 4096, flags=2) == -1
    assert call(p, 4096, sched=None) == -1
    sc.routed = 0
    assert call(p, 4096) == -1
    sc.routed = 0x10
    assert call(_params(topk=0), 4096) == -1


def test_tiered_scratch_size(L):
    # two int32 entries per (b, g, chunk) of the host history, four per slot, four control words
    p = _params(n_hist_chunks=32, hist_head_stride=4096)
    tiles = 1 * 2 * (4096 // 64)
    want = ((2 * tiles + 4 * 100 + 4) * 4 + 255) // 256 * 256
    assert hga.hga_tier_scratch_size(p, 100) == want
    assert hga.hga_tier_scratch_size(p, 0) == 0
    assert hga.hga_tier_scratch_size(_params(topk=0), 100) == 0
    fake = ctypes.c_void_p(0x1000)
    assert L.hga_tier_reset(ctypes.byref(p.c()), 0, fake, None) == -1
    assert L.hga_tier_reset(ctypes.byref(p.c()), 100, None, None) == -1


def test_workspace_size(L):
    p = _params()
    assert hga.hga_attn_bwd_workspace_size(p) >= 4 * 4 * 128
    assert hga.hga_attn_bwd_workspace_size(_params(topk=0)) == 0


def test_decode_shape_checked_on_host(L):
    """A decode call is a one-token segment (seg_len = q_block = 1); other one-token
    shapes and an empty local window are rejected before any launch."""
    ok = _params(seg_len=1, q_block=1).c()
    assert L.hga_attn_decode_workspace_size(ctypes.byref(ok), 64) > 0
    for bad in (dict(seg_len=2, q_block=1), dict(seg_len=64, q_block=1), dict(seg_len=1, q_block=64)):
        p = _params(**bad).c()
        assert L.hga_attn_decode_workspace_size(ctypes.byref(p), 64) == 0, bad
    assert L.hga_attn_decode_workspace_size(ctypes.byref(ok), 0) == 0
    fake = ctypes.c_void_p(0x1000)
    # one-token segments are for hga_attn_decode only
    assert L.hga_attn_fwd(ctypes.byref(ok), fake, fake, fake, fake, fake, fake, fake, fake, None) == -2


def test_decode_workspace_covers_every_partial(L):
    """The decode workspace holds one (m, l, o[D]) fp32 partial per consumer warp (4),
    split, (b, g) and query head of the group; the split count fills about two CTAs per
    SM (148 here, where no device can be queried) without exceeding the unit count."""
    for B, Hq, Hkv, D, k, nc, n_local in ((16, 32, 8, 128, 32, 2047, 64), (1, 8, 2, 64, 6, 5, 130),
                                          (2, 4, 4, 128, 5, 20, 1)):
        p = _params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=D, topk=k, seg_len=1, q_block=1,
                    n_hist_chunks=nc).c()
        units = min(k, nc) + -(-n_local // 64)
        n_split = max(1, min(units, 2 * 148 // (B * Hkv)))
        floats = B * Hkv * n_split * 4 * (Hq // Hkv) * (D + 2)
        want = (floats * 4 + 255) // 256 * 256
        assert L.hga_attn_decode_workspace_size(ctypes.byref(p), n_local) == want, (B, Hq, Hkv, D)
