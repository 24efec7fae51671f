"""Thin ctypes binding of ``libhga.so`` (the C ABI declared in include/hga.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensors are torch tensors (device tensors on the current CUDA
device, page-locked host tensors for the tiered history); the stream is the
caller's current torch stream unless one is given.  A missing or unloadable
library raises ``HGAError`` -- there is no other implementation to fall back
to.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhga.so")

HGA_BF16, HGA_FP32 = 0, 1
HGA_DEV_BAD_INDEX, HGA_DEV_TIMEOUT, HGA_DEV_STAGE_FULL = 1, 2, 4
HGA_TIER_RESET, HGA_TIER_CHAIN = 1, 2
STATUS = {0: "HGA_OK", -1: "HGA_ERR_INVALID_ARG", -2: "HGA_ERR_UNSUPPORTED", -3: "HGA_ERR_CUDA",
          -4: "HGA_ERR_DEVICE_CHECK", -5: "HGA_ERR_TIMEOUT"}

EXPORTED = ("hga_build_summaries", "hga_route", "hga_route_causal", "hga_route_groups", "hga_route_groups_tiered",
            "hga_attn_fwd",
            "hga_route_attn_fwd",
            "hga_attn_bwd_workspace_size", "hga_attn_bwd", "hga_attn_fwd_groups", "hga_attn_bwd_groups",
            "hga_attn_causal_workspace_size", "hga_attn_fwd_causal", "hga_attn_bwd_causal",
            "hga_attn_bwd_noalloc", "hga_attn_decode_workspace_size", "hga_attn_decode", "hga_tier_scratch_size",
            "hga_tier_reset", "hga_fetch_tiered", "hga_tier_offload", "hga_attn_fwd_tiered", "hga_segment_fwd_tiered",
            "hga_segment_fwd",
            "hga_get_device_status", "hga_selftest_wait_timeout", "hga_status_string", "hga_last_error")


class HGAError(RuntimeError):
    def __init__(self, code: int, what: str, detail: str = ""):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}" + (f" ({detail})" if detail else ""))


class CParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("chunk", ctypes.c_int), ("q_block", ctypes.c_int),
                ("topk", ctypes.c_int), ("seg_len", ctypes.c_int), ("n_hist_chunks", ctypes.c_int),
                ("dtype", ctypes.c_int), ("hist_head_stride", ctypes.c_longlong),
                ("seg_head_stride", ctypes.c_longlong), ("qblock_begin", ctypes.c_int),
                ("qblock_end", ctypes.c_int), ("sink_chunks", ctypes.c_int)]


@dataclasses.dataclass
class Params:
    """Mirror of ``hga_params_t`` (strides in tokens; 0/0 block range = all blocks)."""
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    topk: int
    seg_len: int
    n_hist_chunks: int
    dtype: int = HGA_BF16
    hist_head_stride: int = -1  # -1: n_hist_chunks * chunk
    seg_head_stride: int = -1   # -1: seg_len
    chunk: int = 64
    q_block: int = 64
    qblock_begin: int = 0
    qblock_end: int = 0
    sink_chunks: int = 0  # attention-sink window: chunks always routed

    def c(self) -> CParams:
        hs = self.hist_head_stride if self.hist_head_stride >= 0 else self.n_hist_chunks * self.chunk
        ss = self.seg_head_stride if self.seg_head_stride >= 0 else self.seg_len
        return CParams(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim, self.chunk, self.q_block,
                       self.topk, self.seg_len, self.n_hist_chunks, self.dtype, hs, ss, self.qblock_begin,
                       self.qblock_end, self.sink_chunks)


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libhga.so (raises HGAError if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise HGAError(-2, "libhga.so is not built",
                           "run `python -m hierarchical_sparse_long_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, ll, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
        pp = ctypes.POINTER(CParams)
        L.hga_build_summaries.argtypes = [vp, ll, i, i, i, i, i, i, i, vp, i, vp]
        L.hga_route.argtypes = [pp, vp, vp, i, vp, vp]
        L.hga_route_causal.argtypes = [pp, vp, vp, i, vp, vp]
        L.hga_route_groups.argtypes = [pp, vp, vp, i, vp, i, i, vp, vp]
        L.hga_route_groups_tiered.argtypes = [pp, vp, vp, i, vp, i, i, vp, vp, i, vp, vp, vp, vp]
        L.hga_attn_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.hga_route_attn_fwd.argtypes = [pp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp, vp]
        L.hga_attn_fwd_groups.argtypes = [pp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp]
        L.hga_attn_bwd_groups.argtypes = [pp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.hga_attn_causal_workspace_size.argtypes = [pp, i]
        L.hga_attn_causal_workspace_size.restype = sz
        L.hga_attn_fwd_causal.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.hga_attn_bwd_causal.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.hga_attn_bwd_workspace_size.argtypes = [pp]
        L.hga_attn_bwd_workspace_size.restype = sz
        L.hga_attn_bwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.hga_attn_bwd_noalloc.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.hga_attn_decode_workspace_size.argtypes = [pp, i]
        L.hga_attn_decode_workspace_size.restype = sz
        L.hga_attn_decode.argtypes = [pp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp, sz, vp]
        L.hga_tier_scratch_size.argtypes = [pp, i]
        L.hga_tier_scratch_size.restype = sz
        L.hga_tier_reset.argtypes = [pp, i, vp, vp]
        L.hga_fetch_tiered.argtypes = [pp, vp, vp, vp, i, i, vp, vp, i, vp, vp, vp, vp, vp]
        L.hga_tier_offload.argtypes = [pp, vp, vp, vp, vp, ll, vp]
        L.hga_attn_fwd_tiered.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, i, i, vp, vp,
                                          vp, ctypes.POINTER(_TierSchedC)]
        L.hga_segment_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, i, vp, vp,
                                      ctypes.POINTER(_TierSchedC)]
        L.hga_segment_fwd_tiered.argtypes = [pp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, i,
                                             i, vp, vp, vp, vp, vp, ctypes.POINTER(_TierSchedC)]
        L.hga_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
        L.hga_selftest_wait_timeout.argtypes = [ll, vp]
        L.hga_selftest_wait_timeout.restype = ctypes.c_int
        L.hga_status_string.argtypes = [i]
        L.hga_status_string.restype = ctypes.c_char_p
        L.hga_last_error.restype = ctypes.c_char_p
        for f in ("hga_build_summaries", "hga_route", "hga_route_causal", "hga_route_groups",
                  "hga_route_groups_tiered", "hga_attn_fwd",
                  "hga_attn_bwd", "hga_attn_bwd_noalloc", "hga_attn_fwd_groups", "hga_attn_bwd_groups",
                  "hga_route_attn_fwd",
                  "hga_attn_fwd_causal", "hga_attn_bwd_causal",
                  "hga_attn_decode", "hga_tier_reset", "hga_fetch_tiered", "hga_tier_offload", "hga_attn_fwd_tiered",
                  "hga_get_device_status"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        detail = lib().hga_last_error().decode() if rc == -3 else ""
        raise HGAError(rc, what, detail)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return HGA_BF16
    if t.dtype == torch.float32:
        return HGA_FP32
    raise HGAError(-1, "unsupported tensor dtype", str(t.dtype))


def hga_build_summaries(k, head_stride: int, batch: int, n_kv_heads: int, head_dim: int, chunk: int,
                        first_chunk: int, n_chunks: int, summ, summ_cap_chunks: int, stream=None):
    """Chunk summaries (mean of keys) for chunks [first_chunk, first_chunk + n_chunks)."""
    _check(lib().hga_build_summaries(_ptr(k), head_stride, batch, n_kv_heads, head_dim, chunk, first_chunk,
                                     n_chunks, dtype_code(k), _ptr(summ), summ_cap_chunks, _stream(stream)),
           "hga_build_summaries")


def hga_route(p: Params, q, summ, summ_cap_chunks: int, idx, stream=None):
    """Top-k chunk routing per (batch, kv head, query block) into idx (int32)."""
    cp = p.c()
    _check(lib().hga_route(ctypes.byref(cp), _ptr(q), _ptr(summ), summ_cap_chunks, _ptr(idx), _stream(stream)),
           "hga_route")


def hga_route_causal(p: Params, q, summ, summ_cap_chunks: int, idx, stream=None):
    """Strictly causal routing: one route per token into idx [B][Hkv][S][k] (int32)."""
    cp = p.c()
    _check(lib().hga_route_causal(ctypes.byref(cp), _ptr(q), _ptr(summ), summ_cap_chunks, _ptr(idx),
                                  _stream(stream)), "hga_route_causal")


def hga_route_groups(p: Params, q, gsumm, gsumm_cap_groups: int, idx, group: int, topg: int, gidx, stream=None):
    """Second routing stage: the topg best groups of `group` tokens inside each block's
    chosen chunks into gidx [B][Hkv][S/q_block][topg] (int32)."""
    cp = p.c()
    _check(lib().hga_route_groups(ctypes.byref(cp), _ptr(q), _ptr(gsumm), gsumm_cap_groups, _ptr(idx), group,
                                  topg, _ptr(gidx), _stream(stream)), "hga_route_groups")


def hga_route_groups_tiered(p: Params, q, host_gsumm, gsumm_cap_groups: int, idx, group: int, topg: int, gidx,
                            stage_gsumm, stage_slots: int, scratch, idx_remapped, n_fetched=None, stream=None):
    """hga_route_groups from a device cache of group summaries whose misses are
    fetched from pinned host memory (p.hist_head_stride = gsumm_cap_groups * group)."""
    cp = p.c()
    _check(lib().hga_route_groups_tiered(ctypes.byref(cp), _ptr(q), _ptr(host_gsumm), gsumm_cap_groups, _ptr(idx),
                                         group, topg, _ptr(gidx), _ptr(stage_gsumm), stage_slots, _ptr(scratch),
                                         _ptr(idx_remapped), _ptr(n_fetched), _stream(stream)),
           "hga_route_groups_tiered")


def hga_attn_fwd(p: Params, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, stream=None):
    """Exact-token attention forward over routed chunks + the causal segment."""
    cp = p.c()
    _check(lib().hga_attn_fwd(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_seg), _ptr(v_seg),
                              _ptr(idx), _ptr(out), _ptr(lse), _stream(stream)), "hga_attn_fwd")


def hga_route_attn_fwd(p: Params, q, summ, summ_cap_chunks: int, idx, k_hist, v_hist, k_seg, v_seg, out, lse,
                       stream=None):
    """Route, then attend, in one call: the attention overlaps the route's tail
    (routes into idx as hga_route; out/lse as hga_attn_fwd within rounding)."""
    cp = p.c()
    _check(lib().hga_route_attn_fwd(ctypes.byref(cp), _ptr(q), _ptr(summ), summ_cap_chunks, _ptr(idx),
                                    _ptr(k_hist), _ptr(v_hist), _ptr(k_seg), _ptr(v_seg), _ptr(out), _ptr(lse),
                                    _stream(stream)), "hga_route_attn_fwd")


def hga_attn_fwd_groups(p: Params, q, k_hist, v_hist, k_seg, v_seg, gidx, group: int, topg: int, out, lse,
                        stream=None):
    """Attention over the routed groups (hga_route_groups) + the causal segment."""
    cp = p.c()
    _check(lib().hga_attn_fwd_groups(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_seg),
                                     _ptr(v_seg), _ptr(gidx), group, topg, _ptr(out), _ptr(lse), _stream(stream)),
           "hga_attn_fwd_groups")


def hga_attn_bwd_groups(p: Params, q, k_hist, v_hist, k_seg, v_seg, gidx, group: int, topg: int, out, lse, dout,
                        dq, dk_seg, dv_seg, workspace, stream=None):
    """Backward of hga_attn_fwd_groups: dq over routed groups and segment, dk/dv of the segment."""
    cp = p.c()
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().hga_attn_bwd_groups(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_seg),
                                     _ptr(v_seg), _ptr(gidx), group, topg, _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                     _ptr(dk_seg), _ptr(dv_seg), _ptr(workspace), nbytes, _stream(stream)),
           "hga_attn_bwd_groups")


def hga_attn_causal_workspace_size(p: Params, backward: bool = False) -> int:
    cp = p.c()
    return int(lib().hga_attn_causal_workspace_size(ctypes.byref(cp), 1 if backward else 0))


def hga_attn_fwd_causal(p: Params, q, k_hist, v_hist, k_seg, v_seg, idx_tok, out, lse, workspace, stream=None):
    """Attention over per-token (strictly causal) routes [B][Hkv][S][k] + the causal segment."""
    cp = p.c()
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().hga_attn_fwd_causal(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_seg),
                                     _ptr(v_seg), _ptr(idx_tok), _ptr(out), _ptr(lse), _ptr(workspace), nbytes,
                                     _stream(stream)), "hga_attn_fwd_causal")


def hga_attn_bwd_causal(p: Params, q, k_hist, v_hist, k_seg, v_seg, idx_tok, out, lse, dout, dq, dk_seg, dv_seg,
                        workspace, stream=None):
    """Backward of hga_attn_fwd_causal."""
    cp = p.c()
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().hga_attn_bwd_causal(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_seg),
                                     _ptr(v_seg), _ptr(idx_tok), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                     _ptr(dk_seg), _ptr(dv_seg), _ptr(workspace), nbytes, _stream(stream)),
           "hga_attn_bwd_causal")


def hga_attn_decode_workspace_size(p: Params, n_local: int) -> int:
    cp = p.c()
    return int(lib().hga_attn_decode_workspace_size(ctypes.byref(cp), n_local))


def hga_attn_decode(p: Params, q, k_hist, v_hist, k_local, v_local, n_local: int, idx, out, lse, workspace,
                    stream=None):
    """One new token per sequence: attention over its routed chunks and its n_local-token local window."""
    cp = p.c()
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().hga_attn_decode(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_local),
                                 _ptr(v_local), n_local, _ptr(idx), _ptr(out), _ptr(lse), _ptr(workspace), nbytes,
                                 _stream(stream)), "hga_attn_decode")


def hga_attn_bwd_workspace_size(p: Params) -> int:
    cp = p.c()
    return int(lib().hga_attn_bwd_workspace_size(ctypes.byref(cp)))


def hga_attn_bwd(p: Params, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, dout, dq, dk_seg, dv_seg,
                 workspace, stream=None):
    """Backward with frozen routes: dq (history + segment keys), dk/dv of the segment only."""
    cp = p.c()
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().hga_attn_bwd(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_seg), _ptr(v_seg),
                              _ptr(idx), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk_seg), _ptr(dv_seg),
                              _ptr(workspace), nbytes, _stream(stream)), "hga_attn_bwd")


def hga_attn_bwd_noalloc(p: Params, q, k_hist, v_hist, k_seg, v_seg, idx, out, lse, dout, dq, dk_seg, dv_seg,
                         stream=None):
    """hga_attn_bwd for callers that cannot allocate device memory: the
    workspace is a fixed array inside the library (batch * q heads * segment
    length <= 1,048,576).  Calls on one device share that array, so calls
    that overlap on the GPU must be serialised by the caller."""
    cp = p.c()
    _check(lib().hga_attn_bwd_noalloc(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_seg),
                                      _ptr(v_seg), _ptr(idx), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                      _ptr(dk_seg), _ptr(dv_seg), _stream(stream)), "hga_attn_bwd_noalloc")


def hga_tier_scratch_size(p: Params, stage_slots: int) -> int:
    """Bytes of int32 scratch the tiered staging cache of stage_slots tiles needs."""
    cp = p.c()
    return int(lib().hga_tier_scratch_size(ctypes.byref(cp), stage_slots))


def hga_tier_reset(p: Params, stage_slots: int, scratch, stream=None):
    """Marks every slot of the staging cache empty."""
    cp = p.c()
    _check(lib().hga_tier_reset(ctypes.byref(cp), stage_slots, _ptr(scratch), _stream(stream)), "hga_tier_reset")


def hga_fetch_tiered(p: Params, host_k, host_v, idx, qblock_begin: int, qblock_end: int, stage_k, stage_v,
                     stage_slots: int, scratch, idx_remapped, n_fetched=None, copy_stream=None, done=None):
    """One fetch wave: the routed tiles of blocks [qblock_begin, qblock_end) the staging
    cache does not hold are copied from pinned host memory; idx_remapped gets slots."""
    cp = p.c()
    ev = None if done is None else ctypes.c_void_p(done.cuda_event)
    _check(lib().hga_fetch_tiered(ctypes.byref(cp), _ptr(host_k), _ptr(host_v), _ptr(idx), qblock_begin,
                                  qblock_end, _ptr(stage_k), _ptr(stage_v), stage_slots, _ptr(scratch),
                                  _ptr(idx_remapped), _ptr(n_fetched), _stream(copy_stream), ev),
           "hga_fetch_tiered")


def hga_tier_offload(p: Params, k_seg, v_seg, host_k, host_v, dst_token: int, stream=None):
    """Copies the segment's K/V (every (b, g) slice) into the pinned host history at dst_token."""
    cp = p.c()
    _check(lib().hga_tier_offload(ctypes.byref(cp), _ptr(k_seg), _ptr(v_seg), _ptr(host_k), _ptr(host_v),
                                  dst_token, _stream(stream)), "hga_tier_offload")


class _TierSchedC(ctypes.Structure):
    _fields_ = [("start", ctypes.c_void_p), ("fetched", ctypes.c_void_p), ("consumed", ctypes.c_void_p * 4),
                ("inputs", ctypes.c_void_p), ("offloaded", ctypes.c_void_p * 2), ("routed", ctypes.c_void_p),
                ("idx_free", ctypes.c_void_p * 2), ("lag", ctypes.c_int),
                ("wave", ctypes.c_longlong), ("segment", ctypes.c_longlong)]


class TierSched:
    """hga_tier_sched_t: the cross-stream schedule of hga_attn_fwd_tiered over one
    staging cache -- torch events the library records, the lag (the fetch of wave h
    waits for the attention of wave h - lag) and the wave counter it advances."""

    MAX_LAG = 4

    def __init__(self, lag: int = 2):
        import torch
        if not 2 <= lag <= self.MAX_LAG:
            raise ValueError(f"lag must be in 2..{self.MAX_LAG}")
        self.events = [torch.cuda.Event() for _ in range(8 + lag)]
        for e in self.events:  # torch creates its CUDA event on the first record
            e.record()
        h = [e.cuda_event for e in self.events]
        self.c = _TierSchedC()
        self.c.start, self.c.fetched, self.c.inputs, self.c.routed = h[0], h[1], h[2], h[3]
        self.c.offloaded[0], self.c.offloaded[1] = h[4], h[5]
        self.c.idx_free[0], self.c.idx_free[1] = h[6], h[7]
        for i in range(lag):
            self.c.consumed[i] = h[8 + i]
        self.c.lag = lag
        self.c.wave = 0
        self.c.segment = 0

    @property
    def lag(self) -> int:
        return self.c.lag

    @property
    def wave(self) -> int:
        return self.c.wave

    @property
    def segment(self) -> int:
        return self.c.segment


def hga_attn_fwd_tiered(p: Params, q, host_k, host_v, k_seg, v_seg, idx, out, lse, stage_k, stage_v,
                        stage_slots: int, scratch, idx_remapped, wave_blocks: int, sched: TierSched,
                        reset_cache=False, chain=False, n_fetched=None, stream=None, copy_stream=None,
                        prev_k_seg=None, prev_v_seg=None):
    """Attention over host-resident history: fetch waves on copy_stream overlapped with
    earlier waves' attention on stream, ordered by sched (a TierSched); the previous
    segment's chunks are copied from prev_k_seg / prev_v_seg when given."""
    cp = p.c()
    flags = (HGA_TIER_RESET if reset_cache else 0) | (HGA_TIER_CHAIN if chain else 0)
    _check(lib().hga_attn_fwd_tiered(ctypes.byref(cp), _ptr(q), _ptr(host_k), _ptr(host_v), _ptr(k_seg),
                                     _ptr(v_seg), _ptr(prev_k_seg), _ptr(prev_v_seg), _ptr(idx), _ptr(out),
                                     _ptr(lse), _ptr(stage_k), _ptr(stage_v),
                                     stage_slots, _ptr(scratch), _ptr(idx_remapped), wave_blocks, flags,
                                     _ptr(n_fetched), _stream(stream), _stream(copy_stream), ctypes.byref(sched.c)),
           "hga_attn_fwd_tiered")


def hga_segment_fwd(p: Params, q, k_hist, v_hist, k_seg, v_seg, summ, summ_cap_chunks: int, idx, out, lse,
                    sched: TierSched, reset=False, stream=None, route_stream=None):
    """One segment of an evaluation over resident history: route and summary append on
    route_stream, attention on stream (a segment's route runs under the previous
    segment's attention)."""
    cp = p.c()
    _check(lib().hga_segment_fwd(ctypes.byref(cp), _ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(k_seg), _ptr(v_seg),
                                 _ptr(summ), summ_cap_chunks, _ptr(idx), _ptr(out), _ptr(lse),
                                 HGA_TIER_RESET if reset else 0, _stream(stream), _stream(route_stream),
                                 ctypes.byref(sched.c)), "hga_segment_fwd")


def hga_segment_fwd_tiered(p: Params, q, k_seg, v_seg, summ, summ_cap_chunks: int, idx, host_k, host_v, out, lse,
                           stage_k, stage_v, stage_slots: int, scratch, idx_remapped, wave_blocks: int,
                           sched: TierSched, reset=False, n_fetched=None, stream=None, copy_stream=None,
                           route_stream=None, offload_stream=None, prev_k_seg=None, prev_v_seg=None):
    """One segment of a tiered evaluation: route and summary append on route_stream,
    fetches on copy_stream (the previous segment's chunks from prev_k_seg / prev_v_seg
    when given), the K/V offload on offload_stream, attention on stream."""
    cp = p.c()
    _check(lib().hga_segment_fwd_tiered(ctypes.byref(cp), _ptr(q), _ptr(k_seg), _ptr(v_seg), _ptr(prev_k_seg),
                                        _ptr(prev_v_seg), _ptr(summ),
                                        summ_cap_chunks, _ptr(idx), _ptr(host_k), _ptr(host_v), _ptr(out), _ptr(lse),
                                        _ptr(stage_k), _ptr(stage_v), stage_slots, _ptr(scratch),
                                        _ptr(idx_remapped), wave_blocks, HGA_TIER_RESET if reset else 0,
                                        _ptr(n_fetched), _stream(stream), _stream(copy_stream),
                                        _stream(route_stream), _stream(offload_stream), ctypes.byref(sched.c)),
           "hga_segment_fwd_tiered")


def hga_selftest_wait_timeout(wait_cycles: int, stream=None):
    """Launches a wait that can never complete, bounded to wait_cycles; the device
    status then carries HGA_DEV_TIMEOUT (see hga_get_device_status)."""
    _check(lib().hga_selftest_wait_timeout(wait_cycles, _stream(stream)), "hga_selftest_wait_timeout")


def hga_get_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status bits."""
    bits = ctypes.c_uint(0)
    rc = lib().hga_get_device_status(_stream(stream), ctypes.byref(bits))
    if rc not in (0, -4, -5):
        _check(rc, "hga_get_device_status")
    return bits.value
