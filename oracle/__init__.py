"""ctypes front end of the fp64 CPU oracle (``hga_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use this module; the CUDA library and its Python
binding never import it.  Inputs are converted to float64 exactly (every bf16
and fp32 value is a double) before the C code sees them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hga_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "n_q_heads", "n_kv_heads", "head_dim", "chunk", "q_block", "topk", "seg_len",
        "n_hist_chunks", "sink_chunks", "group", "topg")]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no BLAS, no OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(_LIB_DIR, exist_ok=True)
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_summaries.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_longlong, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, _dp]
        _lib.oracle_route.argtypes = [ctypes.POINTER(Shape), _dp, _dp, _ip, _dp, _dp]
        _lib.oracle_attn_fwd.argtypes = [ctypes.POINTER(Shape), _dp, _dp, _dp, _dp, _dp, _ip,
                                         ctypes.POINTER(ctypes.c_longlong), ctypes.c_longlong, _dp, _dp]
        _lib.oracle_attn_bwd.argtypes = [ctypes.POINTER(Shape), _dp, _dp, _dp, _dp, _dp, _ip, _dp,
                                         ctypes.c_void_p, ctypes.c_void_p, _dp, _dp, _dp]
        _lib.oracle_dense_causal.argtypes = [ctypes.POINTER(Shape), _dp, _dp, _dp, _dp, _dp]
        _lib.oracle_route_groups.argtypes = [ctypes.POINTER(Shape), _dp, _dp, _ip, _ip, _dp]
        _lib.oracle_route_causal.argtypes = [ctypes.POINTER(Shape), _dp, _dp, _ip, _dp]
        for f in ("oracle_summaries", "oracle_route", "oracle_attn_fwd", "oracle_attn_bwd",
                  "oracle_dense_causal", "oracle_route_groups", "oracle_route_causal"):
            getattr(_lib, f).restype = ctypes.c_int
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


def shape(batch, n_q_heads, n_kv_heads, head_dim, chunk, q_block, topk, seg_len, n_hist_chunks,
          sink_chunks=0, group=0, topg=0) -> Shape:
    """group > 0 turns on the group stage: attention reads group routes (topg
    groups of `group` tokens per query block) instead of chunk routes."""
    return Shape(batch, n_q_heads, n_kv_heads, head_dim, chunk, q_block, topk, seg_len, n_hist_chunks,
                 sink_chunks, group, topg)


def summaries(k, chunk: int, n_chunks: int | None = None) -> np.ndarray:
    """Chunk summaries (mean of keys) of k [B][Hkv][T][D] -> [B][Hkv][Nc][D]."""
    k = _f64(k)
    B, H, T, D = k.shape
    nc = T // chunk if n_chunks is None else n_chunks
    out = np.zeros((B, H, nc, D), dtype=np.float64)
    _check(lib().oracle_summaries(_p(k), B, H, T, D, chunk, nc, _p(out)), "oracle_summaries")
    return out


def route(sh: Shape, q, summ, with_scores: bool = False):
    """Routes: (idx int32 [B][Hkv][nqb][k], gap [B][Hkv][nqb], scores or None)."""
    q, summ = _f64(q), _f64(summ)
    nqb = sh.seg_len // sh.q_block
    idx = np.zeros((sh.batch, sh.n_kv_heads, nqb, sh.topk), dtype=np.int32)
    gap = np.zeros((sh.batch, sh.n_kv_heads, nqb), dtype=np.float64)
    scores = np.zeros((sh.batch, sh.n_kv_heads, nqb, max(sh.n_hist_chunks, 1)), dtype=np.float64) \
        if with_scores else None
    _check(lib().oracle_route(ctypes.byref(sh), _p(q), _p(summ), idx.ctypes.data_as(_ip), _p(gap),
                              _p(scores) if scores is not None else None), "oracle_route")
    if scores is not None:
        scores = scores[..., :sh.n_hist_chunks]
    return idx, gap, scores


def route_causal(sh: Shape, q, summ):
    """Strictly causal routes, one per token: (idx int32 [B][Hkv][S][k], gap [B][Hkv][S]).

    Token i routes by the mean of its block's queries up to itself; attend with
    a copy of the shape whose q_block is 1.
    """
    q, summ = _f64(q), _f64(summ)
    idx = np.zeros((sh.batch, sh.n_kv_heads, sh.seg_len, sh.topk), dtype=np.int32)
    gap = np.zeros((sh.batch, sh.n_kv_heads, sh.seg_len), dtype=np.float64)
    _check(lib().oracle_route_causal(ctypes.byref(sh), _p(q), _p(summ), idx.ctypes.data_as(_ip), _p(gap)),
           "oracle_route_causal")
    return idx, gap


def route_groups(sh: Shape, q, gsumm, idx):
    """Second routing stage: (gidx int32 [B][Hkv][nqb][topg], gap [B][Hkv][nqb]).

    gsumm: group summaries [B][Hkv][Nc * chunk / group][D] (``summaries(k, group)``);
    idx: the chunk routes of ``route``.
    """
    q, gsumm = _f64(q), _f64(gsumm)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    nqb = sh.seg_len // sh.q_block
    gidx = np.zeros((sh.batch, sh.n_kv_heads, nqb, sh.topg), dtype=np.int32)
    gap = np.zeros((sh.batch, sh.n_kv_heads, nqb), dtype=np.float64)
    _check(lib().oracle_route_groups(ctypes.byref(sh), _p(q), _p(gsumm), idx.ctypes.data_as(_ip),
                                     gidx.ctypes.data_as(_ip), _p(gap)), "oracle_route_groups")
    return gidx, gap


def attn_fwd(sh: Shape, q, k_hist, v_hist, k_seg, v_seg, idx, rows=None):
    """Exact-token attention forward -> (out [B][Hq][S][D], lse [B][Hq][S]).

    rows: optional flat query indices (b*Hq + h)*S + i; other rows stay NaN.
    """
    q, kh, vh, ks, vs = (_f64(a) for a in (q, k_hist, v_hist, k_seg, v_seg))
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.full(q.shape, np.nan)
    lse = np.full(q.shape[:3], np.nan)
    if rows is None:
        rp, nr = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        rp, nr = rows.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)), len(rows)
    _check(lib().oracle_attn_fwd(ctypes.byref(sh), _p(q), _p(kh), _p(vh), _p(ks), _p(vs),
                                 idx.ctypes.data_as(_ip), rp, nr, _p(out), _p(lse)), "oracle_attn_fwd")
    return out, lse


def attn_bwd(sh: Shape, q, k_hist, v_hist, k_seg, v_seg, idx, dout, q_need=None, key_need=None):
    """Backward with frozen routes -> (dq, dk_seg, dv_seg); history gets no grads."""
    q, kh, vh, ks, vs, do = (_f64(a) for a in (q, k_hist, v_hist, k_seg, v_seg, dout))
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    dq = np.zeros_like(q)
    dk = np.zeros_like(ks)
    dv = np.zeros_like(vs)
    qn = None if q_need is None else np.ascontiguousarray(q_need, dtype=np.uint8)
    kn = None if key_need is None else np.ascontiguousarray(key_need, dtype=np.uint8)
    _check(lib().oracle_attn_bwd(ctypes.byref(sh), _p(q), _p(kh), _p(vh), _p(ks), _p(vs),
                                 idx.ctypes.data_as(_ip), _p(do),
                                 qn.ctypes.data if qn is not None else None,
                                 kn.ctypes.data if kn is not None else None,
                                 _p(dq), _p(dk), _p(dv)), "oracle_attn_bwd")
    return dq, dk, dv


def dense_causal(sh: Shape, q, k_all, v_all):
    """Dense causal attention over [history | segment] -> (out, lse)."""
    q, ka, va = _f64(q), _f64(k_all), _f64(v_all)
    out = np.zeros_like(q)
    lse = np.zeros(q.shape[:3])
    _check(lib().oracle_dense_causal(ctypes.byref(sh), _p(q), _p(ka), _p(va), _p(out), _p(lse)),
           "oracle_dense_causal")
    return out, lse
