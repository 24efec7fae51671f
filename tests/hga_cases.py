"""Shared helpers of the GPU parity tests: seeded segment inputs, the CUDA path
through the C ABI, and the oracle on the same numbers."""
from __future__ import annotations

import functools
import os

import numpy as np
import torch

import oracle
from inputs import gen

TOL = {"bf16": dict(max_abs=2e-2, mean_abs=2e-3), "fp32": dict(max_abs=1e-4, mean_abs=1e-4)}
NEAR_TIE = 1e-5


def ensure_built():
    from hierarchical_sparse_long_b200 import build
    build.build()
    oracle.build()


@functools.lru_cache(maxsize=4)
def segment_arrays(w: gen.Workload, seg: int):
    """Host arrays (float32, values exactly representable in the workload dtype) for one segment."""
    T, S = w.seg_starts[seg], w.seg_len
    q = gen.queries(w, T, T + S)
    k_all = gen.keys(w, 0, T + S)
    v_all = gen.values(w, 0, T + S)
    dout = gen.grad_out(w, T, T + S) if w.backward else None
    return dict(T=T, q=q, k_all=k_all, v_all=v_all, dout=dout)


def torch_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_dev(a, w):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(torch_dtype(w)).contiguous()


def params(w, T, **kw):
    import hierarchical_sparse_long_b200 as hga
    p = hga.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                   topk=w.topk, seg_len=w.seg_len, n_hist_chunks=T // w.chunk,
                   dtype=hga.HGA_BF16 if w.dtype == "bf16" else hga.HGA_FP32,
                   hist_head_stride=T + w.seg_len, seg_head_stride=T + w.seg_len, chunk=w.chunk,
                   q_block=w.q_block, sink_chunks=w.sink_chunks)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


class GpuSegment:
    """Device tensors of one segment: K/V of [history | segment] in one buffer per head."""

    def __init__(self, w, arrs):
        self.w = w
        self.T = arrs["T"]
        self.q = to_dev(arrs["q"], w)
        self.k_all = to_dev(arrs["k_all"], w)
        self.v_all = to_dev(arrs["v_all"], w)
        self.dout = to_dev(arrs["dout"], w) if arrs["dout"] is not None else None
        self.p = params(w, self.T)
        self.nc = self.T // w.chunk
        self.cap = max(self.nc, 1)

    @property
    def k_seg(self):
        return self.k_all[:, :, self.T:]

    @property
    def v_seg(self):
        return self.v_all[:, :, self.T:]

    def summaries(self):
        import hierarchical_sparse_long_b200 as hga
        w = self.w
        summ = torch.zeros(w.batch, w.n_kv_heads, self.cap, w.head_dim, device="cuda", dtype=torch.float32)
        hga.hga_build_summaries(self.k_all, self.T + w.seg_len, w.batch, w.n_kv_heads, w.head_dim, w.chunk, 0,
                                self.nc, summ, self.cap)
        return summ

    def route(self, summ):
        import hierarchical_sparse_long_b200 as hga
        w = self.w
        idx = torch.empty(w.batch, w.n_kv_heads, w.seg_len // w.q_block, w.topk, device="cuda", dtype=torch.int32)
        hga.hga_route(self.p, self.q, summ, self.cap, idx)
        return idx

    def fwd(self, idx):
        import hierarchical_sparse_long_b200 as hga
        out = torch.empty_like(self.q)
        lse = torch.empty(self.q.shape[:3], device="cuda", dtype=torch.float32)
        hga.hga_attn_fwd(self.p, self.q, self.k_all, self.v_all, self.k_seg, self.v_seg, idx, out, lse)
        return out, lse

    def bwd(self, idx, out, lse, dout=None):
        import hierarchical_sparse_long_b200 as hga
        dout = self.dout if dout is None else dout
        dq = torch.empty(self.q.shape, device="cuda", dtype=torch.float32)
        w = self.w
        dk = torch.empty(w.batch, w.n_kv_heads, w.seg_len, w.head_dim, device="cuda", dtype=torch.float32)
        dv = torch.empty_like(dk)
        ws = torch.empty(hga.hga_attn_bwd_workspace_size(self.p) // 4 + 1, device="cuda", dtype=torch.float32)
        hga.hga_attn_bwd(self.p, self.q, self.k_all, self.v_all, self.k_seg, self.v_seg, idx, out, lse, dout, dq,
                         dk, dv, ws)
        return dq, dk, dv


def oracle_shape(w, T):
    return oracle.shape(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.q_block, w.topk, w.seg_len,
                        T // w.chunk, w.sink_chunks)


def oracle_route(w, arrs):
    T = arrs["T"]
    sh = oracle_shape(w, T)
    kh = arrs["k_all"][:, :, :T]
    summ = oracle.summaries(kh, w.chunk) if T else np.zeros((w.batch, w.n_kv_heads, 0, w.head_dim))
    idx, gap, _ = oracle.route(sh, arrs["q"], summ)
    return sh, summ, idx, gap


def compare(got, want, kind, what=""):
    """Max-abs / mean-abs parity; returns the two errors."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    tol = TOL[kind]
    assert mx <= tol["max_abs"], f"{what}: max-abs {mx:.3e} > {tol['max_abs']}"
    assert mean <= tol["mean_abs"], f"{what}: mean-abs {mean:.3e} > {tol['mean_abs']}"
    return mx, mean


def route_mismatches(idx_gpu, idx_oracle, gap):
    """(hard mismatches, exempt near-tie mismatches) between two route tables."""
    diff = np.any(idx_gpu != idx_oracle, axis=-1)
    near = gap < NEAR_TIE
    return int(np.sum(diff & ~near)), int(np.sum(diff & near))


def f32(t):
    return t.detach().float().cpu().numpy()
