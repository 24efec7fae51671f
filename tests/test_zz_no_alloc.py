"""hga_attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (a runtime that owns every byte through its own pool and only hands
the library tensors and a stream, or a hot path that must not call
cudaMalloc).  Its workspace is a fixed array inside the library.

Checked through the C ABI against hga_attn_bwd with a caller-allocated
workspace, on two calls in a row (the second call reuses the array the first
one left behind), within the parity tolerance the other tests use.  This file
is collected last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

from inputs import gen
from tests import hga_cases as hc

pytestmark = pytest.mark.gpu

W = gen.custom("noalloc_bf16", n_q_heads=8, n_kv_heads=2, head_dim=128, topk=4, seg_len=256, seq_len=1088,
               seg_starts=(832,), dtype="bf16", seed=21, backward=True)


def test_noalloc_backward_matches_allocating_backward():
    import hierarchical_sparse_long_b200 as hga
    hc.ensure_built()
    arrs = hc.segment_arrays(W, 0)
    g = hc.GpuSegment(W, arrs)
    idx = g.route(g.summaries())
    out, lse = g.fwd(idx)
    ref = [t.clone() for t in g.bwd(idx, out, lse)]
    torch.cuda.synchronize()
    for call in range(2):
        dq = torch.full_like(ref[0], float("nan"))
        dk = torch.full_like(ref[1], float("nan"))
        dv = torch.full_like(ref[2], float("nan"))
        hga.hga_attn_bwd_noalloc(g.p, g.q, g.k_all, g.v_all, g.k_seg, g.v_seg, idx, out, lse, g.dout, dq, dk, dv)
        torch.cuda.synchronize()
        for got, want, name in ((dq, ref[0], "dq"), (dk, ref[1], "dk"), (dv, ref[2], "dv")):
            hc.compare(hc.f32(got), hc.f32(want), "bf16", f"call {call} {name}")
    assert hga.hga_get_device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import hierarchical_sparse_long_b200 as hga
    hc.ensure_built()
    L = hga.lib()
    # 32 q heads x 65,536-token segment = 2,097,152 rows > the 1,048,576-row scratch
    p = hga.Params(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, topk=16, seg_len=65536,
                   n_hist_chunks=0).c()
    fake = ctypes.c_void_p(0x1000)
    rc = L.hga_attn_bwd_noalloc(ctypes.byref(p), fake, None, None, fake, fake, fake, fake, fake, fake, fake, fake,
                                fake, None)
    assert rc == -1
    assert b"scratch" in L.hga_last_error()
