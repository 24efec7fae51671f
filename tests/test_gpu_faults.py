"""Failure handling on the GPU without faulting it: a pipeline wait that can
never complete gives up after its cycle limit, the status word reports it,
and the context keeps working; out-of-range route indices are reported the
same way (see also test_gpu_parity.py)."""
import pytest
import torch

from inputs import gen
from tests import hga_cases as hc

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import hierarchical_sparse_long_b200 as hga
    hc.ensure_built()
    assert hga.hga_get_device_status() == 0
    hga.hga_selftest_wait_timeout(100_000_000)  # about 0.05 s at B200 clocks
    bits = hga.hga_get_device_status()
    assert bits & hga.HGA_DEV_TIMEOUT
    assert hga.hga_get_device_status() == 0  # reading clears it
    # the context is still usable: a normal forward runs and reports nothing
    w = gen.custom("after_timeout", n_q_heads=8, n_kv_heads=2, head_dim=128, topk=2, seg_len=128, seq_len=384,
                   seg_starts=(256,), dtype="bf16", seed=31)
    g = hc.GpuSegment(w, hc.segment_arrays(w, 0))
    out, lse = g.fwd(g.route(g.summaries()))
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    assert hga.hga_get_device_status() == 0


def test_selftest_rejects_unbounded_limits():
    import hierarchical_sparse_long_b200 as hga
    hc.ensure_built()
    with pytest.raises(hga.HGAError):
        hga.hga_selftest_wait_timeout(1 << 40)
