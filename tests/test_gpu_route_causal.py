"""GPU parity of strictly causal routing (hga_route_causal, through the C ABI) against the oracle's
per-token prefix routes: bit-exact except oracle near-ties.

Token i of a block routes by the mean over its G heads of the block's queries up to
i (the limits section of the technical summary proposes a strictly causal variant of
the block-shared route); cases cover fp32 and bf16, a sink window, k > Nc, and a
2,047-chunk history scored in passes of 16 tokens.
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
    # (name, dtype, D, Hq, Hkv, k, S, T, sink, seed)
    ("causal_tiny_fp32", "fp32", 64, 2, 1, 4, 128, 1024, 0, 81),
    ("causal_bf16_g4", "bf16", 128, 8, 2, 8, 192, 40 * 64, 0, 82),
    ("causal_sink2", "bf16", 128, 8, 2, 8, 128, 40 * 64, 2, 83),
    ("causal_k_above_nc", "bf16", 128, 4, 1, 16, 64, 8 * 64, 0, 84),
    ("causal_long_tp16", "bf16", 128, 4, 1, 32, 64, 2047 * 64, 0, 85),   # 16 tokens per pass
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_causal_route_matches_oracle(case):
    import hierarchical_sparse_long_b200 as hga
    name, dtype, D, Hq, Hkv, k, S, T, sink, seed = case
    w = gen.custom(name, dtype=dtype, head_dim=D, n_q_heads=Hq, n_kv_heads=Hkv, topk=k, seg_len=S,
                   seq_len=T + S, seg_starts=(T,), seed=seed)
    nc = T // 64
    q = gen.queries(w, T, T + S)
    kh = gen.keys(w, 0, T)
    sh = oracle.shape(1, Hq, Hkv, D, 64, 64, k, S, nc, sink)
    summ_o = oracle.summaries(kh, 64)
    idx_o, gap = oracle.route_causal(sh, q, summ_o)
    kd = hc.to_dev(kh, w)
    summ = torch.zeros(1, Hkv, nc, D, device="cuda")
    hga.hga_build_summaries(kd, T, 1, Hkv, D, 64, 0, nc, summ, nc)
    p = hga.Params(batch=1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=D, topk=k, seg_len=S, n_hist_chunks=nc,
                   dtype=hga.HGA_BF16 if dtype == "bf16" else hga.HGA_FP32, sink_chunks=sink)
    idx = torch.full((1, Hkv, S, k), -7, device="cuda", dtype=torch.int32)
    hga.hga_route_causal(p, hc.to_dev(q, w), summ, nc, idx)
    torch.cuda.synchronize()
    assert hga.hga_get_device_status() == 0
    hard, exempt = hc.route_mismatches(hc.f32(idx).astype(np.int32), idx_o, gap)
    assert hard == 0
    print(f"{name}: near-tie exemptions {exempt}")
