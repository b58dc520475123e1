"""Seeded input generator: determinism, shapes, dtypes and structure. CPU only."""

import torch

from hierarchical_sparse_attention_pyramid_b200 import synth


def test_head_inputs_deterministic_and_shaped():
    w = synth.WORKLOADS["tiny_4k_fp32"]
    a = synth.head_inputs(w, 0)
    b = synth.head_inputs(w, 0)
    for n in ("q", "k", "v", "dy"):
        assert a[n].shape == (w.N, w.d) and a[n].dtype == torch.float32
        assert torch.equal(a[n], b[n])
    assert not torch.equal(a["q"], a["k"])
    assert abs(float(a["q"].float().std()) - 1.0) < 0.02


def test_bf16_and_lognormal_structure():
    w = synth.WORKLOADS["lognorm_32k"].with_(N=4096, H=2)
    h = synth.head_inputs(w, 1)
    assert h["q"].dtype == torch.bfloat16
    # one scalar per token multiplies q, k and v: the row-norm ratios agree
    rq = h["q"].float().norm(dim=1) / h["k"].float().norm(dim=1)
    assert float(rq.log().std()) < 0.5
    lr = h["q"].float().norm(dim=1).log()
    assert float(lr.std()) > 0.35  # log-normal spread of the per-token scale


def test_outlier_positions_shared_and_scaled():
    w = synth.WORKLOADS["outlier_1m"].with_(N=20000, H=2)
    pos = synth.outlier_positions(w)
    assert len(pos) == 200 and len(set(pos.tolist())) == 200
    h0, h1 = synth.head_inputs(w, 0), synth.head_inputs(w, 1)
    for h in (h0, h1):
        n = h["v"].float().norm(dim=1)
        mask = torch.zeros(w.N, dtype=torch.bool)
        mask[pos] = True
        assert float(n[mask].mean() / n[~mask].mean()) > 3.5
