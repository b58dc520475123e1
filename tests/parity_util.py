"""Helpers shared by the GPU parity tests: seeded, gap-repaired inputs, the
oracle per head, and the tolerance check.

Tolerance (stated for bf16 inputs with fp32 accumulation): per element
    err = |gpu - oracle| / max(1, rms(oracle), |oracle|)
must have max <= 2e-2 and mean <= 2e-3.  bf16 storage alone rounds by up to
2^-9 (0.2%) of a value, so an absolute bound can only hold at unit scale; above
it the same numbers bound the relative error.
"""

from __future__ import annotations

import numpy as np
import torch

from hierarchical_sparse_attention_pyramid_b200 import synth
from oracle import gap_repair
from oracle import lighthouse_oracle as lo

MAX_ERR = 2e-2
MEAN_ERR = 2e-3


def err_stats(got, want):
    g = np.asarray(got, np.float64)
    w = np.asarray(want, np.float64)
    assert g.shape == w.shape, (g.shape, w.shape)
    rms = float(np.sqrt(np.mean(w * w))) if w.size else 0.0
    den = np.maximum(np.maximum(1.0, rms), np.abs(w))
    e = np.abs(g - w) / den
    return float(e.max()) if e.size else 0.0, float(e.mean()) if e.size else 0.0


def assert_close(got, want, name, max_err=MAX_ERR, mean_err=MEAN_ERR):
    mx, mn = err_stats(got, want)
    assert np.all(np.isfinite(np.asarray(got, np.float64))), f"{name}: non-finite values"
    assert mx <= max_err and mn <= mean_err, f"{name}: max err {mx:.3e} (<= {max_err}), mean err {mn:.3e} (<= {mean_err})"
    return mx, mn


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype != torch.float64 else t.cpu().numpy()


def head_case(w: synth.Workload, bh: int):
    """CPU inputs of one head with the top-k near-ties removed (dtype of w)."""
    h = synth.head_inputs(w, bh)
    if w.L > 1:
        h["q"], h["k"], n = gap_repair.repair_head(h["q"], h["k"], w.p, w.L, w.k, w.chunk, w.scorer,
                                                   selection=getattr(w, "selection", "parents"))
        h["repaired"] = n
    return h


def all_heads_case(w: synth.Workload):
    """All heads on the CPU, [B, H, N, d] (small workloads)."""
    heads = [head_case(w, bh) for bh in range(w.B * w.H)]
    return {n: torch.stack([h[n] for h in heads]).reshape(w.B, w.H, w.N, w.d) for n in ("q", "k", "v", "dy")}


def oracle_head(w: synth.Workload, q, k, v, dy=None):
    """fp64 oracle of one head from [N, d] tensors."""
    Y, sv = lo.forward_head(to_np(q), to_np(k), to_np(v), w.p, w.L, w.k, w.chunk, w.scorer,
                            selection=getattr(w, "selection", "parents"))
    out = dict(Y=Y, saved=sv)
    if dy is not None:
        dQ, dK, dV, ex = lo.backward_head(to_np(dy), sv)
        out.update(dQ=dQ, dK=dK, dV=dV, **ex)
    return out


def oracle_sel_flat(w: synth.Workload, sv) -> np.ndarray:
    return np.concatenate([np.asarray(s, np.int64) for s in sv["sel"]]) if w.L > 1 else np.zeros(0, np.int64)


def oracle_seq_map(sv) -> np.ndarray:
    return (sv["seq_level"].astype(np.int64) << 28) | sv["seq_index"].astype(np.int64)


def oracle_slot_of(sv) -> np.ndarray:
    return np.concatenate([t for t in sv["slot_of"]]).astype(np.int64)
