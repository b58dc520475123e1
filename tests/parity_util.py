"""Helpers shared by the GPU parity tests: seeded, gap-repaired inputs, the
oracle per head, and the tolerance check.

Tolerance (the layer's stated bar for bf16 inputs with fp32 accumulation:
max-abs 2e-2, mean-abs 2e-3).  Every element must satisfy

    |gpu - oracle| <= 2e-2 + ulp_out(oracle) / 2

and the mean over the tensor

    mean |gpu - oracle| <= 2e-3 + mean(ulp_out(oracle) / 2)

where ulp_out(x) is the unit in the last place of the tensor's STORED dtype at
|x|.  The only allowance beyond the absolute bar is the rounding of the final
store: the GPU writes a bf16 output (Y, dQ, dK, dV, the pyramid, Qs/Ks/Vs,
dOs), which rounds the value it computed to the nearest bf16, an error of up
to half an ulp that no arithmetic can avoid.  For fp32 outputs (Os, the
attention gradients) that allowance is ~1e-7 relative, so the bar is the
absolute one.

Every check records its achieved errors; tests/conftest.py prints them as a
table at the end of the run (and writes them as JSON lines to the file that
LH_PARITY_LOG names, if set).
"""

from __future__ import annotations

import numpy as np
import torch

from hierarchical_sparse_attention_pyramid_b200 import synth
from oracle import gap_repair
from oracle import lighthouse_oracle as lo

MAX_ABS = 2e-2
MEAN_ABS = 2e-3

# explicit mantissa bits and smallest normal exponent of the stored dtypes
_FORMATS = {"bf16": (7, -126), "fp16": (10, -14), "fp32": (23, -126), "fp64": (52, -1022)}
_TORCH_NAMES = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32", torch.float64: "fp64"}

# (name, dtype, n, max_abs, mean_abs, max_ratio, mean_ratio, rms_ref, kind) of every check this process ran
RESULTS: list[dict] = []


def half_ulp(w: np.ndarray, dtype: str) -> np.ndarray:
    """Half the spacing of `dtype` numbers at |w| (subnormals: the spacing at the smallest normal)."""
    mant, emin = _FORMATS[dtype]
    _, ex = np.frexp(np.abs(np.asarray(w, np.float64)))  # |w| = m 2^ex, m in [0.5, 1)
    binade = np.maximum(ex - 1, emin)
    return np.ldexp(0.5, (binade - mant).astype(np.int64))


def _as_np(x) -> tuple[np.ndarray, str | None]:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy(), _TORCH_NAMES.get(x.dtype)
    return np.asarray(x, np.float64), None


def err_stats(got, want, dtype: str | None = None, max_abs: float = MAX_ABS, mean_abs: float = MEAN_ABS) -> dict:
    g, gd = _as_np(got)
    w = np.asarray(want, np.float64)
    dtype = dtype or gd or "fp32"
    assert g.shape == w.shape, (g.shape, w.shape)
    if g.size == 0:
        return dict(dtype=dtype, n=0, max_abs=0.0, mean_abs=0.0, max_ratio=0.0, mean_ratio=0.0, max_abs_unit=0.0,
                    rms_ref=0.0, finite=True)
    err = np.abs(g - w)
    hu = half_ulp(w, dtype)
    bound = max_abs + hu
    # the elements at unit scale, where the store's rounding is small next to
    # the absolute bar: their largest error shows the arithmetic's own margin
    unit = np.abs(w) <= 1.0
    return dict(dtype=dtype, n=int(g.size), max_abs=float(err.max()), mean_abs=float(err.mean()),
                max_ratio=float((err / bound).max()), mean_ratio=float(err.mean() / (mean_abs + hu.mean())),
                max_abs_unit=float(err[unit].max()) if unit.any() else 0.0,
                rms_ref=float(np.sqrt(np.mean(w * w))), finite=bool(np.all(np.isfinite(g))))


def assert_close(got, want, name, dtype: str | None = None, max_abs: float = MAX_ABS, mean_abs: float = MEAN_ABS):
    """Check `got` (a torch tensor: its dtype is the stored dtype; or an array
    with `dtype` given) against the fp64 oracle values `want`."""
    s = err_stats(got, want, dtype, max_abs, mean_abs)
    RESULTS.append(dict(name=name, kind="check", bar=[max_abs, mean_abs], **s))
    assert s["finite"], f"{name}: non-finite values"
    assert s["max_ratio"] <= 1.0 and s["mean_ratio"] <= 1.0, (
        f"{name}: max-abs {s['max_abs']:.3e} ({s['max_ratio']:.2f} of the bound {max_abs} + half an ulp of "
        f"{s['dtype']}), mean-abs {s['mean_abs']:.3e} ({s['mean_ratio']:.2f} of {mean_abs} + mean half ulp)")
    return s


def assert_all_close(items):
    """assert_close over (got, want, name) triples, recording every one before
    reporting all that failed (so the error table is complete)."""
    bad = []
    for got, want, name in items:
        try:
            assert_close(got, want, name)
        except AssertionError as e:
            bad.append(str(e))
    assert not bad, "; ".join(bad)


def record_info(got, want, name, dtype: str | None = None):
    """Errors for information only (no assertion), e.g. against the oracle
    run without the 16-bit rounding of the attention's inputs."""
    s = err_stats(got, want, dtype)
    RESULTS.append(dict(name=name, kind="info", bar=[MAX_ABS, MEAN_ABS], **s))
    return s


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


def oracle_head(w: synth.Workload, q, k, v, dy=None, attn_dtype="bf16"):
    """fp64 oracle of one head from [N, d] tensors.  attn_dtype=None runs it
    without the bf16 rounding of the attention's inputs (for information)."""
    Y, sv = lo.forward_head(to_np(q), to_np(k), to_np(v), w.p, w.L, w.k, w.chunk, w.scorer,
                            selection=getattr(w, "selection", "parents"), attn_dtype=attn_dtype)
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
