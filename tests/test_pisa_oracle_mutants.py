"""Planted mistakes in the PISA oracle must each fail at least one pin.

Each mutant swaps one function of oracle/pisa_oracle.py for a plausible wrong
version (a shifted visibility rule, a dropped log-sum-exp, an off-by-one
expansion, the wrong tie order, unrounded or summed pooled keys, a dropped
scale) on the CPU, runs the pins of test_pisa_oracle_pins.py, and expects one
of them to fail.  CPU only.
"""

import numpy as np
import pytest

from oracle import pisa_oracle as po
import tests.test_pisa_oracle_pins as pins
from tests.test_oracle_mutants import _run_pins as _run_with

PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]

orig = {n: getattr(po, n) for n in dir(po) if not n.startswith("_")}


def m_visible_first_token(l, j, i, p):
    return np.asarray(j) * p ** l <= np.asarray(i)


def m_visible_strict(l, j, i, p):
    return (np.asarray(j) + 1) * p ** l - 1 < np.asarray(i)


def _masked_logits(Qg, i0, keys, l, b, C, p, scale=True):
    G, d = Qg.shape
    j = np.arange(b * C, (b + 1) * C)
    i = i0 + np.arange(G)
    mask = po.visible(l, j[None, :], i[:, None], p)
    s = Qg @ keys[j].T / (np.sqrt(d) if scale else 1.0)
    return s, mask


def m_score_mean(Qg, i0, keys, l, b, C, p):
    s, mask = _masked_logits(Qg, i0, keys, l, b, C, p)
    return float(s[mask].mean()) if mask.any() else -np.inf


def m_score_max(Qg, i0, keys, l, b, C, p):
    s, mask = _masked_logits(Qg, i0, keys, l, b, C, p)
    return float(s[mask].max()) if mask.any() else -np.inf


def m_score_unmasked(Qg, i0, keys, l, b, C, p):
    s, _ = _masked_logits(Qg, i0, keys, l, b, C, p)
    m = s.max()
    return float(m + np.log(np.exp(s - m).sum()))


def m_score_unscaled(Qg, i0, keys, l, b, C, p):
    s, mask = _masked_logits(Qg, i0, keys, l, b, C, p, scale=False)
    if not mask.any():
        return -np.inf
    v = s[mask]
    return float(v.max() + np.log(np.exp(v - v.max()).sum()))


def m_sub_blocks_unscaled(kept, p):
    kept = np.asarray(kept, np.int64)
    return np.unique((kept[:, None] + np.arange(p)[None, :]).reshape(-1))


def m_top_ties_high(cands, scores, K):
    cands = np.asarray(cands, np.int64)
    scores = np.asarray(scores, np.float64)
    order = sorted(range(len(cands)), key=lambda t: (-scores[t], -cands[t]))
    keep = sorted(order[:min(K, len(cands))], key=lambda t: cands[t])
    return cands[keep], scores[keep]


def m_pyramid_unrounded(K, p, L):
    K = np.asarray(K, np.float64)
    N, d = K.shape
    return [K] + [K.reshape(N // p ** l, p ** l, d).mean(axis=1) for l in range(1, L)]


def m_pyramid_sum(K, p, L):
    K = np.asarray(K, np.float64)
    N, d = K.shape
    return [K] + [po.round_bf16(K.reshape(N // p ** l, p ** l, d).sum(axis=1)) for l in range(1, L)]


MUTANTS = {
    "visible_first_token": ("visible", m_visible_first_token),
    "visible_strict": ("visible", m_visible_strict),
    "score_mean": ("block_score", m_score_mean),
    "score_max": ("block_score", m_score_max),
    "score_unmasked": ("block_score", m_score_unmasked),
    "score_unscaled": ("block_score", m_score_unscaled),
    "sub_blocks_unscaled": ("sub_blocks", m_sub_blocks_unscaled),
    "top_ties_high": ("top_blocks", m_top_ties_high),
    "pyramid_unrounded": ("key_pyramid", m_pyramid_unrounded),
    "pyramid_sum": ("key_pyramid", m_pyramid_sum),
}


def _run_pins():
    import tests.test_oracle_mutants as tm
    saved = tm.PINS
    tm.PINS = PINS
    try:
        return _run_with()
    finally:
        tm.PINS = saved


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(po, attr, fn)
    failed = _run_pins()
    assert failed, f"no pin caught the planted mistake {name}"


def test_unmutated_oracle_passes_every_pin():
    assert _run_pins() == []
