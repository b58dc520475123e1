"""Planted mistakes in the oracle must each fail at least one pin.

Each mutant swaps one oracle function for a plausible wrong version (a
dropped term, a wrong shift, sign or tie order) on the CPU, runs the pins of
test_oracle_pins.py, and expects one of them to fail.  CPU only.
"""

import numpy as np
import pytest

from oracle import lighthouse_oracle as lo
import tests.test_oracle_pins as pins

PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _run_pins():
    failed = []
    for f in PINS:
        params = getattr(f, "pytestmark", [])
        cases = [()]
        for m in params:
            if m.name == "parametrize":
                names, values = m.args[0], m.args[1]
                if "," in names:
                    cases = [tuple(v) for v in values]
                else:
                    cases = [(v,) for v in values]
        for args in cases:
            try:
                f(*args)
            except (AssertionError, ValueError, IndexError) as e:  # noqa: PERF203
                failed.append((f.__name__, type(e).__name__))
                break
    return failed


def m_shift_full_block(l, i, p, N):
    b = p ** l
    return min(N, (i + 1) * b), min(N, (i + 2) * b)


def m_order_fine_first(entries, p):
    lv = np.concatenate([np.full(len(e), l, np.int64) for l, e in enumerate(entries)])
    ix = np.concatenate([np.asarray(e, np.int64) for e in entries])
    last = (ix + 1) * (np.int64(p) ** lv) - 1
    order = np.lexsort((lv, last))
    return lv[order], ix[order]


def m_attention_no_scale(Qs, Ks, Vs):
    d = Qs.shape[1]
    return lo_orig["causal_attention"](Qs * np.sqrt(d), Ks, Vs)


def m_pool_adjoint_no_div(dlevels, p):
    acc = dlevels[-1]
    for l in range(len(dlevels) - 2, -1, -1):
        acc = dlevels[l] + np.repeat(acc, p, axis=0)
    return acc


def m_topk_ties_high(scores, k, T=lo.DEFAULT_CHUNK):
    M = scores.shape[0]
    kp = min(k, M)
    sizes = lo.chunk_sizes(M, T)
    qs = lo.quotas(kp, len(sizes))
    kept, start = [], 0
    for size, q in zip(sizes, qs):
        idx = np.arange(start, start + size)
        order = np.lexsort((-idx, -scores[start:start + size]))
        kept.append(np.sort(idx[order[:q]]))
        start += size
    return np.concatenate(kept)


def m_score_mean_pool(s0, p, L):
    levels = [np.asarray(s0, np.float64)]
    for _ in range(1, L):
        levels.append(levels[-1].reshape(-1, p).mean(axis=1))
    return levels


def m_scores_squared(Q, K, scorer="qk_sum"):
    nq = np.sum(np.asarray(Q) ** 2, axis=1)
    nk = np.sum(np.asarray(K) ** 2, axis=1)
    return {"qk_sum": nq + nk, "k": nk, "q": nq}[scorer]


def m_backward_no_rowsum(Qs, Ks, Vs, dOs):
    S, d = Qs.shape
    scale = 1.0 / np.sqrt(d)
    logits = scale * (Qs @ Ks.T)
    logits = np.where(np.tri(S, dtype=bool), logits, -np.inf)
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    P = e / e.sum(axis=1, keepdims=True)
    dP = dOs @ Vs.T
    dZ = P * dP
    return scale * dZ @ Ks, scale * dZ.T @ Qs, P.T @ dOs


def m_budget_no_min(N, p, L, k, selection="parents"):
    return [k for _ in range(L - 1)]


lo_orig = {n: getattr(lo, n) for n in dir(lo) if not n.startswith("_")}

MUTANTS = {
    "shifted_range": m_shift_full_block,
    "causal_order": m_order_fine_first,
    "causal_attention": m_attention_no_scale,
    "pyramid_pool_adjoint": m_pool_adjoint_no_div,
    "stratified_topk": m_topk_ties_high,
    "score_pyramid": m_score_mean_pool,
    "level0_scores": m_scores_squared,
    "causal_attention_backward": m_backward_no_rowsum,
    "budgets": m_budget_no_min,
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    monkeypatch.setattr(lo, name, MUTANTS[name])
    failed = _run_pins()
    assert failed, f"no pin caught the planted mistake in {name}"
