"""Pins of the PISA selection oracle to facts outside itself (CPU only).

  * a selection worked by hand (tests/golden/pisa_hand_example.json);
  * with K at least the number of level-1 blocks every coarse level keeps
    everything, so the result must equal a flat exhaustive top-K over all
    level-0 blocks, computed here independently (dense score matrix, scipy's
    logsumexp, numpy's lexsort);
  * with Q = 0 every logit is 0, so a block's score is the log of its count
    of visible pairs, counted here one pair at a time;
  * the kept set of every level is the unique set that beats every other
    candidate under (score desc, index asc), found by exhaustive search;
  * a group's selection does not depend on keys after its last query;
  * pooled keys are exact means rounded to bf16, ties to even.
"""

import itertools
import json
import math
import pathlib

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle import pisa_oracle as po

GOLDEN = json.loads((pathlib.Path(__file__).parent / "golden" / "pisa_hand_example.json").read_text())


def _closed_form(expr: str) -> float:
    return eval(expr, {"__builtins__": {}}, {"ln": math.log, "exp": math.exp})  # noqa: S307


def _rand_qk(seed, N, d, scale=1.0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((N, d)) * scale
    K = rng.standard_normal((N, d)) * scale
    # bf16-valued inputs, as the GPU path takes them
    return po.round_bf16(Q), po.round_bf16(K)


def test_hand_example():
    g = GOLDEN
    N, d, p, L, C, G = g["N"], g["d"], g["p"], g["L"], g["C"], g["G"]
    K = np.array(g["keys"], np.float64).reshape(N, d)
    Q = np.full((N, d), float(g["query"]))
    for case in g["cases"]:
        idx, sco = po.select(Q, K, p, L, C, G, case["K"])
        for lev, kept in case["kept"].items():
            lv = int(lev)
            got = [int(x) for x in idx[0, lv] if x >= 0]
            assert got == kept, (case["K"], lv, got, kept)
            want = [_closed_form(e) for e in case["scores"][lev]]
            np.testing.assert_allclose(sco[0, lv, :len(want)], want, rtol=0, atol=1e-12)
        if "level1_all_scores" in case:
            levels = po.key_pyramid(K, p, L)
            s = po.block_scores(Q[:G], 0, levels, 1, np.arange(2), C, p)
            want = [_closed_form(case["level1_all_scores"][str(b)]) for b in range(2)]
            np.testing.assert_allclose(s, want, rtol=0, atol=1e-12)
        if "flat_kept" in case:
            flat = _flat_topk(Q, K, C, G, case["K"])[0][0]
            assert list(flat) == case["flat_kept"]


def _flat_topk(Q, K, C, G, Kb):
    """Exhaustive block selection over level 0, written independently of the
    oracle: dense logits, causal mask by token index, scipy logsumexp per
    block, ranking by numpy lexsort (score desc, block asc)."""
    N, d = Q.shape
    nb = N // C
    out_idx, out_sc = [], []
    for g in range(N // G):
        rows = np.arange(g * G, (g + 1) * G)
        logits = Q[rows] @ K.T / math.sqrt(d)
        mask = np.arange(N)[None, :] <= rows[:, None]
        sc = np.empty(nb)
        for b in range(nb):
            m = mask[:, b * C:(b + 1) * C]
            sc[b] = logsumexp(logits[:, b * C:(b + 1) * C][m]) if m.any() else -np.inf
        order = np.lexsort((np.arange(nb), -sc))[:min(Kb, nb)]
        keep = np.sort(order)
        out_idx.append(keep)
        out_sc.append(sc[keep])
    return out_idx, out_sc


@pytest.mark.parametrize("N,d,p,L,C,G,seed", [
    (256, 8, 2, 3, 8, 32, 0),
    (512, 16, 4, 2, 16, 64, 1),
    (384, 4, 2, 1, 8, 48, 2),
    (512, 8, 2, 4, 4, 16, 3),
])
def test_flat_equivalence_when_coarse_levels_keep_everything(N, d, p, L, C, G, seed):
    Q, K = _rand_qk(seed, N, d, scale=1.5)
    nblk = po.level_blocks(N, p, L, C)
    Kb = nblk[1] if L > 1 else 5
    idx, sco = po.select(Q, K, p, L, C, G, Kb)
    fidx, fsc = _flat_topk(Q, K, C, G, Kb)
    for g in range(N // G):
        got = idx[g, 0][idx[g, 0] >= 0]
        assert np.array_equal(got, fidx[g]), (g, got, fidx[g])
        np.testing.assert_allclose(sco[g, 0, :len(got)], fsc[g], rtol=1e-12, atol=1e-12)
        for l in range(1, L):
            assert np.array_equal(idx[g, l][idx[g, l] >= 0], np.arange(nblk[l]))


@pytest.mark.parametrize("N,p,L,C,G,Kb", [(64, 2, 3, 4, 8, 2), (128, 4, 2, 8, 16, 3), (96, 2, 2, 6, 12, 4)])
def test_zero_queries_score_counts_visible_pairs(N, p, L, C, G, Kb):
    d = 4
    rng = np.random.default_rng(7)
    K = po.round_bf16(rng.standard_normal((N, d)))
    Q = np.zeros((N, d))
    levels = po.key_pyramid(K, p, L)
    for g in range(N // G):
        for l in range(L):
            w = p ** l
            nb = N // (C * w)
            got = po.block_scores(Q[g * G:(g + 1) * G], g * G, levels, l, np.arange(nb), C, p)
            for b in range(nb):
                count = 0
                for i in range(g * G, (g + 1) * G):
                    for j in range(b * C, (b + 1) * C):
                        tokens = range(j * w, (j + 1) * w)  # what entry j of level l averages
                        if all(t <= i for t in tokens):
                            count += 1
                want = math.log(count) if count else -math.inf
                assert got[b] == pytest.approx(want, abs=1e-12), (g, l, b)
    # all-equal scores: ties go to the lower block index at every level
    idx, _ = po.select(Q, K, p, L, C, G, Kb)
    assert idx.shape == (N // G, L, Kb)


def _brute_keep(cands, scores, K):
    n = len(cands)
    Kp = min(K, n)
    winners = []
    for sub in itertools.combinations(range(n), Kp):
        s = set(sub)
        ok = all((scores[a] > scores[b]) or (scores[a] == scores[b] and cands[a] < cands[b])
                 for a in s for b in range(n) if b not in s)
        if ok:
            winners.append(sorted(cands[a] for a in sub))
    return winners


@pytest.mark.parametrize("seed", range(6))
def test_top_blocks_is_the_unique_dominating_set(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 9))
    cands = np.sort(rng.choice(64, size=n, replace=False))
    scores = rng.choice([-np.inf, 0.5, 1.0, 1.0, 2.0, 3.0], size=n)
    for K in range(1, n + 2):
        kept, ks = po.top_blocks(cands, scores, K)
        winners = _brute_keep(cands, scores, K)
        assert len(winners) == 1
        assert list(kept) == winners[0]
        assert np.array_equal(ks, scores[np.searchsorted(cands, kept)])


@pytest.mark.parametrize("N,d,p,L,C,G,Kb,seed", [
    (512, 8, 2, 4, 4, 32, 3, 11),
    (1024, 8, 4, 3, 8, 64, 2, 12),
    (768, 4, 2, 3, 8, 96, 5, 13),
])
def test_selection_invariants(N, d, p, L, C, G, Kb, seed):
    Q, K = _rand_qk(seed, N, d)
    idx, sco = po.select(Q, K, p, L, C, G, Kb)
    nblk = po.level_blocks(N, p, L, C)
    levels = po.key_pyramid(K, p, L)
    for g in range(N // G):
        cands = np.arange(nblk[L - 1])
        for l in range(L - 1, -1, -1):
            kept = idx[g, l][idx[g, l] >= 0]
            assert len(kept) == min(Kb, len(cands))
            assert np.all(np.diff(kept) > 0)
            assert np.all(np.isin(kept, cands))
            assert np.all(idx[g, l, len(kept):] == -1) and np.all(np.isneginf(sco[g, l, len(kept):]))
            # every kept block beats every candidate left out
            sc = po.block_scores(Q[g * G:(g + 1) * G], g * G, levels, l, cands, C, p)
            out = ~np.isin(cands, kept)
            if out.any():
                assert sco[g, l, :len(kept)].min() >= sc[out].max()
            cands = np.concatenate([np.arange(b * p, b * p + p) for b in kept])


def test_selection_ignores_keys_after_the_group():
    N, d, p, L, C, G, Kb = 512, 8, 2, 4, 4, 64, 3
    Q, K = _rand_qk(21, N, d)
    idx, sco = po.select(Q, K, p, L, C, G, Kb)
    rng = np.random.default_rng(22)
    for g in range(N // G):
        K2 = K.copy()
        last = (g + 1) * G - 1
        K2[last + 1:] = po.round_bf16(rng.standard_normal((N - last - 1, d)) * 3)
        idx2, sco2 = po.select(Q, K2, p, L, C, G, Kb)
        assert np.array_equal(idx2[g], idx[g])
        np.testing.assert_array_equal(sco2[g], sco[g])


def test_key_pyramid_is_the_mean_rounded_to_bf16_ties_to_even():
    # integer keys: pair means are multiples of 1/2 and exact in bf16
    rng = np.random.default_rng(5)
    K = rng.integers(-8, 9, size=(64, 4)).astype(np.float64)
    lv = po.key_pyramid(K, 2, 2)
    np.testing.assert_array_equal(lv[1], K.reshape(32, 2, 4).mean(axis=1))
    np.testing.assert_array_equal(lv[0], K)
    # halfway cases: 1 + 2^-8 lies midway between 1 and 1 + 2^-7 (even: 1);
    # 1 + 3*2^-8 lies midway between 1 + 2^-7 and 1 + 2^-6 (even: 1 + 2^-6)
    K = np.array([[1.0], [1 + 2 ** -7], [1 + 2 ** -7], [1 + 2 ** -6]])
    lv = po.key_pyramid(K, 2, 2)
    assert lv[1][0, 0] == 1.0
    assert lv[1][1, 0] == 1 + 2 ** -6
    # p = 4, two levels up: mean of 16 tokens
    K = np.arange(64, dtype=np.float64).reshape(64, 1)
    lv = po.key_pyramid(K, 4, 3)
    np.testing.assert_array_equal(lv[2][:, 0], [7.5, 23.5, 39.5, 55.5])
