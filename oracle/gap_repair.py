"""Near-tie repair of seeded inputs, so that top-k decisions are unambiguous.

TEST INFRASTRUCTURE ONLY (see lighthouse_oracle.py).  Parity on selected
indices is bit-exact, but the GPU scores tokens in fp32 and the oracle in
fp64.  For every (head, level, chunk) whose quota q is below the chunk size,
the q-th and (q+1)-th highest candidate scores are compared in fp64 on the
rounded data; if they are closer than ``rel_gap`` (relative), the Q and K rows
of the level-0 token that attains the (q+1)-th score are scaled by 0.98 and
rounded again to the input dtype.  This repeats until no chunk has a near
tie.  The selection rule itself is the oracle's (stratified top-k with
max-pooled level-0 l2-norm scores; LH-summary Technical details (2)).
"""

from __future__ import annotations

import numpy as np
import torch

from . import lighthouse_oracle as lo


def _decisions(Q, K, p, L, k, T, scorer, selection):
    """Every top-k the selection makes: (level of the candidates, their level
    indices in ascending order, their scores, the budget over them)."""
    N = Q.shape[0]
    s0 = lo.level0_scores(Q, K, scorer)
    spyr = lo.score_pyramid(s0, p, L)
    kp = lo.budgets(N, p, L, k, selection)
    out = []
    if selection == "parents":
        for l in range(L - 1):
            out.append((l + 1, np.arange(spyr[l + 1].shape[0]), spyr[l + 1], kp[l]))
    elif selection == "direct":
        for l in range(L - 1):
            out.append((l, np.arange(spyr[l].shape[0]), spyr[l], p * kp[l]))
    else:
        kept = np.arange(N // p ** (L - 1))
        for l in range(L - 2, -1, -1):
            sc = spyr[l + 1][kept]
            out.append((l + 1, kept, sc, kp[l]))
            sel = kept[lo.stratified_topk(sc, kp[l], T)]
            kept = (sel[:, None] * p + np.arange(p)[None, :]).reshape(-1)
    return s0, out


def near_ties(Q, K, p, L, k, T=lo.DEFAULT_CHUNK, scorer="qk_sum", rel_gap=1e-5, selection="parents"):
    """Level-0 tokens to push down: one per chunk whose q-th/(q+1)-th gap is small."""
    s0, decisions = _decisions(Q, K, p, L, k, T, scorer, selection)
    tokens = []
    for lvl, cand, scores, budget in decisions:
        M = scores.shape[0]
        sizes = lo.chunk_sizes(M, T)
        qs = lo.quotas(min(budget, M), len(sizes))
        start = 0
        for size, q in zip(sizes, qs):
            if 0 < q < size:
                idx = np.arange(start, start + size)
                order = np.lexsort((idx, -scores[start:start + size]))
                a = scores[start + order[q - 1]]
                b = scores[start + order[q]]
                if a <= 0 or (a - b) / a < rel_gap:
                    m = int(cand[start + int(order[q])])
                    block = p ** lvl
                    t0 = m * block
                    tokens.append(t0 + int(np.argmax(s0[t0:t0 + block])))
            start += size
    return sorted(set(tokens))


def repair_head(Q: torch.Tensor, K: torch.Tensor, p, L, k, T=lo.DEFAULT_CHUNK, scorer="qk_sum",
                rel_gap=1e-5, max_rounds=16, factor=0.98, selection="parents"):
    """Repair one head's [N, d] Q and K (CPU tensors, any float dtype).
    Returns (Q, K, rows_repaired)."""
    Q = Q.clone()
    K = K.clone()
    repaired = 0
    for _ in range(max_rounds):
        toks = near_ties(Q.double().numpy(), K.double().numpy(), p, L, k, T, scorer, rel_gap, selection)
        if not toks:
            return Q, K, repaired
        t = torch.tensor(toks, dtype=torch.long)
        Q[t] = (Q[t].double() * factor).to(Q.dtype)
        K[t] = (K[t].double() * factor).to(K.dtype)
        repaired += len(toks)
    if near_ties(Q.double().numpy(), K.double().numpy(), p, L, k, T, scorer, rel_gap):
        raise RuntimeError("gap repair did not converge")
    return Q, K, repaired
