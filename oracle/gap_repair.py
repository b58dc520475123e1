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


def near_ties(Q, K, p, L, k, T=lo.DEFAULT_CHUNK, scorer="qk_sum", rel_gap=1e-5):
    """Level-0 tokens to push down: one per chunk whose q-th/(q+1)-th gap is small."""
    s0 = lo.level0_scores(Q, K, scorer)
    spyr = lo.score_pyramid(s0, p, L)
    tokens = []
    for l in range(L - 1):
        scores = spyr[l + 1]
        M = scores.shape[0]
        sizes = lo.chunk_sizes(M, T)
        qs = lo.quotas(min(k, M), len(sizes))
        start = 0
        for size, q in zip(sizes, qs):
            if 0 < q < size:
                idx = np.arange(start, start + size)
                order = np.lexsort((idx, -scores[start:start + size]))
                a = scores[start + order[q - 1]]
                b = scores[start + order[q]]
                if a <= 0 or (a - b) / a < rel_gap:
                    m = start + int(order[q])
                    block = p ** (l + 1)
                    t0 = m * block
                    tokens.append(t0 + int(np.argmax(s0[t0:t0 + block])))
            start += size
    return sorted(set(tokens))


def repair_head(Q: torch.Tensor, K: torch.Tensor, p, L, k, T=lo.DEFAULT_CHUNK, scorer="qk_sum",
                rel_gap=1e-5, max_rounds=16, factor=0.98):
    """Repair one head's [N, d] Q and K (CPU tensors, any float dtype).
    Returns (Q, K, rows_repaired)."""
    Q = Q.clone()
    K = K.clone()
    repaired = 0
    for _ in range(max_rounds):
        toks = near_ties(Q.double().numpy(), K.double().numpy(), p, L, k, T, scorer, rel_gap)
        if not toks:
            return Q, K, repaired
        t = torch.tensor(toks, dtype=torch.long)
        Q[t] = (Q[t].double() * factor).to(Q.dtype)
        K[t] = (K[t].double() * factor).to(K.dtype)
        repaired += len(toks)
    if near_ties(Q.double().numpy(), K.double().numpy(), p, L, k, T, scorer, rel_gap):
        raise RuntimeError("gap repair did not converge")
    return Q, K, repaired
