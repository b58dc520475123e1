"""fp64 CPU oracle for PISA block selection (coarse-to-fine top-K with LSE scores).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code with the CUDA library.

Source: PISA-review = the blog.secrett2633.cloud review "[논문리뷰] Block Sparse
Attention with Log-Linear Complexity" (Pyramid Sparse Attention, PISA),
sections "1. Key Terms & Definitions", "2. Motivation & Problem Statement",
"3. Method & Key Results".

What the page fixes (section 3): the key blocks are pooled into a
fine-to-coarse hierarchy; selection starts at the coarsest level; at every
level a LogSumExp score is computed for a limited candidate set, the top-K
candidates are kept and expanded into their sub-blocks at the next finer
level, down to the finest level; the cost is O(N log N) (section 3, second
paragraph); block sparse attention splits the keys into contiguous blocks
and selects some of them per query (section 1, "Block Sparse Attention").

Readings of what it leaves open:
  P1  the hierarchy is the mean-pooled key pyramid with factor p: level-l entry
      j is the mean of keys [j p^l, (j+1) p^l); level 0 holds the keys as given.
      Pooled keys are stored in bf16, rounded to nearest even from the exact
      mean (the precision the tensor cores read them in).
  P2  a block is C consecutive entries of one level; block b of level l spans
      the same tokens as blocks p b .. p b + p - 1 of level l-1 (its
      sub-blocks).  Every level has the same block size C, which is what keeps
      a candidate's score O(C d) and the whole selection O(N log N).
  P3  queries are grouped in blocks of G consecutive queries; each group makes
      one selection (block sparse attention is blocked on both axes).
  P4  the LSE score of block b at level l for group g is
          log sum_{i in g} sum_{j in b, visible(i, j)} exp(q_i . k^(l)_j / sqrt(d)),
      over the C entries of the block ("scores of the keys themselves": the
      entries are the original keys at level 0).  Entry j of level l is
      visible to query i when every token it averages is at or before i:
      (j+1) p^l - 1 <= i.  A block with no visible pair scores -inf.
  P5  the candidates of the coarsest level L-1 are all its blocks; every finer
      level's candidates are the sub-blocks of the blocks kept one level up.
      A level keeps K' = min(K, candidates) blocks by score, higher first;
      equal scores (the -inf ones included) go to the lower block index.
  P6  the output of each level is its kept blocks in ascending block order
      with their scores; the level-0 set is the selection.

All arithmetic is float64 numpy.  One head at a time: Q, K are [N, d].
"""

from __future__ import annotations

import numpy as np

from .lighthouse_oracle import round_bf16


# ----------------------------------------------------------------------------
# sizes
# ----------------------------------------------------------------------------

def check_shape(N: int, d: int, p: int, L: int, C: int, G: int) -> None:
    """Readings P1-P3: N must split into whole blocks at every level and into
    whole query groups."""
    if L < 1 or p < 2 or C < 1 or G < 1 or d < 1:
        raise ValueError("need L >= 1, p >= 2, C >= 1, G >= 1, d >= 1")
    if N % (C * p ** (L - 1)) != 0:
        raise ValueError(f"N={N} is not divisible by C*p^(L-1)={C * p ** (L - 1)}")
    if N % G != 0:
        raise ValueError(f"N={N} is not divisible by the group size G={G}")


def level_blocks(N: int, p: int, L: int, C: int) -> list[int]:
    """Blocks per level: N / (C p^l) (reading P2)."""
    return [N // (C * p ** l) for l in range(L)]


# ----------------------------------------------------------------------------
# the key hierarchy (PISA-review section 3: pooling builds fine-to-coarse key blocks)
# ----------------------------------------------------------------------------

def key_pyramid(K: np.ndarray, p: int, L: int) -> list[np.ndarray]:
    """Reading P1: level l entry j = mean of K[j p^l : (j+1) p^l], taken
    exactly in float64 from the level-0 keys and rounded once to bf16."""
    K = np.asarray(K, np.float64)
    N, d = K.shape
    levels = [K]
    for l in range(1, L):
        w = p ** l
        levels.append(round_bf16(K.reshape(N // w, w, d).mean(axis=1)))
    return levels


# ----------------------------------------------------------------------------
# LSE block score (PISA-review section 1 "LogSumExp (LSE)"; section 3)
# ----------------------------------------------------------------------------

def visible(l: int, j: np.ndarray, i: np.ndarray, p: int) -> np.ndarray:
    """Reading P4: entry j of level l is visible to query i when its last
    averaged token (j+1) p^l - 1 is at or before i.  Broadcasts j against i."""
    return (np.asarray(j) + 1) * p ** l - 1 <= np.asarray(i)


def block_score(Qg: np.ndarray, i0: int, keys: np.ndarray, l: int, b: int, C: int, p: int) -> float:
    """Reading P4: log of the summed exp(q.k / sqrt(d)) over every visible
    (query, entry) pair of query group Qg (queries i0 .. i0+G-1) and block b
    of level l (entries bC .. bC+C-1 of `keys`)."""
    G, d = Qg.shape
    j = np.arange(b * C, (b + 1) * C)
    i = i0 + np.arange(G)
    mask = visible(l, j[None, :], i[:, None], p)
    if not mask.any():
        return -np.inf
    s = (Qg @ keys[j].T) / np.sqrt(d)
    v = s[mask]
    m = v.max()
    return float(m + np.log(np.sum(np.exp(v - m))))


def block_scores(Qg, i0, levels, l, cands, C, p) -> np.ndarray:
    """Scores of the candidate blocks `cands` of level l for one group."""
    return np.array([block_score(Qg, i0, levels[l], l, int(b), C, p) for b in cands], np.float64)


# ----------------------------------------------------------------------------
# top-K and expansion (PISA-review section 3)
# ----------------------------------------------------------------------------

def top_blocks(cands: np.ndarray, scores: np.ndarray, K: int) -> tuple[np.ndarray, np.ndarray]:
    """Reading P5: keep K' = min(K, len(cands)) candidates, higher score first,
    equal scores to the lower block index; return them in ascending block order
    with their scores (reading P6)."""
    cands = np.asarray(cands, np.int64)
    scores = np.asarray(scores, np.float64)
    order = sorted(range(len(cands)), key=lambda t: (-scores[t], cands[t]))
    keep = sorted(order[:min(K, len(cands))], key=lambda t: cands[t])
    return cands[keep], scores[keep]


def sub_blocks(kept: np.ndarray, p: int) -> np.ndarray:
    """Reading P2: the sub-blocks of block b one level down are p b .. p b + p - 1."""
    kept = np.asarray(kept, np.int64)
    return (kept[:, None] * p + np.arange(p)[None, :]).reshape(-1)


def select_group(Q, levels, g: int, G: int, C: int, p: int, L: int, K: int):
    """Coarse-to-fine selection for query group g (PISA-review section 3):
    score the candidates of the coarsest level (all its blocks), keep the
    top K, expand them into sub-blocks, and repeat down to level 0.
    Returns [(kept, scores)] indexed by level."""
    Qg = np.asarray(Q[g * G:(g + 1) * G], np.float64)
    i0 = g * G
    out = [None] * L
    cands = np.arange(levels[L - 1].shape[0] // C)
    for l in range(L - 1, -1, -1):
        sc = block_scores(Qg, i0, levels, l, cands, C, p)
        kept, ks = top_blocks(cands, sc, K)
        out[l] = (kept, ks)
        if l > 0:
            cands = sub_blocks(kept, p)
    return out


def select(Q, Kmat, p: int, L: int, C: int, G: int, K: int):
    """All groups of one head.  Returns (kept_idx [n_groups, L, K] int64 padded
    with -1, kept_score [n_groups, L, K] float64 padded with -inf)."""
    Q = np.asarray(Q, np.float64)
    N, d = Q.shape
    check_shape(N, d, p, L, C, G)
    levels = key_pyramid(Kmat, p, L)
    nG = N // G
    idx = np.full((nG, L, K), -1, np.int64)
    sco = np.full((nG, L, K), -np.inf, np.float64)
    for g in range(nG):
        for l, (kept, ks) in enumerate(select_group(Q, levels, g, G, C, p, L, K)):
            idx[g, l, :len(kept)] = kept
            sco[g, l, :len(kept)] = ks
    return idx, sco
