"""fp64 CPU oracle for one Lighthouse attention layer, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code with the CUDA library and does not
import the product package.

Sources (web pages describing Lighthouse Attention, arXiv:2605.06554):
  LH-summary = the aitrends.kr summary of Lighthouse Attention (article 58400),
               sections "Key contributions", "Method", "Technical details".
  LH-post    = the techllm.github.io post "Lighthouse Attention: long-context
               pretraining", sections "How it works", "Key formulas",
               "Limitations and caveats".

The method is an approximation (a selection), so this oracle follows the
algorithm's own steps in the pages' order, written plainly in float64:

  1. pyramid pooling of Q, K, V          (LH-post How it works (1); LH-summary Technical details (1))
  2. level-0 l2-norm scores, max-pooled up the pyramid
                                         (LH-summary Technical details (2); LH-post How it works (2))
  3. stratified chunked top-k per level  (LH-post How it works (2); Limitations, "stratified top-K" bullet)
  4. gather into one causally ordered sequence of length S
                                         (LH-post How it works (3); Key formulas)
  5. dense causal softmax attention on S (LH-summary Technical details (3))
  6. scatter-back to the shifted ranges R(l,i), summed per position
                                         (LH-summary Technical details (4); LH-post How it works (4))
  7. backward by hand-derived adjoints; top-k passes no gradient
                                         (LH-summary Method step 5; LH-post How it works (2))

Readings of points the pages leave open:
  R1  N must be divisible by p^(L-1).
  R2  scorer: "qk_sum" = ||Q_t|| + ||K_t|| (default), "k" = ||K_t|| (the
      projection-norm run), "q" = ||Q_t||.
  R3  for each level l = 0..L-2 the candidates are the entries of level l+1
      (scored by their max-pooled score); k' = min(k, M) of them are kept,
      stratified over C = max(1, M // T) contiguous chunks; each kept parent
      brings its p children at level l, so level l adds p*k' entries.  The top
      level L-1 is kept whole.  Ties go to the lower index.
  R5  sequence order: key (e, -l) ascending, e = (i+1)*p^l - 1 the entry's
      last covered token.
  R6  softmax scale 1/sqrt(d); slot t attends to slots <= t.
  R7  entry (l,i) returns its output to R(l,i) = [(i+1)p^l - 1, (i+2)p^l - 1)
      clipped to [0, N); every position sums what it receives.
  R9  selection is per (batch, head).
  R11 the pages run the gathered sequence through stock FlashAttention, a
      16-bit kernel (LH-summary Technical details (3); LH-post How it works
      (3)), so the attention inputs Qs, Ks, Vs, and the output gradient dOs
      that its backward takes, are rounded to bf16 (round to nearest even);
      the backward passes gradients through those casts unchanged.
      attn_dtype=None keeps them exact.

What pins each step (tests/test_oracle_pins.py; planted mistakes in
tests/test_oracle_mutants.py): pooling, norms, max-pooling and the scatter sum
against their definitions computed another way; the top-k against brute force
over all subsets; S and the entry count against hand-worked values; L = 1
against torch's causal attention; the backward against finite differences,
adjoint identities and torch autograd of an independent forward.  Two
readings are pinned only to their own statement, because the pages give no
value to check them against: the chunk length T = 2048 of R3 (parity unpinned
against the pages' own top-K kernel) and the shift of R7 beyond the causality
it must keep (parity unpinned against the pages' own scatter).

All arrays are float64 numpy arrays; one head at a time is ``[N, d]``.
"""

from __future__ import annotations

import numpy as np

SCORERS = ("qk_sum", "k", "q")
DEFAULT_CHUNK = 2048


# ----------------------------------------------------------------------------
# sizes (LH-summary Key contributions: entry count; LH-post Key formulas: S)
# ----------------------------------------------------------------------------

def check_shape(N: int, p: int, L: int) -> None:
    """Reading R1: the pyramid needs N divisible by p^(L-1)."""
    if L < 1 or p < 2:
        raise ValueError("need L >= 1 and p >= 2")
    if N % (p ** (L - 1)) != 0:
        raise ValueError(f"N={N} is not divisible by p^(L-1)={p ** (L - 1)}")


def level_lengths(N: int, p: int, L: int) -> list[int]:
    """Entries per level: N / p^l for l = 0..L-1 (LH-summary Key contributions)."""
    check_shape(N, p, L)
    return [N // p ** l for l in range(L)]


def pyramid_entry_count(N: int, p: int, L: int) -> int:
    """Total pyramid entries, the sum over l of N / p^l (LH-summary Key contributions)."""
    return sum(level_lengths(N, p, L))


# The three readings of what a level keeps (reading C2).  "parents" (R3, the
# default): k'_l parents at level l+1, chosen by their max-pooled scores among
# all N/p^(l+1) entries, each bringing its p children.  "direct": p*k'_l
# entries of level l chosen by their own scores among all N/p^l.  "nested"
# (coarse to fine): as "parents", but the candidate parents at level l+1 are
# only the entries kept there (the whole top level for l = L-2).
SELECTIONS = ("parents", "direct", "nested")


def budgets(N: int, p: int, L: int, k: int, selection: str = "parents") -> list[int]:
    """k'_l for l = 0..L-2: min(k, candidates).  parents / direct: N/p^(l+1)
    candidates (reading R3 / C4); nested: the p k'_(l+1) kept entries of level
    l+1, or the N/p^(L-1) top entries for l = L-2."""
    check_shape(N, p, L)
    if selection not in SELECTIONS:
        raise ValueError(f"unknown selection {selection!r}")
    if selection != "nested":
        return [min(k, N // p ** (l + 1)) for l in range(L - 1)]
    out = [0] * (L - 1)
    cand = N // p ** (L - 1)
    for lvl in range(L - 2, -1, -1):
        out[lvl] = min(k, cand)
        cand = p * out[lvl]
    return out


def gathered_length(N: int, p: int, L: int, k: int, selection: str = "parents") -> int:
    """S = N/p^(L-1) + sum_l p*k'_l  (LH-post Key formulas, with k' = min(k, candidates))."""
    return N // p ** (L - 1) + sum(p * kp for kp in budgets(N, p, L, k, selection))


# ----------------------------------------------------------------------------
# 1. pyramid pooling (LH-post How it works (1); LH-summary Technical details (1))
# ----------------------------------------------------------------------------

def pyramid_pool(X: np.ndarray, p: int, L: int) -> list[np.ndarray]:
    """Average-pool X level by level with window p: level l+1 entry i is the
    mean of level-l entries p*i .. p*i+p-1.  Level 0 is X itself.  The same
    call is made for Q, K and V, which is what makes the pooling symmetric."""
    N = X.shape[0]
    check_shape(N, p, L)
    levels = [np.asarray(X, dtype=np.float64)]
    for _ in range(1, L):
        prev = levels[-1]
        levels.append(prev.reshape(prev.shape[0] // p, p, prev.shape[1]).mean(axis=1))
    return levels


# ----------------------------------------------------------------------------
# 2. scores (LH-summary Technical details (2))
# ----------------------------------------------------------------------------

def level0_scores(Q: np.ndarray, K: np.ndarray, scorer: str = "qk_sum") -> np.ndarray:
    """Parameter-free level-0 score of token t from ||Q_t||_2 and ||K_t||_2 (reading R2)."""
    nq = np.sqrt(np.sum(np.asarray(Q, np.float64) ** 2, axis=1))
    nk = np.sqrt(np.sum(np.asarray(K, np.float64) ** 2, axis=1))
    if scorer == "qk_sum":
        return nq + nk
    if scorer == "k":
        return nk
    if scorer == "q":
        return nq
    raise ValueError(f"unknown scorer {scorer!r}")


def score_pyramid(s0: np.ndarray, p: int, L: int) -> list[np.ndarray]:
    """Coarser levels take the max over their p children (max-pooling)."""
    check_shape(s0.shape[0], p, L)
    levels = [np.asarray(s0, np.float64)]
    for _ in range(1, L):
        prev = levels[-1]
        levels.append(prev.reshape(-1, p).max(axis=1))
    return levels


# ----------------------------------------------------------------------------
# 3. stratified chunked top-k (LH-post How it works (2); Limitations: the top-K
#    is stratified, every interval contributes a fixed number)
# ----------------------------------------------------------------------------

def chunk_sizes(M: int, T: int = DEFAULT_CHUNK) -> list[int]:
    """C = max(1, M // T) contiguous chunks; the first M mod C are one longer."""
    C = max(1, M // T)
    return [M // C + (1 if c < M % C else 0) for c in range(C)]


def quotas(kp: int, C: int) -> list[int]:
    """q_c = floor(k'/C) + [c < k' mod C]."""
    return [kp // C + (1 if c < kp % C else 0) for c in range(C)]


def stratified_topk(scores: np.ndarray, k: int, T: int = DEFAULT_CHUNK) -> np.ndarray:
    """Keep the q_c highest-scored candidates of every chunk (ties: lower index).
    Returns the kept candidate indices in ascending order (int64)."""
    M = scores.shape[0]
    kp = min(k, M)
    sizes = chunk_sizes(M, T)
    qs = quotas(kp, len(sizes))
    kept = []
    start = 0
    for size, q in zip(sizes, qs):
        idx = np.arange(start, start + size)
        # primary key: score descending; secondary: index ascending
        order = np.lexsort((idx, -scores[start:start + size]))
        kept.append(np.sort(idx[order[:q]]))
        start += size
    return np.concatenate(kept) if kept else np.zeros(0, np.int64)


def select(Q, K, p: int, L: int, k: int, T: int = DEFAULT_CHUNK, scorer: str = "qk_sum",
           selection: str = "parents"):
    """Selection for one head.  Returns (sel, spyr); spyr is the score pyramid.
    parents / nested: sel[l] are the kept parent indices at level l+1
    (ascending) for l = 0..L-2; direct: sel[l] are the kept level-l entries."""
    N = np.asarray(Q).shape[0]
    spyr = score_pyramid(level0_scores(Q, K, scorer), p, L)
    kp = budgets(N, p, L, k, selection)
    if selection == "parents":
        sel = [stratified_topk(spyr[l + 1], kp[l], T) for l in range(L - 1)]
    elif selection == "direct":
        sel = [stratified_topk(spyr[l], p * kp[l], T) for l in range(L - 1)]
    else:
        # top down: the candidates of level l+1 are its kept entries, chunked
        # and ranked by position in that ascending list (ties: lower index)
        sel = [None] * (L - 1)
        kept = np.arange(N // p ** (L - 1), dtype=np.int64)
        for lvl in range(L - 2, -1, -1):
            pos = stratified_topk(spyr[lvl + 1][kept], kp[lvl], T)
            sel[lvl] = kept[pos]
            kept = (sel[lvl][:, None] * p + np.arange(p)[None, :]).reshape(-1)
    return sel, spyr


def selected_entries(sel, N: int, p: int, L: int, selection: str = "parents") -> list[np.ndarray]:
    """Entries kept at every level: for l < L-1 the p children of each kept
    parent (parents, nested) or the kept entries themselves (direct); and the
    whole top level (LH-post Key formulas: the first term of S is the top
    level, kept entirely)."""
    out = []
    for l in range(L - 1):
        kept = np.asarray(sel[l], np.int64)
        if selection != "direct":
            kept = (kept[:, None] * p + np.arange(p)[None, :]).reshape(-1)
        out.append(kept)
    out.append(np.arange(N // p ** (L - 1), dtype=np.int64))
    return out


# ----------------------------------------------------------------------------
# 4. gather into a causally ordered sequence (LH-post How it works (3))
# ----------------------------------------------------------------------------

def causal_order(entries, p: int):
    """Sort all kept entries by (e ascending, level descending), e = (i+1)p^l - 1
    (reading R5).  Returns (seq_level, seq_index), each of length S."""
    lv = np.concatenate([np.full(len(e), l, np.int64) for l, e in enumerate(entries)])
    ix = np.concatenate([np.asarray(e, np.int64) for e in entries])
    last = (ix + 1) * (np.int64(p) ** lv) - 1
    order = np.lexsort((-lv, last))
    return lv[order], ix[order]


def slot_table(seq_level, seq_index, N: int, p: int, L: int) -> list[np.ndarray]:
    """slot_of[l][i] = position of entry (l,i) in the sequence, -1 if not kept."""
    tables = [np.full(n, -1, np.int64) for n in level_lengths(N, p, L)]
    for s, (l, i) in enumerate(zip(seq_level, seq_index)):
        tables[int(l)][int(i)] = s
    return tables


def gather(levels, seq_level, seq_index) -> np.ndarray:
    """Row s of the sequence is the pyramid entry (seq_level[s], seq_index[s])."""
    d = levels[0].shape[1]
    out = np.empty((len(seq_level), d), np.float64)
    for s, (l, i) in enumerate(zip(seq_level, seq_index)):
        out[s] = levels[int(l)][int(i)]
    return out


# ----------------------------------------------------------------------------
# 5. dense causal softmax attention on the sequence (LH-summary Technical details (3))
# ----------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (8 significant bits), ties to even,
    straight from float64 (reading R11).  Exact for the normal bf16 range
    (|x| >= 2^-126); the layer's values never come near it."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)  # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


ROW_BLOCK = 512  # rows are independent; blocks only bound memory


def causal_attention(Qs, Ks, Vs):
    """O = softmax(Qs Ks^T / sqrt(d) + causal mask) Vs, with an explicit softmax
    per row; also returns LSE_t = log sum_{u<=t} exp(q_t.k_u / sqrt(d)).
    Columns u > t hold exact zeros in P and are not computed."""
    S, d = Qs.shape
    scale = 1.0 / np.sqrt(d)
    O = np.empty((S, Vs.shape[1]), np.float64)
    lse = np.empty(S, np.float64)
    for r0 in range(0, S, ROW_BLOCK):
        r1 = min(S, r0 + ROW_BLOCK)
        logits = scale * (Qs[r0:r1] @ Ks[:r1].T)
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(r1)[None, :]
        logits = np.where(cols <= rows, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        z = e.sum(axis=1, keepdims=True)
        O[r0:r1] = (e / z) @ Vs[:r1]
        lse[r0:r1] = (m + np.log(z))[:, 0]
    return O, lse


# ----------------------------------------------------------------------------
# 6. scatter-back (LH-summary Technical details (4); LH-post How it works (4))
# ----------------------------------------------------------------------------

def shifted_range(l: int, i: int, p: int, N: int) -> tuple[int, int]:
    """R(l,i) = [(i+1)p^l - 1, (i+2)p^l - 1) clipped to [0, N) (reading R7)."""
    b = p ** l
    return min(N, (i + 1) * b - 1), min(N, (i + 2) * b - 1)


def scatter_back(Os, seq_level, seq_index, N: int, p: int, L: int) -> np.ndarray:
    """Every slot adds its output row to each position of its shifted range;
    contributions are summed level by level, l = 0 first."""
    Y = np.zeros((N, Os.shape[1]), np.float64)
    for l in range(L):
        for s in np.nonzero(seq_level == l)[0]:
            a, b = shifted_range(l, int(seq_index[s]), p, N)
            Y[a:b] += Os[s]
    return Y


# ----------------------------------------------------------------------------
# forward for one head
# ----------------------------------------------------------------------------

def forward_head(Q, K, V, p: int, L: int, k: int, T: int = DEFAULT_CHUNK, scorer: str = "qk_sum",
                 sel=None, attn_dtype="bf16", selection: str = "parents"):
    """One head of the layer.  Returns (Y, saved) with everything the backward
    and the parity tests need.  ``sel`` freezes the selection (used by the
    causality and finite-difference checks); by default it is computed.
    ``attn_dtype`` = "bf16" rounds the attention inputs (reading R11); None
    keeps them exact.  ``selection`` is the reading of C2 (see SELECTIONS)."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    N = Q.shape[0]
    pq, pk, pv = (pyramid_pool(X, p, L) for X in (Q, K, V))
    if sel is None:
        sel, spyr = select(Q, K, p, L, k, T, scorer, selection)
    else:
        spyr = None
    seq_level, seq_index = causal_order(selected_entries(sel, N, p, L, selection), p)
    Qs, Ks, Vs = gather(pq, seq_level, seq_index), gather(pk, seq_level, seq_index), gather(pv, seq_level, seq_index)
    if attn_dtype == "bf16":
        Qs, Ks, Vs = round_bf16(Qs), round_bf16(Ks), round_bf16(Vs)
    elif attn_dtype is not None:
        raise ValueError(f"unknown attn_dtype {attn_dtype!r}")
    Os, lse = causal_attention(Qs, Ks, Vs)
    Y = scatter_back(Os, seq_level, seq_index, N, p, L)
    saved = dict(N=N, p=p, L=L, k=k, T=T, scorer=scorer, attn_dtype=attn_dtype, selection=selection, sel=sel, spyr=spyr,
                 pyr_q=pq, pyr_k=pk, pyr_v=pv,
                 seq_level=seq_level, seq_index=seq_index,
                 slot_of=slot_table(seq_level, seq_index, N, p, L),
                 Qs=Qs, Ks=Ks, Vs=Vs, Os=Os, lse=lse)
    return Y, saved


# ----------------------------------------------------------------------------
# 7. backward by hand-derived adjoints (LH-summary Method step 5: gradients run
#    back through scatter, gather and the attention; none reaches the indices)
# ----------------------------------------------------------------------------

def scatter_adjoint(dY, seq_level, seq_index, N: int, p: int) -> np.ndarray:
    """Adjoint of scatter_back: dOs[s] = sum of dY_j over j in R(l,i), ascending j."""
    dOs = np.zeros((len(seq_level), dY.shape[1]), np.float64)
    for s, (l, i) in enumerate(zip(seq_level, seq_index)):
        a, b = shifted_range(int(l), int(i), p, N)
        if b > a:
            dOs[s] = dY[a:b].sum(axis=0)
    return dOs


def causal_attention_backward(Qs, Ks, Vs, dOs):
    """Adjoint of causal_attention for fixed inputs, recomputing P per row:
        dV = P^T dO;  dP = dO V^T;  dZ = P * (dP - rowsum(P * dP));
        dQ = dZ K / sqrt(d);  dK = dZ^T Q / sqrt(d)."""
    S, d = Qs.shape
    scale = 1.0 / np.sqrt(d)
    dQ = np.zeros_like(Qs)
    dK = np.zeros_like(Ks)
    dV = np.zeros_like(Vs)
    for r0 in range(0, S, ROW_BLOCK):
        r1 = min(S, r0 + ROW_BLOCK)
        logits = scale * (Qs[r0:r1] @ Ks[:r1].T)
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(r1)[None, :]
        logits = np.where(cols <= rows, logits, -np.inf)
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        P = e / e.sum(axis=1, keepdims=True)
        dP = dOs[r0:r1] @ Vs[:r1].T
        dZ = P * (dP - np.sum(P * dP, axis=1, keepdims=True))
        dV[:r1] += P.T @ dOs[r0:r1]
        dQ[r0:r1] = scale * (dZ @ Ks[:r1])
        dK[:r1] += scale * (dZ.T @ Qs[r0:r1])
    return dQ, dK, dV


def gather_adjoint(dXs, seq_level, seq_index, N: int, p: int, L: int) -> list[np.ndarray]:
    """Adjoint of gather: slot gradients go back to their pyramid entries;
    entries that were not kept get zero."""
    d = dXs.shape[1]
    levels = [np.zeros((n, d), np.float64) for n in level_lengths(N, p, L)]
    for s, (l, i) in enumerate(zip(seq_level, seq_index)):
        levels[int(l)][int(i)] += dXs[s]
    return levels


def pyramid_pool_adjoint(dlevels, p: int) -> np.ndarray:
    """Adjoint of pyramid_pool: going down one level, every child receives 1/p
    of its parent's gradient, added to its own."""
    acc = dlevels[-1]
    for l in range(len(dlevels) - 2, -1, -1):
        n, d = acc.shape
        child = np.array(dlevels[l], dtype=np.float64).reshape(n, p, d)
        child += (acc / p)[:, None, :]
        acc = child.reshape(n * p, d)
    return acc


def backward_head(dY, saved):
    """dQ, dK, dV of one head for upstream gradient dY (selection held fixed)."""
    dY = np.asarray(dY, np.float64)
    N, p, L = saved["N"], saved["p"], saved["L"]
    sl, si = saved["seq_level"], saved["seq_index"]
    dOs = scatter_adjoint(dY, sl, si, N, p)
    if saved.get("attn_dtype") == "bf16":
        dOs = round_bf16(dOs)
    dQs, dKs, dVs = causal_attention_backward(saved["Qs"], saved["Ks"], saved["Vs"], dOs)
    grads = [pyramid_pool_adjoint(gather_adjoint(g, sl, si, N, p, L), p) for g in (dQs, dKs, dVs)]
    return grads[0], grads[1], grads[2], dict(dOs=dOs, dQs=dQs, dKs=dKs, dVs=dVs)


# ----------------------------------------------------------------------------
# several heads: [BH, N, d], selection per head (reading R9)
# ----------------------------------------------------------------------------

def forward(Q, K, V, p: int, L: int, k: int, T: int = DEFAULT_CHUNK, scorer: str = "qk_sum", attn_dtype="bf16",
            selection: str = "parents"):
    Ys, saves = [], []
    for h in range(Q.shape[0]):
        Y, sv = forward_head(Q[h], K[h], V[h], p, L, k, T, scorer, attn_dtype=attn_dtype, selection=selection)
        Ys.append(Y)
        saves.append(sv)
    return np.stack(Ys), saves


def backward(dY, saves):
    outs = [backward_head(dY[h], sv) for h, sv in enumerate(saves)]
    return (np.stack([o[0] for o in outs]), np.stack([o[1] for o in outs]),
            np.stack([o[2] for o in outs]), [o[3] for o in outs])
