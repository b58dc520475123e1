"""Context parallelism for one Lighthouse layer: the host logic that splits the
N tokens of every head over W ranks and exchanges what crosses a shard.

The pages train at 1M tokens with context parallelism on one 8-GPU node
(aitrends.kr summary of Lighthouse Attention, Method step 6 and Limitations).
This module plans and drives that split; the per-rank arithmetic is done by a
stage backend (the CUDA library on a GPU), so every piece here is shape and
index bookkeeping plus torch.distributed collectives.

Partition (each rank r owns tokens [t0, t1) = [r N/W, (r+1) N/W)):
  * N/W must be a multiple of p^(L-1), so every pyramid level tiles each shard
    and a shard pools its own levels with no exchange.
  * Selection reads every score: the level-0 norms are all-gathered (2 floats
    per token) and every rank runs the same global top-k, so all ranks hold
    the same selection and it equals the unsharded one bit for bit.
  * An entry (l, i) has key e = (i+1) p^l - 1 inside the shard that pools it,
    and the sequence is sorted by key, so a shard's kept entries form one
    contiguous segment [off_r, off_r + S_r) of the gathered sequence.  Each
    rank gathers its own segment.
  * The causal attention over S needs every earlier key: the segments of Qs,
    Ks, Vs (and for the backward dOs, LSE, Delta) are all-gathered, and each
    rank computes a window of rows chosen so the causal work is balanced
    (query tile t costs t+1 key tiles; key tile t costs n_tiles - t query
    tiles).  The windows' outputs are all-gathered back so each rank reads the
    rows of its own segment.
  * Halo.  R(l, i) = [e, e + p^l) starts in the entry's own shard and can run
    into the next one: for l >= 1 exactly the entry (l, t1/p^l - 1), whose
    e = t1 - 1, covers the next shard's first p^l - 1 tokens.  Forward: each
    rank adds the Os rows of the previous shard's kept boundary entries to its
    first p^l - 1 rows of Y.  Backward: each rank publishes the sums of dY over
    its first p^l - 1 tokens, and the previous rank adds them to its boundary
    entries' dOs before rounding (and before Delta).

Backend interface (one object per rank; tensors are [BH, ...] per shard):
  pool(q, k, v) -> (levels, norms)             levels: the shard's pyramid; norms [2, BH, n]
  select(norms) -> sel                          global selection from [2, BH, N] norms
  gather(q, k, v, levels, sel_local) -> (seq, (qs, ks, vs))
                                                seq: per head (level, index) of the shard's
                                                segment in causal order (local indices)
  attention(qs, ks, vs, lo, hi) -> (os, lse)    rows [lo, hi) of the causal attention
  scatter(os_seg, seq) -> y                     the shard's Y without the halo
  halo_add_y(y, h, rows, row)                   add one Os row to Y[h, 0:rows]
  scatter_adjoint(dy, seq) -> dos               unrounded sums of dY over each entry's range
                                                inside the shard
  finish_dos(dos, os_seg) -> (dos, delta)       rounding of dOs and Delta = rowsum(dOs * Os)
  attention_bwd_kv(qs, ks, vs, lse, dos, delta, lo, hi) -> (dks, dvs)  key rows [lo, hi)
  attention_bwd_q(qs, ks, vs, lse, dos, delta, lo, hi) -> dqs           query rows [lo, hi)
  pool_adjoint(dqs, dks, dvs, seq) -> (dq, dk, dv)
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

TILE = 128  # rows of an attention tile: windows are tile-aligned


# ---------------------------------------------------------------- partition

@dataclass(frozen=True)
class Shard:
    N: int
    p: int
    L: int
    world: int
    rank: int

    def __post_init__(self):
        check_shardable(self.N, self.p, self.L, self.world)
        if not 0 <= self.rank < self.world:
            raise ValueError("rank outside [0, world)")

    @property
    def n(self) -> int:
        return self.N // self.world

    @property
    def t0(self) -> int:
        return self.rank * self.n

    @property
    def t1(self) -> int:
        return self.t0 + self.n

    def level_range(self, l: int) -> tuple[int, int]:
        """Entries of level l pooled inside this shard."""
        b = self.p ** l
        return self.t0 // b, self.t1 // b


def check_shardable(N: int, p: int, L: int, world: int) -> None:
    if world < 1 or N % world:
        raise ValueError(f"N={N} is not divisible by world={world}")
    if (N // world) % (p ** (L - 1)):
        raise ValueError(f"N/world={N // world} is not a multiple of p^(L-1)={p ** (L - 1)}: "
                         "a top-level block would straddle two shards")


def kept_entries(sel, N: int, p: int, L: int, selection: str = "parents") -> list[np.ndarray]:
    """Kept entry indices of every level (ascending) from one head's selection:
    the p children of each kept parent (or the listed entries, direct) and the
    whole top level."""
    out = []
    for l in range(L - 1):
        s = np.asarray(sel[l], np.int64)
        out.append(s if selection == "direct" else (s[:, None] * p + np.arange(p)[None, :]).reshape(-1))
    out.append(np.arange(N // p ** (L - 1), dtype=np.int64))
    return out


def segment_counts(kept, N: int, p: int, L: int, world: int) -> np.ndarray:
    """S_r: kept entries pooled inside each shard (their keys lie in it)."""
    n = N // world
    counts = np.zeros(world, np.int64)
    for l in range(L):
        b = p ** l
        edges = np.arange(world + 1, dtype=np.int64) * (n // b)
        counts += np.diff(np.searchsorted(kept[l], edges))
    return counts


def local_selection(sel, shard: Shard, selection: str = "parents") -> list[np.ndarray]:
    """The shard's part of one head's selection, in shard-local indices: kept
    parents at level l+1 (or kept level-l entries, direct) inside the shard."""
    out = []
    for l in range(shard.L - 1):
        s = np.asarray(sel[l], np.int64)
        lv = l if selection == "direct" else l + 1
        a, b = shard.level_range(lv)
        out.append(s[(s >= a) & (s < b)] - a)
    return out


def global_slot(kept, l: int, i: int, p: int) -> int:
    """Position of kept entry (l, i) in the causal order: the kept entries of
    every level with a smaller key (e, -l)."""
    e = (i + 1) * p ** l - 1
    slot = 0
    for lv, ent in enumerate(kept):
        b = p ** lv
        # keys (e', -lv) < (e, -l): e' < e, or e' == e and lv > l
        lim = (e + 1) // b if lv > l else (e // b if lv < l else i)
        if lv == l:
            slot += int(np.searchsorted(ent, i))
        else:
            slot += int(np.searchsorted(ent, lim))
    return slot


def halo_in(kept, shard: Shard) -> list[tuple[int, int, int]]:
    """Entries of the previous shard whose ranges run into this one, as
    (level, global slot, rows covered here): for l >= 1 the kept entry
    (l, t0/p^l - 1), covering this shard's first p^l - 1 rows."""
    if shard.rank == 0:
        return []
    out = []
    for l in range(1, shard.L):
        i = shard.t0 // shard.p ** l - 1
        ent = kept[l]
        j = int(np.searchsorted(ent, i))
        if j < len(ent) and ent[j] == i:
            out.append((l, global_slot(kept, l, i, shard.p), shard.p ** l - 1))
    return out


def halo_out_entries(seq_level, seq_index, shard: Shard) -> list[tuple[int, int]]:
    """This shard's kept boundary entries (l >= 1, local index n/p^l - 1) as
    (level, local slot); the next shard's first p^l - 1 dY rows belong to them."""
    out = []
    if shard.rank == shard.world - 1:
        return out
    for s, (l, i) in enumerate(zip(seq_level, seq_index)):
        l, i = int(l), int(i)
        if l >= 1 and i == shard.n // shard.p ** l - 1:
            out.append((l, s))
    return out


def balanced_windows(S: int, world: int, kind: str = "query") -> list[tuple[int, int]]:
    """Tile-aligned row windows [lo, hi) covering [0, S) whose causal work is
    about equal: query tile t costs t+1 key tiles (forward, dQ); key tile t
    costs n_tiles - t query tiles (dK, dV)."""
    nt = (S + TILE - 1) // TILE
    t = np.arange(nt)
    cost = (t + 1) if kind == "query" else (nt - t)
    cum = np.concatenate([[0], np.cumsum(cost)])
    total = cum[-1]
    cuts = [0]
    for r in range(1, world):
        target = total * r / world
        i = int(np.searchsorted(cum, target))  # first cut at or past the target
        if i > 0 and target - cum[i - 1] < cum[min(i, nt)] - target:
            i -= 1  # the nearer of the two tile boundaries
        cuts.append(i)
    cuts.append(nt)
    cuts = np.maximum.accumulate(np.minimum(np.array(cuts), nt))
    return [(int(min(S, cuts[r] * TILE)), int(min(S, cuts[r + 1] * TILE))) for r in range(world)]


# ---------------------------------------------------------------- exchanges

def allgather_cat(x: torch.Tensor, dim: int, group=None) -> torch.Tensor:
    """Equal-sized pieces, concatenated in rank order along `dim`."""
    import torch.distributed as dist
    parts = [torch.empty_like(x) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.cat(parts, dim=dim)


def allgather_rows(x: torch.Tensor, counts, group=None) -> torch.Tensor:
    """Pieces of `counts[r]` rows along dim 1 (padded to the largest for the
    collective), concatenated in rank order: [BH, sum(counts), ...]."""
    import torch.distributed as dist
    mx = int(max(counts))
    pad = torch.zeros((x.shape[0], mx) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
    pad[:, :x.shape[1]] = x
    parts = [torch.empty_like(pad) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:, :int(c)] for p, c in zip(parts, counts)], dim=1)


# ---------------------------------------------------------------- driver

@dataclass
class CpContext:
    """What the backward needs from the forward on one rank."""
    seq: list                # per head: (seq_level, seq_index) of the segment, local indices
    kept: list               # per head: global kept entries per level
    counts: np.ndarray       # [world, BH]: segment lengths
    off: np.ndarray          # [BH]: this rank's segment start
    qs: torch.Tensor         # all-gathered sequence tensors [BH, S, d]
    ks: torch.Tensor
    vs: torch.Tensor
    os: torch.Tensor         # [BH, S, d]
    lse: torch.Tensor        # [BH, S]


def _segment_rows(full: torch.Tensor, off, counts_r) -> torch.Tensor:
    """Rows [off_h, off_h + S_r,h) of every head (same count for every head is
    not assumed: heads are padded to the largest with zeros)."""
    mx = int(max(counts_r))
    out = torch.zeros((full.shape[0], mx) + tuple(full.shape[2:]), dtype=full.dtype, device=full.device)
    for h in range(full.shape[0]):
        out[h, :int(counts_r[h])] = full[h, int(off[h]):int(off[h]) + int(counts_r[h])]
    return out


def cp_forward(backend, shard: Shard, q, k, v, selection: str = "parents", group=None):
    """Forward of this rank's shard.  q, k, v: [BH, n, d] (the shard's tokens).
    Returns (y [BH, n, d], CpContext)."""
    BH = q.shape[0]
    N, p, L, W, r = shard.N, shard.p, shard.L, shard.world, shard.rank
    levels, norms = backend.pool(q, k, v)
    sel = backend.select(allgather_cat(norms, dim=-1, group=group))  # same on every rank
    kept = [kept_entries(sel[h], N, p, L, selection) for h in range(BH)]
    counts = np.stack([segment_counts(kept[h], N, p, L, W) for h in range(BH)], axis=1)  # [W, BH]
    off = counts[:r].sum(axis=0)
    sel_loc = [local_selection(sel[h], shard, selection) for h in range(BH)]
    seq, (qs_r, ks_r, vs_r) = backend.gather(q, k, v, levels, sel_loc)
    # the whole sequence on every rank (heads differ in S_r: gathered per head)
    full = []
    for t in (qs_r, ks_r, vs_r):
        full.append(torch.stack([allgather_rows(t[h:h + 1, :int(counts[r, h])], counts[:, h], group)[0]
                                 for h in range(BH)]))
    qs, ks, vs = full
    S = qs.shape[1]
    lo, hi = balanced_windows(S, W, "query")[r]
    os_w, lse_w = backend.attention(qs, ks, vs, lo, hi)
    win = [b - a for a, b in balanced_windows(S, W, "query")]
    os_f = allgather_rows(os_w, win, group)
    lse_f = allgather_rows(lse_w[..., None], win, group)[..., 0]
    y = backend.scatter(_segment_rows(os_f, off, counts[r]), seq)
    for h in range(BH):
        for l, slot, rows in halo_in(kept[h], shard):
            backend.halo_add_y(y, h, rows, os_f[h, slot])
    ctx = CpContext(seq=seq, kept=kept, counts=counts, off=off, qs=qs, ks=ks, vs=vs, os=os_f, lse=lse_f)
    return y, ctx


def cp_backward(backend, shard: Shard, dy, ctx: CpContext, group=None):
    """Backward of this rank's shard.  dy: [BH, n, d].  Returns dq, dk, dv [BH, n, d]."""
    BH = dy.shape[0]
    W, r, p, L = shard.world, shard.rank, shard.p, shard.L
    # halo: sums of dY over this shard's first p^l - 1 tokens, for the previous shard
    heads = torch.stack([dy[:, :p ** l - 1].sum(dim=1) for l in range(1, L)], dim=1) if L > 1 else \
        torch.zeros((BH, 0, dy.shape[2]), dtype=dy.dtype, device=dy.device)
    heads_all = allgather_cat(heads[None], dim=0, group=group)  # [W, BH, L-1, d]
    dos = backend.scatter_adjoint(dy, ctx.seq)
    if r + 1 < W:
        for h in range(BH):
            lv, ix = ctx.seq[h]
            for l, s in halo_out_entries(lv, ix, shard):
                dos[h, s] += heads_all[r + 1, h, l - 1]
    dos, delta = backend.finish_dos(dos, _segment_rows(ctx.os, ctx.off, ctx.counts[r]))
    dos_f = torch.stack([allgather_rows(dos[h:h + 1, :int(ctx.counts[r, h])], ctx.counts[:, h], group)[0]
                         for h in range(BH)])
    delta_f = torch.stack([allgather_rows(delta[h:h + 1, :int(ctx.counts[r, h]), None], ctx.counts[:, h],
                                          group)[0, :, 0] for h in range(BH)])
    S = ctx.qs.shape[1]
    klo, khi = balanced_windows(S, W, "key")[r]
    qlo, qhi = balanced_windows(S, W, "query")[r]
    dks_w, dvs_w = backend.attention_bwd_kv(ctx.qs, ctx.ks, ctx.vs, ctx.lse, dos_f, delta_f, klo, khi)
    dqs_w = backend.attention_bwd_q(ctx.qs, ctx.ks, ctx.vs, ctx.lse, dos_f, delta_f, qlo, qhi)
    kwin = [b - a for a, b in balanced_windows(S, W, "key")]
    qwin = [b - a for a, b in balanced_windows(S, W, "query")]
    dks = _segment_rows(allgather_rows(dks_w, kwin, group), ctx.off, ctx.counts[r])
    dvs = _segment_rows(allgather_rows(dvs_w, kwin, group), ctx.off, ctx.counts[r])
    dqs = _segment_rows(allgather_rows(dqs_w, qwin, group), ctx.off, ctx.counts[r])
    return backend.pool_adjoint(dqs, dks, dvs, ctx.seq)
