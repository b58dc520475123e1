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
    Ks, Vs (and for the backward dOs, Delta) are all-gathered, and each
    rank computes a window of rows chosen so the causal work is balanced
    (query tile t costs t+1 key tiles; key tile t costs n_tiles - t query
    tiles).  The windows' outputs go back point to point: each rank receives
    only the rows of its own segment (and, for Os, its halo rows) from the
    ranks whose windows hold them; LSE, which every window's backward reads,
    is all-gathered.
  * Halo.  R(l, i) = [e, e + p^l) starts in the entry's own shard and can run
    into the next one: for l >= 1 exactly the entry (l, t1/p^l - 1), whose
    e = t1 - 1, covers the next shard's first p^l - 1 tokens.  Forward: each
    rank adds the Os rows of the previous shard's kept boundary entries to its
    first p^l - 1 rows of Y.  Backward: each rank publishes the sums of dY over
    its first p^l - 1 tokens, and the previous rank adds them to its boundary
    entries' dOs before rounding (and before Delta).

Backend interface (one object per rank; tensors are [BH, ...] per shard):
  pool(q, k, v) -> (levels, norms)             levels: the shard's pyramid; norms [2, BH, n]
  select(norms) -> sel                          global selection from [2, BH, N] norms, as per
                                                head and level lists of kept parents (or entries)
  gather(q, k, v, levels, sel_local) -> (seq, (qs, ks, vs))
                                                seq: per head (level, index) of the shard's
                                                segment in causal order (local indices)
  attention(qs, ks, vs, lo, hi) -> (os, lse)    rows [lo, hi) of the causal attention
  scatter(os_seg, seq, halo) -> y              the shard's Y; halo: per head the previous
                                                shard's kept boundary entries (level, Os row
                                                [d], rows), summed into the first rows
  head_sums(dy) -> [BH, L-1, d]                 sums of dY over the shard's first p^l - 1 rows
  scatter_adjoint(dy, seq, os_seg, nxt) -> (dos, delta)
                                                dOs over each entry's range inside the shard,
                                                plus nxt[h, l-1] (the next shard's head_sums,
                                                None on the last shard) for the boundary
                                                entries, rounded; Delta = rowsum(dOs * Os)
  attention_bwd_kv(qs, ks, vs, lse, dos, delta, lo, hi) -> (dks, dvs)  key rows [lo, hi)
  attention_bwd_q(qs, ks, vs, lse, dos, delta, lo, hi) -> dqs           query rows [lo, hi)
  pool_adjoint(dqs, dks, dvs, seq) -> (dq, dk, dv)
The driver itself only moves rows (all-gathers, segment copies) and keeps the
index bookkeeping; all arithmetic is in the backend.
"""

from __future__ import annotations

import ctypes

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

# the exchanges of one layer, in the order the driver issues them: all-gathers
# (norms, qkv, lse, head_sums, dos, delta) and point-to-point row moves from
# the attention windows to the segments (os, dkv, dq)
EXCHANGES = ("norms", "qkv", "os", "lse", "head_sums", "dos", "delta", "dkv", "dq")
# element sizes under the CUDA backend: fp32 norms, bf16 Qs|Ks|Vs, fp32 Os,
# LSE, head sums and Delta, fp16 dOs (bf16 values), fp32 gradients
CUDA_ELEMENT_BYTES = dict(norms=4, qkv=2, os=4, lse=4, head_sums=4, dos=2, delta=4, dkv=4, dq=4)
# when a list, every exchange appends the elements this rank received
EXCHANGE_LOG: list | None = None


def _log(n: int) -> None:
    if EXCHANGE_LOG is not None:
        EXCHANGE_LOG.append(int(n))


def segment_rows(counts: np.ndarray, rank: int) -> list[np.ndarray]:
    """Per head, the sequence rows of a rank's segment."""
    off = counts[:rank].sum(axis=0)
    return [np.arange(off[h], off[h] + counts[rank, h], dtype=np.int64) for h in range(counts.shape[1])]


def os_rows_needed(kept, counts: np.ndarray, shard: "Shard") -> list[np.ndarray]:
    """Per head, the Os rows a rank reads: its segment, then the previous
    shard's kept boundary entries (halo_in order)."""
    seg = segment_rows(counts, shard.rank)
    return [np.concatenate([seg[h], np.array([slot for _, slot, _ in halo_in(kept[h], shard)], np.int64)])
            for h in range(counts.shape[1])]


def exchange_elements(BH: int, N: int, d: int, L: int, S: int, world: int, rank: int, counts: np.ndarray,
                      os_need) -> dict:
    """Elements one rank receives in each exchange of a layer (forward and
    backward).  counts: [world, BH] segment lengths; os_need: this rank's
    os_rows_needed.  An all-gather brings world - 1 pieces padded to the
    longest piece; a row move brings the needed rows that lie outside this
    rank's own window."""
    seg_rows = max(1, int(counts.max()))
    qwin, kwin = balanced_windows(S, world, "query"), balanced_windows(S, world, "key")

    def outside(rows, win):
        lo, hi = win[rank]
        return sum(int(((r < lo) | (r >= hi)).sum()) for r in rows)

    seg = segment_rows(counts, rank)
    wq = max(b - a for a, b in qwin)
    out = dict(norms=(world - 1) * 2 * BH * (N // world), qkv=(world - 1) * BH * seg_rows * 3 * d,
               os=outside(os_need, qwin) * d, lse=(world - 1) * BH * wq)
    if L > 1:
        out["head_sums"] = (world - 1) * BH * (L - 1) * d
    out.update(dos=(world - 1) * BH * seg_rows * d, delta=(world - 1) * BH * seg_rows,
               dkv=outside(seg, kwin) * 2 * d, dq=outside(seg, qwin) * d)
    return out


def _all_gather(parts, x: torch.Tensor, group=None) -> None:
    """dist.all_gather; CUDA tensors go through host copies when the group's
    backend is gloo (which gathers host memory), e.g. ranks sharing one GPU in
    a test."""
    import torch.distributed as dist
    _log((len(parts) - 1) * x.numel())
    if x.is_cuda and dist.get_backend(group) == "gloo":
        host = [torch.empty(x.shape, dtype=x.dtype) for _ in parts]
        dist.all_gather(host, x.cpu(), group=group)
        for p, h in zip(parts, host):
            p.copy_(h)
    else:
        dist.all_gather(parts, x, group=group)


def allgather_cat(x: torch.Tensor, dim: int, group=None) -> torch.Tensor:
    """Equal-sized pieces, concatenated in rank order along `dim`."""
    import torch.distributed as dist
    parts = [torch.empty_like(x) for _ in range(dist.get_world_size(group))]
    _all_gather(parts, x.contiguous(), group=group)
    return torch.cat(parts, dim=dim)


def allgather_rows(x: torch.Tensor, counts, group=None) -> torch.Tensor:
    """Pieces of `counts[r]` rows along dim 1 (padded to the largest for the
    collective), concatenated in rank order: [BH, sum(counts), ...]."""
    import torch.distributed as dist
    mx = int(max(counts))
    pad = torch.zeros((x.shape[0], mx) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
    pad[:, :x.shape[1]] = x
    parts = [torch.empty_like(pad) for _ in range(dist.get_world_size(group))]
    _all_gather(parts, pad, group=group)
    return torch.cat([p[:, :int(c)] for p, c in zip(parts, counts)], dim=1)


def segment_index(counts: np.ndarray, mx: int) -> np.ndarray:
    """Where each head's sequence rows sit once every rank's segments are
    gathered as one [W, BH, mx] block of rows: for head h and sequence row s,
    the flat row r*BH*mx + h*mx + j of segment row j of rank r.  [BH, S]."""
    W, BH = counts.shape
    return np.stack([np.concatenate([r * BH * mx + h * mx + np.arange(int(counts[r, h]), dtype=np.int64)
                                     for r in range(W)]) for h in range(BH)])


def allgather_segments(x: torch.Tensor, counts: np.ndarray, group=None) -> torch.Tensor:
    """The whole sequence of every head from each rank's segments, in one
    collective.  x on rank r: [BH, >= counts[r, h], ...], rows past a head's
    count ignored; counts: [W, BH], every head's column summing to the same S.
    Returns [BH, S, ...]."""
    import torch.distributed as dist
    W, BH = counts.shape
    mx = max(1, int(counts.max()))
    rest = tuple(x.shape[2:])
    pad = torch.zeros((BH, mx) + rest, dtype=x.dtype, device=x.device)
    m = min(mx, x.shape[1])
    pad[:, :m] = x[:, :m]
    parts = [torch.empty_like(pad) for _ in range(dist.get_world_size(group))]
    _all_gather(parts, pad, group=group)
    idx = torch.from_numpy(segment_index(counts, mx)).to(x.device)
    return torch.stack(parts).reshape((W * BH * mx,) + rest)[idx.reshape(-1)].reshape((BH, idx.shape[1]) + rest)


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
    os: torch.Tensor         # [BH, max segment, d]: Os rows of this rank's segment
    lse: torch.Tensor        # [BH, S]


def redistribute_rows(x_w: torch.Tensor, windows, need, group=None) -> torch.Tensor:
    """Move the rows of window-distributed tensors to the ranks that read them.
    x_w: this rank's rows [lo, hi) of its window, every head: [BH, hi - lo, ...]
    (windows[rank] = (lo, hi)); need[q][h]: the sequence rows rank q reads of
    head h (every rank passes the same windows and need).  Each rank sends
    each other rank, in one batch of point-to-point transfers, the rows it
    needs from this window, packed head by head, and copies its own.  Returns
    [BH, max_h len(need[rank][h]), ...]: row j of head h holds sequence row
    need[rank][h][j] (zeros past a head's rows)."""
    import torch.distributed as dist
    W, r = dist.get_world_size(group), dist.get_rank(group)
    lo, hi = windows[r]
    BH, rest, dev = x_w.shape[0], tuple(x_w.shape[2:]), x_w.device
    mx = max(1, max(len(n) for n in need[r]))
    out = torch.zeros((BH * mx,) + rest, dtype=x_w.dtype, device=dev)
    src = x_w.contiguous().reshape((BH * (hi - lo),) + rest)

    def inside(rows_of_heads, a, b):  # per head: (positions in the list, rows) inside [a, b)
        return [(np.nonzero((rows >= a) & (rows < b))[0], rows[(rows >= a) & (rows < b)]) for rows in rows_of_heads]

    def index(parts, row_of):  # flat indices, head by head
        return torch.from_numpy(np.concatenate([row_of(h, j, rows) for h, (j, rows) in enumerate(parts)]
                                               + [np.zeros(0, np.int64)]).astype(np.int64)).to(dev)

    def src_index(parts):  # rows of this window
        return index(parts, lambda h, j, rows: h * (hi - lo) + (rows - lo))

    def dst_index(parts):  # positions in this rank's list
        return index(parts, lambda h, j, rows: h * mx + j)

    own = inside(need[r], lo, hi)
    if sum(len(j) for j, _ in own):
        out[dst_index(own)] = src[src_index(own)]
    # gloo moves host memory: stage through it (ranks sharing a GPU in a test)
    stage = torch.device("cpu") if dist.get_backend(group) == "gloo" else dev
    ops, recvs = [], []
    for q in range(W):
        if q == r:
            continue
        peer = q if group is None else dist.get_global_rank(group, q)
        send = inside(need[q], lo, hi)
        if sum(len(j) for j, _ in send):
            ops.append(dist.P2POp(dist.isend, src[src_index(send)].to(stage), peer, group))
        recv = inside(need[r], *windows[q])
        n = sum(len(j) for j, _ in recv)
        if n:
            buf = torch.empty((n,) + rest, dtype=x_w.dtype, device=stage)
            ops.append(dist.P2POp(dist.irecv, buf, peer, group))
            recvs.append((buf, dst_index(recv)))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    _log(sum(b.numel() for b, _ in recvs))
    for buf, idx in recvs:
        out[idx] = buf.to(dev)
    return out.reshape((BH, mx) + rest)


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
    # the whole sequence on every rank: one collective for Qs, Ks and Vs of all heads
    qkv = allgather_segments(torch.stack((qs_r, ks_r, vs_r), dim=2), counts, group)
    qs, ks, vs = (qkv[:, :, t].contiguous() for t in range(3))
    S = qs.shape[1]
    qwin = balanced_windows(S, W, "query")
    lo, hi = qwin[r]
    os_w, lse_w = backend.attention(qs, ks, vs, lo, hi)
    # Os rows go to the ranks that read them (their segments and halo rows);
    # LSE, read by every window of the backward, to every rank
    need = [os_rows_needed(kept, counts, Shard(N, p, L, W, q_)) for q_ in range(W)]
    os_need = redistribute_rows(os_w, qwin, need, group)
    lse_f = allgather_rows(lse_w[..., None], [b - a for a, b in qwin], group)[..., 0]
    mxs = int(counts[r].max())
    os_seg = os_need[:, :mxs].clone()
    os_seg[torch.from_numpy(np.arange(mxs)[None, :] >= counts[r][:, None]).to(os_seg.device)] = 0
    halo = [[(l, os_need[h, int(counts[r, h]) + i], rows) for i, (l, _, rows) in enumerate(halo_in(kept[h], shard))]
            for h in range(BH)]
    y = backend.scatter(os_seg, seq, halo)
    ctx = CpContext(seq=seq, kept=kept, counts=counts, off=off, qs=qs, ks=ks, vs=vs, os=os_seg, lse=lse_f)
    return y, ctx


def cp_backward(backend, shard: Shard, dy, ctx: CpContext, group=None):
    """Backward of this rank's shard.  dy: [BH, n, d].  Returns dq, dk, dv [BH, n, d]."""
    W, r, L = shard.world, shard.rank, shard.L
    # halo: sums of dY over this shard's first p^l - 1 tokens, for the previous shard
    nxt = None
    if L > 1:
        heads_all = allgather_cat(backend.head_sums(dy)[None], dim=0, group=group)  # [W, BH, L-1, d]
        nxt = heads_all[r + 1] if r + 1 < W else None
    dos, delta = backend.scatter_adjoint(dy, ctx.seq, ctx.os, nxt)
    dos_f = allgather_segments(dos, ctx.counts, group)
    delta_f = allgather_segments(delta, ctx.counts, group)
    S = ctx.qs.shape[1]
    klo, khi = balanced_windows(S, W, "key")[r]
    qlo, qhi = balanced_windows(S, W, "query")[r]
    dks_w, dvs_w = backend.attention_bwd_kv(ctx.qs, ctx.ks, ctx.vs, ctx.lse, dos_f, delta_f, klo, khi)
    dqs_w = backend.attention_bwd_q(ctx.qs, ctx.ks, ctx.vs, ctx.lse, dos_f, delta_f, qlo, qhi)
    # each gradient row goes to the rank whose segment holds it
    seg = [segment_rows(ctx.counts, q_) for q_ in range(W)]
    dkv = redistribute_rows(torch.stack((dks_w, dvs_w), dim=2), balanced_windows(S, W, "key"), seg, group)
    dks, dvs = dkv[:, :, 0].contiguous(), dkv[:, :, 1].contiguous()
    dqs = redistribute_rows(dqs_w, balanced_windows(S, W, "query"), seg, group)
    return backend.pool_adjoint(dqs, dks, dvs, ctx.seq)


# ---------------------------------------------------------------- the CUDA backend

def _contiguous(*ts):
    """Contiguous forms of the tensors, held by the caller until its library
    call has been issued: a pointer taken from a temporary `.contiguous()`
    copy dangles once the copy is freed, and the allocator hands that memory
    to the next copy."""
    return tuple(t.contiguous() for t in ts)


class CudaBackend:
    """The per-rank arithmetic in the library's kernels: the whole-layer stage
    calls on the shard (pool, selection), the shard forms of the gather,
    scatter-back, its adjoint and the pool adjoint (halo rows included), and
    the row-window forms of the attention.  bf16 rows of 128 channels (the
    scatter-back's halo path).  `layer` is the whole layer; tensors are CUDA."""

    def __init__(self, layer, shard: Shard):
        from . import api
        if layer.dtype != "bf16" or layer.d != 128:
            raise ValueError("the CUDA context-parallel backend takes bf16 rows of 128 channels")
        self.api = api
        self.layer = layer
        self.shard = shard
        self.local = api.Layer(layer.B, layer.H, shard.n, layer.d, layer.L, layer.p, layer.k, layer.chunk,
                               layer.dtype, layer.scorer, layer.selection)
        self.info = api.plan(layer)
        self.local_info = api.plan(self.local)

    def _shape4(self, x):
        return x.reshape(self.layer.B, self.layer.H, *x.shape[1:])

    def pool(self, q, k, v):
        pq, pk, pv, norms = self.api.pyramid_pool(self.local, self._shape4(q.contiguous()),
                                                  self._shape4(k.contiguous()), self._shape4(v.contiguous()))
        return (pq, pk, pv), norms

    def select(self, norms):
        self.sel = self.api.score_topk(self.layer, norms.contiguous())
        host = self.sel.cpu().numpy()
        I, L, p = self.info, self.layer.L, self.layer.p
        direct = self.layer.selection == "direct"
        out = []
        for h in range(host.shape[0]):
            per = []
            for l in range(L - 1):
                n = int(I.kprime[l]) * (p if direct else 1)
                per.append(host[h, int(I.sel_off[l]):int(I.sel_off[l]) + n].astype(np.int64))
            out.append(per)
        self.sel_lists = out
        return out

    def gather(self, q, k, v, levels, sel_local):
        from . import _lib
        sh, lay = self.shard, self.layer
        kept = [kept_entries(self.sel_lists[h], lay.N, lay.p, lay.L, lay.selection) for h in range(lay.BH)]
        counts = np.stack([segment_counts(kept[h], lay.N, lay.p, lay.L, sh.world) for h in range(lay.BH)], axis=1)
        self.counts_r = counts[sh.rank]
        self.seg_rows = max(1, int(self.counts_r.max()))
        dev = q.device
        seg_off = torch.from_numpy(counts[:sh.rank].sum(axis=0).astype(np.int64)).to(dev)
        qs, ks, vs = (torch.zeros((lay.BH, self.seg_rows, lay.d), dtype=torch.bfloat16, device=dev) for _ in range(3))
        # rows past a head's segment hold an entry with an empty range
        self.seq_map = torch.full((lay.BH, self.seg_rows), sh.n, dtype=torch.int32, device=dev)
        self.slot_of = torch.empty((lay.BH, self.local_info.pyr_entries), dtype=torch.int32, device=dev)
        pq, pk, pv = levels
        q, k, v = _contiguous(q, k, v)
        p_ = self.api._p
        _lib.call("lh_gather_shard", ctypes.byref(lay.cfg()), ctypes.c_int64(sh.t0), ctypes.c_int64(sh.t1),
                  p_(seg_off), ctypes.c_int64(self.seg_rows), p_(q), p_(k), p_(v), p_(pq), p_(pk), p_(pv),
                  p_(self.sel), p_(qs), p_(ks), p_(vs), p_(self.seq_map), p_(self.slot_of), self.api._stream())
        sm = self.seq_map.cpu().numpy().astype(np.int64)
        seq = [((sm[h, :c] >> 28), (sm[h, :c] & ((1 << 28) - 1))) for h, c in enumerate(self.counts_r)]
        return seq, (qs, ks, vs)

    def attention(self, qs, ks, vs, lo, hi):
        os_, lse = self.api.attn_fwd_rows(self.layer, qs.contiguous(), ks.contiguous(), vs.contiguous(), lo, hi)
        return os_[:, lo:hi], lse[:, lo:hi]

    def scatter(self, os_seg, seq, halo):
        from . import _lib
        lay = self.layer
        hal = torch.zeros((lay.BH, max(lay.L - 1, 1), lay.d), dtype=torch.float32, device=os_seg.device)
        for h, ents in enumerate(halo):
            for l, row, rows in ents:
                hal[h, l - 1] = row
        y = torch.empty((lay.B, lay.H, self.shard.n, lay.d), dtype=torch.bfloat16, device=os_seg.device)
        (os_seg,) = _contiguous(os_seg)
        p_ = self.api._p
        _lib.call("lh_scatter_back_shard", ctypes.byref(self.local.cfg()), ctypes.c_int64(self.seg_rows),
                  p_(os_seg), p_(self.slot_of), p_(hal), p_(y), self.api._stream())
        return y.reshape(lay.BH, self.shard.n, lay.d)

    def head_sums(self, dy):
        from . import _lib
        lay = self.layer
        sums = torch.empty((lay.BH, lay.L - 1, lay.d), dtype=torch.float32, device=dy.device)
        (dy,) = _contiguous(dy)
        _lib.call("lh_head_sums", ctypes.byref(self.local.cfg()), self.api._p(dy), self.api._p(sums),
                  self.api._stream())
        return sums

    def scatter_adjoint(self, dy, seq, os_seg, nxt):
        from . import _lib
        lay = self.layer
        dos = torch.zeros((lay.BH, self.seg_rows, lay.d), dtype=torch.float16, device=dy.device)
        delta = torch.zeros((lay.BH, self.seg_rows), dtype=torch.float32, device=dy.device)
        dy, os_seg = _contiguous(dy, os_seg)
        if nxt is not None:
            (nxt,) = _contiguous(nxt)
        p_ = self.api._p
        _lib.call("lh_scatter_back_adjoint_shard", ctypes.byref(self.local.cfg()), ctypes.c_int64(self.seg_rows),
                  p_(dy), p_(self.seq_map), p_(os_seg), p_(nxt) if nxt is not None else None, p_(dos), p_(delta),
                  self.api._stream())
        return dos, delta

    def _bwd(self, qs, ks, vs, lse, dos, delta, q_rows, k_rows):
        return self.api.attn_bwd_rows(self.layer, qs.contiguous(), ks.contiguous(), vs.contiguous(),
                                      lse.contiguous(), dos.contiguous(), delta.contiguous(), q_rows, k_rows)

    def attention_bwd_kv(self, qs, ks, vs, lse, dos, delta, lo, hi):
        _, dks, dvs = self._bwd(qs, ks, vs, lse, dos, delta, (0, 0), (lo, hi))
        return dks[:, lo:hi], dvs[:, lo:hi]

    def attention_bwd_q(self, qs, ks, vs, lse, dos, delta, lo, hi):
        dqs, _, _ = self._bwd(qs, ks, vs, lse, dos, delta, (lo, hi), (0, 0))
        return dqs[:, lo:hi]

    def pool_adjoint(self, dqs, dks, dvs, seq):
        from . import _lib
        lay = self.layer
        shp = (lay.B, lay.H, self.shard.n, lay.d)
        dq, dk, dv = (torch.empty(shp, dtype=torch.bfloat16, device=dqs.device) for _ in range(3))
        dqs, dks, dvs = _contiguous(dqs, dks, dvs)
        p_ = self.api._p
        _lib.call("lh_pool_adjoint_shard", ctypes.byref(self.local.cfg()), ctypes.c_int64(self.seg_rows),
                  p_(dqs), p_(dks), p_(dvs), p_(self.slot_of), p_(dq), p_(dk), p_(dv), self.api._stream())
        return tuple(t.reshape(lay.BH, self.shard.n, lay.d) for t in (dq, dk, dv))
