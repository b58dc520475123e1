"""Context parallelism host logic (hierarchical_sparse_attention_pyramid_b200
.context_parallel), on the CPU: the partition bookkeeping against the oracle's
unsharded causal order, and the whole sharded forward and backward over 2 and
4 gloo ranks against the unsharded oracle.  Each rank's arithmetic is done by
a backend built from the oracle's stage functions (fp64, the attention inputs
not rounded), so a mismatch can only come from the partition, the exchanges,
the halo adds or the attention windows."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from hierarchical_sparse_attention_pyramid_b200 import context_parallel as cp
from oracle import lighthouse_oracle as lo

CASES = {
    # name: (N, d, L, p, k, chunk, H, selection, scorer)
    "p2_L3": (1024, 16, 3, 2, 20, 64, 2, "parents", "qk_sum"),
    "p4_L4": (2048, 16, 4, 4, 12, 64, 2, "parents", "k"),
    "direct_p2_L4": (1024, 8, 4, 2, 24, 64, 1, "direct", "qk_sum"),
    "nested_p2_L4": (1024, 8, 4, 2, 10, 32, 1, "nested", "q"),
}


def _inputs(N, d, H, seed):
    g = np.random.default_rng(seed)
    scale = np.exp(0.5 * g.standard_normal((H, N, 1)))  # per-token norm spread, like the log-normal workload
    q, k, v, dy = (g.standard_normal((H, N, d)) for _ in range(4))
    return q * scale, k * scale, v * scale, dy


def _oracle(case, q, k, v, dy):
    N, d, L, p, kk, T, H, selection, scorer = case
    out = []
    for h in range(H):
        Y, sv = lo.forward_head(q[h], k[h], v[h], p, L, kk, T, scorer, attn_dtype=None, selection=selection)
        dQ, dK, dV, _ = lo.backward_head(dy[h], sv)
        out.append((Y, dQ, dK, dV, sv))
    return out


# ---------------------------------------------------------------- bookkeeping

@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("world", [2, 4])
def test_segments_are_the_unsharded_order(name, world):
    """Every shard's kept entries are one contiguous run of the unsharded
    sequence, in the same order, with the counts and offsets the plan gives;
    the previous shard's boundary entries sit at the global slots halo_in
    names; the windows tile [0, S)."""
    N, d, L, p, kk, T, H, selection, scorer = case = CASES[name]
    q, k, v, dy = _inputs(N, d, H, 5)
    for h, (_, _, _, _, sv) in enumerate(_oracle(case, q, k, v, dy)):
        kept = cp.kept_entries(sv["sel"], N, p, L, selection)
        counts = cp.segment_counts(kept, N, p, L, world)
        S = len(sv["seq_level"])
        assert counts.sum() == S == lo.gathered_length(N, p, L, kk, selection)
        off = 0
        for r in range(world):
            shard = cp.Shard(N, p, L, world, r)
            seg_l = sv["seq_level"][off:off + counts[r]]
            seg_i = sv["seq_index"][off:off + counts[r]]
            # keys of the segment lie in the shard
            e = (seg_i + 1) * p ** seg_l - 1
            assert np.all((e >= shard.t0) & (e < shard.t1))
            # the local selection reproduces the segment in local indices
            ents = lo.selected_entries(cp.local_selection(sv["sel"], shard, selection), shard.n, p, L, selection)
            ll, li = lo.causal_order(ents, p)
            np.testing.assert_array_equal(ll, seg_l)
            np.testing.assert_array_equal(li + 0, seg_i - (shard.t0 // p ** seg_l))
            # global slots of the halo entries
            for l, slot, rows in cp.halo_in(kept, shard):
                assert sv["seq_level"][slot] == l and sv["seq_index"][slot] == shard.t0 // p ** l - 1
                assert rows == p ** l - 1
            off += counts[r]
        for kind in ("query", "key"):
            win = cp.balanced_windows(S, world, kind)
            assert win[0][0] == 0 and win[-1][1] == S
            assert all(a[1] == b[0] for a, b in zip(win, win[1:]))


def test_global_slot_matches_oracle():
    N, d, L, p, kk, T, H, selection, scorer = case = CASES["p4_L4"]
    q, k, v, dy = _inputs(N, d, H, 9)
    sv = _oracle(case, q, k, v, dy)[0][4]
    kept = cp.kept_entries(sv["sel"], N, p, L, selection)
    for s in range(0, len(sv["seq_level"]), 7):
        assert cp.global_slot(kept, int(sv["seq_level"][s]), int(sv["seq_index"][s]), p) == s


def test_shards_must_hold_whole_top_blocks():
    with pytest.raises(ValueError):
        cp.Shard(1024, 4, 5, 8, 0)  # 128 tokens per shard, top blocks of 256
    with pytest.raises(ValueError):
        cp.Shard(1000, 2, 2, 3, 0)
    cp.Shard(1024, 4, 4, 16, 3)


def test_balanced_windows_balance_the_causal_work():
    S = 29696
    for kind in ("query", "key"):
        win = cp.balanced_windows(S, 8, kind)
        nt = (S + 127) // 128
        cost = []
        for a, b in win:
            t = np.arange(a // 128, (b + 127) // 128)
            cost.append(((t + 1) if kind == "query" else (nt - t)).sum())
        assert max(cost) / (sum(cost) / 8) < 1.05


# ---------------------------------------------------------------- the sharded layer on gloo ranks

class OracleBackend:
    """The per-rank arithmetic from the oracle's stage functions, fp64."""

    def __init__(self, case, shard):
        (self.N, self.d, self.L, self.p, self.k, self.T, self.H, self.selection, self.scorer) = case
        self.shard = shard
        self.n = shard.n

    def pool(self, q, k, v):
        levels = [[lo.pyramid_pool(x[h].numpy(), self.p, self.L) for x in (q, k, v)] for h in range(q.shape[0])]
        norms = torch.stack([torch.linalg.vector_norm(q, dim=-1), torch.linalg.vector_norm(k, dim=-1)])
        return levels, norms

    def select(self, norms):
        sel = []
        for h in range(norms.shape[1]):
            nq, nk = norms[0, h].numpy(), norms[1, h].numpy()
            s0 = {"qk_sum": nq + nk, "k": nk, "q": nq}[self.scorer]
            spyr = lo.score_pyramid(s0, self.p, self.L)
            kp = lo.budgets(self.N, self.p, self.L, self.k, self.selection)
            if self.selection == "parents":
                sel.append([lo.stratified_topk(spyr[l + 1], kp[l], self.T) for l in range(self.L - 1)])
            elif self.selection == "direct":
                sel.append([lo.stratified_topk(spyr[l], self.p * kp[l], self.T) for l in range(self.L - 1)])
            else:
                s = [None] * (self.L - 1)
                kept = np.arange(self.N // self.p ** (self.L - 1), dtype=np.int64)
                for lvl in range(self.L - 2, -1, -1):
                    s[lvl] = kept[lo.stratified_topk(spyr[lvl + 1][kept], kp[lvl], self.T)]
                    kept = (s[lvl][:, None] * self.p + np.arange(self.p)[None, :]).reshape(-1)
                sel.append(s)
        return sel

    def gather(self, q, k, v, levels, sel_loc):
        seq, rows = [], [[], [], []]
        for h in range(q.shape[0]):
            ents = lo.selected_entries(sel_loc[h], self.n, self.p, self.L, self.selection)
            lv, ix = lo.causal_order(ents, self.p)
            seq.append((lv, ix))
            for t in range(3):
                rows[t].append(lo.gather(levels[h][t], lv, ix))
        mx = max(len(s[0]) for s in seq)
        out = []
        for t in range(3):
            x = torch.zeros((q.shape[0], mx, self.d), dtype=torch.float64)
            for h, r in enumerate(rows[t]):
                x[h, :len(r)] = torch.from_numpy(r)
            out.append(x)
        return seq, tuple(out)

    def attention(self, qs, ks, vs, a, b):
        os_, lse = [], []
        for h in range(qs.shape[0]):
            O, ls = lo.causal_attention(qs[h].numpy(), ks[h].numpy(), vs[h].numpy())
            os_.append(torch.from_numpy(O[a:b]))
            lse.append(torch.from_numpy(ls[a:b]))
        return torch.stack(os_), torch.stack(lse)

    def scatter(self, os_seg, seq, halo):
        y = torch.stack([torch.from_numpy(lo.scatter_back(os_seg[h, :len(lv)].numpy(), lv, ix, self.n, self.p,
                                                          self.L)) for h, (lv, ix) in enumerate(seq)])
        for h, ents in enumerate(halo):
            for l, row, rows in ents:
                y[h, :rows] += row
        return y

    def head_sums(self, dy):
        return torch.stack([dy[:, :self.p ** l - 1].sum(dim=1) for l in range(1, self.L)], dim=1)

    def scatter_adjoint(self, dy, seq, os_seg, nxt):
        mx = max(len(s[0]) for s in seq)
        dos = torch.zeros((dy.shape[0], mx, self.d), dtype=torch.float64)
        for h, (lv, ix) in enumerate(seq):
            dos[h, :len(lv)] = torch.from_numpy(lo.scatter_adjoint(dy[h].numpy(), lv, ix, self.n, self.p))
            if nxt is not None:
                for l, s in cp.halo_out_entries(lv, ix, self.shard):
                    dos[h, s] += nxt[h, l - 1]
        return dos, (dos * os_seg).sum(-1)

    def _bwd(self, qs, ks, vs, dos):
        return [lo.causal_attention_backward(qs[h].numpy(), ks[h].numpy(), vs[h].numpy(), dos[h].numpy())
                for h in range(qs.shape[0])]

    def attention_bwd_kv(self, qs, ks, vs, lse, dos, delta, a, b):
        g = self._bwd(qs, ks, vs, dos)
        return (torch.stack([torch.from_numpy(x[1][a:b]) for x in g]),
                torch.stack([torch.from_numpy(x[2][a:b]) for x in g]))

    def attention_bwd_q(self, qs, ks, vs, lse, dos, delta, a, b):
        return torch.stack([torch.from_numpy(x[0][a:b]) for x in self._bwd(qs, ks, vs, dos)])

    def pool_adjoint(self, dqs, dks, dvs, seq):
        out = []
        for t in (dqs, dks, dvs):
            out.append(torch.stack([torch.from_numpy(lo.pyramid_pool_adjoint(
                lo.gather_adjoint(t[h, :len(lv)].numpy(), lv, ix, self.n, self.p, self.L), self.p))
                for h, (lv, ix) in enumerate(seq)]))
        return tuple(out)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, name, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        case = CASES[name]
        N, d, L, p, kk, T, H, selection, scorer = case
        q, k, v, dy = (torch.from_numpy(x) for x in _inputs(N, d, H, 3))
        shard = cp.Shard(N, p, L, world, rank)
        sl = slice(shard.t0, shard.t1)
        be = OracleBackend(case, shard)
        y, ctx = cp.cp_forward(be, shard, q[:, sl], k[:, sl], v[:, sl], selection)
        dq, dk, dv = cp.cp_backward(be, shard, dy[:, sl].contiguous(), ctx)
        out[rank] = tuple(t.numpy() for t in (y, dq, dk, dv))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,world", [(n, w) for n in sorted(CASES) for w in (2, 4)] + [("p4_L4", 8)])
def test_sharded_layer_matches_unsharded_oracle(name, world):
    case = CASES[name]
    N, d, L, p, kk, T, H, selection, scorer = case
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), name, out), nprocs=world, join=True)
    q, k, v, dy = _inputs(N, d, H, 3)
    want = _oracle(case, q, k, v, dy)
    for t, nm in enumerate(("Y", "dQ", "dK", "dV")):
        got = np.concatenate([out[r][t] for r in range(world)], axis=1)
        for h in range(H):
            np.testing.assert_allclose(got[h], want[h][t], rtol=1e-9, atol=1e-11, err_msg=f"{name} {nm} head {h}")


def _count_main(rank, world, port, name, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    calls = cp.EXCHANGE_LOG = []
    try:
        case = CASES[name]
        N, d, L, p, kk, T, H, selection, scorer = case
        q, k, v, dy = (torch.from_numpy(x) for x in _inputs(N, d, H, 3))
        shard = cp.Shard(N, p, L, world, rank)
        sl = slice(shard.t0, shard.t1)
        be = OracleBackend(case, shard)
        y, ctx = cp.cp_forward(be, shard, q[:, sl], k[:, sl], v[:, sl], selection)
        n_fwd = len(calls)
        cp.cp_backward(be, shard, dy[:, sl].contiguous(), ctx)
        need = cp.os_rows_needed(ctx.kept, ctx.counts, shard)
        want = cp.exchange_elements(H, N, d, L, ctx.qs.shape[1], world, rank, ctx.counts, need)
        out[rank] = (n_fwd, len(calls) - n_fwd, calls == [want[n] for n in cp.EXCHANGES if n in want])
    finally:
        cp.EXCHANGE_LOG = None
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["p2_L3", "direct_p2_L4"])
def test_collectives_per_layer_do_not_grow_with_heads(name):
    """One exchange per quantity, whatever the number of heads: forward norms,
    Qs|Ks|Vs (all-gathers), Os (rows to the ranks that read them), LSE;
    backward head sums, dOs, Delta (all-gathers), dKs|dVs, dQs (rows to the
    segments' ranks); each rank receiving what exchange_elements predicts."""
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_count_main, args=(2, _free_port(), name, out), nprocs=2, join=True)
    assert [out[r] for r in range(2)] == [(4, 5, True), (4, 5, True)]


def _redistribute_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        g = np.random.default_rng(11)  # the same draws on every rank
        ok = []
        for dtype in (torch.float32, torch.bfloat16, torch.float16):
            BH, S = 3, 700
            X = torch.from_numpy(g.standard_normal((BH, S, 2, 5))).to(dtype)
            # windows tile [0, S), one of them empty
            cuts = np.sort(g.choice(np.arange(1, S), world - 2, replace=False))
            cuts = [0, 0] + list(cuts) + [S] if world > 2 else [0, 0, S]
            windows = list(zip(cuts[:-1], cuts[1:]))[:world]
            windows[-1] = (windows[-1][0], S)
            # every rank reads an arbitrary, unsorted set of rows per head (some none)
            need = [[g.permutation(S)[:g.integers(0, 200)] for _ in range(BH)] for _ in range(world)]
            lo, hi = windows[rank]
            got = cp.redistribute_rows(X[:, lo:hi], windows, need, None)
            mx = max(1, max(len(n) for n in need[rank]))
            want = torch.zeros((BH, mx, 2, 5), dtype=dtype)
            for h in range(BH):
                want[h, :len(need[rank][h])] = X[h, torch.from_numpy(need[rank][h])]
            ok.append(got.dtype == dtype and torch.equal(got, want))
        out[rank] = all(ok)
    finally:
        dist.destroy_process_group()


def test_redistribute_rows_delivers_every_needed_row():
    """Each rank gets exactly the rows it asks for, in its own order, from
    whichever rank's window holds them (an empty window included), for the
    dtypes the CUDA backend exchanges; rows past a head's list are zero."""
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_redistribute_main, args=(3, _free_port(), out), nprocs=3, join=True)
    assert [out[r] for r in range(3)] == [True] * 3
