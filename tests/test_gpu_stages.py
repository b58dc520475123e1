"""GPU parity, stage by stage, through the C ABI (liblh.so) against the fp64
oracle.  Where a stage needs upstream results, the test feeds it the
oracle's values, so a failure points at one kernel.  Index outputs must be
bit-exact; float outputs meet the tolerance of parity_util."""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_pyramid_b200 as lh
from hierarchical_sparse_attention_pyramid_b200 import synth
from hierarchical_sparse_attention_pyramid_b200.synth import Workload
from oracle import lighthouse_oracle as lo
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

SMALL = {
    w.name: w
    for w in (
        synth.WORKLOADS["tiny_4k_fp32"],
        Workload("chunked_lognorm", 1, 2, 8192, 128, 3, 4, 96, "bf16", "qk_sum", "lognormal_token", 11, chunk=512),
        Workload("ragged", 1, 2, 1000, 128, 3, 2, 37, "bf16", "qk_sum", "iid", 12, chunk=64),
        # N not a multiple of the pool's 8-row batches or 16-row stages, with level-1 block ends in the last stage
        Workload("odd_rows_p2", 1, 1, 1002, 64, 2, 2, 37, "bf16", "qk_sum", "iid", 21, chunk=64),
        Workload("deep_p4", 1, 1, 8192, 128, 6, 4, 5, "bf16", "qk_sum", "outlier_tokens", 13),
        Workload("keep_all_kscore", 2, 1, 512, 64, 3, 2, 1000, "bf16", "k", "iid", 14),
        Workload("dense_L1", 1, 2, 700, 64, 1, 2, 1, "bf16", "qk_sum", "iid", 15),
        Workload("qscore_fp32_d128", 1, 1, 2048, 128, 4, 2, 20, "fp32", "q", "iid", 16, chunk=128),
        # the two other readings of what a level keeps
        Workload("direct_sel", 1, 2, 8192, 128, 4, 2, 48, "bf16", "qk_sum", "iid", 18, chunk=512,
                 selection="direct"),
        Workload("nested_sel", 1, 2, 8192, 64, 5, 2, 40, "bf16", "k", "lognormal_token", 19, chunk=32,
                 selection="nested"),
        # bf16 rows of 128 (the pool pair and scatter-back stream kernels) at L = 2 with p = 8 and at L = 5 with
        # p = 2 (tasks of 64 rows holding several top-level blocks), N not a multiple of the 64-row task
        Workload("two_levels_p8", 1, 2, 4000, 128, 2, 8, 64, "bf16", "qk_sum", "iid", 22, chunk=128),
        Workload("five_levels_p2", 2, 1, 4080, 128, 5, 2, 24, "bf16", "qk_sum", "lognormal_token", 23, chunk=256),
    )
}

_cache = {}


def case(name):
    """Inputs on the GPU plus the oracle of every head (cached per module)."""
    if name not in _cache:
        w = SMALL[name]
        x = pu.all_heads_case(w)
        heads = []
        for b in range(w.B):
            for h in range(w.H):
                heads.append(pu.oracle_head(w, x["q"][b, h], x["k"][b, h], x["v"][b, h], x["dy"][b, h]))
        gpu = {n: t.cuda() for n, t in x.items()}
        _cache[name] = (w, gpu, heads)
    return _cache[name]


def layer_of(w):
    return lh.Layer.of(w)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_pool(name):
    w, x, heads = case(name)
    L = layer_of(w)
    info = lh.plan(L)
    pq, pk, pv, norms = lh.pyramid_pool(L, x["q"], x["k"], x["v"])
    torch.cuda.synchronize()
    for bh, o in enumerate(heads):
        sv = o["saved"]
        nq = np.linalg.norm(sv["pyr_q"][0], axis=1)
        nk = np.linalg.norm(sv["pyr_k"][0], axis=1)
        np.testing.assert_allclose(pu.to_np(norms[0, bh]), nq, rtol=2e-6)
        np.testing.assert_allclose(pu.to_np(norms[1, bh]), nk, rtol=2e-6)
        for lvl in range(1, w.L):
            a, n = info.upper_off[lvl], info.level_len[lvl]
            for got, want, t in ((pq, sv["pyr_q"], "q"), (pk, sv["pyr_k"], "k"), (pv, sv["pyr_v"], "v")):
                pu.assert_close(got[bh, a:a + n], want[lvl], f"{name} pyr_{t} level {lvl}")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_score_topk_bit_exact(name):
    w, x, heads = case(name)
    if w.L == 1:
        pytest.skip("no selection with one level")
    L = layer_of(w)
    _, _, _, norms = lh.pyramid_pool(L, x["q"], x["k"], x["v"])
    sel = lh.score_topk(L, norms)
    torch.cuda.synchronize()
    for bh, o in enumerate(heads):
        np.testing.assert_array_equal(sel[bh].cpu().numpy().astype(np.int64), pu.oracle_sel_flat(w, o["saved"]))


@pytest.mark.parametrize("N,L,p,k", [(131072, 3, 2, 512), (65536, 4, 4, 100)])
def test_score_topk_global_chunk_bit_exact(N, L, p, k):
    """An exact global top-k per level (one chunk of every candidate): the
    65536-candidate level is read from the score pyramid in every radix pass,
    the smaller ones are staged in shared memory; indices must match the
    oracle's sort exactly (selection only, after gap repair)."""
    w = Workload("global_topk", 1, 2, N, 64, L, p, k, "bf16", "qk_sum", "iid", 17, chunk=1 << 20)
    L_ = layer_of(w)
    heads = [pu.head_case(w, bh) for bh in range(w.H)]
    q = torch.stack([h["q"] for h in heads]).cuda()
    kk = torch.stack([h["k"] for h in heads]).cuda()
    _, _, _, norms = lh.pyramid_pool(L_, q, kk, kk)
    sel = lh.score_topk(L_, norms)
    torch.cuda.synchronize()
    for bh, h in enumerate(heads):
        want, _ = lo.select(pu.to_np(h["q"]), pu.to_np(h["k"]), w.p, w.L, w.k, w.chunk, w.scorer)
        np.testing.assert_array_equal(sel[bh].cpu().numpy().astype(np.int64),
                                      np.concatenate([np.asarray(x, np.int64) for x in want]))


@pytest.mark.parametrize("name", sorted(SMALL))
def test_gather(name):
    w, x, heads = case(name)
    L = layer_of(w)
    pq, pk, pv, norms = lh.pyramid_pool(L, x["q"], x["k"], x["v"])
    sel = lh.score_topk(L, norms) if w.L > 1 else torch.zeros(1, dtype=torch.int32, device="cuda")
    qs, ks, vs, seq_map, slot_of = lh.gather(L, x["q"], x["k"], x["v"], pq, pk, pv, sel)
    torch.cuda.synchronize()
    for bh, o in enumerate(heads):
        sv = o["saved"]
        np.testing.assert_array_equal(seq_map[bh].cpu().numpy().astype(np.int64), pu.oracle_seq_map(sv))
        np.testing.assert_array_equal(slot_of[bh].cpu().numpy().astype(np.int64), pu.oracle_slot_of(sv))
        for got, want, t in ((qs, sv["Qs"], "Qs"), (ks, sv["Ks"], "Ks"), (vs, sv["Vs"], "Vs")):
            pu.assert_close(got[bh], want, f"{name} {t}")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_pool_from_and_gather_from(name):
    """The stage calls lh_forward makes: the pool writes levels >= first_level
    only (the rows below stay as they were), the norms are unchanged, and the
    gather that averages the lower levels from level 0 matches the oracle, for
    every admissible first_level (the plan's choice included)."""
    w, x, heads = case(name)
    L = layer_of(w)
    info = lh.plan(L)
    assert 1 <= info.first_level <= max(1, w.L - 1)
    _, _, _, norms_full = lh.pyramid_pool(L, x["q"], x["k"], x["v"])
    sel = lh.score_topk(L, norms_full) if w.L > 1 else torch.zeros(1, dtype=torch.int32, device="cuda")
    for first in range(1, max(1, w.L - 1) + 1):
        pq, pk, pv, norms = lh.pyramid_pool(L, x["q"], x["k"], x["v"], first_level=first)
        qs, ks, vs, seq_map, slot_of = lh.gather(L, x["q"], x["k"], x["v"], pq, pk, pv, sel, first_level=first)
        torch.cuda.synchronize()
        assert torch.equal(norms, norms_full), f"{name} first_level {first}: norms differ"
        for bh, o in enumerate(heads):
            sv = o["saved"]
            for lvl in range(1, w.L):
                a, n = info.upper_off[lvl], info.level_len[lvl]
                for got, want, t in ((pq, sv["pyr_q"], "q"), (pk, sv["pyr_k"], "k"), (pv, sv["pyr_v"], "v")):
                    if lvl >= first:
                        pu.assert_close(got[bh, a:a + n], want[lvl], f"{name} from {first} pyr_{t} {lvl}")
                    else:
                        assert not got[bh, a:a + n].any(), f"{name} from {first}: level {lvl} of pyr_{t} written"
            np.testing.assert_array_equal(seq_map[bh].cpu().numpy().astype(np.int64), pu.oracle_seq_map(sv))
            np.testing.assert_array_equal(slot_of[bh].cpu().numpy().astype(np.int64), pu.oracle_slot_of(sv))
            for got, want, t in ((qs, sv["Qs"], "Qs"), (ks, sv["Ks"], "Ks"), (vs, sv["Vs"], "Vs")):
                pu.assert_close(got[bh], want, f"{name} from {first} {t}")


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


ATTN_SHAPES = [(1, 128, 64), (2, 300, 64), (2, 1000, 128), (3, 640, 128), (1, 2048, 128), (1, 77, 128)]


@pytest.mark.parametrize("BH,S,d", ATTN_SHAPES)
def test_attn_fwd(BH, S, d):
    g = torch.Generator().manual_seed(1000 + S + d)
    q, k, v = (torch.randn(BH, S, d, generator=g).to(torch.bfloat16) for _ in range(3))
    L = lh.Layer(1, BH, 4096, d, 3, 2, 8)
    os_, lse = lh.attn_fwd(L, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    for h in range(BH):
        O, ls = lo.causal_attention(pu.to_np(q[h]), pu.to_np(k[h]), pu.to_np(v[h]))
        pu.assert_close(os_[h], O, f"O head {h}")
        np.testing.assert_allclose(pu.to_np(lse[h]), ls, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("BH,S,d", ATTN_SHAPES)
def test_attn_bwd(BH, S, d):
    g = torch.Generator().manual_seed(2000 + S + d)
    q, k, v, do = (torch.randn(BH, S, d, generator=g).to(torch.bfloat16) for _ in range(4))
    lse = torch.empty(BH, S, dtype=torch.float32)
    delta = torch.empty(BH, S, dtype=torch.float32)
    want = []
    for h in range(BH):
        O, ls = lo.causal_attention(pu.to_np(q[h]), pu.to_np(k[h]), pu.to_np(v[h]))
        lse[h] = torch.from_numpy(ls)
        delta[h] = torch.from_numpy(np.sum(pu.to_np(do[h]) * O, axis=1))
        want.append(lo.causal_attention_backward(pu.to_np(q[h]), pu.to_np(k[h]), pu.to_np(v[h]), pu.to_np(do[h])))
    L = lh.Layer(1, BH, 4096, d, 3, 2, 8)
    # dOs is passed as fp16 holding the bf16 values (exact), as the scatter adjoint writes it
    dqs, dks, dvs = lh.attn_bwd(L, q.cuda(), k.cuda(), v.cuda(), lse.cuda(), do.half().cuda(), delta.cuda())
    torch.cuda.synchronize()
    for h in range(BH):
        for got, wnt, t in zip((dqs, dks, dvs), want[h], ("dQ", "dK", "dV")):
            pu.assert_close(got[h], wnt, f"{t} head {h}")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_scatter_back(name):
    w, x, heads = case(name)
    L = layer_of(w)
    info = lh.plan(L)
    os_ = torch.stack([torch.from_numpy(o["saved"]["Os"]).float() for o in heads]).cuda()
    slot_of = torch.stack([torch.from_numpy(pu.oracle_slot_of(o["saved"]).astype(np.int32)) for o in heads]).cuda()
    y = lh.scatter_back(L, os_, slot_of)
    torch.cuda.synchronize()
    yf = y.reshape(w.B * w.H, w.N, w.d)
    for bh, o in enumerate(heads):
        sv = o["saved"]
        want = lo.scatter_back(pu.to_np(os_[bh].cpu()), sv["seq_level"], sv["seq_index"], w.N, w.p, w.L)
        pu.assert_close(yf[bh], want, f"{name} Y", max_abs=1e-2, mean_abs=1e-3)
    assert info.S == os_.shape[1]


@pytest.mark.parametrize("name", sorted(SMALL))
def test_scatter_adjoint(name):
    w, x, heads = case(name)
    L = layer_of(w)
    os_ = torch.stack([torch.from_numpy(o["saved"]["Os"]).float() for o in heads]).cuda()
    seq_map = torch.stack([torch.from_numpy(pu.oracle_seq_map(o["saved"]).astype(np.int32)) for o in heads]).cuda()
    dos, delta = lh.scatter_back_adjoint(L, x["dy"], seq_map, os_)
    torch.cuda.synchronize()
    dyf = x["dy"].reshape(w.B * w.H, w.N, w.d)
    for bh, o in enumerate(heads):
        sv = o["saved"]
        want = lo.scatter_adjoint(pu.to_np(dyf[bh]), sv["seq_level"], sv["seq_index"], w.N, w.p)
        # stored in fp16 but rounded to bf16 first (the attention's 16-bit input)
        pu.assert_close(dos[bh], want, f"{name} dOs", dtype="bf16")
        dl = np.sum(pu.to_np(dos[bh]) * pu.to_np(os_[bh]), axis=1)
        np.testing.assert_allclose(pu.to_np(delta[bh]), dl, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_pool_adjoint(name):
    w, x, heads = case(name)
    L = layer_of(w)
    grads = [torch.stack([torch.from_numpy(o[t]).float() for o in heads]).cuda() for t in ("dQs", "dKs", "dVs")]
    slot_of = torch.stack([torch.from_numpy(pu.oracle_slot_of(o["saved"]).astype(np.int32)) for o in heads]).cuda()
    dq, dk, dv = lh.pool_adjoint(L, grads[0], grads[1], grads[2], slot_of)
    torch.cuda.synchronize()
    for bh, o in enumerate(heads):
        sv = o["saved"]
        for got, src, t in ((dq, "dQs", "dQ"), (dk, "dKs", "dK"), (dv, "dVs", "dV")):
            lv = lo.gather_adjoint(np.float32(o[src]).astype(np.float64), sv["seq_level"], sv["seq_index"], w.N, w.p, w.L)
            want = lo.pyramid_pool_adjoint(lv, w.p)
            pu.assert_close(got.reshape(w.B * w.H, w.N, w.d)[bh], want, f"{name} {t}")


@pytest.mark.parametrize("BH,S,d,cuts", [(2, 1000, 128, (0, 384, 640, 1000)), (1, 300, 64, (0, 128, 300)),
                                         (3, 777, 128, (0, 0, 256, 777))])
def test_attn_row_windows(BH, S, d, cuts):
    """The attention over row windows (the pieces context parallelism runs on
    different GPUs) equals the whole-sequence kernels bit for bit, row by row,
    whatever the cuts (empty windows included)."""
    g = torch.Generator().manual_seed(S + d)
    qs, ks, vs = (torch.randn(BH, S, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    L = lh.Layer(1, BH, 4096, d, 3, 2, 8)
    os_full, lse_full = lh.attn_fwd(L, qs, ks, vs)
    os_w = torch.full_like(os_full, float("nan"))
    lse_w = torch.full_like(lse_full, float("nan"))
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        lh.attn_fwd_rows(L, qs, ks, vs, lo, hi, os_w, lse_w)
    torch.cuda.synchronize()
    assert torch.equal(os_w, os_full) and torch.equal(lse_w, lse_full)
    dos = torch.randn(BH, S, d, generator=g).to(torch.bfloat16).to(torch.float16).cuda()
    delta = (dos.float() * os_full).sum(-1).contiguous()
    dq, dk, dv = lh.attn_bwd(L, qs, ks, vs, lse_full, dos, delta)
    dq_w, dk_w, dv_w = (torch.full_like(dq, float("nan")) for _ in range(3))
    # query windows in order, key windows in reverse order (independent pieces)
    for (qlo, qhi), (klo, khi) in zip(zip(cuts[:-1], cuts[1:]), reversed(list(zip(cuts[:-1], cuts[1:])))):
        lh.attn_bwd_rows(L, qs, ks, vs, lse_full, dos, delta, (qlo, qhi), (klo, khi), dq_w, dk_w, dv_w)
    torch.cuda.synchronize()
    assert torch.equal(dq_w, dq) and torch.equal(dk_w, dk) and torch.equal(dv_w, dv)
