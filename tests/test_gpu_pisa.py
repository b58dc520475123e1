"""GPU parity of the PISA block selection (lh_pisa_pool_keys, lh_pisa_select)
against the fp64 oracle, through the C ABI.

The key pyramid must be bit-exact: both sides round the exact mean to bf16.

The selection is an integer result decided by float scores, and the GPU's
scores are fp32 (tensor-core dot products, ex2/lg2 approximations, fp32
sums) where the oracle's are fp64.  So every level of every checked group is
re-scored by the oracle on the candidates the GPU had at that level (the
coarsest level's blocks, then the sub-blocks of the GPU's kept blocks one
level up), and:
  * the GPU's kept scores equal the oracle's to EPS (absolute, natural log);
  * the GPU's kept set equals the oracle's top-K of those candidates unless
    the oracle's K-th and (K+1)-th scores are within EPS (a near tie), where
    it must still be a valid top-K to EPS;
  * the kept lists are ascending, padded with -1 / -inf, and the first level
    scores all of the coarsest blocks.
EPS = 2e-3: the score is ln of a sum of up to G*C exponentials of logits
q.k/sqrt(d).  bf16 products are exact in fp32; a 128-term fp32 dot product is
off by at most 128 * 2^-24 of sum|q_k k_k| (about 6e-4 in logit units for
rows of norm sqrt(d) scaled by the LogNormal(0, 0.5) factors, far less in
practice); ex2 / lg2 approximations add about 2^-22 relative each and the
fp32 sums of at most 16384 terms about 1e-3 relative at worst.  All three are
far below EPS on these inputs, and the gaps between candidate scores are far
above it but for a few near ties per thousand decisions.
"""

import numpy as np
import pytest
import torch

from hierarchical_sparse_attention_pyramid_b200 import pisa, synth
from hierarchical_sparse_attention_pyramid_b200.synth import PisaWorkload
from oracle import pisa_oracle as po
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

EPS = 2e-3

SMALL = {
    w.name: w
    for w in (
        synth.PISA_WORKLOADS["pisa_small_8k"],
        PisaWorkload("p2_deep_d64", 1, 1, 8192, 64, 2, 6, 64, 128, 4, "iid", 30),
        PisaWorkload("block128_outliers", 2, 1, 4096, 128, 2, 3, 128, 128, 3, "outlier_tokens", 31),
        PisaWorkload("flat_L1", 1, 2, 2048, 64, 2, 1, 64, 128, 5, "iid", 32),
        PisaWorkload("keep_all_padded", 1, 1, 1024, 128, 2, 3, 64, 128, 64, "lognormal_token", 33),
        PisaWorkload("wide_top_256", 1, 1, 32768, 64, 2, 2, 64, 128, 2, "iid", 34),
        PisaWorkload("p8_K1", 1, 1, 32768, 128, 8, 3, 64, 128, 1, "lognormal_token", 35),
    )
}
# groups the oracle recomputes (None = all)
GROUPS = {"wide_top_256": (0, 1, 37, 100, 200, 255), "p8_K1": (0, 3, 64, 128, 255)}

_cache = {}


def inputs(w):
    if w.name not in _cache:
        heads = [synth.head_inputs(w, bh) for bh in range(w.B * w.H)]
        q = torch.stack([h["q"] for h in heads]).reshape(w.B, w.H, w.N, w.d)
        k = torch.stack([h["k"] for h in heads]).reshape(w.B, w.H, w.N, w.d)
        _cache[w.name] = (q, k)
    return _cache[w.name]


def sel_of(w):
    return pisa.Pisa(w.B, w.H, w.N, w.d, w.p, w.L, w.block, w.group, w.topk)


def check_group(Qh, levels, w, g, idx, sco):
    """Re-score every level of group g along the GPU's path; return True when
    the GPU took the oracle's own decision at every level."""
    C, p, G, K, L = w.block, w.p, w.group, w.topk, w.L
    Qg = Qh[g * G:(g + 1) * G]
    cands = np.arange(levels[L - 1].shape[0] // C)
    exact = True
    for lv in range(L - 1, -1, -1):
        kk = min(K, len(cands))
        kept = idx[lv, :kk].astype(np.int64)
        assert np.all(idx[lv, kk:] == -1) and np.all(np.isneginf(sco[lv, kk:])), (g, lv)
        assert np.all(np.diff(kept) > 0) and np.all(np.isin(kept, cands)), (g, lv, kept)
        sc = po.block_scores(Qg, g * G, levels, lv, cands, C, p)
        pos = np.searchsorted(cands, kept)
        want = sc[pos]
        got = sco[lv, :kk].astype(np.float64)
        both_inf = np.isneginf(want) & np.isneginf(got)
        with np.errstate(invalid="ignore"):
            diff = np.abs(np.where(both_inf, 0.0, got - want))
        assert np.all(diff <= EPS), (g, lv, got, want)
        o_kept, _ = po.top_blocks(cands, sc, K)
        if not np.array_equal(o_kept, kept):
            exact = False
            order = np.sort(sc)[::-1]
            assert kk < len(cands) and order[kk - 1] - order[kk] <= EPS, (g, lv, "decision differs without a near tie")
            out = ~np.isin(cands, kept)
            assert want.min() >= sc[out].max() - EPS, (g, lv)
        cands = po.sub_blocks(kept, p)
    return exact


@pytest.mark.parametrize("name", sorted(SMALL))
def test_key_pyramid_bit_exact(name):
    w = SMALL[name]
    if w.L == 1:
        pytest.skip("no pyramid at L = 1")
    q, k = inputs(w)
    s = sel_of(w)
    info = pisa.plan(s)
    kp = pisa.pool_keys(s, k.cuda().contiguous())
    torch.cuda.synchronize()
    kp = kp.float().cpu().numpy()
    for bh in range(w.B * w.H):
        levels = po.key_pyramid(pu.to_np(k.reshape(-1, w.N, w.d)[bh]), w.p, w.L)
        for lv in range(1, w.L):
            rows = kp[bh, info.level_off[lv]:info.level_off[lv] + w.N // w.p ** lv]
            np.testing.assert_array_equal(rows, levels[lv], err_msg=f"{name} head {bh} level {lv}")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_selection_parity(name):
    w = SMALL[name]
    q, k = inputs(w)
    s = sel_of(w)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    idx, sco = pisa.select(s, q.cuda().contiguous(), k.cuda().contiguous(),
                           pisa.pool_keys(s, k.cuda().contiguous()), ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    idx = idx.cpu().numpy()
    sco = sco.cpu().numpy()
    groups = GROUPS.get(name) or range(w.N // w.group)
    n_exact = n = 0
    for bh in range(w.B * w.H):
        Qh = pu.to_np(q.reshape(-1, w.N, w.d)[bh])
        levels = po.key_pyramid(pu.to_np(k.reshape(-1, w.N, w.d)[bh]), w.p, w.L)
        for g in groups:
            n_exact += check_group(Qh, levels, w, g, idx[bh, g], sco[bh, g])
            n += 1
    # near ties are rare: the GPU follows the oracle's own path almost everywhere
    assert n_exact >= 0.9 * n, (n_exact, n)


def test_selection_is_deterministic_and_ignores_future_keys():
    w = SMALL["pisa_small_8k"]
    q, k = inputs(w)
    s = sel_of(w)
    qc, kc = q.cuda().contiguous(), k.cuda().contiguous()
    a = pisa.block_select(s, qc, kc)
    b = pisa.block_select(s, qc, kc)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    # keys after a group's last query change nothing for that group
    g = 20
    k2 = kc.clone()
    k2[:, :, (g + 1) * w.group:] = torch.randn_like(k2[:, :, (g + 1) * w.group:], dtype=torch.float32).to(k2.dtype)
    c = pisa.block_select(s, qc, k2)
    assert torch.equal(a[0][:, :g + 1], c[0][:, :g + 1]) and torch.equal(a[1][:, :g + 1], c[1][:, :g + 1])


@pytest.mark.slow
@pytest.mark.parametrize("name,heads,groups", [("pisa_128k", (0, 11), (0, 1, 300, 777, 1023)),
                                               ("pisa_256k", (5,), (0, 2047))])
def test_full_size_sampled(name, heads, groups):
    w = synth.PISA_WORKLOADS[name]
    x = synth.cuda_inputs(w, "cuda")
    cases = {}
    for bh in heads:
        h = synth.head_inputs(w, bh)
        b, hh = divmod(bh, w.H)
        x["q"][b, hh] = h["q"].cuda()
        x["k"][b, hh] = h["k"].cuda()
        cases[bh] = h
    s = sel_of(w)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    idx, sco = pisa.select(s, x["q"], x["k"], pisa.pool_keys(s, x["k"]), ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    # every group of every head: level 0 holds K ascending blocks with finite or -inf scores
    lvl0 = idx[:, :, 0]
    assert bool((lvl0[..., 1:] > lvl0[..., :-1]).all())
    assert not bool(torch.isnan(sco).any())
    idx = idx.cpu().numpy()
    sco = sco.cpu().numpy()
    for bh, h in cases.items():
        Qh = pu.to_np(h["q"])
        levels = po.key_pyramid(pu.to_np(h["k"]), w.p, w.L)
        for g in groups:
            check_group(Qh, levels, w, g, idx[bh, g], sco[bh, g])
