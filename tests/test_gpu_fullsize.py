"""GPU parity at the full workload sizes, through lh_forward / lh_backward as
bench.py calls them.  All heads run on the GPU; the sampled heads are drawn
on the CPU (and gap-repaired) so the fp64 oracle can recompute them one by
one, and are compared element by element.  Every head is checked for the
properties that hold at any size: the sequence map is a permutation that
slot_of inverts, each level keeps p*k' entries plus the whole top level, and
all outputs are finite."""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_pyramid_b200 as lh
from hierarchical_sparse_attention_pyramid_b200 import synth
from tests import parity_util as pu

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLED = {
    "lognorm_32k": (0, 5),
    "kscore_128k": (7,),
    "sparse64_512k": (0, 15),
    "outlier_1m": (3,),
}


@pytest.mark.parametrize("name", sorted(SAMPLED))
def test_full_size(name):
    w = synth.WORKLOADS[name]
    L = lh.Layer.of(w)
    info = lh.plan(L)
    x = synth.cuda_inputs(w, "cuda")
    cases = {}
    for bh in SAMPLED[name]:
        h = pu.head_case(w, bh)
        b, hh = divmod(bh, w.H)
        for n in ("q", "k", "v", "dy"):
            x[n][b, hh] = h[n].cuda()
        cases[bh] = h
    y, bufs = lh.forward(L, x["q"], x["k"], x["v"])
    dq, dk, dv = lh.backward(L, x["dy"], bufs)
    lh.check_error(bufs)
    v = bufs.ctx_views()
    S = info.S

    # properties of every head
    for t in (y, dq, dk, dv):
        assert torch.isfinite(t).all()
    seq = v["seq_map"].long()
    lvl, idx = seq >> 28, seq & ((1 << 28) - 1)
    off = torch.tensor([info.level_off[i] for i in range(w.L)], device="cuda")
    rows = off[lvl] + idx
    back = torch.gather(v["slot_of"].long(), 1, rows)
    assert torch.equal(back, torch.arange(S, device="cuda").expand_as(back))
    assert int((v["slot_of"] >= 0).sum()) == w.B * w.H * S
    counts = torch.stack([(lvl == i).sum(1) for i in range(w.L)], 1)
    want_counts = [w.p * info.kprime[i] for i in range(w.L - 1)] + [info.level_len[w.L - 1]]
    assert torch.equal(counts, torch.tensor(want_counts, device="cuda").expand_as(counts))

    # sampled heads against the oracle
    flat = lambda t: t.reshape(w.B * w.H, w.N, w.d)  # noqa: E731
    checks = []
    for bh, h in cases.items():
        o = pu.oracle_head(w, h["q"], h["k"], h["v"], h["dy"])
        sv = o["saved"]
        np.testing.assert_array_equal(v["sel"][bh].cpu().numpy().astype(np.int64), pu.oracle_sel_flat(w, sv))
        np.testing.assert_array_equal(v["seq_map"][bh].cpu().numpy().astype(np.int64), pu.oracle_seq_map(sv))
        np.testing.assert_array_equal(v["slot_of"][bh].cpu().numpy().astype(np.int64), pu.oracle_slot_of(sv))
        checks += [(v["os"][bh], sv["Os"], f"{name} head {bh} Os"), (flat(y)[bh], o["Y"], f"{name} head {bh} Y"),
                   (flat(dq)[bh], o["dQ"], f"{name} head {bh} dQ"), (flat(dk)[bh], o["dK"], f"{name} head {bh} dK"),
                   (flat(dv)[bh], o["dV"], f"{name} head {bh} dV")]
        if bh == SAMPLED[name][0]:
            # for information: against the oracle without the bf16 rounding of
            # the attention's inputs
            ox = pu.oracle_head(w, h["q"], h["k"], h["v"], h["dy"], attn_dtype=None)
            pu.record_info(v["os"][bh], ox["saved"]["Os"], f"{name} head {bh} Os [exact attention inputs]")
            for t, n in ((y, "Y"), (dq, "dQ"), (dk, "dK"), (dv, "dV")):
                pu.record_info(flat(t)[bh], ox[n], f"{name} head {bh} {n} [exact attention inputs]")
    pu.assert_all_close(checks)
