"""GPU parity of the whole layer (lh_forward / lh_backward through the C ABI)
against the fp64 oracle on small workloads: selected indices bit-exact, Y and
dQ, dK, dV within the tolerance of parity_util."""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_pyramid_b200 as lh
from tests import parity_util as pu
from tests.test_gpu_stages import SMALL, case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", sorted(SMALL))
def test_forward_backward(name):
    w, x, heads = case(name)
    L = lh.Layer.of(w)
    y, bufs = lh.forward(L, x["q"], x["k"], x["v"])
    dq, dk, dv = lh.backward(L, x["dy"], bufs)
    lh.check_error(bufs)
    v = bufs.ctx_views()
    flat = lambda t: t.reshape(w.B * w.H, w.N, w.d)  # noqa: E731
    checks = []
    for bh, o in enumerate(heads):
        sv = o["saved"]
        if w.L > 1:
            np.testing.assert_array_equal(v["sel"][bh].cpu().numpy().astype(np.int64), pu.oracle_sel_flat(w, sv))
        np.testing.assert_array_equal(v["seq_map"][bh].cpu().numpy().astype(np.int64), pu.oracle_seq_map(sv))
        np.testing.assert_array_equal(v["slot_of"][bh].cpu().numpy().astype(np.int64), pu.oracle_slot_of(sv))
        checks += [(v["os"][bh], sv["Os"], f"{name} head {bh} Os"), (flat(y)[bh], o["Y"], f"{name} head {bh} Y"),
                   (flat(dq)[bh], o["dQ"], f"{name} head {bh} dQ"), (flat(dk)[bh], o["dK"], f"{name} head {bh} dK"),
                   (flat(dv)[bh], o["dV"], f"{name} head {bh} dV")]
        # for information: the same outputs against the oracle run without the
        # bf16 rounding of the attention's inputs (how far that reading moves
        # the reference point)
        ox = pu.oracle_head(w, x["q"][bh // w.H, bh % w.H], x["k"][bh // w.H, bh % w.H], x["v"][bh // w.H, bh % w.H],
                            x["dy"][bh // w.H, bh % w.H], attn_dtype=None)
        pu.record_info(v["os"][bh], ox["saved"]["Os"], f"{name} head {bh} Os [exact attention inputs]")
        for t, n in ((y, "Y"), (dq, "dQ"), (dk, "dK"), (dv, "dV")):
            pu.record_info(flat(t)[bh], ox[n], f"{name} head {bh} {n} [exact attention inputs]")
    pu.assert_all_close(checks)


def test_forward_is_deterministic():
    w, x, _ = case("chunked_lognorm")
    L = lh.Layer.of(w)
    y1, b1 = lh.forward(L, x["q"], x["k"], x["v"])
    g1 = lh.backward(L, x["dy"], b1)
    y2, b2 = lh.forward(L, x["q"], x["k"], x["v"])
    g2 = lh.backward(L, x["dy"], b2)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(b1.ctx, b2.ctx)
    # every output row has one writer and a fixed summation order (no atomics
    # anywhere): repeated runs agree bit for bit
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_autograd_function_matches_direct_calls():
    w, x, _ = case("ragged")
    q, k, v = (x[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    y = lh.lighthouse_attention(q, k, v, L=w.L, p=w.p, k_budget=w.k, chunk=w.chunk, scorer=w.scorer)
    y.backward(x["dy"])
    L = lh.Layer.of(w)
    y2, bufs = lh.forward(L, x["q"], x["k"], x["v"])
    dq2, dk2, dv2 = lh.backward(L, x["dy"], bufs)
    torch.cuda.synchronize()
    assert torch.equal(y.detach(), y2)
    assert torch.equal(q.grad, dq2) and torch.equal(k.grad, dk2) and torch.equal(v.grad, dv2)


@pytest.mark.parametrize("what", ["dy", "v"])
def test_fp16_range_of_the_backward_is_reported(what):
    """dOs and Vs enter the backward's dV and dP products in fp16: a value
    beyond 65504 is reported as LH_ERR_DEVICE by check_error, not passed on
    silently."""
    w, x, _ = case("ragged")
    L = lh.Layer.of(w)
    q, k, v, dy = (x[n] for n in ("q", "k", "v", "dy"))
    if what == "dy":
        dy = torch.full_like(dy, 30000.0)  # a top-level slot sums 4 rows: 120000
    else:
        v = torch.full_like(v, 70000.0)
    y, bufs = lh.forward(L, q, k, v)
    lh.backward(L, dy, bufs)
    with pytest.raises(Exception, match="LH_ERR_DEVICE"):
        lh.check_error(bufs)
    # the word is cleared and ordinary inputs run clean again
    y, bufs = lh.forward(L, x["q"], x["k"], x["v"])
    lh.backward(L, x["dy"], bufs)
    lh.check_error(bufs)
