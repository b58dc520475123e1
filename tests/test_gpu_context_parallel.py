"""Context parallelism with the CUDA backend: the layer's tokens split over 2
ranks (processes sharing this GPU, with a gloo group for the exchanges), each
rank running its shard through the library's kernels (the shard forms of the
gather, scatter-back, adjoint and pool adjoint, the row-window attention), and
the concatenated shards compared with the unsharded GPU layer and the fp64
oracle at the parity bar."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import hierarchical_sparse_attention_pyramid_b200 as lh
from hierarchical_sparse_attention_pyramid_b200 import context_parallel as cp
from hierarchical_sparse_attention_pyramid_b200.synth import Workload
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

# N/2 a multiple of p^(L-1); bf16 rows of 128; two heads with different segment lengths
CASES = {
    "parents_p2": Workload("cp_parents_p2", 1, 2, 8192, 128, 4, 2, 48, "bf16", "qk_sum", "lognormal_token", 31,
                           chunk=512),
    "direct_p4": Workload("cp_direct_p4", 1, 2, 8192, 128, 3, 4, 64, "bf16", "qk_sum", "iid", 32, chunk=1024,
                          selection="direct"),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, name, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        w = CASES[name]
        x = pu.all_heads_case(w)
        shard = cp.Shard(w.N, w.p, w.L, world, rank)
        sl = slice(shard.t0, shard.t1)
        q, k, v, dy = (x[n].reshape(w.B * w.H, w.N, w.d)[:, sl].contiguous().cuda() for n in ("q", "k", "v", "dy"))
        be = cp.CudaBackend(lh.Layer.of(w), shard)
        y, ctx = cp.cp_forward(be, shard, q, k, v, w.selection)
        dq, dk, dv = cp.cp_backward(be, shard, dy, ctx)
        torch.cuda.synchronize()
        out[rank] = tuple(t.float().cpu().numpy() for t in (y, dq, dk, dv))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", sorted(CASES))
def test_sharded_layer_matches_unsharded(name):
    w = CASES[name]
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), name, out), nprocs=world, join=True)
    x = pu.all_heads_case(w)
    L = lh.Layer.of(w)
    y, bufs = lh.forward(L, *(x[n].cuda() for n in ("q", "k", "v")))
    grads = lh.backward(L, x["dy"].cuda(), bufs)
    lh.check_error(bufs)
    whole = [t.reshape(w.B * w.H, w.N, w.d).float().cpu().numpy() for t in (y, *grads)]
    for t, nm in enumerate(("Y", "dQ", "dK", "dV")):
        got = np.concatenate([out[r][t] for r in range(world)], axis=1)
        for bh in range(w.B * w.H):
            o = pu.oracle_head(w, x["q"][0, bh], x["k"][0, bh], x["v"][0, bh], x["dy"][0, bh])
            pu.assert_close(torch.from_numpy(got[bh]).to(torch.bfloat16), o[nm], f"{name} sharded {nm} head {bh}")
            # against the unsharded kernels: only the summation order at the shard edge differs
            pu.assert_close(torch.from_numpy(got[bh]).to(torch.bfloat16), whole[t][bh],
                            f"{name} sharded vs whole {nm} head {bh}")
