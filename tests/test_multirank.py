"""Host logic of bench.py under torchrun, as two gloo ranks on the CPU: the
process-group setup from the launcher's environment, the barrier, and the
max-over-ranks step time from which the whole-job throughput is computed.
The layer has no collective on its data path (each rank runs its own
layer), so nothing else crosses ranks."""

import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist

    w, r, local = bench.dist_setup()
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    # each rank's own step time; the job's time is the slowest rank's
    ms = 10.0 + 5.0 * rank
    out[rank] = bench.max_over_ranks(ms, w, "cpu")
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_max_step_time():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}
    # whole-job tokens/s: both ranks' tokens over the slowest rank's time
    n = 524288
    assert world * n / (out[0] / 1e3) == 2 * n / 0.015
