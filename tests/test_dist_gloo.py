"""Data-parallel calibration with two gloo ranks on the CPU: each rank
calibrates on its own shard of the calibration tokens, the ranges are
max-all-reduced, and every rank ends with the range of the whole set (and so
the same smoothing factor)."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch

    import oracle
    import sq_inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = sq_inputs.WORKLOADS["tiny_ln"]
    rows = wl.calib // world
    shard = sq_inputs.calib_rows(wl, rank * rows, rows)
    a = oracle.calibrate_absmax(shard, gamma=sq_inputs.gamma(wl), beta=sq_inputs.beta(wl))
    t = torch.from_numpy(a)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    s, _ = oracle.smooth(t.numpy(), oracle.calibrate_absmax(sq_inputs.weight(wl)), wl.alpha)
    out[rank] = (t.numpy().copy(), s)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_calibration_matches_whole_set():
    import oracle
    import sq_inputs
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    wl = sq_inputs.WORKLOADS["tiny_ln"]
    whole = oracle.calibrate_absmax(sq_inputs.calib_rows(wl), gamma=sq_inputs.gamma(wl),
                                    beta=sq_inputs.beta(wl))
    for r in range(world):
        amax, s = out[r]
        assert np.array_equal(amax, whole)
    assert np.array_equal(out[0][1], out[1][1])
