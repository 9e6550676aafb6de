"""Tensor-parallel layers on two gloo ranks on the CPU (the compute steps
through the oracle, the collectives through torch.distributed): the
column-parallel layer's gathered output and the row-parallel layer's reduced
output equal the unsharded layer bit for bit."""
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

    import sq_inputs
    from tp_oracle_ops import OracleOps
    from w8a8_int8_linear_channel_b200.tp import (ColumnParallelSmoothQuantLinear, DistComm,
                                                  RowParallelSmoothQuantLinear, shard_range)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ops, comm = OracleOps(), DistComm()
    T = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a))

    # column-parallel, LayerNorm folded (the attention-projection construction)
    wl = sq_inputs.WORKLOADS["tiny_ln"]
    w, calib, h = sq_inputs.weight(wl), sq_inputs.calib_rows(wl), sq_inputs.run_rows(wl, 0, wl.M)
    bias = (np.arange(wl.N) % 7 - 3).astype(np.float16) * np.float16(0.25)
    lo, hi = shard_range(wl.N, rank, world)
    col = ColumnParallelSmoothQuantLinear.from_float(
        T(w[lo:hi]), T(calib), wl.alpha, T(sq_inputs.gamma(wl)), T(sq_inputs.beta(wl)), T(bias[lo:hi]),
        ops=ops, comm=comm)
    y_col = col.forward_gather(T(h)).numpy()

    # row-parallel, smoothing by 1/s at run time (the FFN-down construction)
    wl2 = sq_inputs.WORKLOADS["tiny"]
    w2, calib2, h2 = sq_inputs.weight(wl2), sq_inputs.calib_rows(wl2), sq_inputs.run_rows(wl2, 0, wl2.M)
    lo, hi = shard_range(wl2.K, rank, world)
    row = RowParallelSmoothQuantLinear.from_float(T(w2[:, lo:hi]), T(calib2[:, lo:hi]), wl2.alpha, T(bias),
                                                  ops=ops, comm=comm)
    y_row = row.forward(T(h2[:, lo:hi])).numpy()
    out[rank] = (y_col, y_row, row.sw.numpy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_rank_tensor_parallel_equals_unsharded():
    import oracle
    import sq_inputs
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")

    wl = sq_inputs.WORKLOADS["tiny_ln"]
    bias = (np.arange(wl.N) % 7 - 3).astype(np.float16) * np.float16(0.25)
    ref = oracle.run_step(sq_inputs.calib_rows(wl), sq_inputs.weight(wl), sq_inputs.run_rows(wl, 0, wl.M),
                          sq_inputs.gamma(wl), sq_inputs.beta(wl), bias, wl.alpha)
    wl2 = sq_inputs.WORKLOADS["tiny"]
    ref2 = oracle.run_step(sq_inputs.calib_rows(wl2), sq_inputs.weight(wl2), sq_inputs.run_rows(wl2, 0, wl2.M),
                           None, None, bias, wl2.alpha)
    for r in range(world):
        y_col, y_row, sw = out[r]
        assert np.array_equal(y_col.view(np.uint16), ref["y"].view(np.uint16))
        assert np.array_equal(sw, ref2["sw"])  # the weight scales span every input channel
        assert np.array_equal(y_row.view(np.uint16), ref2["y"].view(np.uint16))


def _worker_k_overflow(rank, world, port, out):
    import torch

    from tp_oracle_ops import OracleOps
    from w8a8_int8_linear_channel_b200 import MAX_K
    from w8a8_int8_linear_channel_b200.tp import DistComm, RowParallelSmoothQuantLinear
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    k_rank = (MAX_K // 2 // 16 + 2) * 16  # each slice fits, their sum does not
    assert k_rank <= MAX_K < world * k_rank
    w = torch.zeros((1, k_rank), dtype=torch.float16)
    try:
        RowParallelSmoothQuantLinear.from_float(w, w.clone(), 0.5, ops=OracleOps(), comm=DistComm())
        out[rank] = "no error"
    except ValueError as e:
        out[rank] = str(e)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_row_parallel_rejects_total_k_beyond_int32_bound():
    """Each rank's K slice is within MAX_K but their sum is not: every rank refuses before any
    compute, since the summed int32 accumulators could wrap."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker_k_overflow, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for r in range(world):
        assert "exceeds" in out[r], out[r]
