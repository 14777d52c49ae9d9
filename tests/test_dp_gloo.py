"""Two gloo ranks on CPU: row sharding plus the all-reduce of the weight gradients
reproduce the single-process backward (fp64 oracle on each shard)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from block_diagonal_linear_b200 import dp, synthetic


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, shape, rows, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = dict(shape, rows=rows, dtype="f32")
        inp = synthetic.make_inputs(w, seed=77)
        a, b = dp.shard_rows(rows, rank, world)
        dX, dR, dL = oracle.backward(shape, inp["dY"].f64[a:b], inp["X"].f64[a:b], inp["R"].f64,
                                     inp["L"].f64, nthreads=1)
        tR, tL = torch.from_numpy(dR), torch.from_numpy(dL)
        dp.allreduce_weight_grads(tR, tL)
        np.save(os.path.join(out_dir, "dX_%d.npy" % rank), dX)
        np.save(os.path.join(out_dir, "dR_%d.npy" % rank), tR.numpy())
        np.save(os.path.join(out_dir, "dL_%d.npy" % rank), tL.numpy())
    finally:
        dist.destroy_process_group()


def test_shard_rows_partition():
    for rows in (0, 1, 7, 16384):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_rows(rows, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            assert max(b - a for a, b in spans) - min(b - a for a, b in spans) <= 1
    with pytest.raises(ValueError):
        dp.shard_rows(4, 2, 2)


def test_two_rank_backward_matches_single_process(tmp_path):
    shape = dict(nb1=4, in1=4, out1=4, nb2=4, in2=4, out2=4, out_transpose=1)
    rows, world = 37, 2
    mp.start_processes(_worker, args=(world, _free_port(), shape, rows, str(tmp_path)),
                       nprocs=world, start_method="spawn")
    w = dict(shape, rows=rows, dtype="f32")
    inp = synthetic.make_inputs(w, seed=77)
    rX, rR, rL = oracle.backward(shape, inp["dY"].f64, inp["X"].f64, inp["R"].f64, inp["L"].f64)
    dX = np.concatenate([np.load(tmp_path / ("dX_%d.npy" % r)) for r in range(world)])
    np.testing.assert_allclose(dX, rX, rtol=1e-12, atol=1e-12)
    for r in range(world):
        np.testing.assert_allclose(np.load(tmp_path / ("dR_%d.npy" % r)), rR, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(np.load(tmp_path / ("dL_%d.npy" % r)), rL, rtol=1e-12, atol=1e-12)
