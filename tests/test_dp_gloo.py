"""Multi-process checks of the data-parallel plumbing (gloo, CPU, two ranks).

The exchange logic of compressive_fine_tuning_b200.dp is exercised with the
oracle standing in for each rank's kernels: the sum of per-rank LUT gradients
over a token-sharded batch must equal the gradient of the whole batch, and the
row-sharded forward, gathered, must equal the unsharded forward, and the
sketching stage sharded over calibration tokens and then rows must give the
same index map and LUTs as one process.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from compressive_fine_tuning_b200 import dp, synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))


def _dlut_worker(rank, world, port, ntask, average):
    _init(rank, world, port)
    try:
        c = synth.layer_case(7, n=24, d=128, bits=3, gpr=2, T=37, ntask=ntask, with_task=ntask > 1)
        full = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k, c.task, ntask)
        s = dp.token_shard(c.T, rank, world)
        task = None if c.task is None else c.task[s]
        part = oracle.backward_lut(c.x[s], c.dy[s], c.idx, c.gpr, c.k, task, ntask)
        g = torch.from_numpy(np.ascontiguousarray(part, dtype=np.float32))
        red = dp.LutGradReducer(average=average)
        red.submit(g)
        red.wait()
        want = full / world if average else full
        err = np.abs(g.numpy() - want).max()
        assert err <= 1e-6 * (np.abs(want).max() + 1e-30), err
    finally:
        dist.destroy_process_group()


def _fwd_worker(rank, world, port):
    _init(rank, world, port)
    try:
        c = synth.layer_case(11, n=40, d=64, bits=4, gpr=1, T=5, ntask=3, with_task=True)
        full = oracle.forward(c.x, c.idx, c.lut, c.task)
        rows = dp.row_shard(c.n, rank, world)
        y_loc = oracle.forward(c.x, c.idx[rows], c.lut[:, rows], c.task)
        y = dp.gather_rows(torch.from_numpy(y_loc), c.n)
        assert y.shape == full.shape
        assert np.array_equal(y.numpy(), full)
    finally:
        dist.destroy_process_group()


def _sketch_worker(rank, world, port):
    """Calibration tokens sharded for the Gram matrix (one all-reduce), rows
    sharded for Lloyd and the mapping, row blocks gathered: the same index map
    and LUTs as the whole stage on one process."""
    _init(rank, world, port)
    try:
        n, d, gpr, bits = 24, 64, 2, 2
        c = synth.sketch_case(21, n, d, 300)
        idx_ref, lut_ref = oracle.sketch_layer(c.theta, c.x, bits, gpr)
        toks = dp.token_shard(c.s, rank, world)
        h = dp.reduce_gram(torch.from_numpy(oracle.gram(c.x[toks])))
        np.testing.assert_allclose(h.numpy(), oracle.gram(c.x), rtol=1e-12, atol=1e-9)
        u, hd = oracle.inverse_factor(oracle.damped(h.numpy(), 0.01))
        rows = dp.row_shard(n, rank, world)
        lut_loc = oracle.lloyd_luts(c.theta[rows], hd, bits, gpr, 100)
        idx_loc = oracle.sketch_round(c.theta[rows], u, lut_loc)
        lut = dp.gather_row_blocks(torch.from_numpy(lut_loc), n).numpy()
        idx = dp.gather_row_blocks(torch.from_numpy(idx_loc), n).numpy()
        assert np.array_equal(lut.view(np.uint16), lut_ref.view(np.uint16))
        assert np.array_equal(idx, idx_ref)
    finally:
        dist.destroy_process_group()


def test_sketching_stage_shards_tokens_then_rows():
    mp.spawn(_sketch_worker, args=(2, _free_port()), nprocs=2, join=True)


@pytest.mark.parametrize("ntask,average", [(1, False), (3, False), (1, True)])
def test_token_sharded_lut_gradient_sums_to_whole_batch(ntask, average):
    mp.spawn(_dlut_worker, args=(2, _free_port(), ntask, average), nprocs=2, join=True)


def test_row_sharded_forward_gathers_to_whole_output():
    mp.spawn(_fwd_worker, args=(2, _free_port()), nprocs=2, join=True)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shards_partition_exactly(world):
    for T in (0, 1, 7, 8192, 8193):
        cover = []
        for r in range(world):
            s = dp.token_shard(T, r, world)
            cover.extend(range(T)[s])
            assert (s.stop - s.start) in (T // world, T // world + 1)
        assert cover == list(range(T))
    for n in (8, 4096, 11008, 1024):
        cover = []
        for r in range(world):
            s = dp.row_shard(n, r, world)
            assert s.start % 8 == 0 and s.stop % 8 == 0
            cover.extend(range(n)[s])
        assert cover == list(range(n))
    with pytest.raises(ValueError):
        dp.row_shard(12, 0, world)
