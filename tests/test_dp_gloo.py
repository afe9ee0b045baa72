"""The data-parallel path on CPU with two gloo ranks: each rank owns its own tokens, the fp32
weight-gradient partials are summed across ranks and re-quantized, and step times are combined
as the maximum over ranks. The per-rank compute is the oracle (the product kernels need a B200);
what is under test is the decomposition and the collective logic of
``int8_fully_quantized_b200.parallel``."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import oracle as O
    from inputs import synthetic as S
    from int8_fully_quantized_b200 import parallel as P
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, N, K = 128, 96, 64
        rng = np.random.default_rng(P.shard_seed(0, rank))
        dy = O.quantize_block(S.grad(rng, M, N))
        x = O.quantize_block(S.activation(rng, M, K, 2, 20.0))
        partial = torch.from_numpy(O.linear_wgrad(*dy, *x).copy())
        P.allreduce_wgrad_(partial)
        t = P.max_over_ranks(1.5 + rank)
        np.save(os.path.join(out_dir, f"dw_{rank}.npy"), partial.numpy())
        np.save(os.path.join(out_dir, f"t_{rank}.npy"), np.array([t]))
        np.save(os.path.join(out_dir, f"dy_{rank}.npy"), dy[0]); np.save(os.path.join(out_dir, f"dys_{rank}.npy"), dy[1])
        np.save(os.path.join(out_dir, f"x_{rank}.npy"), x[0]); np.save(os.path.join(out_dir, f"xs_{rank}.npy"), x[1])
        assert P.world() == (rank, world)
    finally:
        dist.destroy_process_group()


def test_dp_wgrad_allreduce_two_ranks(tmp_path):
    import oracle as O
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    dws = [np.load(tmp_path / f"dw_{r}.npy") for r in range(world)]
    assert np.array_equal(dws[0], dws[1])                      # every rank holds the same sum
    assert [float(np.load(tmp_path / f"t_{r}.npy")[0]) for r in range(world)] == [2.5, 2.5]
    # the summed partials equal the weight gradient over all ranks' tokens
    dyq = np.concatenate([np.load(tmp_path / f"dy_{r}.npy") for r in range(world)])
    dys = np.concatenate([np.load(tmp_path / f"dys_{r}.npy") for r in range(world)])
    xq = np.concatenate([np.load(tmp_path / f"x_{r}.npy") for r in range(world)])
    xs = np.concatenate([np.load(tmp_path / f"xs_{r}.npy") for r in range(world)])
    full = O.linear_wgrad(dyq, dys, xq, xs)
    # two fp32 partials summed once: within a few ulps of the partials, far below any index error
    assert np.allclose(dws[0], full, rtol=1e-6, atol=1e-6 * np.abs(full).max())
    q, s = O.requantize(dws[0])
    qr, sr = O.requantize(full)
    d = np.abs(q.astype(np.int32) - qr)
    assert d.max() <= 1 and np.count_nonzero(d) <= 1e-3 * d.size


def test_single_rank_helpers_are_noops():
    from int8_fully_quantized_b200 import parallel as P
    t = torch.ones(4)
    assert P.allreduce_wgrad_(t) is t and torch.equal(t, torch.ones(4))
    assert P.max_over_ranks(3.0) == 3.0
    assert P.world() == (0, 1)
    assert P.shard_seed(0, 0) != P.shard_seed(0, 1)
