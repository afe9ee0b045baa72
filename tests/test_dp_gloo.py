"""The data-parallel path on CPU with two gloo ranks: each rank owns its own tokens, the fp32
weight-gradient partials are summed across ranks and re-quantized, and step times are combined
as the maximum over ranks. The per-rank compute is the oracle (the product kernels need a B200);
what is under test is the decomposition and the collective logic of
``int8_fully_quantized_b200.parallel``: the plain all-reduce and the overlapped exchange
(WgradExchange) that the multi-GPU step uses, whose re-quantized dW must match the oracle's
weight gradient over all ranks' tokens."""
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


def _overlap_worker(rank, world, port, out_dir):
    """Two layers' weight gradients, as in the layer step: the first partial's all-reduce is started,
    more work runs while it is in flight, the second is started, and both are re-quantized at the end."""
    import sys
    sys.path.insert(0, ROOT)
    import oracle as O
    from inputs import synthetic as S
    from int8_fully_quantized_b200 import parallel as P
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(P.shard_seed(7, rank))
        dy2 = O.quantize_block(S.grad(rng, 64, 96))
        g = O.quantize_block(S.activation(rng, 64, 160, 2, 10.0))
        dy1 = O.quantize_block(S.grad(rng, 64, 160))
        x = O.quantize_block(S.activation(rng, 64, 96, 2, 20.0))
        ex = P.WgradExchange()
        ex.start(torch.from_numpy(O.linear_wgrad(*dy2, *g).copy()), "dW2")    # [96, 160]
        O.linear_dgrad(*dy1, *O.quantize_block(S.weight(rng, 160, 96)))       # work while it is in flight
        ex.start(torch.from_numpy(O.linear_wgrad(*dy1, *x).copy()), "dW1")    # [160, 96]
        res = ex.finish(lambda tag, dw: (tag, O.requantize(dw.numpy())))
        assert [t for t, _ in res] == ["dW2", "dW1"]
        for tag, (q, s) in res:
            np.save(os.path.join(out_dir, f"{tag}_q_{rank}.npy"), q)
            np.save(os.path.join(out_dir, f"{tag}_s_{rank}.npy"), s)
        for name, t in (("dy2", dy2), ("g", g), ("dy1", dy1), ("x", x)):
            np.save(os.path.join(out_dir, f"{name}_q_{rank}.npy"), t[0])
            np.save(os.path.join(out_dir, f"{name}_s_{rank}.npy"), t[1])
    finally:
        dist.destroy_process_group()


def test_dp_overlapped_exchange_requantized_two_ranks(tmp_path):
    import oracle as O
    world = 2
    mp.start_processes(_overlap_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    cat = lambda name, part: np.concatenate([np.load(tmp_path / f"{name}_{part}_{r}.npy") for r in range(world)])
    full = {"dW2": O.linear_wgrad(cat("dy2", "q"), cat("dy2", "s"), cat("g", "q"), cat("g", "s")),
            "dW1": O.linear_wgrad(cat("dy1", "q"), cat("dy1", "s"), cat("x", "q"), cat("x", "s"))}
    for tag in ("dW2", "dW1"):
        q = [np.load(tmp_path / f"{tag}_q_{r}.npy") for r in range(world)]
        s = [np.load(tmp_path / f"{tag}_s_{r}.npy") for r in range(world)]
        assert np.array_equal(q[0], q[1]) and np.array_equal(s[0], s[1])   # every rank re-quantizes the same sum
        qr, sr = O.requantize(full[tag])
        d = np.abs(q[0].astype(np.int32) - qr)
        assert d.max() <= 1 and np.count_nonzero(d) <= 1e-3 * d.size, tag
        assert np.all(np.abs(s[0].astype(np.float64) - sr) <= 1e-5 * sr), tag


def test_single_rank_helpers_are_noops():
    from int8_fully_quantized_b200 import parallel as P
    t = torch.ones(4)
    assert P.allreduce_wgrad_(t) is t and torch.equal(t, torch.ones(4))
    assert P.max_over_ranks(3.0) == 3.0
    assert P.world() == (0, 1)
    assert P.shard_seed(0, 0) != P.shard_seed(0, 1)
    ex = P.WgradExchange()
    ex.start(t, "a")
    assert ex.finish(lambda tag, dw: (tag, dw is t)) == [("a", True)]
