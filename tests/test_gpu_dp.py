"""The data-parallel layer step of bench.py on the GPU: two ranks, each with its own tokens and the
same weights, run `GpuStep.run_data_parallel` (fp32 weight-gradient partials from the GEMM kernel,
their all-reduce started as soon as each exists, re-quantization of the sums with the GPU quantizer).
Both ranks run on cuda:0 over a gloo process group: the all-reduce is host-mediated, so no kernel of
one rank waits on another rank's kernels. Checked against the oracle: every rank holds the same
summed partials and codes, the sums are the two ranks' own partials added, the codes are the
quantizer rule applied to the sums, and the sums are the weight gradient over both ranks' tokens."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DIMS = (256, 256, 512)   # tokens per rank M, hidden H, inner F


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import int8_fully_quantized_b200 as jf
        from int8_fully_quantized_b200 import parallel as P
        jf.load_library()
        host = bench.host_inputs(P.shard_seed(0, rank), seed_weight=0, dims=DIMS)
        step = bench.GpuStep(host, world)
        step.run_data_parallel()
        torch.cuda.synchronize()
        # this rank's own partials: the same two weight-gradient GEMMs on its tokens, no exchange
        p2, p1 = torch.empty_like(step.dw2_f32), torch.empty_like(step.dw1_f32)
        jf.jf_linear_wgrad(step.dY2, step.G, None, p2)
        jf.jf_linear_wgrad(step.dY1, step.Xn, None, p1)
        torch.cuda.synchronize()
        arrays = {"dW2_q": step.dW2.q, "dW2_s": step.dW2.s, "dW1_q": step.dW1.q, "dW1_s": step.dW1.s,
                  "sum2": step.dw2_f32, "sum1": step.dw1_f32, "own2": p2, "own1": p1,
                  "dY2_q": step.dY2.q, "dY2_s": step.dY2.s, "G_q": step.G.q, "G_s": step.G.s,
                  "dY1_q": step.dY1.q, "dY1_s": step.dY1.s, "Xn_q": step.Xn.q, "Xn_s": step.Xn.s}
        for k, v in arrays.items():
            np.save(os.path.join(out_dir, f"{k}_{rank}.npy"), v.cpu().numpy())
        np.save(os.path.join(out_dir, f"status_{rank}.npy"), np.array([jf.jf_device_status()]))
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
@pytest.mark.timeout(600)
def test_data_parallel_step_two_ranks(tmp_path):
    import oracle as O
    from gpu_common import assert_gemm_f32_close
    world = 2
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    ld = lambda name, r: np.load(tmp_path / f"{name}_{r}.npy")
    assert [int(ld("status", r)[0]) for r in range(world)] == [0, 0]
    for tag, a, b in (("2", "dY2", "G"), ("1", "dY1", "Xn")):
        # every rank holds the same sum and the same codes
        for name in (f"sum{tag}", f"dW{tag}_q", f"dW{tag}_s"):
            assert np.array_equal(ld(name, 0), ld(name, 1)), name
        s = ld(f"sum{tag}", 0)
        # the sum is the two ranks' own fp32 partials added (one rounding, in either order)
        assert np.array_equal(s, ld(f"own{tag}", 0) + ld(f"own{tag}", 1)), f"sum{tag}"
        # the codes are the quantizer rule applied to the sum
        q, sc = O.quantize_block(s)
        assert np.array_equal(ld(f"dW{tag}_q", 0), q) and np.array_equal(ld(f"dW{tag}_s", 0), sc), f"dW{tag}"
        # the sum is the weight gradient over both ranks' tokens
        cat = lambda n: np.concatenate([ld(n, r) for r in range(world)])
        Aq, As, Bq, Bs = cat(f"{a}_q"), cat(f"{a}_s"), cat(f"{b}_q"), cat(f"{b}_s")
        ref = O.linear_wgrad(Aq, As, Bq, Bs)
        mag = O.linear_wgrad(np.abs(Aq.astype(np.int16)).astype(np.int8), As,
                             np.abs(Bq.astype(np.int16)).astype(np.int8), Bs)
        assert_gemm_f32_close(s, ref, mag, f"dW{tag}")
