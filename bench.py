#!/usr/bin/env python
"""Benchmark of the per-block INT8 data-flow hot path on B200.

One step = one training pass (forward and backward) of the hidden-4096 transformer MLP layer on INT8
blocks, M = 8192 tokens, hidden H = 4096, inner F = 16384 (the hidden-4096 layer of the Jetfire
summary's "Key results" and "Measured effects" table): X ~ N(0,1) with 4 outlier channels x50, W1 and
W2 ~ N(0, 0.02), the upstream gradient dY ~ N(0, 1e-3), all bf16 on entry:

    forward:  quantize X -> LayerNorm_i8 -> fc1 (Y1 = Xn W1^T) -> GELU_i8 -> fc2 (Y2 = G W2^T)
              (quantize W1, W2 beside them)
    backward: quantize dY -> fc2 dgrad (dG = dY W2) and wgrad (dW2 = dY^T G) -> GELU_i8 backward
              -> fc1 dgrad (dXn = dY1 W1) and wgrad (dW1 = dY1^T Xn) -> LayerNorm_i8 backward
              (dX, dgamma, dbeta) -> dequantize dX to bf16

Every operator reads and writes INT8 blocks with per-block scales; six block-scaled INT8 GEMMs of
2 * 8192 * 4096 * 16384 int8 ops each. Inputs are resident in HBM when the timed region starts; L2
is flushed between steps (a 256 MiB write outside the timed events). ``value`` is the whole-step
throughput in TOPS counted on the six GEMMs over the step time, summed over ranks. ``--gpus N``
(under torchrun) runs N data-parallel ranks, each with its own 8192 tokens; the fp32 weight-gradient
partials are summed with NCCL all-reduces that overlap the rest of the backward, then re-quantized
(weak scaling).

``--impl reference`` times the CPU oracle (the method written out plainly in numpy) on a bounded
sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "per-block INT8 GEMM TOPS (% INT8 peak); quantize/GELU/LN GB/s (% HBM)"
WORKLOAD_NAME = ("hidden-4096 MLP layer on INT8 blocks, forward and backward: LayerNorm_i8 -> fc1 4096->16384 -> "
                 "GELU_i8 -> fc2 16384->4096, six block-scaled INT8 GEMMs (fwd, dgrad, wgrad of fc1 and fc2), "
                 "quantize, GELU_i8 and LayerNorm_i8 backward, dequantize (per rank)")
NOMINAL_I8_OVER_BF16 = 2.0       # dense int8 (4.5 POPS) / dense bf16 (2.25 PFLOP/s), nominal B200
NOMINAL_I8_TOPS = 4500.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
ALU_LANES_PER_CLK_PER_SM = 128   # 4 warp schedulers x 32 lanes, one issue per scheduler per clock
B200_SMS = 148


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    p.add_argument("--no-sweep", action="store_true", help="skip the memory-bound sweep in the main line")
    p.add_argument("--eager", action="store_true", help="time eager launches instead of the step's CUDA graph")
    p.add_argument("--configs", action="store_true",
                   help="time the single-linear, hidden-4096 GEMM and hidden-4096 MLP-block workloads (one JSON line)")
    p.add_argument("--cpu-sample-blocks", type=int, default=16,
                   help="oracle sample: this many x this many output blocks of each GEMM")
    p.add_argument("--sweep", action="store_true",
                   help="time the memory-bound kernels on the M x 4096 sweep instead of the step")
    p.add_argument("--profile-gemm", action="store_true",
                   help="run the three block-scaled GEMM modes on the GPT2-medium fc1 shapes (M=4096, K=1024, "
                        "N=4096) --steps times each, L2 flushed before each launch: a small case for ncu captures")
    p.add_argument("--sweep-m", type=int, nargs="*", default=[1024, 8192, 65536])
    p.add_argument("--sweep-ops", nargs="*", default=["quantize_bf16", "dequantize_bf16", "gelu_i8", "layernorm_i8",
                                                      "gelu_i8_bwd", "layernorm_i8_bwd", "fused_fc1",
                                                      "granularity_mse", "mxfp8_fc1"])
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if any(k not in d for k in ("hbm_gbs", "bf16_tflops")):
            raise KeyError("incomplete peaks file")
        return {**FALLBACK_PEAKS, **{k: float(d[k]) for k in FALLBACK_PEAKS if k in d}}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# --------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
               0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                for i in range(pynvml.nvmlDeviceGetCount()):
                    hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                    u = pynvml.nvmlDeviceGetUUID(hh)
                    u = u.decode() if isinstance(u, bytes) else u
                    if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                        h = hh
            self.h = h if h is not None else pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - only without NVML
            self.nvml = None
            self.error = str(e)

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "window": "warm-up and timed steps, NVML every 5 ms"}


# --------------------------------------------------------------------------------------------
# host inputs
# --------------------------------------------------------------------------------------------
def layer_dims():
    from inputs import synthetic as S
    w = S.WORKLOADS["h4096_fc1"]
    return w["M"], w["K"], w["N"]          # tokens M, hidden H, inner F


def host_inputs(seed_tokens, seed_weight, dims=None):
    """bf16 bit patterns of X [M, H], dY [M, H], W1 [F, H], W2 [H, F]; fp32 gamma, beta [H]
    (dims = (M, H, F), the layer's by default)."""
    from inputs import synthetic as S
    M, H, F = dims or layer_dims()
    n_out, fac = S.WORKLOADS["h4096_fc1"]["x_outliers"]
    rng = np.random.default_rng(seed_tokens)
    x = S.activation(rng, M, H, n_out, fac)
    dy = S.grad(rng, M, H)
    rw = np.random.default_rng(seed_weight)
    w1 = S.weight(rw, F, H)
    w2 = S.weight(rw, H, F)
    gamma = rw.uniform(0.5, 1.5, H).astype(np.float32)
    beta = rw.normal(0, 0.1, H).astype(np.float32)
    return {"x": S.to_bf16_bits(x), "dy": S.to_bf16_bits(dy), "w1": S.to_bf16_bits(w1), "w2": S.to_bf16_bits(w2),
            "gamma": gamma, "beta": beta}


def gpt2m_inputs(seed):
    """GPT2-medium fc1 operands (M=4096, K=1024, N=4096; X with 10 channels x30) for the side measurements."""
    from inputs import synthetic as S
    w = S.WORKLOADS["gpt2m_fc1"]
    M, K, N = w["M"], w["K"], w["N"]
    rng = np.random.default_rng(seed)
    n_out, fac = w["x_outliers"]
    x = S.activation(rng, M, K, n_out, fac)
    wt = S.weight(np.random.default_rng(seed + 100), N, K)
    return M, K, N, {"x": S.to_bf16_bits(x), "w": S.to_bf16_bits(wt)}


def sbytes(r, c):
    return (r // 32) * (c // 32) * 4


def bytes_quant(r, c, in_bytes):  # read input, write codes + scales
    return r * c * (in_bytes + 1) + sbytes(r, c)


def bytes_i8_op(r, c, extra=0):  # read codes + scales, write codes + scales
    return 2 * (r * c + sbytes(r, c)) + extra


# --------------------------------------------------------------------------------------------
# our implementation
# --------------------------------------------------------------------------------------------
class GpuStep:
    OPS = ["quantize_x", "layernorm_i8", "quantize_w1", "quantize_w2", "fc1_fwd", "gelu_i8", "fc2_fwd",
           "quantize_dy", "fc2_dgrad", "fc2_wgrad", "gelu_i8_bwd", "fc1_dgrad", "fc1_wgrad", "layernorm_i8_bwd",
           "dequantize_dx"]
    GEMMS = ["fc1_fwd", "fc2_fwd", "fc2_dgrad", "fc2_wgrad", "fc1_dgrad", "fc1_wgrad"]

    def __init__(self, host, world_size):
        import torch
        import int8_fully_quantized_b200 as jf
        self.jf, self.torch = jf, torch
        (M, H), F = host["x"].shape, host["w1"].shape[0]   # the layer's sizes, from its inputs
        self.M, self.H, self.F, self.world = M, H, F, world_size
        dev = torch.device("cuda", torch.cuda.current_device())
        bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        self.xb, self.dyb, self.w1b, self.w2b = bf(host["x"]), bf(host["dy"]), bf(host["w1"]), bf(host["w2"])
        self.gamma = torch.from_numpy(host["gamma"]).to(dev)
        self.beta = torch.from_numpy(host["beta"]).to(dev)
        e = lambda r, c: jf.empty_qtensor(r, c, dev)
        self.Xq, self.Xn, self.W1, self.W2 = e(M, H), e(M, H), e(F, H), e(H, F)
        self.Y1, self.G, self.Y2 = e(M, F), e(M, F), e(M, H)
        self.dY2, self.dG, self.dW2, self.dY1, self.dXn, self.dW1, self.dX = \
            e(M, H), e(M, F), e(H, F), e(M, F), e(M, H), e(F, H), e(M, H)
        self.dgamma = torch.empty(H, dtype=torch.float32, device=dev)
        self.dbeta = torch.empty(H, dtype=torch.float32, device=dev)
        self.ln_ws = torch.empty(jf.jf_layernorm_i8_bwd_workspace_bytes(M, H), dtype=torch.uint8, device=dev)
        self.dx_bf16 = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        if world_size > 1:
            self.dw1_f32 = torch.empty((F, H), dtype=torch.float32, device=dev)
            self.dw2_f32 = torch.empty((H, F), dtype=torch.float32, device=dev)
        self.launches_per_step = (16 if world_size == 1 else 19)   # kernels of ours (LN backward: two)
        self.bytes = {
            "quantize_x": bytes_quant(M, H, 2), "quantize_w1": bytes_quant(F, H, 2),
            "quantize_w2": bytes_quant(H, F, 2), "quantize_dy": bytes_quant(M, H, 2),
            "layernorm_i8": bytes_i8_op(M, H, 8 * H), "gelu_i8": bytes_i8_op(M, F),
            "gelu_i8_bwd": bytes_i8_op(M, F, M * F + sbytes(M, F)),
            "layernorm_i8_bwd": bytes_i8_op(M, H, M * H + sbytes(M, H) + 12 * H),
            "dequantize_dx": M * H * 3 + sbytes(M, H),
        }
        self.ops = {g: 2 * M * H * F for g in self.GEMMS}
        self.side = torch.cuda.Stream(device=dev)
        self.ev = {k: torch.cuda.Event() for k in ("w1", "w2", "dy", "g", "dy1")}
        self.graph = None

    # the operators, one call each (the weight gradients in fp32 for the data-parallel sum)
    def _op(self, name):
        jf = self.jf
        if name == "quantize_x": jf.jf_quantize_block(self.xb, self.Xq.q, self.Xq.s)
        elif name == "layernorm_i8": jf.jf_layernorm_i8(self.Xq, self.gamma, self.beta, 1e-5, self.Xn)
        elif name == "quantize_w1": jf.jf_quantize_block(self.w1b, self.W1.q, self.W1.s)
        elif name == "quantize_w2": jf.jf_quantize_block(self.w2b, self.W2.q, self.W2.s)
        elif name == "fc1_fwd": jf.jf_linear_fwd(self.Xn, self.W1, self.Y1)
        elif name == "gelu_i8": jf.jf_gelu_i8(self.Y1, self.G)
        elif name == "fc2_fwd": jf.jf_linear_fwd(self.G, self.W2, self.Y2)
        elif name == "quantize_dy": jf.jf_quantize_block(self.dyb, self.dY2.q, self.dY2.s)
        elif name == "fc2_dgrad": jf.jf_linear_dgrad(self.dY2, self.W2, self.dG)
        elif name == "fc2_wgrad":
            if self.world > 1: jf.jf_linear_wgrad(self.dY2, self.G, None, self.dw2_f32)
            else: jf.jf_linear_wgrad(self.dY2, self.G, self.dW2)
        elif name == "gelu_i8_bwd": jf.jf_gelu_i8_bwd(self.Y1, self.dG, self.dY1)
        elif name == "fc1_dgrad": jf.jf_linear_dgrad(self.dY1, self.W1, self.dXn)
        elif name == "fc1_wgrad":
            if self.world > 1: jf.jf_linear_wgrad(self.dY1, self.Xn, None, self.dw1_f32)
            else: jf.jf_linear_wgrad(self.dY1, self.Xn, self.dW1)
        elif name == "layernorm_i8_bwd":
            jf.jf_layernorm_i8_bwd(self.Xq, self.dXn, self.gamma, 1e-5, self.dX, self.dgamma, self.dbeta, self.ln_ws)
        elif name == "dequantize_dx": jf.jf_dequantize_block(self.dX.q, self.dX.s, self.dx_bf16)
        else: raise KeyError(name)

    def run_overlapped(self):
        """The step on two streams, ordered by its data dependences: the three bf16 quantizers of the
        weights and the upstream gradient, and the two weight-gradient GEMMs, run on a side stream
        beside the forward and the input-gradient chain (one GPU; captured as a CUDA graph)."""
        t, ev = self.torch, self.ev
        main = t.cuda.current_stream()
        self.side.wait_stream(main)
        with t.cuda.stream(self.side):
            self._op("quantize_w1"); ev["w1"].record()
            self._op("quantize_w2"); ev["w2"].record()
            self._op("quantize_dy"); ev["dy"].record()
        self._op("quantize_x")
        self._op("layernorm_i8")
        main.wait_event(ev["w1"])
        self._op("fc1_fwd")
        self._op("gelu_i8")
        ev["g"].record()
        main.wait_event(ev["w2"])
        self._op("fc2_fwd")
        main.wait_event(ev["dy"])
        self._op("fc2_dgrad")
        with t.cuda.stream(self.side):
            self.side.wait_event(ev["g"])
            self._op("fc2_wgrad")
        self._op("gelu_i8_bwd")
        ev["dy1"].record()
        self._op("fc1_dgrad")
        with t.cuda.stream(self.side):
            self.side.wait_event(ev["dy1"])
            self._op("fc1_wgrad")
        self._op("layernorm_i8_bwd")
        self._op("dequantize_dx")
        main.wait_stream(self.side)

    def run_data_parallel(self):
        """The step on several ranks: each weight gradient is an fp32 partial over this rank's tokens;
        its NCCL all-reduce is issued as soon as the partial exists and runs beside the rest of the
        backward (WgradExchange); each summed gradient is re-quantized per block once its
        all-reduce has landed."""
        from int8_fully_quantized_b200.parallel import WgradExchange
        ex = WgradExchange()
        for op in ("quantize_x", "layernorm_i8", "quantize_w1", "quantize_w2", "fc1_fwd", "gelu_i8", "fc2_fwd",
                   "quantize_dy", "fc2_dgrad", "fc2_wgrad"):
            self._op(op)
        ex.start(self.dw2_f32, self.dW2)
        for op in ("gelu_i8_bwd", "fc1_dgrad", "fc1_wgrad"):
            self._op(op)
        ex.start(self.dw1_f32, self.dW1)
        self._op("layernorm_i8_bwd")
        self._op("dequantize_dx")
        ex.finish(lambda dst, dw: self.jf.jf_quantize_block(dw, dst.q, dst.s))

    def step(self):
        if self.world > 1:
            self.run_data_parallel()
        elif self.graph is not None:
            self.graph.replay()
        else:
            self.run_overlapped()

    def capture(self):
        """CUDA graph of run_overlapped (single GPU): one replay launches the step's kernels with no
        host work in between."""
        t = self.torch
        self.graph = t.cuda.CUDAGraph()
        with t.cuda.graph(self.graph):
            self.run_overlapped()

    def run_serialized(self, ev):
        """Every operator on one stream, bracketed by events (the per-kernel times)."""
        ev[0].record()
        for i, op in enumerate(self.OPS):
            self._op(op)
            ev[i + 1].record()


def _device_ms(fn, flush, reps=10):
    """Median CUDA-event time of fn over reps launches, L2 flushed (256 MiB write) before each."""
    import torch
    for _ in range(3):
        flush.zero_()
        fn()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(); fn(); b.record()
        ts.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ts)


def tensor_ceiling(jf, flush, i8_peak):
    """The plain INT8 product (jf_gemm_i8_s32: the same TMA / tcgen05 machinery, int32 result, no
    per-block rescale) at the fc1 and fc2 shapes of the layer: the tensor core's measured INT8 rate."""
    import torch
    M, H, F = layer_dims()
    g = torch.Generator(device="cuda").manual_seed(1)
    out = {}
    for name, (m, n, k) in (("fc1_shape", (M, F, H)), ("fc2_shape", (M, H, F))):
        a = torch.randint(-127, 128, (m, k), dtype=torch.int8, device="cuda", generator=g)
        b = torch.randint(-127, 128, (n, k), dtype=torch.int8, device="cuda", generator=g)
        c = torch.empty((m, n), dtype=torch.int32, device="cuda")
        ms = _device_ms(lambda: jf.jf_gemm_i8_s32(a, b, c), flush, reps=10)
        tops = 2 * m * n * k / (ms * 1e-3) / 1e12
        out[name] = {"M": m, "N": n, "K": k, "ms": round(ms, 4), "TOPS": round(tops, 1),
                     "frac_of_peak": round(tops / i8_peak, 4), "frac_of_nominal_4500": round(tops / NOMINAL_I8_TOPS, 4)}
        del a, b, c
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    import int8_fully_quantized_b200 as jf
    from int8_fully_quantized_b200 import parallel as P

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    jf.load_library()
    host = host_inputs(P.shard_seed(0, rank), seed_weight=0)
    step = GpuStep(host, world)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")   # 256 MiB > L2

    use_graph = world == 1 and not args.eager
    sampler = ClockSampler(local)
    with sampler:
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            step.step()
        torch.cuda.synchronize()
        if use_graph:
            step.capture()
            for _ in range(max(3, args.warmup)):
                flush.zero_()
                step.step()
        st = jf.jf_device_status()
        if st != 0:
            raise RuntimeError(f"device status after warm-up: {jf.jf_strerror(st)}")
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        # timed region: whole steps (graph replays on one GPU, eager launches on several)
        bounds = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            bounds[i][0].record()
            step.step()
            bounds[i][1].record()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        # per-kernel times: the operators serialized on one stream, each bracketed by events
        n_ops = max(3, min(args.steps, 5))
        op_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(GpuStep.OPS) + 1)] for _ in range(n_ops)]
        for i in range(n_ops):
            flush.zero_()
            step.run_serialized(op_evs[i])
        torch.cuda.synchronize()
    st = jf.jf_device_status()
    if st != 0:
        raise RuntimeError(f"device status after the timed steps: {jf.jf_strerror(st)}")
    per_op = {op: [op_evs[i][j].elapsed_time(op_evs[i][j + 1]) for i in range(n_ops)]
              for j, op in enumerate(GpuStep.OPS)}
    step_ms_local = sum(a.elapsed_time(b) for a, b in bounds) / args.steps
    step_ms = P.max_over_ranks(step_ms_local, device="cuda")
    ops_per_step = sum(step.ops.values())
    value = world * ops_per_step / (step_ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    i8_peak = peaks["bf16_tflops"] * NOMINAL_I8_OVER_BF16
    i8_peak_sustained = peaks["bf16_tflops_sustained"] * NOMINAL_I8_OVER_BF16
    kernels = {}
    for op, ts in per_op.items():
        ms = statistics.mean(ts)
        if op in step.ops:
            tops = step.ops[op] / (ms * 1e-3) / 1e12
            kernels[op] = {"ms": round(ms, 4), "TOPS": round(tops, 1), "frac_i8_peak": round(tops / i8_peak, 4)}
        else:
            gbs = step.bytes[op] / (ms * 1e-3) / 1e9
            kernels[op] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    dom = max(step.GEMMS, key=lambda o: statistics.mean(per_op[o]))
    dom_ms = statistics.mean(per_op[dom])
    achieved = step.ops[dom] / (dom_ms * 1e-3) / 1e12
    # The same launch seen as issue work: per output element and 32-deep contraction block an int32 ->
    # fp32 conversion and an FMA (M*N*K/16 lane-instructions per launch), against 4 x 32 lane-instructions
    # per clock per SM: the CUDA-core ceiling of the per-block rescale.
    alu_work = step.ops[dom] // 32
    alu_peak = ALU_LANES_PER_CLK_PER_SM * B200_SMS * peaks["sm_max_mhz"] * 1e6 / 1e12
    alu_achieved = alu_work / (dom_ms * 1e-3) / 1e12
    world_ok = world == 1
    ceiling = tensor_ceiling(jf, flush, i8_peak) if world_ok else None
    roofline = {"kernel": f"gemm_i8_kernel ({dom})", "bound": "tensor", "achieved": round(achieved, 1),
                "peak": round(i8_peak, 1), "unit": "TOPS", "frac": round(achieved / i8_peak, 4),
                "traffic": _load_traffic(dom),
                "peak_source": f"{peak_src} bf16 dense burst {peaks['bf16_tflops']:g} TFLOP/s x nominal int8/bf16 "
                               f"ratio {NOMINAL_I8_OVER_BF16:g}",
                "algorithmic": f"2*M*N*K = {step.ops[dom]} int8 ops per launch (M=8192, N*K=4096*16384)",
                "frac_of_sustained_peak": round(achieved / i8_peak_sustained, 4),
                "frac_of_nominal_4500": round(achieved / NOMINAL_I8_TOPS, 4),
                "measured_tensor_ceiling": ceiling,
                "alu_view": {"achieved": round(alu_achieved, 2), "peak": round(alu_peak, 2),
                             "unit": "T lane-instructions/s", "frac": round(alu_achieved / alu_peak, 4),
                             "work": "2 per output element per 32-deep block = M*N*K/16 per launch",
                             "peak_source": f"{ALU_LANES_PER_CLK_PER_SM} lane-instructions/clk/SM x {B200_SMS} SMs x "
                                            f"{peaks['sm_max_mhz']:g} MHz (derived)"}}
    M, H, F = step.M, step.H, step.F
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(step_ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAME, "M": M, "H": H, "F": F, "block": 32,
                   "inputs": "bf16 X ~N(0,1) with 4 channels x50, W1, W2 ~N(0,0.02), dY ~N(0,1e-3)",
                   "parallelism": f"dp{world}", "l2": "flushed between steps (256 MiB write, outside timed events)"},
        "kernels": kernels, "roofline": roofline,
        "execution": ("CUDA graph of the step on two streams ordered by data dependences (the three bf16 quantizers "
                      "of W1, W2, dY and the two weight-gradient GEMMs beside the forward and input-gradient chain); "
                      "per-kernel times from the operators serialized on one stream"
                      if use_graph else "eager launches; fp32 weight-gradient all-reduces (NCCL) overlap the rest "
                                        "of the backward; per-kernel events serialized"),
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": sampler.summary(),
    }
    if not args.no_e2e:
        result["e2e"] = run_e2e(step, host, args, world, flush)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and world == 1:
        del step
        torch.cuda.empty_cache()
        if not args.no_sweep:
            result["sweep"] = memory_sweep(jf, [8192, 65536], SWEEP_OPS, flush, peaks)
        if not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(args.cpu_sample_blocks)
    if rank == 0:
        print(json.dumps(result), flush=True)


def _load_traffic(kernel_op):
    """DRAM read + write bytes per launch of the dominant kernel from the committed ncu capture
    (profiles/gemm_traffic.json), or None when that capture was taken of other GEMM kernel sources."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    try:
        from int8_fully_quantized_b200 import build_lib
        with open(path) as f:
            d = json.load(f)
        if d.get("kernel_source_hash") != build_lib.kernel_source_hash():
            return None
        v = d.get(kernel_op)
        return None if v is None else int(v)
    except Exception:
        return None


def run_e2e(step, host, args, world, flush):
    """Same step through the public API with host buffers. Every step copies its batch (X and the
    upstream gradient dY, bf16) from pinned host memory to the device, runs the layer's forward and
    backward, and reads its results back to pinned host memory: dX (bf16), the re-quantized weight
    gradients dW1, dW2 (codes and scales) and dgamma, dbeta. The weights are model state, resident
    on the device. The steps are pipelined the way a training loop feeds a GPU: two device
    input/output slots, the host->device copies of step i+1 on a copy stream and the device->host
    reads of step i on a third stream while step i+1 computes. The timed window runs from the first
    input copy to the last result read; ms_per_step = window / steps. The L2 flush before each
    step's operators is inside the window."""
    import torch
    from int8_fully_quantized_b200 import parallel as P
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    hx, hdy = pin(host["x"]), pin(host["dy"])
    outs = [step.dx_bf16, step.dW1.q, step.dW1.s, step.dW2.q, step.dW2.s, step.dgamma, step.dbeta]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in (hx, hdy))
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    slots = [step, GpuStep(host, world)]
    use_graph = world == 1 and not args.eager
    if use_graph:
        for s in slots:
            if s.graph is None:
                s.capture()
    main = torch.cuda.current_stream()
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    ready = [torch.cuda.Event() for _ in slots]      # the slot's inputs have landed
    computed = [torch.cuda.Event() for _ in slots]   # the slot's operators have finished
    read = [torch.cuda.Event() for _ in slots]       # the slot's results are on the host

    def copy_in(i, started=None):
        k = i % 2
        with torch.cuda.stream(h2d_stream):
            if started is not None:
                h2d_stream.wait_event(started)
            if i >= 2:
                h2d_stream.wait_event(computed[k])   # step i-2 has finished reading this slot
            s = slots[k]
            s.xb.copy_(hx, non_blocking=True)
            s.dyb.copy_(hdy, non_blocking=True)
            ready[k].record(h2d_stream)

    def compute_and_read(i):
        k = i % 2
        s = slots[k]
        main.wait_event(ready[k])
        if i >= 2:
            main.wait_event(read[k])   # step i-2's results have left this slot
        flush.zero_()
        s.step()
        computed[k].record(main)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(computed[k])
            for dst, src in zip(host_out, [s.dx_bf16, s.dW1.q, s.dW1.s, s.dW2.q, s.dW2.s, s.dgamma, s.dbeta]):
                dst.copy_(src, non_blocking=True)
            read[k].record(d2h_stream)

    def pipeline(n, started=None):
        copy_in(0, started)
        if n > 1:
            copy_in(1)
        for i in range(n):
            compute_and_read(i)
            if i + 2 < n:
                copy_in(i + 2)
        main.wait_stream(d2h_stream)
        main.wait_stream(h2d_stream)

    pipeline(max(3, args.warmup))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(main)
    pipeline(args.steps, started=t0)
    t1.record(main)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    ms = P.max_over_ranks(ms, device="cuda")
    ops = sum(step.ops.values())
    del slots[1]
    return {"value": round(world * ops / (ms * 1e-3) / 1e12, 2), "unit": "TOPS", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pipelining": "two slots; step i+1's host->device copies and step i's device->host reads overlap the "
                          "operators; window from the first input copy to the last result read"}


# --------------------------------------------------------------------------------------------
# memory-bound sweep (also reported in the main line at M = 8192 and 65536)
# --------------------------------------------------------------------------------------------
SWEEP_OPS = ["quantize_bf16", "dequantize_bf16", "gelu_i8", "layernorm_i8", "gelu_i8_bwd", "layernorm_i8_bwd"]


def memory_sweep(jf, ms_list, op_names, flush, peaks, reps=10):
    """quantize (bf16 in), dequantize (bf16 out), GELU_i8, LayerNorm_i8 and their INT8 backward on
    M x 4096 tensors, N(0,1) with 1% of the channels x100. GB/s from algorithmic bytes (every input
    read once, every output written once) over the median CUDA-event time, L2 flushed before each
    launch, and the fraction of the measured HBM copy bandwidth."""
    import torch
    from inputs import synthetic as S
    H = 4096
    out = {}
    for M in ms_list:
        x = S.to_bf16_bits(S.memory_sweep_input(0, M, H))
        xb = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
        del x
        Q = jf.quantize_block(xb)
        D = jf.quantize_block(torch.from_numpy(S.to_bf16_bits(S.memory_sweep_input(1, M, H)).view(np.int16)).cuda()
                              .view(torch.bfloat16))
        Y = jf.empty_qtensor(M, H)
        yb = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
        gamma = torch.ones(H, device="cuda")
        beta = torch.zeros(H, device="cuda")
        dgam, dbet = torch.empty(H, device="cuda"), torch.empty(H, device="cuda")
        ws = torch.empty(jf.jf_layernorm_i8_bwd_workspace_bytes(M, H), dtype=torch.uint8, device="cuda")
        ops = {
            "quantize_bf16": (lambda: jf.jf_quantize_block(xb, Y.q, Y.s), bytes_quant(M, H, 2)),
            "dequantize_bf16": (lambda: jf.jf_dequantize_block(Q.q, Q.s, yb), M * H * 3 + sbytes(M, H)),
            "gelu_i8": (lambda: jf.jf_gelu_i8(Q, Y), bytes_i8_op(M, H)),
            "layernorm_i8": (lambda: jf.jf_layernorm_i8(Q, gamma, beta, 1e-5, Y), bytes_i8_op(M, H, 8 * H)),
            "gelu_i8_bwd": (lambda: jf.jf_gelu_i8_bwd(Q, D, Y), bytes_i8_op(M, H, M * H + sbytes(M, H))),
            "layernorm_i8_bwd": (lambda: jf.jf_layernorm_i8_bwd(Q, D, gamma, 1e-5, Y, dgam, dbet, ws),
                                 bytes_i8_op(M, H, M * H + sbytes(M, H) + 12 * H)),
        }
        for name, (fn, nbytes) in ops.items():
            if name not in op_names:
                continue
            ms = _device_ms(fn, flush, reps=reps)
            gbs = nbytes / (ms * 1e-3) / 1e9
            out[f"{name}@M={M}"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        del xb, Q, D, Y, yb, ws
        torch.cuda.empty_cache()
    assert jf.jf_device_status() == 0
    return out


def run_sweep(args):
    """The memory-bound sweep at M in {1024, 8192, 65536} (one JSON line); with "fused_fc1",
    "granularity_mse" and "mxfp8_fc1" also the f1 fused epilogue, the f3 granularity MSEs and the f4
    MXFP8 comparison on the GPT2-medium fc1 shapes."""
    import torch
    import int8_fully_quantized_b200 as jf
    torch.cuda.set_device(0)
    jf.load_library()
    peaks, peak_src = load_peaks()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    out = memory_sweep(jf, args.sweep_m, args.sweep_ops, flush, peaks, reps=max(5, args.steps // 5))
    if "fused_fc1" in args.sweep_ops:
        out.update(_sweep_fused_fc1(jf, flush))
    if "granularity_mse" in args.sweep_ops:
        out["granularity_mse"] = _granularity_mse(jf)
    if "mxfp8_fc1" in args.sweep_ops:
        out["mxfp8_vs_int8_fc1"] = _mxfp8_vs_int8(jf, flush)
    assert jf.jf_device_status() == 0
    print(json.dumps({"sweep": out, "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": peak_src,
                      "l2": "flushed before every timed launch"}), flush=True)


# --------------------------------------------------------------------------------------------
# CPU oracle timings (the baseline leg, and the --impl reference arm)
# --------------------------------------------------------------------------------------------
_ORACLE_OPERANDS = {}


def _oracle_operands():
    """Quantized operands of the layer's six GEMMs and one 32-token strip of its memory-bound operators,
    drawn with the workload's distributions and quantized by the oracle itself (values do not change
    the oracle's cost; none of them comes from the GPU). Cached: built once, outside any timing."""
    if _ORACLE_OPERANDS:
        return _ORACLE_OPERANDS
    import oracle as O
    from inputs import synthetic as S
    M, H, F = layer_dims()
    rng = np.random.default_rng(3)
    q = lambda a: O.quantize_block(a)
    X = q(S.activation(rng, M, H, 4, 50.0))      # Xn stand-in [M, H]
    G = q(S.activation(rng, M, F, 0, 1.0))       # GELU output stand-in [M, F]
    W1, W2 = q(S.weight(rng, F, H)), q(S.weight(rng, H, F))
    dY2, dY1 = q(S.grad(rng, M, H)), q(S.grad(rng, M, F))
    _ORACLE_OPERANDS.update(
        gemms=[("fc1_fwd", O.linear_fwd, X, W1, M, F), ("fc2_fwd", O.linear_fwd, G, W2, M, H),
               ("fc2_dgrad", O.linear_dgrad, dY2, W2, M, F), ("fc2_wgrad", O.linear_wgrad, dY2, G, H, F),
               ("fc1_dgrad", O.linear_dgrad, dY1, W1, M, H), ("fc1_wgrad", O.linear_wgrad, dY1, X, F, H)],
        strip_x=S.activation(rng, 32, H, 4, 50.0), strip_dy=S.grad(rng, 32, H), strip_g=S.activation(rng, 32, F, 0, 1.0),
        gamma=np.ones(H, np.float32), beta=np.zeros(H, np.float32), H=H, F=F)
    return _ORACLE_OPERANDS


def _oracle_sample(nblk, seed=0):
    """The oracle on a bounded sample of one step: nblk x nblk output blocks (evenly spread) of each of
    the six GEMMs with their full contraction, plus quantize, LayerNorm_i8 and its backward, GELU_i8
    and its backward and dequantize on one 32-token strip. Returns (GEMM int8 ops done, seconds)."""
    import oracle as O
    d = _oracle_operands()
    t0 = time.perf_counter()
    ops = 0
    for _, fn, A, B, rows, cols in d["gemms"]:
        rb = list(np.linspace(0, rows // 32 - 1, nblk).astype(int))
        cb = list(np.linspace(0, cols // 32 - 1, nblk).astype(int))
        O.requantize(fn(*A, *B, rb, cb))
        depth = A[0].shape[1] if fn is not O.linear_wgrad else A[0].shape[0]
        ops += 2 * (32 * nblk) * (32 * nblk) * depth
    xq, xs = O.quantize_block(d["strip_x"])
    O.layernorm_i8(xq, xs, d["gamma"], d["beta"], 1e-5)
    dq, ds = O.quantize_block(d["strip_dy"])
    O.layernorm_i8_bwd(xq, xs, dq, ds, d["gamma"], 1e-5)
    gq, gs = O.quantize_block(d["strip_g"])
    O.gelu_i8(gq, gs)
    O.gelu_i8_bwd(gq, gs, gq, gs)
    O.dequantize_block(xq, xs, "bf16")
    return ops, time.perf_counter() - t0


def _cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(nblk):
    _oracle_operands()
    ops, dt = _oracle_sample(nblk)
    return {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": _cpu_cores(), "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"{nblk}x{nblk} output blocks of each of the six GEMMs (full contraction) plus one 32-token "
                      f"strip of every memory-bound operator; GEMM int8 ops done / wall time"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    nblk = 6
    _oracle_operands()
    for _ in range(max(3, args.warmup)):
        _oracle_sample(nblk)
    times, ops = [], 0
    for _ in range(args.steps):
        ops, dt = _oracle_sample(nblk)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = ops / (ms * 1e-3) / 1e12
    cores = _cpu_cores()
    M, H, F = layer_dims()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAME, "M": M, "H": H, "F": F, "block": 32, "parallelism": "oracle on host"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {nblk}x{nblk} output blocks of each of the six GEMMs (full "
                                   f"contraction) plus one 32-token strip of every memory-bound operator"},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _mxfp8_vs_int8(jf, flush):
    """The GPT2-medium fc1 forward (M=4096, K=1024, N=4096, bf16 inputs) two ways: Jetfire's 32x32
    INT8 blocks (quantize X and W, block-scaled INT8 GEMM with fp32 output) and MXFP8 (1x32 E8M0
    blocks, E4M3 elements, the tensor core's block-scaled MMA). Device times (L2 flushed before each
    launch) and the relative Frobenius error of each fp32 output against the exact product of the
    bf16 inputs (fp64 on the host)."""
    import torch
    M, K, N, host = gpt2m_inputs(0)
    xb = torch.from_numpy(host["x"].view(np.int16)).cuda().view(torch.bfloat16)
    wb = torch.from_numpy(host["w"].view(np.int16)).cuda().view(torch.bfloat16)
    ref = (xb.cpu().double().numpy() @ wb.cpu().double().numpy().T)

    def timed(fn, reps=10):
        for _ in range(3):
            flush.zero_()
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(); fn(); b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ts)

    res = {}
    X, W = jf.quantize_block(xb), jf.quantize_block(wb)
    Y, yf = jf.empty_qtensor(M, N), torch.empty((M, N), dtype=torch.float32, device="cuda")
    q_ms = timed(lambda: (jf.jf_quantize_block(xb, X.q, X.s), jf.jf_quantize_block(wb, W.q, W.s)))
    g_ms = timed(lambda: jf.jf_linear_fwd(X, W, None, yf))
    err = float(np.linalg.norm(yf.cpu().double().numpy() - ref) / np.linalg.norm(ref))
    res["int8_32x32"] = {"quantize_ms": round(q_ms, 4), "gemm_ms": round(g_ms, 4),
                         "gemm_TOPS": round(2 * M * N * K / (g_ms * 1e-3) / 1e12, 1), "rel_error": float(f"{err:.4g}")}
    (Aq, As), (Bq, Bs) = jf.mx_quantize(xb), jf.mx_quantize(wb)
    q_ms = timed(lambda: (jf.jf_mx_quantize(xb, Aq, As), jf.jf_mx_quantize(wb, Bq, Bs)))
    g_ms = timed(lambda: jf.jf_mx_linear_fwd(Aq, As, Bq, Bs, yf))
    err = float(np.linalg.norm(yf.cpu().double().numpy() - ref) / np.linalg.norm(ref))
    res["mxfp8_1x32"] = {"quantize_ms": round(q_ms, 4), "gemm_ms": round(g_ms, 4),
                         "gemm_TOPS": round(2 * M * N * K / (g_ms * 1e-3) / 1e12, 1), "rel_error": float(f"{err:.4g}")}
    return res


def _granularity_mse(jf):
    """Quantization MSE at each scale granularity, computed on the GPU (quantize, then the fp64 error
    sums), on the GPT2-medium fc1 activations (10 of 1024 channels x30) and on the sweep input
    (8192 x 4096, 1% of the channels x100): the ablation of the summary's measured effects."""
    import torch
    from inputs import synthetic as S
    res = {}
    _, _, _, host = gpt2m_inputs(0)
    cases = {"gpt2m_fc1_X": torch.from_numpy(host["x"].view(np.int16)).cuda().view(torch.bfloat16),
             "sweep_8192x4096": torch.from_numpy(S.to_bf16_bits(S.memory_sweep_input(0, 8192, 4096)).view(np.int16))
             .cuda().view(torch.bfloat16)}
    for name, x in cases.items():
        mse = {g: jf.quantization_mse(x, g) for g in ["block", "token", "channel", "tensor"]}
        res[name] = {"mse": {g: float(f"{v:.6g}") for g, v in mse.items()},
                     "token_over_block": round(mse["token"] / mse["block"], 2)}
    return res


def _sweep_fused_fc1(jf, flush):
    """GPT2-medium fc1 forward (M=4096, K=1024, N=4096): GELU fused into the GEMM epilogue versus the
    forward GEMM followed by GELU_i8 (device time of each variant, L2 flushed before each)."""
    import torch
    M, K, N, host = gpt2m_inputs(0)
    X = jf.quantize_block(torch.from_numpy(host["x"].view(np.int16)).cuda().view(torch.bfloat16))
    W = jf.quantize_block(torch.from_numpy(host["w"].view(np.int16)).cuda().view(torch.bfloat16))
    Y, G, P = jf.empty_qtensor(M, N), jf.empty_qtensor(M, N), jf.empty_qtensor(M, N)
    variants = {
        "fc1_fwd_then_gelu_i8": lambda: (jf.jf_linear_fwd(X, W, Y), jf.jf_gelu_i8(Y, G)),
        "fc1_fwd_gelu_fused": lambda: jf.jf_linear_fwd_gelu(X, W, G),
        "fc1_fwd_gelu_fused_with_pre": lambda: jf.jf_linear_fwd_gelu(X, W, G, P),
    }
    res = {}
    for name, fn in variants.items():
        for _ in range(3):
            flush.zero_()
            fn()
        ts = []
        for _ in range(10):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(); fn(); b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        ms = statistics.median(a.elapsed_time(b) for a, b in ts)
        res[name] = {"ms": round(ms, 4), "TOPS": round(2 * M * N * K / (ms * 1e-3) / 1e12, 1)}
    return res


def run_configs(args):
    """The workloads besides the headline step, each timed on the device (L2 flushed before every
    launch) with the CPU oracle beside it on the same inputs (whole where it finishes in seconds,
    else a stated sample):
      single_linear_256: quantize X and W (fp32 256x256) and the forward, a latency case;
      h4096_fc1 / h4096_fc2: forward, input- and weight-gradient GEMMs of the hidden-4096 layer;
      h4096_mlp_block: LayerNorm_i8 -> fc1 -> GELU_i8 -> fc2 on INT8 blocks (M = 8192), and the
      same with GELU fused into fc1's epilogue."""
    import torch
    import int8_fully_quantized_b200 as jf
    import oracle as O
    from inputs import synthetic as S
    torch.cuda.set_device(0)
    jf.load_library()
    peaks, peak_src = load_peaks()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    alu_peak = ALU_LANES_PER_CLK_PER_SM * B200_SMS * peaks["sm_max_mhz"] * 1e6
    i8_peak = peaks["bf16_tflops"] * NOMINAL_I8_OVER_BF16
    out = {}
    # ---- single linear, 256^3, fp32 inputs
    d = S.workload("linear_256", 0)
    x, w = torch.from_numpy(d["X"]).cuda(), torch.from_numpy(d["W"]).cuda()
    X, W, Y = jf.empty_qtensor(256, 256), jf.empty_qtensor(256, 256), jf.empty_qtensor(256, 256)
    ms = _device_ms(lambda: (jf.jf_quantize_block(x, X.q, X.s), jf.jf_quantize_block(w, W.q, W.s),
                             jf.jf_linear_fwd(X, W, Y)), flush, reps=20)
    t0 = time.perf_counter()
    xq, xs = O.quantize_block(d["X"]); wq, ws = O.quantize_block(d["W"])
    O.requantize(O.linear_fwd(xq, xs, wq, ws))
    cpu_s = time.perf_counter() - t0
    out["single_linear_256"] = {"device_us": round(ms * 1e3, 2), "oracle_ms": round(cpu_s * 1e3, 2),
                                "note": "three launches (quantize X, quantize W, forward); latency-bound"}
    del x, w, X, W, Y
    # ---- hidden-4096 GEMMs
    for name in ("h4096_fc1", "h4096_fc2"):
        wl = S.WORKLOADS[name]
        M, K, N = wl["M"], wl["K"], wl["N"]
        g = torch.Generator(device="cuda").manual_seed(0)
        qt = lambda r, c: jf.QTensor(torch.randint(-127, 128, (r, c), dtype=torch.int8, device="cuda", generator=g),
                                     torch.rand((r // 32, c // 32), device="cuda", generator=g) * 0.01 + 1e-3)
        A, B, dY = qt(M, K), qt(N, K), qt(M, N)
        res = {}
        for mode, fn, rows, cols in (("fwd", lambda o: jf.jf_linear_fwd(A, B, o), M, N),
                                     ("dgrad", lambda o: jf.jf_linear_dgrad(dY, B, o), M, K),
                                     ("wgrad", lambda o: jf.jf_linear_wgrad(dY, A, o), N, K)):
            o = jf.empty_qtensor(rows, cols)
            ms = _device_ms(lambda: fn(o), flush, reps=5)
            ops = 2 * M * N * K
            res[mode] = {"ms": round(ms, 3), "TOPS": round(ops / (ms * 1e-3) / 1e12, 1),
                         "alu_frac": round(ops / 32 / (ms * 1e-3) / alu_peak, 4),
                         "tensor_frac": round(ops / (ms * 1e-3) / 1e12 / i8_peak, 4)}
            del o
        # oracle: one 32x32 output block of the forward, timed, and its cost for the full output
        Xh, Wh = host_q(A), host_q(B)
        t0 = time.perf_counter()
        O.linear_fwd(*Xh, *Wh, [0], [0])
        blk = time.perf_counter() - t0
        res["oracle"] = {"one_block_ms": round(blk * 1e3, 2),
                         "full_fwd_s_extrapolated": round(blk * (M // 32) * (N // 32), 1)}
        out[name] = res
        del A, B, dY
    # ---- hidden-4096 MLP block on INT8 blocks
    wl1, wl2 = S.WORKLOADS["h4096_fc1"], S.WORKLOADS["h4096_fc2"]
    M, H, F = wl1["M"], wl1["K"], wl1["N"]
    rng = np.random.default_rng(0)
    xin = torch.from_numpy(S.to_bf16_bits(S.activation(rng, M, H, 4, 50.0)).view(np.int16)).cuda().view(torch.bfloat16)
    Xq = jf.quantize_block(xin)
    W1 = jf.quantize_block(torch.from_numpy(S.to_bf16_bits(S.weight(rng, F, H)).view(np.int16)).cuda().view(torch.bfloat16))
    W2 = jf.quantize_block(torch.from_numpy(S.to_bf16_bits(S.weight(rng, H, F)).view(np.int16)).cuda().view(torch.bfloat16))
    gamma, beta = torch.ones(H, device="cuda"), torch.zeros(H, device="cuda")
    Xn, Y1, G, Y2 = jf.empty_qtensor(M, H), jf.empty_qtensor(M, F), jf.empty_qtensor(M, F), jf.empty_qtensor(M, H)
    chain = lambda: (jf.jf_layernorm_i8(Xq, gamma, beta, 1e-5, Xn), jf.jf_linear_fwd(Xn, W1, Y1), jf.jf_gelu_i8(Y1, G),
                     jf.jf_linear_fwd(G, W2, Y2))
    fused = lambda: (jf.jf_layernorm_i8(Xq, gamma, beta, 1e-5, Xn), jf.jf_linear_fwd_gelu(Xn, W1, G),
                     jf.jf_linear_fwd(G, W2, Y2))
    ops = 2 * M * F * H * 2
    ms, msf = _device_ms(chain, flush, reps=5), _device_ms(fused, flush, reps=5)
    out["h4096_mlp_block"] = {"ms": round(ms, 3), "TOPS": round(ops / (ms * 1e-3) / 1e12, 1),
                              "fused_gelu_ms": round(msf, 3), "fused_gelu_TOPS": round(ops / (msf * 1e-3) / 1e12, 1),
                              "note": "GEMM int8 ops of fc1 + fc2 over the block's device time"}
    assert jf.jf_device_status() == 0
    print(json.dumps({"configs": out, "peaks": {"alu_T_lane_instr_s": round(alu_peak / 1e12, 2),
                                                 "int8_tops": round(i8_peak, 1), "source": peak_src},
                      "l2": "flushed before every timed launch", "cpu_threads": _cpu_cores()}), flush=True)


def host_q(t):
    """(codes, scales) of a device QTensor as host numpy arrays."""
    return t.q.cpu().numpy(), t.s.cpu().numpy()


def run_profile_gemm(args):
    """fwd, dgrad and wgrad of the GPT2-medium fc1 shapes, each launched --steps times in that order
    (3 warm-up launches of each first), with the L2 flushed before every launch; prints the median
    device time of each. A small, fixed launch sequence for profiler captures of the GEMM kernel."""
    import torch
    import int8_fully_quantized_b200 as jf
    torch.cuda.set_device(0)
    jf.load_library()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    M, K, N, host = gpt2m_inputs(0)
    X = jf.quantize_block(torch.from_numpy(host["x"].view(np.int16)).cuda().view(torch.bfloat16))
    W = jf.quantize_block(torch.from_numpy(host["w"].view(np.int16)).cuda().view(torch.bfloat16))
    from inputs import synthetic as S
    dY = jf.quantize_block(torch.from_numpy(S.to_bf16_bits(S.grad(np.random.default_rng(5), M, N)).view(np.int16))
                           .cuda().view(torch.bfloat16))
    Y, dX, dW = jf.empty_qtensor(M, N), jf.empty_qtensor(M, K), jf.empty_qtensor(N, K)
    out = {}
    for name, fn in (("fwd", lambda: jf.jf_linear_fwd(X, W, Y)), ("dgrad", lambda: jf.jf_linear_dgrad(dY, W, dX)),
                     ("wgrad", lambda: jf.jf_linear_wgrad(dY, X, dW))):
        ms = _device_ms(fn, flush, reps=max(1, args.steps))
        out[name] = {"ms": round(ms, 4), "TOPS": round(2 * M * N * K / (ms * 1e-3) / 1e12, 1)}
    assert jf.jf_device_status() == 0
    print(json.dumps({"profile_gemm": out, "M": M, "K": K, "N": N}), flush=True)


def main():
    args = parse_args()
    if args.profile_gemm:
        run_profile_gemm(args)
        return
    if args.configs:
        run_configs(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
