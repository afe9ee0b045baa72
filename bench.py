#!/usr/bin/env python
"""Benchmark of the per-block INT8 data-flow hot path on B200.

One step = one pass of every operator of the path over one batch of the GPT2-medium MLP linear
workload (tokens M = 4096, hidden K = 1024, N = 4096; X ~ N(0,1) with 1% of the channels x30,
W ~ N(0, 0.02), dY ~ N(0, 1e-3), bf16 on entry):

    quantize X -> LayerNorm_i8 -> quantize W -> linear fwd (Y = X W^T) -> GELU_i8
    quantize dY -> dgrad (dX = dY W) -> wgrad (dW = dY^T X) -> dequantize dX to bf16

Inputs are resident in HBM when the timed region starts; L2 is flushed between steps (a 256 MiB
write outside the timed events). ``value`` is the whole-step throughput in TOPS counted on the
three GEMMs (3 x 2MNK int8 ops per step and rank) over the step time, summed over ranks.
``--gpus N`` (under torchrun) runs N data-parallel ranks, each with its own M = 4096 tokens; the
fp32 weight-gradient partials are summed with NCCL and re-quantized (weak scaling).

``--impl reference`` times the CPU oracle (the method written out plainly in numpy) on a bounded
token sample of the same workload, on rank 0 only.
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
WORKLOAD = "gpt2m_fc1"
NOMINAL_I8_OVER_BF16 = 2.0       # dense int8 (4.5 POPS) / dense bf16 (2.25 PFLOP/s), nominal B200
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    p.add_argument("--eager", action="store_true", help="time eager launches instead of the step's CUDA graph")
    p.add_argument("--configs", action="store_true",
                   help="time the single-linear, hidden-4096 GEMM and hidden-4096 MLP-block workloads (one JSON line)")
    p.add_argument("--cpu-sample-tokens", type=int, default=1024)
    p.add_argument("--sweep", action="store_true",
                   help="time the memory-bound kernels on the M x 4096 sweep instead of the step")
    p.add_argument("--sweep-m", type=int, nargs="*", default=[1024, 8192, 65536])
    p.add_argument("--sweep-ops", nargs="*", default=["quantize_bf16", "dequantize_bf16", "gelu_i8", "layernorm_i8",
                                                      "gelu_i8_bwd", "layernorm_i8_bwd", "fused_fc1",
                                                      "granularity_mse", "mxfp8_fc1"])
    return p.parse_args()


ALU_LANES_PER_CLK_PER_SM = 128   # 4 warp schedulers x 32 lanes, one issue per scheduler per clock
B200_SMS = 148


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
def host_inputs(M, K, N, seed_tokens, seed_weight):
    from inputs import synthetic as S
    w = S.WORKLOADS[WORKLOAD]
    rng = np.random.default_rng(seed_tokens)
    n_out, fac = w["x_outliers"]
    x = S.activation(rng, M, K, n_out, fac)
    dy = S.grad(rng, M, N)
    wt = S.weight(np.random.default_rng(seed_weight), N, K)
    rng_ln = np.random.default_rng(seed_weight + 7)
    gamma = rng_ln.uniform(0.5, 1.5, K).astype(np.float32)
    beta = rng_ln.normal(0, 0.1, K).astype(np.float32)
    return {"x": S.to_bf16_bits(x), "w": S.to_bf16_bits(wt), "dy": S.to_bf16_bits(dy), "gamma": gamma, "beta": beta}


def bytes_quant(r, c, in_bytes):  # read input, write codes + scales
    return r * c * (in_bytes + 1) + (r // 32) * (c // 32) * 4


def bytes_i8_op(r, c, extra=0):  # read codes + scales, write codes + scales
    return 2 * (r * c + (r // 32) * (c // 32) * 4) + extra


# --------------------------------------------------------------------------------------------
# our implementation
# --------------------------------------------------------------------------------------------
class GpuStep:
    OPS = ["quantize_x", "layernorm_i8", "quantize_w", "linear_fwd", "gelu_i8", "quantize_dy",
           "linear_dgrad", "linear_wgrad", "dequantize_dx"]

    def __init__(self, M, K, N, host, world_size):
        import torch
        import int8_fully_quantized_b200 as jf
        self.jf, self.torch = jf, torch
        self.M, self.K, self.N, self.world = M, K, N, world_size
        dev = torch.device("cuda", torch.cuda.current_device())
        bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        self.xb, self.wb, self.dyb = bf(host["x"]), bf(host["w"]), bf(host["dy"])
        self.gamma = torch.from_numpy(host["gamma"]).to(dev)
        self.beta = torch.from_numpy(host["beta"]).to(dev)
        e = lambda r, c: jf.empty_qtensor(r, c, dev)
        self.Xq, self.Xn, self.Wq, self.Y, self.G = e(M, K), e(M, K), e(N, K), e(M, N), e(M, N)
        self.dYq, self.dX, self.dW = e(M, N), e(M, K), e(N, K)
        self.dx_bf16 = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.dw_f32 = torch.empty((N, K), dtype=torch.float32, device=dev) if world_size > 1 else None
        self.launches_per_step = 9 + (1 if world_size > 1 else 0)
        self.bytes = {
            "quantize_x": bytes_quant(M, K, 2), "quantize_w": bytes_quant(N, K, 2), "quantize_dy": bytes_quant(M, N, 2),
            "layernorm_i8": bytes_i8_op(M, K, 8 * K), "gelu_i8": bytes_i8_op(M, N),
            "dequantize_dx": M * K * 3 + (M // 32) * (K // 32) * 4,
        }
        self.ops = {"linear_fwd": 2 * M * N * K, "linear_dgrad": 2 * M * K * N, "linear_wgrad": 2 * N * K * M}
        self.side = torch.cuda.Stream(device=dev)
        self.w_ready, self.dy_ready, self.xn_ready = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
        self.graph = None

    def run_overlapped(self):
        """The same nine operators on two streams, ordered by their data dependences only: quantize W
        and quantize dY run beside quantize X and LayerNorm_i8, and the weight gradient (dY^T Xn)
        needs neither the forward nor GELU, so it runs beside them and the input gradient; the
        persistent GEMMs then fill each other's last partial wave of tiles."""
        jf, t = self.jf, self.torch
        main = t.cuda.current_stream()
        self.side.wait_stream(main)
        with t.cuda.stream(self.side):
            jf.jf_quantize_block(self.wb, self.Wq.q, self.Wq.s)
            self.w_ready.record()
            jf.jf_quantize_block(self.dyb, self.dYq.q, self.dYq.s)
            self.dy_ready.record()
        jf.jf_quantize_block(self.xb, self.Xq.q, self.Xq.s)
        jf.jf_layernorm_i8(self.Xq, self.gamma, self.beta, 1e-5, self.Xn)
        self.xn_ready.record()
        with t.cuda.stream(self.side):
            self.side.wait_event(self.xn_ready)
            jf.jf_linear_wgrad(self.dYq, self.Xn, self.dW, None)
        main.wait_event(self.w_ready)
        jf.jf_linear_fwd(self.Xn, self.Wq, self.Y, None)
        jf.jf_gelu_i8(self.Y, self.G)
        main.wait_event(self.dy_ready)
        jf.jf_linear_dgrad(self.dYq, self.Wq, self.dX, None)
        jf.jf_dequantize_block(self.dX.q, self.dX.s, self.dx_bf16)
        main.wait_stream(self.side)

    def capture(self):
        """CUDA graph of run_overlapped (single GPU): one replay launches the step's kernels with no
        host work in between."""
        t = self.torch
        self.graph = t.cuda.CUDAGraph()
        with t.cuda.graph(self.graph):
            self.run_overlapped()

    def run(self, ev=None):
        jf, t = self.jf, self.torch
        mark = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        mark(0)
        jf.jf_quantize_block(self.xb, self.Xq.q, self.Xq.s)
        mark(1)
        jf.jf_layernorm_i8(self.Xq, self.gamma, self.beta, 1e-5, self.Xn)
        mark(2)
        jf.jf_quantize_block(self.wb, self.Wq.q, self.Wq.s)
        mark(3)
        jf.jf_linear_fwd(self.Xn, self.Wq, self.Y, None)
        mark(4)
        jf.jf_gelu_i8(self.Y, self.G)
        mark(5)
        jf.jf_quantize_block(self.dyb, self.dYq.q, self.dYq.s)
        mark(6)
        jf.jf_linear_dgrad(self.dYq, self.Wq, self.dX, None)
        mark(7)
        if self.world > 1:
            from int8_fully_quantized_b200.parallel import allreduce_wgrad_
            jf.jf_linear_wgrad(self.dYq, self.Xn, None, self.dw_f32)
            allreduce_wgrad_(self.dw_f32)
            jf.jf_quantize_block(self.dw_f32, self.dW.q, self.dW.s)
        else:
            jf.jf_linear_wgrad(self.dYq, self.Xn, self.dW, None)
        mark(8)
        jf.jf_dequantize_block(self.dX.q, self.dX.s, self.dx_bf16)
        mark(9)


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
    wl = __import__("inputs.synthetic", fromlist=["WORKLOADS"]).WORKLOADS[WORKLOAD]
    M, K, N = wl["M"], wl["K"], wl["N"]
    host = host_inputs(M, K, N, P.shard_seed(0, rank), seed_weight=0)
    step = GpuStep(M, K, N, host, world)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")   # 256 MiB > L2
    stream = torch.cuda.current_stream()

    use_graph = world == 1 and not args.eager
    sampler = ClockSampler(local)
    with sampler:
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            step.run() if not use_graph else step.run_overlapped()
        torch.cuda.synchronize()
        if use_graph:
            step.capture()
            for _ in range(max(3, args.warmup)):
                flush.zero_()
                step.graph.replay()
        st = jf.jf_device_status()
        if st != 0:
            raise RuntimeError(f"device status after warm-up: {jf.jf_strerror(st)}")
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        # timed region: whole steps (graph replays on one GPU, eager launches on several)
        bounds = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(10)] for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            if use_graph:
                bounds[i][0].record()
                step.graph.replay()
                bounds[i][1].record()
            else:
                step.run(evs[i])
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        # per-kernel times: the operators serialized on one stream, each bracketed by events
        n_ops = max(3, min(args.steps, 20))
        op_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(10)] for _ in range(n_ops)] if use_graph else evs
        if use_graph:
            for i in range(n_ops):
                flush.zero_()
                step.run(op_evs[i])
            torch.cuda.synchronize()
    st = jf.jf_device_status()
    if st != 0:
        raise RuntimeError(f"device status after the timed steps: {jf.jf_strerror(st)}")
    per_op = {op: [op_evs[i][j].elapsed_time(op_evs[i][j + 1]) for i in range(len(op_evs))]
              for j, op in enumerate(GpuStep.OPS)}
    if use_graph:
        step_ms_local = sum(a.elapsed_time(b) for a, b in bounds) / args.steps
    else:
        step_ms_local = sum(evs[i][0].elapsed_time(evs[i][9]) for i in range(args.steps)) / args.steps
    step_ms = P.max_over_ranks(step_ms_local, device="cuda")
    ops_per_step = sum(step.ops.values())
    value = world * ops_per_step / (step_ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    i8_peak_burst = peaks["bf16_tflops"] * NOMINAL_I8_OVER_BF16
    kernels = {}
    for op, ts in per_op.items():
        ms = statistics.mean(ts)
        if op in step.ops:
            tops = step.ops[op] / (ms * 1e-3) / 1e12
            kernels[op] = {"ms": round(ms, 4), "TOPS": round(tops, 1), "frac_i8_peak": round(tops / i8_peak_burst, 4)}
        else:
            gbs = step.bytes[op] / (ms * 1e-3) / 1e9
            kernels[op] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    gemm_ops = [op for op in step.ops]
    dom = max(gemm_ops, key=lambda o: statistics.mean(per_op[o]))
    dom_ms = statistics.mean(per_op[dom])
    achieved = step.ops[dom] / (dom_ms * 1e-3) / 1e12
    traffic = _load_traffic(dom)
    # The binding roofline of the block-scaled GEMM is the SM issue rate, not the tensor pipe: every
    # output element needs, per 32-deep contraction block, an int32 -> fp32 convert and an FMA (two
    # lane-instructions), i.e. M*N*K/16 per launch, and an SM issues at most 4 x 32 lane-instructions
    # per clock. That ceiling (about 1.19 int8 POPS at 1965 MHz) lies below the tensor peak.
    alu_work = step.ops[dom] // 32                      # 2*M*N*K / 32 = 2 instructions per (element, block)
    alu_peak = ALU_LANES_PER_CLK_PER_SM * peaks.get("sm_count", B200_SMS) * peaks["sm_max_mhz"] * 1e6 / 1e12
    alu_achieved = alu_work / (dom_ms * 1e-3) / 1e12
    roofline = {"kernel": f"gemm_i8_kernel ({dom})", "bound": "alu", "achieved": round(alu_achieved, 2),
                "peak": round(alu_peak, 2), "unit": "T lane-instructions/s", "frac": round(alu_achieved / alu_peak, 4),
                "traffic": traffic,
                "peak_source": f"{ALU_LANES_PER_CLK_PER_SM} lane-instructions/clk/SM (4 schedulers x 32 lanes) x "
                               f"{B200_SMS} SMs x {peaks['sm_max_mhz']:g} MHz",
                "algorithmic": f"2 per output element per 32-deep block = M*N*K/16 = {alu_work} per launch",
                "tensor_view": {"achieved": round(achieved, 1), "peak": round(i8_peak_burst, 1), "unit": "TOPS",
                                "frac": round(achieved / i8_peak_burst, 4),
                                "peak_source": f"{peak_src} bf16 dense burst x {NOMINAL_I8_OVER_BF16:g}"}}

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(step_ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": "GPT2-medium MLP fc1 linear fwd+dgrad+wgrad with quantize, LayerNorm_i8, GELU_i8 "
                               "and dequantize (per rank)", "M": M, "K": K, "N": N, "block": 32,
                   "inputs": "bf16 X ~N(0,1) with 10 channels x30, W ~N(0,0.02), dY ~N(0,1e-3)",
                   "parallelism": f"dp{world}", "l2": "flushed between steps (256 MiB write, outside timed events)"},
        "kernels": kernels, "roofline": roofline,
        "execution": ("CUDA graph of the step on two streams ordered by data dependences (quantize W, quantize dY "
                      "and the weight gradient beside quantize X, LayerNorm_i8, the forward, GELU_i8 and the input "
                      "gradient); per-kernel times from the nine operators serialized on one stream"
                      if use_graph else "eager launches on one stream, per-kernel events"),
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": sampler.summary(),
    }
    if not args.no_e2e:
        result["e2e"] = run_e2e(step, host, args, world, flush)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(args.cpu_sample_tokens, host)
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
    """Same step through the public API with host buffers. Every step copies its X, W and dY from
    pinned host memory to the device, runs the nine operators, and reads dX (bf16) and dW (codes
    and scales) back to pinned host memory. The steps are pipelined the way a training loop feeds
    a GPU: two device input/output slots, the host->device copies of step i+1 on a copy stream and
    the device->host reads of step i on a third stream while step i+1 computes. The timed window
    runs from the first input copy to the last result read; ms_per_step = window / steps. The L2
    flush before each step's operators is inside the window."""
    import torch
    from int8_fully_quantized_b200 import parallel as P
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    hx, hw, hdy = pin(host["x"]), pin(host["w"]), pin(host["dy"])
    out_dx = torch.empty(step.dx_bf16.shape, dtype=torch.bfloat16).pin_memory()
    out_wq = torch.empty(step.dW.q.shape, dtype=torch.int8).pin_memory()
    out_ws = torch.empty(step.dW.s.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hx, hw, hdy))
    d2h = sum(t.numel() * t.element_size() for t in (out_dx, out_wq, out_ws))

    slots = [step, GpuStep(step.M, step.K, step.N, host, world)]
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
            s.wb.copy_(hw, non_blocking=True)
            s.dyb.copy_(hdy, non_blocking=True)
            ready[k].record(h2d_stream)

    def compute_and_read(i):
        k = i % 2
        s = slots[k]
        main.wait_event(ready[k])
        if i >= 2:
            main.wait_event(read[k])   # step i-2's results have left this slot
        flush.zero_()
        if use_graph:
            s.graph.replay()
        else:
            s.run()
        computed[k].record(main)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(computed[k])
            out_dx.copy_(s.dx_bf16, non_blocking=True)
            out_wq.copy_(s.dW.q, non_blocking=True)
            out_ws.copy_(s.dW.s, non_blocking=True)
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
    return {"value": round(world * ops / (ms * 1e-3) / 1e12, 2), "unit": "TOPS", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pipelining": "two slots; step i+1's host->device copies and step i's device->host reads overlap the "
                          "operators; window from the first input copy to the last result read"}


# --------------------------------------------------------------------------------------------
# CPU oracle timings (the baseline leg, and the --impl reference arm)
# --------------------------------------------------------------------------------------------
def _oracle_step(host, tokens):
    """The whole step in the CPU oracle on the first `tokens` tokens of the batch (W in full).
    Returns the GEMM int8 ops it performed."""
    import oracle as O
    K = host["x"].shape[1]
    N = host["w"].shape[0]
    x = O.bf16_bits_to_f32(host["x"][:tokens])
    w = O.bf16_bits_to_f32(host["w"])
    dy = O.bf16_bits_to_f32(host["dy"][:tokens])
    Xq, Xs = O.quantize_block(x)
    Xn_q, Xn_s, _ = O.layernorm_i8(Xq, Xs, host["gamma"], host["beta"], 1e-5)
    Wq, Ws = O.quantize_block(w)
    Y = O.linear_fwd(Xn_q, Xn_s, Wq, Ws)
    Yq, Ys = O.requantize(Y)
    O.gelu_i8(Yq, Ys)
    dYq, dYs = O.quantize_block(dy)
    dX = O.linear_dgrad(dYq, dYs, Wq, Ws)
    dXq, dXs = O.requantize(dX)
    O.requantize(O.linear_wgrad(dYq, dYs, Xn_q, Xn_s))
    O.dequantize_block(dXq, dXs, "bf16")
    return 3 * 2 * tokens * N * K


def _cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(tokens, host):
    t0 = time.perf_counter()
    ops = _oracle_step(host, tokens)
    dt = time.perf_counter() - t0
    return {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": _cpu_cores(), "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"one oracle step on the first {tokens} of the 4096 tokens (full W), GEMM int8 ops / wall time"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = __import__("inputs.synthetic", fromlist=["WORKLOADS"]).WORKLOADS[WORKLOAD]
    M, K, N = wl["M"], wl["K"], wl["N"]
    host = host_inputs(M, K, N, 1, seed_weight=0)
    tokens = 256
    for _ in range(max(3, args.warmup)):
        _oracle_step(host, tokens)
    times = []
    ops = 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        ops = _oracle_step(host, tokens)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = ops / (ms * 1e-3) / 1e12
    cores = _cpu_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": "GPT2-medium MLP fc1 linear fwd+dgrad+wgrad with quantize, LayerNorm_i8, GELU_i8 "
                               "and dequantize", "M": M, "K": K, "N": N, "block": 32, "parallelism": "oracle on host"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": f"each step: the oracle's full step on the first {tokens} of the {M} tokens"},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """Memory-bound sweep: quantize (bf16 in), dequantize (bf16 out), GELU_i8, LayerNorm_i8 and their
    INT8 backward on M x 4096 tensors, M in {1024, 8192, 65536}; N(0,1) with 1% of the channels x100.
    One JSON line with GB/s (algorithmic bytes: every input read once, every output written once)
    and the fraction of the measured HBM copy bandwidth per kernel and size. With "fused_fc1" it
    also times the GPT2-medium fc1 forward with GELU fused into the GEMM epilogue against the
    forward GEMM followed by GELU_i8."""
    import torch
    import int8_fully_quantized_b200 as jf
    from inputs import synthetic as S
    torch.cuda.set_device(0)
    jf.load_library()
    peaks, peak_src = load_peaks()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    H = 4096
    out = {}
    for M in args.sweep_m:
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
        ops = {
            "quantize_bf16": (lambda: jf.jf_quantize_block(xb, Y.q, Y.s), bytes_quant(M, H, 2)),
            "dequantize_bf16": (lambda: jf.jf_dequantize_block(Q.q, Q.s, yb), M * H * 3 + (M // 32) * (H // 32) * 4),
            "gelu_i8": (lambda: jf.jf_gelu_i8(Q, Y), bytes_i8_op(M, H)),
            "layernorm_i8": (lambda: jf.jf_layernorm_i8(Q, gamma, beta, 1e-5, Y), bytes_i8_op(M, H, 8 * H)),
            "gelu_i8_bwd": (lambda: jf.jf_gelu_i8_bwd(Q, D, Y), bytes_i8_op(M, H, M * H + (M // 32) * (H // 32) * 4)),
            "layernorm_i8_bwd": (lambda: jf.jf_layernorm_i8_bwd(Q, D, gamma, 1e-5, Y, dgam, dbet, ws),
                                 bytes_i8_op(M, H, M * H + (M // 32) * (H // 32) * 4 + 12 * H)),
        }
        dgam, dbet = torch.empty(H, device="cuda"), torch.empty(H, device="cuda")
        ws = torch.empty(jf.jf_layernorm_i8_bwd_workspace_bytes(M, H), dtype=torch.uint8, device="cuda")
        for name, (fn, nbytes) in ops.items():
            if name not in args.sweep_ops:
                continue
            for _ in range(3):
                flush.zero_()
                fn()
            ts = []
            for _ in range(max(5, args.steps // 5)):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(); fn(); b.record()
                ts.append((a, b))
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in ts)
            gbs = nbytes / (ms * 1e-3) / 1e9
            out[f"{name}@M={M}"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        del xb, Q, D, Y, yb, ws
    if "fused_fc1" in args.sweep_ops:
        out.update(_sweep_fused_fc1(jf, flush))
    if "granularity_mse" in args.sweep_ops:
        out["granularity_mse"] = _granularity_mse(jf)
    if "mxfp8_fc1" in args.sweep_ops:
        out["mxfp8_vs_int8_fc1"] = _mxfp8_vs_int8(jf, flush)
    assert jf.jf_device_status() == 0
    print(json.dumps({"sweep": out, "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": peak_src,
                      "l2": "flushed before every timed launch"}), flush=True)


def _mxfp8_vs_int8(jf, flush):
    """The GPT2-medium fc1 forward (M=4096, K=1024, N=4096, bf16 inputs) two ways: Jetfire's 32x32
    INT8 blocks (quantize X and W, block-scaled INT8 GEMM with fp32 output) and MXFP8 (1x32 E8M0
    blocks, E4M3 elements, the tensor core's block-scaled MMA). Device times (L2 flushed before each
    launch) and the relative Frobenius error of each fp32 output against the exact product of the
    bf16 inputs (fp64 on the host)."""
    import torch
    wl = __import__("inputs.synthetic", fromlist=["WORKLOADS"]).WORKLOADS[WORKLOAD]
    M, K, N = wl["M"], wl["K"], wl["N"]
    host = host_inputs(M, K, N, 0, seed_weight=0)
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
    wl = __import__("inputs.synthetic", fromlist=["WORKLOADS"]).WORKLOADS[WORKLOAD]
    host = host_inputs(wl["M"], wl["K"], wl["N"], 0, seed_weight=0)
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
    wl = __import__("inputs.synthetic", fromlist=["WORKLOADS"]).WORKLOADS[WORKLOAD]
    M, K, N = wl["M"], wl["K"], wl["N"]
    host = host_inputs(M, K, N, 0, seed_weight=0)
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


def main():
    args = parse_args()
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
