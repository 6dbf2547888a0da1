#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 + double-quant linear layer on B200.

Headline: forward + backward of one 4096 x 4096 QLoRA linear at M = 4096
tokens, rank 64, alpha 128 (s = 2), W ~ N(0, 0.02) with 0.1 % outliers x 10,
X and dY ~ N(0, 1) in bf16 -- in TFLOP/s of algorithmic work
    4 M d_in d_out + 6 M r (d_in + d_out)  per step.
A step = one qlora_linear_fwd + one qlora_linear_bwd (the frozen weight is
quantised once, before timing, as in training). With --gpus N > 1 each rank
runs the same step on its own batch (weak scaling) and the adapter gradients
dA, dB are summed over ranks with NCCL, the data-parallel exchange.

Also reported ("components", rank 0 at N = 1): the quantise and dequantise
sweep over 32 Llama-7B-shaped layers (HBM GB/s) and the decode-sized NF4
GEMV over one Llama-7B block at M in {1, 4, 16} (HBM GB/s).

--impl reference times the CPU oracle (plain C + numpy fp64) on a bounded
sample of the same workload; it is the reference arm of this repository.
"""
import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s at M=4096; NF4 GEMV/dequant HBM GB/s"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the library's kernels, as named by its launch bookkeeping
KERNELS = ("k_gemm2sm", "k_dequant", "k_fused_fwd", "k_fused_dgrad", "k_skinny",
           "k_gemv_xa", "k_gemv", "k_gemv_finish", "k_quantize_codes", "k_offset", "k_double_quant", "k_adamw")
# DRAM bytes (read + write) of one launch of the dominant kernel, from an ncu
# capture of the same kernel and workload; update with the kernel.
TRAFFIC_BYTES = {"k_gemm2sm": 79222357}
TRAFFIC_SOURCE = {"k_gemm2sm": "ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum "
                                "--clock-control none -k regex:k_ on bench.py --profile-case l4096 (three fwd + bwd "
                                "steps of this workload): mean of the six k_gemm2sm launches"}
L2_FLUSH_BYTES = 256 << 20        # 2x the 126 MB L2
DEFAULT_PAIR_MIN_M = 128          # the library's default token count for the pair-GEMM route


def l2_flush(buf):
    """Evict the timed kernels' inputs from L2 between timed repetitions (outside the timed
    region): write a buffer twice the L2 size, then read it back. The read leaves L2 holding
    clean lines of the flush buffer; a write alone would leave about 126 MB of dirty lines
    whose write-back the next timed kernel would pay for in DRAM bandwidth."""
    import torch
    buf.zero_()
    buf.view(torch.int32).sum()


def step_flops(M, d_in, d_out, r):
    return 4.0 * M * d_in * d_out + 6.0 * M * r * (d_in + d_out)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and clock-event reasons of this rank's GPU, polled through NVML every
    ~0.5 ms on a background thread (the timed region lasts only a few milliseconds),
    plus one sample taken synchronously when the region ends (right after the final
    synchronise, before the clock can relax); only samples between mark_begin() and
    mark_end() count. Reads the settings only, changes none."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.nv = self.h = None
        self.t0 = self.t1 = None
        self.thread = None
        self.stop_flag = False
        self.max_mhz = None
        self.err = None

    def _handle(self, nv):
        import torch
        try:
            pr = torch.cuda.get_device_properties(self.gpu)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception as e:   # NVML missing: no samples, say why
            self.err = f"nvml unavailable: {e}"
            return
        self.nv, self.h = nv, h

        def poll():
            while not self.stop_flag:
                try:
                    t = time.perf_counter()
                    mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    try:
                        rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                    except Exception:
                        rs = int(nv.nvmlDeviceGetCurrentClocksThrottleReasons(h))
                    self.samples.append((t, mhz, rs))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.0005)
        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        time.sleep(0.01)

    def mark_begin(self):
        self.t0 = time.perf_counter()

    def _sample_now(self):
        nv, h = self.nv, self.h
        if nv is None:
            return
        try:
            mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
            try:
                rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
            except Exception:
                rs = int(nv.nvmlDeviceGetCurrentClocksThrottleReasons(h))
            self.samples.append((time.perf_counter(), mhz, rs))
        except Exception as e:
            self.err = str(e)

    def mark_end(self):
        self._sample_now()
        self.t1 = time.perf_counter()

    def stop(self):
        self.stop_flag = True
        if self.thread is not None:
            self.thread.join(timeout=2)
        t0 = self.t0 if self.t0 is not None else -1e30
        t1 = self.t1 if self.t1 is not None else 1e30
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": [self.err or "no samples in the timed region"], "samples": 0, "source": "nvml"}
        reasons = sorted({name for _, _, rs in inside for bit, name in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(m for _, m, _ in inside), "sm_min_mhz": min(m for _, m, _ in inside),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside), "source": "nvml, 0.5 ms"}


# ------------------------------------------------------------------ distributed
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def allreduce_adapter_grads(dA, dB, world):
    """Data-parallel exchange of the adapter gradients (sum over ranks)."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(dA)
        dist.all_reduce(dB)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    import torch
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ our arm
def rank_batch(wl, li, rank, device):
    """The data-parallel partition of the tokens: rank k trains on its own batch of
    wl.M tokens (X, dY), drawn with the workload's seeds shifted by 7777 k, so the
    global batch of N ranks is the concatenation of the N rank batches in rank order
    (rank 0's batch is the single-GPU workload itself)."""
    import torch
    import synth_inputs as si
    L = wl.layers[li]
    X = si.normal((wl.M, L.d_in), 1.0, si.seed_of(wl, li, "X") + 7777 * rank, device=device, dtype=torch.bfloat16)
    dY = si.normal((wl.M, L.d_out), 1.0, si.seed_of(wl, li, "dY") + 7777 * rank, device=device,
                   dtype=torch.bfloat16)
    return X, dY


def headline_inputs(rank):
    import synth_inputs as si
    wl = si.workload("l4096")
    L = wl.layers[0]
    inp = si.layer_inputs(wl, 0, device="cuda", w_device="cuda")
    if rank:
        # weak scaling: every rank its own batch of tokens
        inp["X"], inp["dY"] = rank_batch(wl, 0, rank, "cuda")
    return wl, L, inp


def run_ours(args, peaks, peak_kind):
    import torch
    import bit_nf4_quantized_double_b200 as q

    world, rank, local = dist_setup(args)
    wl, L, inp = headline_inputs(rank)
    M, d_in, d_out, r, s = wl.M, L.d_in, L.d_out, L.r, L.s
    dev = inp["X"].device
    t = q.qlora_nf4_quantize(inp["W"])
    del inp["W"]
    X, dY, A, B = inp["X"], inp["dY"], inp["A"], inp["B"]
    Y = torch.empty(M, d_out, dtype=torch.bfloat16, device=dev)
    XA = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, d_in, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(d_in, r, dtype=torch.float32, device=dev)
    dB = torch.empty(r, d_out, dtype=torch.float32, device=dev)
    Lb = q.lib()
    ws_f = torch.empty(max(1, Lb.qlora_linear_fwd_workspace(M, d_out, d_in, r)), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(max(1, Lb.qlora_linear_bwd_workspace(M, d_out, d_in, r)), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def layer_step():
        q.qlora_linear_fwd(X, t, A, B, s, Y=Y, XA_save=XA, ws=ws_f)
        q.qlora_linear_bwd(X, dY, t, A, B, s, XA=XA, dX=dX, dA=dA, dB=dB, ws=ws_b)

    def eager_step():
        layer_step()
        allreduce_adapter_grads(dA, dB, world)

    for _ in range(args.warmup):
        eager_step()
    torch.cuda.synchronize()
    status = q.qlora_get_device_status()
    if status != q.QLORA_OK:
        raise RuntimeError(f"device status {status} during warm-up")

    # The layer's fwd + bwd launches are captured once in a CUDA graph and replayed
    # each step (the same kernels on the same buffers; the graph removes the host
    # launch cost). The gradient all-reduce stays outside the graph.
    graph = None
    launches_per_step = None
    if not args.no_graph:
        c0 = q.qlora_launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer_step()
        launches_per_step = q.qlora_launch_count() - c0
        graph.replay()
        torch.cuda.synchronize()

    def step():
        if graph is not None:
            graph.replay()
            allreduce_adapter_grads(dA, dB, world)
        else:
            eager_step()

    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    launches0 = q.qlora_launch_count()
    clocks.mark_begin()
    for i in range(args.steps):
        l2_flush(flush)                     # L2 flush between timed steps (not timed)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    launches = q.qlora_launch_count() - launches0
    if graph is not None:
        launches = launches_per_step * args.steps   # replays launch without the host counter
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier(world)
    clk = clocks.stop()
    total_ms = sum(a.elapsed_time(b) for a, b in evs)
    total_ms = max_over_ranks(total_ms, world)
    status = q.qlora_get_device_status()
    if status != q.QLORA_OK:
        raise RuntimeError(f"device status {status} during timing")

    # Per-kernel breakdown from a second, identical pass with every launch of the
    # library bracketed by CUDA events on its stream (kept out of the timed pass
    # above because the events add a little time per launch).
    q.qlora_profile_read(None)
    q.qlora_profile_enable(True)
    for i in range(args.steps):
        l2_flush(flush)
        eager_step()
    q.qlora_profile_enable(False)
    torch.cuda.synchronize()
    kern = {}
    for name in KERNELS:
        ms, n = q.qlora_profile_read(name)
        if n:
            kern[name] = (ms, n)
    q.qlora_profile_read(None)

    flops = step_flops(M, d_in, d_out, r)
    value = world * args.steps * flops / (total_ms / 1e3) / 1e12
    # dominant kernel: the tensor-core GEMM of the path in use (the CTA-pair GEMM
    # for this batch: forward and dgrad launches, whose flops are equal here)
    dom = "k_gemm2sm" if "k_gemm2sm" in kern else max(("k_fused_fwd", "k_fused_dgrad"), key=lambda k: kern.get(k, (0, 0))[0])
    fwd_flops = 2.0 * M * d_in * d_out + 2.0 * M * r * d_out
    dgrad_flops = 2.0 * M * d_out * d_in + 2.0 * M * r * d_in
    dom_ms, dom_n = kern.get(dom, (0.0, 0))
    per_step = dom_n // args.steps if dom_n else 0
    dom_flops = (fwd_flops + dgrad_flops) / 2 if per_step == 2 else (fwd_flops if dom != "k_fused_dgrad" else dgrad_flops)
    achieved = dom_flops / (dom_ms / dom_n / 1e3) / 1e12 if dom_n else None
    # the timed region lasts milliseconds, so the burst cuBLAS figure is the denominator;
    # the sustained (seconds-long, power-capped) one is reported beside it
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))

    # ---------------------------------------------------------------- e2e
    Xh = X.cpu().pin_memory()
    dYh = dY.cpu().pin_memory()
    dAh = torch.empty(dA.shape, dtype=dA.dtype).pin_memory()
    dBh = torch.empty(dB.shape, dtype=dB.dtype).pin_memory()

    def e2e_step():
        X.copy_(Xh, non_blocking=True)
        dY.copy_(dYh, non_blocking=True)
        step()
        dAh.copy_(dA, non_blocking=True)
        dBh.copy_(dB, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    for i in range(args.steps):
        l2_flush(flush)
        eev[i][0].record(stream)
        e2e_step()
        eev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in eev), world)
    e2e = {"value": world * args.steps * flops / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
           "h2d_bytes_per_step": X.numel() * 2 + dY.numel() * 2,
           "d2h_bytes_per_step": dA.numel() * 4 + dB.numel() * 4}

    components = None
    if world == 1 and not args.no_components:
        del Xh, dYh
        components = run_components(args, peaks, peak_kind, flush)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(M_sample=args.cpu_sample_tokens)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, generated on device)",
        "config": {"workload": "QLoRA linear 4096x4096 (d_in=d_out=4096), M=4096 tokens, r=64, alpha=128 (s=2), "
                               "W ~ N(0,0.02) fp32 with 0.1% x10 outliers quantised once to NF4+DQ, "
                               "X,dY ~ N(0,1) bf16; step = fwd + bwd" + (" + NCCL all-reduce of dA,dB"
                                                                       if world > 1 else ""),
                   "global_batch_tokens": M * world, "l2": "flushed between timed steps (256 MB written, then read back)",
                   "flops_per_step": flops, "parallelism": f"dp{world}" if world > 1 else "single GPU",
                   "launch": "CUDA graph replay of the layer fwd+bwd" if graph is not None else "eager"},
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 2) if achieved else None,
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4) if achieved else None,
                     "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback 1590 TFLOP/s burst",
                     "frac_of_sustained": round(achieved / peak_sustained, 4) if achieved else None,
                     "traffic": TRAFFIC_BYTES.get(dom), "traffic_source": TRAFFIC_SOURCE.get(dom), "flops_per_launch": dom_flops, "launches": dom_n,
                     "kernel_ms_per_step": {k: round(v[0] / args.steps, 5) for k, v in kern.items()},
                     "kernel_launches_per_step": {k: v[1] // args.steps for k, v in kern.items()}},
        "e2e": e2e, "gpu_launches": launches, "clocks": clk,
    }
    if components is not None:
        line["components"] = components
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def _time_graph(fn, reps, flush, stream):
    """Capture fn in a CUDA graph, replay it reps times with an L2 flush before
    each replay; return the average device milliseconds of one replay."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    for _ in range(2):
        g.replay()
    times = []
    for _ in range(reps):
        l2_flush(flush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(torch.cuda.current_stream())
        g.replay()
        b.record(torch.cuda.current_stream())
        times.append((a, b))
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in times) / reps
    del g
    return ms


def _host_time(fn, target_s=2.0, max_reps=10):
    """Seconds per call of fn on the host: one call, then repeats filling about target_s."""
    t0 = time.perf_counter()
    fn()
    one = time.perf_counter() - t0
    reps = max(1, min(max_reps, int(target_s / max(one, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(reps):
        fn()
    return (time.perf_counter() - t0) / reps, reps


def _kernel_ms(names, fn, reps, flush):
    """Per-call device milliseconds of the named library kernels over `reps` eager calls
    of fn (every launch bracketed by CUDA events on its stream, L2 flushed before each)."""
    import torch
    import bit_nf4_quantized_double_b200 as q
    q.qlora_profile_read(None)
    q.qlora_profile_enable(True)
    for _ in range(reps):
        l2_flush(flush)
        fn()
    q.qlora_profile_enable(False)
    torch.cuda.synchronize()
    out = {}
    for n in names:
        ms, k = q.qlora_profile_read(n)
        if k:
            out[n] = {"ms_per_call": round(ms / reps, 5), "launches_per_call": k // reps}
    q.qlora_profile_read(None)
    return out


def run_components(args, peaks, peak_kind, flush):
    import numpy as np
    import torch
    import bit_nf4_quantized_double_b200 as q
    import oracle
    import synth_inputs as si

    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    out = {"hbm_peak_gbs": hbm, "hbm_peak_source": peak_kind}
    stream = torch.cuda.current_stream()
    cores = _cores()

    # --- quantise / dequantise sweep over 32 Llama-7B-shaped layers (bf16 weights), one
    # grouped call per layer (its seven projections)
    n_layers = args.sweep_layers
    wl = si.workload("llama7b", n_layers=n_layers)
    layers = []
    for l0 in range(0, len(wl.layers), 7):
        Ws = [si.layer_inputs(wl, li, device="cuda")["W"] for li in range(l0, l0 + 7)]
        layers.append((Ws, [q.nf4_empty(W.shape[0], W.shape[1]) for W in Ws]))
    n_w = sum(W.numel() for Ws, _ in layers for W in Ws)
    ws_q = torch.empty(q.lib().qlora_nf4_quantize_grouped_workspace(
        7, (q._Tensor * 7)(*[t.ctype() for t in layers[0][1]])), dtype=torch.uint8, device="cuda")
    wh = [torch.empty(W.shape, dtype=torch.bfloat16, device="cuda") for W in layers[0][0]]
    alg_bytes = 2.0 + 0.5 + 1.0 / 64 + 4.0 / 16384       # per weight, bf16 in/out

    def quant_sweep():
        for Ws, Ts in layers:
            q.qlora_nf4_quantize_grouped(Ws, outs=Ts, ws=ws_q)

    def deq_sweep():
        for _, Ts in layers:
            q.qlora_nf4_dequant_grouped(Ts, outs=wh)

    res = {}
    for name, fn, knames in (("quantize", quant_sweep, ("k_quantize_codes", "k_offset", "k_double_quant")),
                             ("dequant", deq_sweep, ("k_dequant",))):
        reps = 3
        ms = _time_graph(fn, reps, flush, stream)
        kern = _kernel_ms(knames, fn, reps, flush)
        kms = sum(v["ms_per_call"] for v in kern.values())
        gbs = n_w * alg_bytes / (ms / 1e3) / 1e9
        res[name] = {"workload": f"{n_layers} Llama-7B layers x 7 projections, {n_w} bf16 weights, "
                                 "one grouped call per layer, CUDA graph replay, L2 flushed",
                     "ms_per_sweep": round(ms, 4), "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 4),
                     "kernels": kern, "kernel_GB/s": round(n_w * alg_bytes / (kms / 1e3) / 1e9, 1) if kms else None,
                     "bytes_per_weight": round(alg_bytes, 5)}
    # the oracle on the host: one projection (4096 x 4096, bf16) quantised and dequantised
    Wq = layers[0][0][0]
    bits = Wq.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    t_q, rq = _host_time(lambda: oracle.quantize_bf16(bits, Wq.shape[0], Wq.shape[1]))
    ref = oracle.quantize_bf16(bits, Wq.shape[0], Wq.shape[1])
    t_d, rd = _host_time(lambda: oracle.dequant(ref))
    nq = Wq.numel()
    for name, t_s, reps in (("quantize", t_q, rq), ("dequant", t_d, rd)):
        res[name]["cpu_baseline"] = {"value": round(nq * alg_bytes / t_s / 1e9, 3), "unit": "GB/s", "cores": cores,
                                     "kind": "oracle", "sample": f"one 4096 x 4096 bf16 projection, {reps} calls"}
    out["llama7b_sweep"] = res
    assert q.qlora_get_device_status() == q.QLORA_OK
    del layers, wh, ws_q
    torch.cuda.empty_cache()

    # --- decode GEMV: one Llama-7B block at M in {1, 4, 16}, forward only
    gem = {}
    for M in (1, 4, 16):
        wl = si.workload("decode7b", M=M)
        items = []
        nbytes = 0
        for li, L in enumerate(wl.layers):
            inp = si.layer_inputs(wl, li, device="cuda")
            T = q.qlora_nf4_quantize(inp["W"])
            Y = torch.empty(M, L.d_out, dtype=torch.bfloat16, device="cuda")
            items.append({"X": inp["X"], "W": T, "A": inp.get("A"), "B": inp.get("B"), "s": L.s, "Y": Y,
                          "Wsrc": inp["W"] if li == 0 else None})
            nbytes += T.nbytes + inp["X"].numel() * 2 + Y.numel() * 2
            if L.r:
                nbytes += inp["A"].numel() * 2 + inp["B"].numel() * 2
            del inp
        # the block's seven projections in one grouped call (one persistent GEMV, X A, finish)
        wsz = q.lib().qlora_linear_fwd_grouped_workspace(
            M, len(items), (q._LinearDesc * len(items))(*[
                q._LinearDesc(None, ctypes.pointer(it["W"].ctype()), None, None,
                              0 if it["A"] is None else it["A"].shape[1], 1.0, None, None) for it in items]))
        ws = torch.empty(max(1, wsz), dtype=torch.uint8, device="cuda")

        def layer():
            q.qlora_linear_fwd_grouped(items, ws=ws)

        ms = _time_graph(layer, 20, flush, stream)
        gbs = nbytes / (ms / 1e3) / 1e9
        kern = _kernel_ms(("k_gemv", "k_gemv_xa", "k_gemv_finish"), layer, 10, flush)
        gem[f"M{M}"] = {"ms_per_layer": round(ms, 5), "bytes": nbytes, "GB/s": round(gbs, 1),
                        "frac": round(gbs / hbm, 4), "kernels": kern}
        if M == 1:
            # the oracle on the host: the q projection at M = 1 (dequantise in C, fp64 product)
            it = items[0]
            L = wl.layers[0]
            bits = it["Wsrc"].view(torch.int16).cpu().numpy().view(np.uint16).ravel()
            ref = oracle.quantize_bf16(bits, L.d_out, L.d_in)
            f64 = lambda t: t.to(torch.float64).cpu().numpy()
            Xn, An, Bn = f64(it["X"]), f64(it["A"]), f64(it["B"])

            def cpu_q():
                Wh = oracle.bf16_bits_to_f32(oracle.dequant(ref)).reshape(L.d_out, L.d_in).astype(np.float64)
                oracle.linear_fwd(Xn, Wh, An, Bn, L.s)
            t_c, reps = _host_time(cpu_q)
            qbytes = it["W"].nbytes + it["X"].numel() * 2 + it["Y"].numel() * 2 + (An.size + Bn.size) * 2
            gem[f"M{M}"]["cpu_baseline"] = {"value": round(qbytes / t_c / 1e9, 3), "unit": "GB/s", "cores": cores,
                                            "kind": "oracle",
                                            "sample": f"the q projection (4096 x 4096, r = 16) at M = 1, {reps} calls"}
        del items
        torch.cuda.empty_cache()
    out["decode7b_gemv"] = {"workload": "one Llama-7B block (q,k,v,o 4096x4096; gate,up 11008x4096; "
                                        "down 4096x11008), r=16 on q,k,v,o, fwd only, one grouped call "
                                        "(qlora_linear_fwd_grouped), CUDA graph replay, L2 flushed", **gem}
    assert q.qlora_get_device_status() == q.QLORA_OK
    out["l70b_layer"] = run_l70b(args, peaks, peak_kind, flush, stream)
    out["merge_4096"] = run_merge(hbm, flush, stream)
    out["fmt4"] = run_fmt4(hbm, flush, stream)
    out["adamw"] = run_adamw(hbm, flush, stream)
    out["large_m_routes"] = run_routes(flush, stream)
    out["mid_m"] = run_mid_m(flush, stream)
    return out


def run_routes(flush, stream):
    """The headline layer's fwd + bwd (4096 x 4096, M = 4096, r = 64) through each of the two
    large-M routes: the default (dequantise W once into bf16 scratch, CTA-pair GEMM) and the
    fused dequant-GEMM kernels forced at every M, which dequantise the codes in the mainloop
    of each 256-token tile."""
    import torch
    import bit_nf4_quantized_double_b200 as q
    wl, L, inp = headline_inputs(0)
    M, d_in, d_out, r, s = wl.M, L.d_in, L.d_out, L.r, L.s
    t = q.qlora_nf4_quantize(inp["W"])
    X, dY, A, B = inp["X"], inp["dY"], inp["A"], inp["B"]
    flops = step_flops(M, d_in, d_out, r)
    out = {"workload": "4096 x 4096 layer, M = 4096, r = 64, fwd + bwd, CUDA graph replay, L2 flushed"}
    for name, P in (("dequant_then_pair_gemm", DEFAULT_PAIR_MIN_M), ("fused_dequant_gemm", 2 ** 63 - 1)):
        q.lib().qlora_linear_set_pair_min_m(P)
        try:
            Y = torch.empty(M, d_out, dtype=torch.bfloat16, device="cuda")
            XA = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
            dX = torch.empty(M, d_in, dtype=torch.bfloat16, device="cuda")
            dA = torch.empty(d_in, r, dtype=torch.float32, device="cuda")
            dB = torch.empty(r, d_out, dtype=torch.float32, device="cuda")
            ws_f = torch.empty(max(1, q.lib().qlora_linear_fwd_workspace(M, d_out, d_in, r)), dtype=torch.uint8,
                               device="cuda")
            ws_b = torch.empty(max(1, q.lib().qlora_linear_bwd_workspace(M, d_out, d_in, r)), dtype=torch.uint8,
                               device="cuda")

            def step():
                q.qlora_linear_fwd(X, t, A, B, s, Y=Y, XA_save=XA, ws=ws_f)
                q.qlora_linear_bwd(X, dY, t, A, B, s, XA=XA, dX=dX, dA=dA, dB=dB, ws=ws_b)

            ms = _time_graph(step, 10, flush, stream)
            kern = _kernel_ms(KERNELS, step, 5, flush)
            out[name] = {"ms_per_step": round(ms, 5), "TFLOP/s": round(flops / (ms / 1e3) / 1e12, 1),
                         "kernels": kern}
        finally:
            q.lib().qlora_linear_set_pair_min_m(DEFAULT_PAIR_MIN_M)
    assert q.qlora_get_device_status() == q.QLORA_OK
    return out


def run_mid_m(flush, stream, M=480, r=64):
    """Mid-sized batches on weights with one narrow side: the default routing (the pair GEMM
    from 128 tokens on, with split K where the tiles are few) against the fused kernels
    everywhere."""
    import torch
    import bit_nf4_quantized_double_b200 as q
    import synth_inputs as si
    out = {"workload": f"fwd + bwd at M = {M}, r = {r}, weights 16384 x 1024 and 1024 x 16384, CUDA graph replay, "
                       "L2 flushed"}
    for rows, cols in ((16384, 1024), (1024, 16384)):
        W = si.normal((rows, cols), 0.02, seed=rows + 3, device="cuda")
        t = q.qlora_nf4_quantize(W)
        del W
        X = si.normal((M, cols), 1.0, seed=5, device="cuda", dtype=torch.bfloat16)
        dY = si.normal((M, rows), 1.0, seed=6, device="cuda", dtype=torch.bfloat16)
        A = si.normal((cols, r), 0.02, seed=7, device="cuda", dtype=torch.bfloat16)
        B = si.normal((r, rows), 0.01, seed=8, device="cuda", dtype=torch.bfloat16)
        flops = step_flops(M, cols, rows, r)
        res = {}
        for name, P in (("default", DEFAULT_PAIR_MIN_M), ("fused_everywhere", 2 ** 63 - 1)):
            q.lib().qlora_linear_set_pair_min_m(P)
            try:
                def step():
                    Y, XA = q.qlora_linear_fwd(X, t, A, B, 2.0)
                    q.qlora_linear_bwd(X, dY, t, A, B, 2.0, XA=XA)
                ms = _time_graph(step, 10, flush, stream)
                res[name] = {"ms_per_step": round(ms, 5), "TFLOP/s": round(flops / (ms / 1e3) / 1e12, 1),
                             "kernels": _kernel_ms(KERNELS + ("k_gemm2sm_reduce",), step, 3, flush)}
            finally:
                q.lib().qlora_linear_set_pair_min_m(DEFAULT_PAIR_MIN_M)
        out[f"{rows}x{cols}"] = res
        del t
    assert q.qlora_get_device_status() == q.QLORA_OK
    return out


def run_adamw(hbm, flush, stream, layers=80):
    """The adapter's optimizer step (AdamW, fp32 state) over the adapters of 80 70B-like
    layers (r = 64 on all seven projections: 10.35 M parameters a layer), in device memory
    and in managed memory brought to the GPU beforehand; 30 bytes per parameter."""
    import numpy as np
    import torch
    import bit_nf4_quantized_double_b200 as q
    import oracle
    import synth_inputs as si
    wl = si.workload("l70b")
    per_layer = sum(L.r * (L.d_in + L.d_out) for L in wl.layers)
    n = per_layer * layers
    res = {"workload": f"AdamW step over the r=64 adapters of {layers} 70B-like layers ({n} fp32 parameters), "
                       "CUDA graph replay", "params": n, "bytes_per_param": 30}
    g = torch.randn(n, device="cuda") * 1e-3
    for kind in ("device", "managed"):
        if kind == "device":
            theta, m, v = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
            tb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        else:
            theta, m, v, tb = q.managed_empty(n), q.managed_empty(n), q.managed_empty(n), q.managed_empty(n, torch.bfloat16)
            for x in (theta, m, v):
                x.zero_()
            for x in (theta, m, v, tb):
                q.qlora_adamw_prefetch(x, to_device=True)
        ms = _time_graph(lambda: q.qlora_adamw_step(theta, g, m, v, 1, 1e-3, theta_bf16=tb), 5, flush, stream)
        gbs = n * 30 / (ms / 1e3) / 1e9
        res[kind] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 4)}
        del theta, m, v, tb
        torch.cuda.empty_cache()
    assert q.qlora_get_device_status() == q.QLORA_OK
    del g
    torch.cuda.empty_cache()
    rng = np.random.default_rng(0)
    th = rng.normal(0, 0.02, per_layer).astype(np.float32)
    gg = rng.normal(0, 1e-3, per_layer).astype(np.float32)
    mm, vv = np.zeros(per_layer, np.float32), np.zeros(per_layer, np.float32)
    t_c, reps = _host_time(lambda: oracle.adamw_step(th, gg, mm, vv, 1, 1e-3, want_bf16=True))
    res["cpu_baseline"] = {"value": round(per_layer * 30 / t_c / 1e9, 3), "unit": "GB/s", "cores": _cores(),
                           "kind": "oracle", "sample": f"one layer's adapters ({per_layer} parameters), {reps} calls"}
    return res


def run_fmt4(hbm, flush, stream):
    """The 4-bit reference formats (Int4, FP4 E2M1, FP4 E3M0) on 2^26 fp32 weights: quantise
    (4 + 1/2 + 4/64 B per weight) and dequantise (1/2 + 4/64 + 2 B per weight) against HBM."""
    import numpy as np
    import torch
    import bit_nf4_quantized_double_b200 as q
    from oracle import formats
    import synth_inputs as si
    n = 1 << 26
    W = si.normal((n,), 0.02, seed=77, device="cuda")
    res = {}
    wn = si.normal((1 << 20,), 0.02, seed=77).numpy()
    for fmt in ("int4", "fp4_e2m1", "fp4_e3m0"):
        codes, absmax = q.qlora_fmt4_quantize(W, fmt)
        outb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        mq = _time_graph(lambda: q.qlora_fmt4_quantize(W, fmt), 5, flush, stream)
        md = _time_graph(lambda: q.qlora_fmt4_dequant(codes, absmax, n, fmt, out=outb), 5, flush, stream)
        bq, bd = n * (4 + 0.5 + 4 / 64), n * (0.5 + 4 / 64 + 2)
        t_c, reps = _host_time(lambda: formats.dequant(*formats.quantize(wn, fmt), fmt), target_s=1.0)
        res[fmt] = {"quantize_ms": round(mq, 4), "quantize_GB/s": round(bq / (mq / 1e3) / 1e9, 1),
                    "quantize_frac": round(bq / (mq / 1e3) / 1e9 / hbm, 4),
                    "dequant_ms": round(md, 4), "dequant_GB/s": round(bd / (md / 1e3) / 1e9, 1),
                    "dequant_frac": round(bd / (md / 1e3) / 1e9 / hbm, 4),
                    "cpu_baseline": {"value": round((1 << 20) * (4 + 0.5 + 4 / 64 + 0.5 + 4 / 64 + 2) / t_c / 1e9, 3),
                                     "unit": "GB/s", "cores": 1, "kind": "oracle",
                                     "sample": f"2^20 weights quantised and dequantised (numpy), {reps} calls"}}
    assert q.qlora_get_device_status() == q.QLORA_OK
    del W
    torch.cuda.empty_cache()
    return {"workload": "2^26 fp32 weights ~ N(0, 0.02^2), 64-weight absmax blocks, CUDA graph replay, L2 flushed",
            **res}


_FLUSH = [None]


def run_merge(hbm, flush, stream):
    """Adapter merge + re-quantisation of the 4096 x 4096 layer (r = 64): time per call
    (CUDA-graph replay, L2 flushed) and the change of the layer output it causes."""
    import torch
    import bit_nf4_quantized_double_b200 as q
    import synth_inputs as si
    _FLUSH[0] = flush
    wl = si.workload("l4096")
    L = wl.layers[0]
    inp = si.layer_inputs(wl, 0, device="cuda")
    t = q.qlora_nf4_quantize(inp["W"])
    out = q.nf4_empty(L.d_out, L.d_in)
    wb = torch.empty(L.d_out, L.d_in, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(q.lib().qlora_nf4_merge_workspace(L.d_out, L.d_in), dtype=torch.uint8, device="cuda")
    ms = _time_graph(lambda: q.qlora_nf4_merge_adapter(t, inp["A"], inp["B"], L.s, out=out, W_bf16=wb, ws=ws),
                     10, flush, stream)
    n = L.d_out * L.d_in
    # NF4 read, merged bf16 written and read back by the quantiser, NF4 written
    alg = n * (2 * (0.5 + 1 / 64 + 4 / 16384) + 2 * 2) + (L.d_in + L.d_out) * L.r * 2
    X = inp["X"][:256]
    Yu, _ = q.qlora_linear_fwd(X, t, inp["A"], inp["B"], L.s)
    Ym, _ = q.qlora_linear_fwd(X, out, None, None, 0.0)
    rel = ((Ym.double() - Yu.double()).norm() / Yu.double().norm()).item()
    assert q.qlora_get_device_status() == q.QLORA_OK
    kern = _kernel_ms(("k_merge_prep", "k_merge_bf16", "k_quantize_codes", "k_offset", "k_double_quant"),
                      lambda: q.qlora_nf4_merge_adapter(t, inp["A"], inp["B"], L.s, out=out, W_bf16=wb, ws=ws), 5,
                      _FLUSH[0])
    # the oracle on the host: merge (C) and re-quantisation of the same weight
    import numpy as np
    import oracle
    ref = oracle.quantize(inp["W"].cpu().numpy())
    wh_bits = oracle.dequant(ref).reshape(L.d_out, L.d_in)
    An = inp["A"].float().cpu().numpy()
    Bn = inp["B"].float().cpu().numpy()

    def cpu_merge():
        m = oracle.merge_bf16(wh_bits, An, Bn, L.s)
        oracle.quantize_bf16(m.ravel(), L.d_out, L.d_in)
    t_c, reps = _host_time(cpu_merge, target_s=3.0)
    return {"workload": "merge s*(AB)^T into the 4096x4096 NF4 weight in bf16 and re-quantise (r=64), "
                        "CUDA graph replay, L2 flushed",
            "ms": round(ms, 4), "GB/s": round(alg / (ms / 1e3) / 1e9, 1), "frac": round(alg / (ms / 1e3) / 1e9 / hbm, 4),
            "kernels": kern,
            "k_merge_bf16_roofline": _merge_roofline(kern, n, L.r),
            "cpu_baseline": {"value": round(alg / t_c / 1e9, 3), "unit": "GB/s", "cores": _cores(), "kind": "oracle",
                             "sample": f"the same merge and re-quantisation, full size, {reps} calls"},
            "output_rel_change_fro": round(rel, 6),
            "output_change_sample": "256 tokens: X W'^T (merged, re-quantised) against X W^T + s (XA) B"}


# fp32 FMA peak of the merge kernel's bound (its r multiply-adds per weight have a fixed
# order, so they run on the FP32 pipes): 148 SMs x 128 FMA lanes x 2 flop x 1.965 GHz
# (the B200's maximum SM clock), a derived figure, not a measured one.
FP32_FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def _merge_roofline(kern, n, r):
    k = kern.get("k_merge_bf16")
    if not k or not k.get("ms_per_call"):
        return None
    achieved = 2.0 * n * r / (k["ms_per_call"] / 1e3) / 1e12
    return {"bound": "alu", "achieved": round(achieved, 2), "peak": round(FP32_FMA_PEAK_TFLOPS, 2),
            "unit": "TFLOP/s", "frac": round(achieved / FP32_FMA_PEAK_TFLOPS, 4),
            "peak_source": "derived: 148 SMs x 128 fp32 FMA lanes x 2 x 1.965 GHz",
            "work": f"2 x {n} weights x r = {r} flop (one fused multiply-add per weight per j)"}


def run_l70b(args, peaks, peak_kind, flush, stream):
    """One 70B-like layer (q,o 8192^2; k,v 1024x8192; gate,up 28672x8192; down
    8192x28672), r = 64 on all seven projections, M = 4096: fwd + bwd of every
    projection, replayed from one CUDA graph, L2 flushed between replays."""
    import torch
    import bit_nf4_quantized_double_b200 as q
    import synth_inputs as si
    wl = si.workload("l70b")
    M = wl.M
    items = []
    flops = 0.0
    for li, L in enumerate(wl.layers):
        inp = si.layer_inputs(wl, li, device="cuda")
        T = q.qlora_nf4_quantize(inp["W"])
        del inp["W"]
        lb = q.lib()
        it = dict(X=inp["X"], dY=inp["dY"], A=inp["A"], B=inp["B"], s=L.s, T=T,
                  Y=torch.empty(M, L.d_out, dtype=torch.bfloat16, device="cuda"),
                  XA=torch.empty(M, L.r, dtype=torch.bfloat16, device="cuda"),
                  dX=torch.empty(M, L.d_in, dtype=torch.bfloat16, device="cuda"),
                  dA=torch.empty(L.d_in, L.r, dtype=torch.float32, device="cuda"),
                  dB=torch.empty(L.r, L.d_out, dtype=torch.float32, device="cuda"))
        items.append(it)
        flops += step_flops(M, L.d_in, L.d_out, L.r)
    # one workspace per direction, sized for the largest projection (calls are stream-ordered)
    wsf = max(lb.qlora_linear_fwd_workspace(M, L.d_out, L.d_in, L.r) for L in wl.layers)
    wsb = max(lb.qlora_linear_bwd_workspace(M, L.d_out, L.d_in, L.r) for L in wl.layers)
    ws_f = torch.empty(max(1, wsf), dtype=torch.uint8, device="cuda")
    ws_b = torch.empty(max(1, wsb), dtype=torch.uint8, device="cuda")

    def layer():
        for it in items:
            q.qlora_linear_fwd(it["X"], it["T"], it["A"], it["B"], it["s"], Y=it["Y"], XA_save=it["XA"], ws=ws_f)
            q.qlora_linear_bwd(it["X"], it["dY"], it["T"], it["A"], it["B"], it["s"], XA=it["XA"], dX=it["dX"],
                               dA=it["dA"], dB=it["dB"], ws=ws_b)

    reps = max(3, min(args.steps, 10))
    # SM clocks and clock-event reasons while the layer replays (seconds of tensor work
    # right after the memory-bound components: the power cap may lower the clock here)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    clocks.mark_begin()
    ms = _time_graph(layer, reps, flush, stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    clk = clocks.stop()
    kern = _kernel_ms(KERNELS, layer, 2, flush)
    assert q.qlora_get_device_status() == q.QLORA_OK
    tf = flops / (ms / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    # the oracle on the host, a bounded sample: the k projection (1024 x 8192, r = 64),
    # dequantised in C; Y and dX on 128 token rows and dA, dB over all 4096 tokens in fp64
    import numpy as np
    import oracle
    li = [l.name for l in wl.layers].index("k")
    L = wl.layers[li]
    it = items[li]
    Wsrc = si.layer_inputs(wl, li, device="cpu", M=0)["W"].numpy()
    ref = oracle.quantize(Wsrc)
    f64 = lambda t: t.to(torch.float64).cpu().numpy()
    Xn, dYn, An, Bn = f64(it["X"]), f64(it["dY"]), f64(it["A"]), f64(it["B"])
    rows = np.random.default_rng(5).choice(M, 128, replace=False)

    def cpu_sample():
        Wh = oracle.bf16_bits_to_f32(oracle.dequant(ref)).reshape(L.d_out, L.d_in).astype(np.float64)
        oracle.linear_fwd(Xn[rows], Wh, An, Bn, L.s)
        oracle.linear_bwd(Xn[rows], dYn[rows], Wh, An, Bn, L.s)
        oracle.adapter_grads(Xn, dYn, An, Bn, L.s)
    t_c, creps = _host_time(cpu_sample, target_s=3.0, max_reps=5)
    K, N, r = L.d_in, L.d_out, L.r
    sample_flops = 4.0 * 128 * K * N + 6.0 * 128 * r * (K + N) + 6.0 * M * r * (K + N)
    cpu = {"value": round(sample_flops / t_c / 1e12, 6), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
           "sample": f"k projection: dequantise, Y and dX on 128 of the 4096 tokens, dA and dB on all, fp64; "
                     f"{creps} calls; the rate extrapolates to the layer"}
    del items, ws_f, ws_b
    torch.cuda.empty_cache()
    return {"workload": "70B-like layer: q,o 8192x8192; k,v 1024x8192; gate,up 28672x8192; down 8192x28672; "
                        "r=64, alpha=128 on all seven; M=4096; fwd+bwd of each, CUDA graph replay, L2 flushed",
            "flops_per_step": flops, "ms_per_step": round(ms, 4), "TFLOP/s": round(tf, 1),
            "frac_of_sustained_bf16": round(tf / peak, 4), "reps": reps, "clocks": clk, "kernels": kern,
            "cpu_baseline": cpu}


# ------------------------------------------------------------------ CPU oracle
def _oracle_problem(M_sample):
    import numpy as np
    import torch
    import oracle
    import synth_inputs as si
    wl = si.workload("l4096")
    L = wl.layers[0]
    inp = si.layer_inputs(wl, 0, device="cpu")
    ref = oracle.quantize(inp["W"].numpy())
    f64 = lambda t: t.to(torch.float64).numpy()
    return (wl, L, ref, f64(inp["X"][:M_sample]), f64(inp["dY"][:M_sample]), f64(inp["A"]), f64(inp["B"]))


def _oracle_step(L, ref, X, dY, A, B):
    import oracle
    Wh = oracle.bf16_bits_to_f32(oracle.dequant(ref)).reshape(L.d_out, L.d_in).astype("float64")
    Y = oracle.linear_fwd(X, Wh, A, B, L.s)
    dX, dA, dB = oracle.linear_bwd(X, dY, Wh, A, B, L.s)
    return Y, dX, dA, dB


def _cores():
    import oracle
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        blas = os.cpu_count()
    return max(oracle.threads(), blas)


def cpu_baseline(M_sample=512, target_s=10.0):
    wl, L, ref, X, dY, A, B = _oracle_problem(M_sample)
    t0 = time.perf_counter()
    _oracle_step(L, ref, X, dY, A, B)
    one = time.perf_counter() - t0
    reps = max(1, min(20, int(target_s / max(one, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(reps):
        _oracle_step(L, ref, X, dY, A, B)
    el = time.perf_counter() - t0
    flops = step_flops(M_sample, L.d_in, L.d_out, L.r)
    return {"value": round(reps * flops / el / 1e12, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"{M_sample} of the 4096 tokens, full 4096x4096 weight: oracle dequant (C) + fp64 "
                      f"fwd + bwd products (numpy), {reps} steps, {el:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl, L, ref, X, dY, A, B = _oracle_problem(args.cpu_sample_tokens)
    for _ in range(args.warmup):
        _oracle_step(L, ref, X, dY, A, B)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(L, ref, X, dY, A, B)
    el = time.perf_counter() - t0
    flops = step_flops(args.cpu_sample_tokens, L.d_in, L.d_out, L.r)
    value = args.steps * flops / el / 1e12
    sample = (f"{args.cpu_sample_tokens} of the 4096 tokens per step, full 4096x4096 weight: oracle dequant (C) "
              f"+ fp64 fwd + bwd products (numpy)")
    n = int(os.environ.get("WORLD_SIZE", "1"))
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": "QLoRA linear 4096x4096, M=4096 tokens, r=64, alpha=128 (s=2); bounded sample "
                                   "per step", "sample_tokens": args.cpu_sample_tokens},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_decode_profile(M, reps=3):
    """A small case for an ncu capture of the decode path: one Llama-7B block at M tokens,
    forward only, through one grouped call, `reps` times with the L2 flushed before each."""
    import torch
    import bit_nf4_quantized_double_b200 as q
    import synth_inputs as si
    wl = si.workload("decode7b", M=M)
    items = []
    for li, L in enumerate(wl.layers):
        inp = si.layer_inputs(wl, li, device="cuda")
        items.append({"X": inp["X"], "W": q.qlora_nf4_quantize(inp["W"]), "A": inp.get("A"), "B": inp.get("B"),
                      "s": L.s, "Y": torch.empty(M, L.d_out, dtype=torch.bfloat16, device="cuda")})
        del inp
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    for _ in range(reps):
        l2_flush(flush)
        q.qlora_linear_fwd_grouped(items)
    torch.cuda.synchronize()
    assert q.qlora_get_device_status() == q.QLORA_OK
    print(json.dumps({"decode_profile": {"M": M, "reps": reps}}), flush=True)


def run_profile_case(name, reps=3):
    """Small cases for ncu captures of one kernel each (a few launches, inputs above the L2
    size, the L2 flushed before each launch): decode1 / decode16 (the decode block's grouped
    forward), layer (one Llama-7B layer quantised and dequantised by the grouped calls),
    adamw (64 M adapter parameters), merge (the 4096^2 adapter merge), fmt4 (the three
    4-bit reference formats on 2^26 weights), l4096 (one fwd + bwd step of the headline layer),
    l4096fused (the same step through the fused dequant-GEMM kernels)."""
    import torch
    import bit_nf4_quantized_double_b200 as q
    import synth_inputs as si
    if name.startswith("decode"):
        run_decode_profile(int(name[len("decode"):]), reps)
        return
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    if name == "layer":
        wl = si.workload("llama7b", n_layers=1)
        Ws = [si.layer_inputs(wl, li, device="cuda")["W"] for li in range(7)]
        Ts = q.qlora_nf4_quantize_grouped(Ws)
        outs = [torch.empty(W.shape, dtype=torch.bfloat16, device="cuda") for W in Ws]
        for _ in range(reps):
            l2_flush(flush)
            q.qlora_nf4_quantize_grouped(Ws, outs=Ts)
            l2_flush(flush)
            q.qlora_nf4_dequant_grouped(Ts, outs=outs)
    elif name == "adamw":
        n = 64 << 20
        theta, g, m, v = (torch.zeros(n, device="cuda") for _ in range(4))
        tb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        for t in range(1, reps + 1):
            l2_flush(flush)
            q.qlora_adamw_step(theta, g, m, v, t, 1e-3, theta_bf16=tb)
    elif name == "merge":
        wl = si.workload("l4096")
        L = wl.layers[0]
        inp = si.layer_inputs(wl, 0, device="cuda")
        t = q.qlora_nf4_quantize(inp["W"])
        for _ in range(reps):
            l2_flush(flush)
            q.qlora_nf4_merge_adapter(t, inp["A"], inp["B"], L.s)
    elif name == "fmt4":
        W = si.normal((1 << 26,), 0.02, seed=77, device="cuda")
        for fmt in ("int4", "fp4_e2m1", "fp4_e3m0"):
            l2_flush(flush)
            codes, absmax = q.qlora_fmt4_quantize(W, fmt)
            l2_flush(flush)
            q.qlora_fmt4_dequant(codes, absmax, W.numel(), fmt)
    elif name == "l4096fused":
        wl, L, inp = headline_inputs(0)
        t = q.qlora_nf4_quantize(inp["W"])
        q.lib().qlora_linear_set_pair_min_m(2 ** 63 - 1)
        for _ in range(reps):
            l2_flush(flush)
            Y, XA = q.qlora_linear_fwd(inp["X"], t, inp["A"], inp["B"], L.s)
            q.qlora_linear_bwd(inp["X"], inp["dY"], t, inp["A"], inp["B"], L.s, XA=XA)
        q.lib().qlora_linear_set_pair_min_m(DEFAULT_PAIR_MIN_M)
    elif name == "l4096":
        wl, L, inp = headline_inputs(0)
        t = q.qlora_nf4_quantize(inp["W"])
        for _ in range(reps):
            l2_flush(flush)
            Y, XA = q.qlora_linear_fwd(inp["X"], t, inp["A"], inp["B"], L.s)
            q.qlora_linear_bwd(inp["X"], inp["dY"], t, inp["A"], inp["B"], L.s, XA=XA)
    else:
        raise SystemExit(f"unknown profile case {name}")
    torch.cuda.synchronize()
    assert q.qlora_get_device_status() == q.QLORA_OK
    print(json.dumps({"profile_case": name, "reps": reps}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep-layers", type=int, default=32)
    ap.add_argument("--cpu-sample-tokens", type=int, default=512)
    ap.add_argument("--no-graph", action="store_true", help="launch every step eagerly instead of replaying a CUDA graph")
    ap.add_argument("--decode-profile", type=int, default=0, metavar="M",
                    help="only run the decode block at M tokens three times (a small case for ncu) and exit")
    ap.add_argument("--profile-case", default="", metavar="NAME",
                    help="only run a small case for an ncu capture (decode1, decode16, layer, adamw, merge, fmt4, "
                         "l4096) and exit")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case)
        return
    if args.decode_profile:
        run_decode_profile(args.decode_profile)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return
    peaks, kind = load_peaks()
    run_ours(args, peaks, kind)


if __name__ == "__main__":
    main()
