"""Benchmark of the blockwise-FP8 linear layer on B200.

One step = the full hot path over one batch: the four linears of one
Qwen3-1.7B-like transformer layer (QKV 2048->4096, O 2048->2048, gate/up
2048->12288, down 6144->2048) at M = 16384 tokens, each with
  forward  quantize_act_dual(X) (row groups for the forward, token groups for
           wgrad, one read of X), quantize_weight(W), GEMM  Y = X W^T
  dgrad    quantize_act_dual(dY) (row groups for dgrad, token groups for
           wgrad),                                GEMM dX = dY W   (W^T read in place)
  wgrad                                           GEMM dW = dY^T X
i.e. 12 quantizer and 12 GEMM launches, 4.948 TFLOP of blockwise-FP8 GEMM.
With --separate-quant the activation layouts come from quantize_act and
quantize_act_t in separate launches (20 quantizer launches).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--scale fp32|ue8m0]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample
    python bench.py --case all|NAME        # single kernels, L2 flushed

Metric: blockwise-FP8 GEMM TFLOP/s of the whole step (GEMM FLOPs / step time
including the quantizers), with the GEMM kernel's roofline (TFLOP/s vs the
FP8 dense peak) and the quantizers' GB/s vs HBM in the same JSON line.
The timed region is one replay of a CUDA graph holding the K steps (L2
flush, an event pair around each step and around each launch); --no-graph
issues the same sequence eagerly.
Inputs are synthetic (seeded), resident in HBM for `value`; `e2e` repeats the
step with the inputs copied from pinned host memory and the outputs copied
back inside the timed region.  Multi-GPU: one process per GPU, each a replica
on its own token batch (data-parallel shards, no collective on the data
path): weak scaling, value summed over ranks, time = max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from blockwise_fp8_linear_fp8bq_b200 import synth  # noqa: E402

M_TOKENS = 16384
METRIC = "blockwise-FP8 GEMM TFLOP/s & % FP8 peak; quantizer GB/s & % HBM (1 B200)"
WORKLOAD = ("qwen3-1.7b layer linears (qkv 2048x4096, o 2048x2048, gate_up 2048x12288, "
            "down 6144x2048) fwd+dgrad+wgrad, M=16384 tokens")
FP8_OVER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor ratio (4.5 / 2.25 PFLOP/s)
FP8_FLOP_PER_SM_CYCLE = 16384  # dense FP8 tensor-core rate of one SM per clock


def linears(M=M_TOKENS):
    return synth.layer_linears(M)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        out = {"hbm_gbs": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
               "bf16_sustained": float(p["bf16_tflops_sustained"]), "source": "measured"}
        # the SM clock the burst peak was measured at, where the file gives one
        for key in ("bf16_sm_mhz", "bf16_clock_mhz", "sm_mhz_burst", "burst_sm_mhz"):
            if isinstance(p.get(key), (int, float)):
                out["sm_mhz"] = float(p[key])
                break
        out["keys"] = sorted(p.keys())
        return out
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every
    5 ms in a background thread while the timed region runs.  Read-only: it
    changes no GPU setting."""

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown")]

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []
        self.reasons = set()
        self.ok = False

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            p = torch.cuda.get_device_properties(self.device)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            self.h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
            return
        self.stop_flag = threading.Event()

        def loop():
            nv = self.nv
            masks = [(n, getattr(nv, c, 0)) for n, c in self.REASONS]
            while not self.stop_flag.is_set():
                try:
                    self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    for n, m in masks:
                        if m and (r & m):
                            self.reasons.add(n)
                except Exception:
                    pass
                self.stop_flag.wait(0.005)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self):
        if not self.ok:
            return None
        self.stop_flag.set()
        self.thread.join()
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(self.samples), "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# -------------------------------------------------------------------- ours --
class LayerStep:
    """Device buffers and the launch sequence of one step."""

    def __init__(self, fp, fmt, seed, device, only=None, dual=True, mx=False, split=True, group=True):
        self.fp = fp
        self.fmt = fmt
        self.dual = dual
        # the forward's input (both layouts) and the weight in one grouped launch
        self.group = group and dual and not mx
        # GEMM workspace: the last round of output tiles may be split along K
        self.ws = fp.gemm_workspace(device) if split else None
        self.mx = mx  # 1x32 MX blocks (UE8M0) on every operand; weights quantized in both orientations
        self.items = []
        sdt = torch.float32 if fmt == fp.SCALE_FP32 else torch.uint8
        e4 = torch.float8_e4m3fn
        g = 32 if mx else 128
        for i, lin in enumerate(linears()):
            if only is not None and lin.name not in only:
                continue
            M, K, N = lin.M, lin.K, lin.N
            s = seed + 100 * i
            it = dict(lin=lin,
                      x=lin.x(s, device=device), w=lin.w(s, device=device), dy=lin.dy(s, device=device),
                      qx=torch.empty(M, K, dtype=e4, device=device),
                      sx=torch.empty(K // g, fp.row_scale_ld(M), dtype=sdt, device=device),
                      qw=torch.empty(N, K, dtype=e4, device=device),
                      sw=(torch.empty(K // 32, fp.row_scale_ld(N), dtype=sdt, device=device) if mx else
                          torch.empty(K // 128, (N + 127) // 128, dtype=sdt, device=device)),
                      qd=torch.empty(M, N, dtype=e4, device=device),
                      sd=torch.empty(N // g, fp.row_scale_ld(M), dtype=sdt, device=device),
                      qdt=torch.empty(N, M, dtype=e4, device=device),
                      sdt=torch.empty(M // g, fp.row_scale_ld(N), dtype=sdt, device=device),
                      qxt=torch.empty(K, M, dtype=e4, device=device),
                      sxt=torch.empty(M // g, fp.row_scale_ld(K), dtype=sdt, device=device),
                      y=torch.empty(M, N, dtype=torch.bfloat16, device=device),
                      dx=torch.empty(M, K, dtype=torch.bfloat16, device=device),
                      dw=torch.empty(N, K, dtype=torch.bfloat16, device=device))
            if mx:  # W^T codes grouped along N, for dgrad
                it["qwt"] = torch.empty(K, N, dtype=e4, device=device)
                it["swt"] = torch.empty(N // 32, fp.row_scale_ld(K), dtype=sdt, device=device)
            self.items.append(it)

    # algorithmic bytes of each quantizer launch (bf16 read, e4m3 write, scales)
    def quant_bytes(self):
        sb = 4 if self.fmt == self.fp.SCALE_FP32 else 1
        tot = 0
        if self.mx:
            for it in self.items:
                lin = it["lin"]
                M, K, N = lin.M, lin.K, lin.N
                tot += 2 * (N * K * 3 + N * K // 32)  # W in both orientations
                tot += M * K * 4 + 2 * M * K // 32     # dual(X)
                tot += M * N * 4 + 2 * M * N // 32     # dual(dY)
            return tot
        for it in self.items:
            lin = it["lin"]
            M, K, N = lin.M, lin.K, lin.N
            tot += N * K * 3 + (K // 128) * ((N + 127) // 128) * sb  # weight(W)
            if self.dual:
                # one bf16 read, both code layouts written
                tot += M * K * 4 + ((K // 128) * M + (M // 128) * K) * sb  # dual(X)
                tot += M * N * 4 + ((N // 128) * M + (M // 128) * N) * sb  # dual(dY)
            else:
                tot += M * K * 3 + (K // 128) * M * sb          # act(X)
                tot += M * N * 3 + (N // 128) * M * sb          # act(dY)
                tot += M * N * 3 + (M // 128) * N * sb          # act_t(dY)
                tot += M * K * 3 + (M // 128) * K * sb          # act_t(X)
        return tot

    def gemm_flops(self):
        return sum(3 * it["lin"].flops for it in self.items)

    def launches(self):
        if self.mx:
            return 7 * len(self.items)
        if self.group:
            return 5 * len(self.items)
        return (6 if self.dual else 8) * len(self.items)

    def run(self, ev=None, external=False):
        """Issue the step on the current stream.  With `ev` (a list), record a
        CUDA event pair around every launch: ev.append((kind, start, end));
        `external` makes them event-record nodes when captured in a graph."""
        fp, f = self.fp, self.fmt
        # one event between consecutive launches: the end of launch i is the
        # start of launch i + 1 (a pair per launch would put two event-record
        # nodes, and their latency, between every two kernels)
        prev = [None]
        if ev is not None:
            prev[0] = torch.cuda.Event(enable_timing=True, external=external)
            prev[0].record()

        def timed(kind, fn):
            if ev is None:
                fn()
                return
            fn()
            b = torch.cuda.Event(enable_timing=True, external=external)
            b.record()
            ev.append((kind, prev[0], b))
            prev[0] = b

        if self.mx:
            for it in self.items:
                timed("quant", lambda: fp.quantize_act_dual_mx(it["x"], it["qx"], it["sx"], it["qxt"], it["sxt"]))
                timed("quant", lambda: fp.quantize_act_mx(it["w"], it["qw"], it["sw"]))
                timed("quant", lambda: fp.quantize_act_t_mx(it["w"], it["qwt"], it["swt"]))
                timed("gemm", lambda: fp.gemm(fp.mx_operand(it["qx"], it["sx"]), fp.mx_operand(it["qw"], it["sw"]),
                                              it["y"], workspace=self.ws))
                timed("quant", lambda: fp.quantize_act_dual_mx(it["dy"], it["qd"], it["sd"], it["qdt"], it["sdt"]))
                timed("gemm", lambda: fp.gemm(fp.mx_operand(it["qd"], it["sd"]), fp.mx_operand(it["qwt"], it["swt"]),
                                              it["dx"], workspace=self.ws))
                timed("gemm", lambda: fp.gemm(fp.mx_operand(it["qdt"], it["sdt"]),
                                              fp.mx_operand(it["qxt"], it["sxt"]), it["dw"], workspace=self.ws))
            return
        for it in self.items:
            if self.group:
                timed("quant", lambda: fp.quantize_group(
                    [("dual", it["x"], (it["qx"], it["sx"], it["qxt"], it["sxt"])), ("weight", it["w"], (it["qw"], it["sw"]))],
                    f))
            elif self.dual:
                timed("quant", lambda: fp.quantize_act_dual(it["x"], f, it["qx"], it["sx"], it["qxt"], it["sxt"]))
            else:
                timed("quant", lambda: fp.quantize_act(it["x"], f, it["qx"], it["sx"]))
            if not self.group:
                timed("quant", lambda: fp.quantize_weight(it["w"], f, it["qw"], it["sw"]))
            timed("gemm", lambda: fp.gemm(fp.row_operand(it["qx"], it["sx"], f),
                                          fp.block_operand(it["qw"], it["sw"], f), it["y"], workspace=self.ws))
            if self.dual:
                timed("quant", lambda: fp.quantize_act_dual(it["dy"], f, it["qd"], it["sd"], it["qdt"], it["sdt"]))
            else:
                timed("quant", lambda: fp.quantize_act(it["dy"], f, it["qd"], it["sd"]))
            timed("gemm", lambda: fp.gemm(fp.row_operand(it["qd"], it["sd"], f),
                                          fp.block_operand(it["qw"], it["sw"], f, transposed=True), it["dx"],
                                          workspace=self.ws))
            if not self.dual:
                timed("quant", lambda: fp.quantize_act_t(it["dy"], f, it["qdt"], it["sdt"]))
                timed("quant", lambda: fp.quantize_act_t(it["x"], f, it["qxt"], it["sxt"]))
            timed("gemm", lambda: fp.gemm(fp.row_operand(it["qdt"], it["sdt"], f),
                                          fp.row_operand(it["qxt"], it["sxt"], f), it["dw"], workspace=self.ws))


def l2_flush(buf):
    buf.zero_()


def measure_step(args, fp, step, dev, dist, flush):
    """Warm up, then time `args.steps` steps of `step` as two CUDA graphs (see
    below).  Returns step / kernel-split times, the NVML clock records of both
    replays, and the SM clock the GEMM kernels themselves counted."""
    for _ in range(args.warmup):
        step.run()
    fp.check()

    # Two graphs of the same K steps, each replayed once.  The timed region
    # (`value`) holds per step the L2 flush and one event pair around the
    # step: nothing sits between the step's kernels.  The kernel split
    # (`roofline`, `gemm`, `quantizers`) comes from the other graph, replayed
    # first, which adds an event between every two launches; those
    # event-record nodes order the kernels strictly, so its step runs a few
    # percent longer.  The host's Python and ctypes work is outside both.  (--no-graph
    # issues the same two sequences eagerly.)  The GEMMs of the kernel-split
    # graph also add up their SM cycles and nanoseconds (clock counters): the
    # clock the tensor cores ran at, which NVML's 5 ms samples do not resolve.
    step_events, split_step_events, kernel_events = [], [], []
    clk = torch.zeros(2, dtype=torch.int64, device=dev)

    def timed_steps(per_launch, external):
        fp.set_clock_counters(clk if per_launch else None)
        for _ in range(args.steps):
            l2_flush(flush)
            a = torch.cuda.Event(enable_timing=True, external=external)
            b = torch.cuda.Event(enable_timing=True, external=external)
            a.record()
            step.run(kernel_events if per_launch else None, external=external)
            b.record()
            (split_step_events if per_launch else step_events).append((a, b))
        fp.set_clock_counters(None)

    graphs = {}
    if not args.no_graph:
        torch.cuda.synchronize()
        for per_launch in (False, True):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                timed_steps(per_launch, True)
            graphs[per_launch] = g
        # no warm-up replay: the events are recorded by the graphs' own
        # nodes, so a graph's first-launch cost falls outside them, and an
        # extra 30-step replay would push the GPU into its power cap first
        torch.cuda.synchronize()

    def replay(per_launch):
        sampler = ClockSampler(dev)
        sampler.start()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        if graphs:
            graphs[per_launch].replay()
        else:
            timed_steps(per_launch, False)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        return sampler.stop()

    clk.zero_()
    clocks_split = replay(True)
    cyc, ns = (int(v) for v in clk.tolist())
    # idle between the two replays, so that the second starts from the power
    # state the first did rather than from the end of a 70 ms burst
    time.sleep(2.0)
    clocks = replay(False)
    fp.check()
    graphs.clear()
    return dict(step_ms=sum(a.elapsed_time(b) for a, b in step_events),
                split_step_ms=sum(a.elapsed_time(b) for a, b in split_step_events),
                gemm_ms=sum(a.elapsed_time(b) for k, a, b in kernel_events if k == "gemm"),
                quant_ms=sum(a.elapsed_time(b) for k, a, b in kernel_events if k == "quant"),
                clocks=clocks, clocks_split=clocks_split,
                gemm_kernel_mhz=(1e3 * cyc / ns) if ns > 0 else None,
                gemm_launches=len([1 for k, _, _ in kernel_events if k == "gemm"]),
                quant_launches=len([1 for k, _, _ in kernel_events if k == "quant"]))


def run_ours(args, rank, world, dist):
    import blockwise_fp8_linear_fp8bq_b200 as fp
    fp.lib()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    fmt = fp.SCALE_FP32 if args.scale == "fp32" else fp.SCALE_UE8M0
    step = LayerStep(fp, fmt, seed=1000 * (rank + 1), device=dev, dual=not args.separate_quant,
                     mx=args.scale == "mx", split=not args.no_split, group=not args.no_group_quant)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    m = measure_step(args, fp, step, dev, dist, flush)
    step_ms, split_step_ms, gemm_ms, quant_ms = m["step_ms"], m["split_step_ms"], m["gemm_ms"], m["quant_ms"]
    clocks, clocks_split = m["clocks"], m["clocks_split"]

    # end to end: every step's inputs (X, W, dY of the four linears) copied
    # from pinned host memory and its outputs (Y, dX, dW) copied back inside
    # the timed region.  One copy stream per PCIe direction: step s+1's
    # inputs travel while step s computes and step s-1's outputs travel back.
    # The device inputs and outputs are double-buffered for that; the codes
    # and scales are not (the step's launches stay in order on one stream).
    e2e = None
    if not args.no_e2e:
        in_keys, out_keys = ("x", "w", "dy"), ("y", "dx", "dw")
        keys = [(i, k) for i in range(len(step.items)) for k in in_keys + out_keys]
        dev_bufs = [{(i, k): step.items[i][k] for i, k in keys},
                    {(i, k): torch.empty_like(step.items[i][k]) for i, k in keys}]
        host_in = {(i, k): step.items[i][k].to("cpu").pin_memory()
                   for i in range(len(step.items)) for k in in_keys}
        host_out = {(i, k): torch.empty_like(step.items[i][k], device="cpu").pin_memory()
                    for i in range(len(step.items)) for k in out_keys}
        bi = sum(h.numel() * h.element_size() for h in host_in.values())
        bo = sum(h.numel() * h.element_size() for h in host_out.values())
        cs = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

        def pipeline(n, start_ev):
            comp, out = [], []
            for s in range(n):
                b = dev_bufs[s % 2]
                ev_in = torch.cuda.Event()
                with torch.cuda.stream(s_in):
                    s_in.wait_event(start_ev)
                    if s >= 2:
                        s_in.wait_event(comp[s - 2])  # step s-2 done reading these inputs
                    for (i, k), h in host_in.items():
                        b[(i, k)].copy_(h, non_blocking=True)
                    ev_in.record(s_in)
                cs.wait_event(ev_in)
                if s >= 2:
                    cs.wait_event(out[s - 2])  # step s-2's outputs are back on the host
                for (i, k), t in b.items():
                    step.items[i][k] = t
                step.run()
                comp.append(torch.cuda.Event())
                comp[-1].record(cs)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(comp[-1])
                    for (i, k), h in host_out.items():
                        h.copy_(b[(i, k)], non_blocking=True)
                    out.append(torch.cuda.Event())
                    out[-1].record(s_out)
            cs.wait_event(out[-1])

        e2e_steps = max(2, min(args.steps, 10))
        ev = torch.cuda.Event()
        ev.record(cs)
        pipeline(2, ev)  # warm-up of the copy path
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(cs)
        pipeline(e2e_steps, t0)
        t1.record(cs)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        for (i, k), t in dev_bufs[0].items():
            step.items[i][k] = t
        e2e_ms = t0.elapsed_time(t1) / e2e_steps
        fp.check()
        e2e = {"ms_per_step": e2e_ms, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": e2e_steps,
               "copies": "one stream per PCIe direction, overlapped with the step's kernels"}

    out = dict(step_ms=step_ms, split_step_ms=split_step_ms, gemm_ms=gemm_ms, quant_ms=quant_ms,
               clocks=clocks, clocks_split=clocks_split, e2e=e2e, gemm_kernel_mhz=m["gemm_kernel_mhz"],
               flops=step.gemm_flops(), qbytes=step.quant_bytes(), launches=step.launches() * args.steps,
               gemm_launches=m["gemm_launches"], quant_launches=m["quant_launches"])
    extras = world == 1 and args.scale == "ue8m0"
    # the same step with FP32 scales (the DeepSeek-V3-style promotion path),
    # measured the same way, as a sub-record of the default line
    if extras and not args.no_fp32_record:
        step32 = LayerStep(fp, fp.SCALE_FP32, seed=1000 * (rank + 1), device=dev, dual=not args.separate_quant,
                           split=not args.no_split, group=not args.no_group_quant)
        time.sleep(2.0)
        m32 = measure_step(args, fp, step32, dev, dist, flush)
        out["fp32"] = dict(m32, flops=step32.gemm_flops(), qbytes=step32.quant_bytes())
        del step32
        torch.cuda.empty_cache()
    # the 28-layer sweep plus the LM head, end to end (quantizers + GEMMs)
    if extras and not args.no_sweep:
        time.sleep(2.0)
        out["sweep"] = run_sweep(args, fp, step, dev, flush)
    if extras:
        out["fp8_ceiling"] = fp8_cublas_ceiling(dev)
    return out


# ------------------------------------------------------------ the sweep --
SWEEP_LAYERS = 28


def sweep_flops(M=M_TOKENS):
    return SWEEP_LAYERS * sum(3 * lin.flops for lin in linears(M)) + synth.LM_HEAD.flops


def run_sweep(args, fp, step, dev, flush, reps=3):
    """The full 28-layer linear sweep with an untied LM head: per layer the
    four linears' forward, dgrad and wgrad with their quantizers (each layer
    its own seeded inputs X, W, dY), then the LM head's weight and input
    quantization and its forward GEMM [16384 x 2048] . [151936 x 2048]^T.
    End to end on the device (quantizers + GEMMs, 562 launches), one CUDA
    graph replayed `reps` times after an L2 flush each; the LM head's output
    is then checked on sampled rows, columns and elements."""
    fmt = step.fmt
    per_layer = []
    for layer in range(1, SWEEP_LAYERS):
        bufs = []
        for i, it in enumerate(step.items):
            lin = it["lin"]
            s = 90000 + 1000 * layer + 100 * i
            bufs.append(dict(x=lin.x(s, device=dev), w=lin.w(s, device=dev), dy=lin.dy(s, device=dev)))
        per_layer.append(bufs)
    per_layer.insert(0, [dict(x=it["x"], w=it["w"], dy=it["dy"]) for it in step.items])
    lm = synth.LM_HEAD
    x_lm, w_lm = lm.x(95000, device=dev), lm.w(95000, device=dev)
    sdt = torch.float32 if fmt == fp.SCALE_FP32 else torch.uint8
    qx_lm = torch.empty(lm.M, lm.K, dtype=torch.float8_e4m3fn, device=dev)
    sx_lm = torch.empty(lm.K // 128, fp.row_scale_ld(lm.M), dtype=sdt, device=dev)
    qw_lm = torch.empty(lm.N, lm.K, dtype=torch.float8_e4m3fn, device=dev)
    sw_lm = torch.empty(lm.K // 128, (lm.N + 127) // 128, dtype=sdt, device=dev)
    y_lm = torch.empty(lm.M, lm.N, dtype=torch.bfloat16, device=dev)
    A_lm, B_lm = fp.row_operand(qx_lm, sx_lm, fmt), fp.block_operand(qw_lm, sw_lm, fmt)

    def one_sweep():
        for bufs in per_layer:
            for it, b in zip(step.items, bufs):
                it["x"], it["w"], it["dy"] = b["x"], b["w"], b["dy"]
            step.run()
        fp.quantize_group([("act", x_lm, (qx_lm, sx_lm)), ("weight", w_lm, (qw_lm, sw_lm))], fmt)
        fp.gemm(A_lm, B_lm, y_lm, workspace=step.ws)

    one_sweep()  # warm-up, and every operand produced once
    fp.check()
    events = []
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        l2_flush(flush)
        a = torch.cuda.Event(enable_timing=True, external=True)
        b = torch.cuda.Event(enable_timing=True, external=True)
        a.record()
        one_sweep()
        b.record()
        events.append((a, b))
    torch.cuda.synchronize()
    times = []
    sampler = ClockSampler(dev)
    sampler.start()
    for _ in range(reps):
        g.replay()
        torch.cuda.synchronize()
        times.append(events[0][0].elapsed_time(events[0][1]))
    clocks = sampler.stop()
    fp.check()
    del g
    # restore the layer-0 inputs the step buffers held
    for it, b in zip(step.items, per_layer[0]):
        it["x"], it["w"], it["dy"] = b["x"], b["w"], b["dy"]
    check = lm_head_check(fp, fmt, qx_lm, sx_lm, qw_lm, sw_lm, y_lm)
    ms = statistics.median(times)
    flops = sweep_flops()
    del per_layer, x_lm, w_lm, y_lm
    torch.cuda.empty_cache()
    return {"layers": SWEEP_LAYERS, "ms": ms, "ms_all": times, "tflops": flops / (ms * 1e-3) / 1e12,
            "flops": flops, "launches": SWEEP_LAYERS * step.launches() + 2, "clocks": clocks,
            "lm_head_check": check,
            "what": "28 layers x (qkv, o, gate_up, down) x (fwd, dgrad, wgrad) with their quantizers at M=16384, "
                    "then the LM head weight + input quantization and forward GEMM; one graph replay per sweep, "
                    "L2 flushed before each"}


def _dequant_rows(q: torch.Tensor, s: torch.Tensor, fmt: int, rows: torch.Tensor) -> torch.Tensor:
    """float64 values of 1x128-group codes q[rows] (scales [K/128][ld])."""
    v = q[rows].float().double()
    sc = s[:, rows].t()
    sc = sc.to(torch.float64) if sc.dtype == torch.float32 else torch.exp2(sc.to(torch.float64) - 127.0)
    return v * sc.repeat_interleave(128, dim=1)


def _dequant_block_rows(q: torch.Tensor, s: torch.Tensor, rows: torch.Tensor) -> torch.Tensor:
    """float64 values of 128x128-block codes q[rows] (scales [K/128][ceil(N/128)])."""
    v = q[rows].float().double()
    sc = s[:, rows // 128].t()
    sc = sc.to(torch.float64) if sc.dtype == torch.float32 else torch.exp2(sc.to(torch.float64) - 127.0)
    return v * sc.repeat_interleave(128, dim=1)


def lm_head_check(fp, fmt, qx, sx, qw, sw, y, nrows=4, ncols=4, nelem=1024, seed=4242):
    """The LM head output against the definition D = deq(A) deq(B)^T in
    float64 (torch on the device), on sampled whole rows, whole columns and
    single elements, with the tests' tolerance: relative Frobenius error
    <= 5e-3 and |diff| <= 1e-2 rms + half a BF16 ulp per element."""
    M, N = y.shape
    dev = y.device
    g = torch.Generator().manual_seed(seed)
    rows = torch.randperm(M, generator=g)[:nrows].tolist() + [M - 1]
    cols = torch.randperm(N, generator=g)[:ncols].tolist() + [N - 1]
    er = torch.randint(0, M, (nelem,), generator=g)
    ec = torch.randint(0, N, (nelem,), generator=g)
    r_t, c_t = torch.tensor(rows, device=dev), torch.tensor(cols, device=dev)
    xa = _dequant_rows(qx, sx, fmt, r_t)
    ref_rows = torch.cat([xa @ _dequant_block_rows(qw, sw, torch.arange(n0, min(n0 + 16384, N), device=dev)).t()
                          for n0 in range(0, N, 16384)], dim=1)
    wb = _dequant_block_rows(qw, sw, c_t)
    ref_cols = torch.cat([_dequant_rows(qx, sx, fmt, torch.arange(m0, min(m0 + 4096, M), device=dev)) @ wb.t()
                          for m0 in range(0, M, 4096)], dim=0)
    er_d, ec_d = er.to(dev), ec.to(dev)
    ref_el = (_dequant_rows(qx, sx, fmt, er_d) * _dequant_block_rows(qw, sw, ec_d)).sum(dim=1)
    got = torch.cat([y[r_t].double().ravel(), y[:, c_t].double().ravel(), y[er_d, ec_d].double()])
    ref = torch.cat([ref_rows.ravel(), ref_cols.ravel(), ref_el])
    diff = got - ref
    rel = float(diff.norm() / ref.norm())
    rms = float(ref.pow(2).mean().sqrt())
    _, e = torch.frexp(ref.abs())
    half_ulp = torch.ldexp(torch.ones_like(ref), (e - 9).to(torch.int32)) * (ref != 0)
    excess = float((diff.abs() - (1e-2 * rms + half_ulp)).max())
    return {"ok": rel <= 5e-3 and excess <= 0.0, "rel_frobenius": rel, "max_excess_over_bound": excess,
            "values_checked": int(ref.numel()), "how": "sampled rows, columns and elements vs float64 torch "
            "dequantize-then-matmul on the device"}


def fp8_cublas_ceiling(dev, n=8192, reps=20):
    """A measured FP8 ceiling beside the BF16 x 2 denominator: cuBLASLt's FP8
    GEMM (torch._scaled_mm, E4M3 x E4M3 -> BF16, per-tensor scales) at
    8192^3, timed with CUDA events after an L2 flush each.  A cross-check of
    the denominator only; nothing of the path runs through it."""
    try:
        g = torch.Generator(device=dev).manual_seed(7)
        a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        one = torch.ones((), device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        f = lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            f()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        return {"tflops": 2.0 * n ** 3 / (ms * 1e-3) / 1e12, "ms": ms, "shape": f"{n}^3",
                "what": "torch._scaled_mm (cuBLASLt FP8 e4m3, bf16 out), median of 20 after an L2 flush each"}
    except Exception as exc:  # pragma: no cover - depends on the box's torch build
        return {"unavailable": str(exc)[:200]}


# --------------------------------------------------------- oracle on CPU --
def oracle_format(args):
    """(scale format, group size) of the oracle sample for --scale."""
    return {"fp32": (0, 128), "ue8m0": (1, 128), "mx": (1, 32)}[args.scale]


def oracle_sample(fmt: int = 0, group: int = 128, size: int = 1):
    """Time the CPU oracle on a bounded sample of the step and extrapolate to
    the whole step: quantizers on 256-row slabs of each tensor (x size), GEMMs
    on whole output rows (size x T rows of each forward GEMM, T = oracle
    threads)."""
    import numpy as np
    import oracle
    oracle.build()
    T = oracle.num_threads()
    rows_per_gemm = max(1, T) * size
    q_elems = q_time = 0.0
    g_flops = g_time = 0.0
    full_q_elems = 0
    full_flops = 0
    for i, lin in enumerate(linears()):
        M, K, N = lin.M, lin.K, lin.N
        s = 7000 + 100 * i
        slab = 256 * size
        x = synth.bf16_bits(synth.activations_bf16(slab, K, s))
        w = synth.bf16_bits(synth.weights_bf16(min(N, slab), K, s + 1))
        dy = synth.bf16_bits(synth.grads_bf16(slab, N, s + 2))
        t = time.perf_counter()
        qx, sx = oracle.quantize_act(x, fmt, group)
        if group == 32:  # MX: the weight in both orientations
            qw, sw = oracle.quantize_act(w, fmt, group)
            qwt, swt = oracle.quantize_act_t(synth.bf16_bits(synth.weights_bf16(slab, min(K, slab), s + 5)), fmt, group)
        else:
            qw, sw = oracle.quantize_weight(w, fmt)
        qd, sd = oracle.quantize_act(dy, fmt, group)
        qdt, sdt = oracle.quantize_act_t(dy, fmt, group)
        qxt, sxt = oracle.quantize_act_t(x, fmt, group)
        q_time += time.perf_counter() - t
        q_elems += 2 * x.size + w.size + 2 * dy.size + (slab * min(K, slab) if group == 32 else 0)
        full_q_elems += 2 * M * K + N * K + 2 * M * N + (N * K if group == 32 else 0)
        # GEMMs: T full output rows of each, operands sized to the real contraction
        xa = synth.bf16_bits(synth.activations_bf16(rows_per_gemm, K, s + 3))
        qa, sa = oracle.quantize_act(xa, fmt, group)
        A = oracle.row_operand(qa, sa, fmt, group)
        wb = synth.bf16_bits(synth.weights_bf16(N, K, s + 4))
        if group == 32:
            B = oracle.row_operand(*oracle.quantize_act(wb, fmt, group), fmt, group)
        else:
            B = oracle.block_operand(*oracle.quantize_weight(wb, fmt), fmt)
        t = time.perf_counter()
        oracle.gemm(A, B)
        g_time += time.perf_counter() - t
        g_flops += 2.0 * rows_per_gemm * N * K
        full_flops += 3 * lin.flops
    # dgrad and wgrad rows cost the same per FLOP as forward rows in the oracle
    # (one dequantized multiply-add per term), so the forward sample stands for all three
    step_s = full_q_elems * (q_time / q_elems) + full_flops * (g_time / g_flops)
    sample = (f"4 linears: {slab}-row slabs through the quantizers and {rows_per_gemm} full output rows "
              f"of each forward GEMM; {q_elems / 1e6:.1f} M quantized elements in {q_time:.2f} s, "
              f"{g_flops / 1e9:.2f} GFLOP in {g_time:.2f} s; extrapolated to the full step")
    return {"step_s": step_s, "tflops": full_flops / step_s / 1e12, "cores": T, "sample": sample,
            "sample_s": q_time + g_time}


def run_reference(args, rank, world):
    if rank != 0:
        return
    steps = []
    t_all = time.perf_counter()
    res = None
    for i in range(args.warmup + args.steps):
        res = oracle_sample(*oracle_format(args))
        if i >= args.warmup:
            steps.append(res["step_s"])
    step_s = statistics.median(steps) if steps else res["step_s"]
    flops = sum(3 * lin.flops for lin in linears())
    value = flops / step_s / 1e12
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "scale_format": args.scale, "tokens": M_TOKENS,
                   "parallelism": f"replicas{world}"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": res["cores"], "kind": "oracle",
                         "sample": res["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t_all,
    }
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------ kernel cases --
def case_launchers(step, fp):
    """name -> (kind, algorithmic units, fn) for every launch of the step; units
    are FLOPs for GEMMs and bytes for quantizers."""
    f = fp.SCALE_FP32 if step.fmt == fp.SCALE_FP32 else fp.SCALE_UE8M0
    sb = 4 if f == fp.SCALE_FP32 else 1
    out = {}
    if step.mx:
        for it in step.items:
            lin = it["lin"]
            M, K, N, n = lin.M, lin.K, lin.N, lin.name
            out[f"quant_dual_mx:x:{n}"] = ("quant", M * K * 4 + 2 * M * K // 32, lambda it=it: fp.quantize_act_dual_mx(
                it["x"], it["qx"], it["sx"], it["qxt"], it["sxt"]))
            out[f"quant_dual_mx:dy:{n}"] = ("quant", M * N * 4 + 2 * M * N // 32, lambda it=it: fp.quantize_act_dual_mx(
                it["dy"], it["qd"], it["sd"], it["qdt"], it["sdt"]))
            out[f"quant_act_mx:w:{n}"] = ("quant", N * K * 3 + N * K // 32,
                                          lambda it=it: fp.quantize_act_mx(it["w"], it["qw"], it["sw"]))
            out[f"quant_act_t_mx:w:{n}"] = ("quant", N * K * 3 + N * K // 32,
                                            lambda it=it: fp.quantize_act_t_mx(it["w"], it["qwt"], it["swt"]))
            out[f"gemm_fwd_mx:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
                fp.mx_operand(it["qx"], it["sx"]), fp.mx_operand(it["qw"], it["sw"]), it["y"], workspace=step.ws))
            out[f"gemm_dgrad_mx:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
                fp.mx_operand(it["qd"], it["sd"]), fp.mx_operand(it["qwt"], it["swt"]), it["dx"], workspace=step.ws))
            out[f"gemm_wgrad_mx:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
                fp.mx_operand(it["qdt"], it["sdt"]), fp.mx_operand(it["qxt"], it["sxt"]), it["dw"], workspace=step.ws))
            it["dwf"] = torch.zeros(N, K, dtype=torch.float32, device=it["dw"].device)
            out[f"gemm_wgrad_acc_mx:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
                fp.mx_operand(it["qdt"], it["sdt"]), fp.mx_operand(it["qxt"], it["sxt"]), it["dwf"], accumulate=True))
        return out
    for it in step.items:
        lin = it["lin"]
        M, K, N, n = lin.M, lin.K, lin.N, lin.name
        out[f"quant_act:x:{n}"] = ("quant", M * K * 3 + (K // 128) * M * sb,
                                   lambda it=it: fp.quantize_act(it["x"], f, it["qx"], it["sx"]))
        out[f"quant_weight:{n}"] = ("quant", N * K * 3 + (K // 128) * ((N + 127) // 128) * sb,
                                    lambda it=it: fp.quantize_weight(it["w"], f, it["qw"], it["sw"]))
        out[f"quant_act:dy:{n}"] = ("quant", M * N * 3 + (N // 128) * M * sb,
                                    lambda it=it: fp.quantize_act(it["dy"], f, it["qd"], it["sd"]))
        out[f"quant_act_t:dy:{n}"] = ("quant", M * N * 3 + (M // 128) * N * sb,
                                      lambda it=it: fp.quantize_act_t(it["dy"], f, it["qdt"], it["sdt"]))
        out[f"quant_act_t:x:{n}"] = ("quant", M * K * 3 + (M // 128) * K * sb,
                                     lambda it=it: fp.quantize_act_t(it["x"], f, it["qxt"], it["sxt"]))
        out[f"quant_dual:x:{n}"] = ("quant", M * K * 4 + ((K // 128) * M + (M // 128) * K) * sb,
                                    lambda it=it: fp.quantize_act_dual(it["x"], f, it["qx"], it["sx"], it["qxt"], it["sxt"]))
        out[f"quant_dual:dy:{n}"] = ("quant", M * N * 4 + ((N // 128) * M + (M // 128) * N) * sb,
                                     lambda it=it: fp.quantize_act_dual(it["dy"], f, it["qd"], it["sd"], it["qdt"], it["sdt"]))
        out[f"quant_group:x_w:{n}"] = ("quant", M * K * 4 + ((K // 128) * M + (M // 128) * K) * sb + N * K * 3
                                       + (K // 128) * ((N + 127) // 128) * sb,
                                       lambda it=it: fp.quantize_group(
                                           [("dual", it["x"], (it["qx"], it["sx"], it["qxt"], it["sxt"])),
                                            ("weight", it["w"], (it["qw"], it["sw"]))], f))
        out[f"gemm_fwd:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
            fp.row_operand(it["qx"], it["sx"], f), fp.block_operand(it["qw"], it["sw"], f), it["y"], workspace=step.ws))
        out[f"gemm_dgrad:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
            fp.row_operand(it["qd"], it["sd"], f), fp.block_operand(it["qw"], it["sw"], f, transposed=True), it["dx"],
            workspace=step.ws))
        out[f"gemm_wgrad:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
            fp.row_operand(it["qdt"], it["sdt"], f), fp.row_operand(it["qxt"], it["sxt"], f), it["dw"],
            workspace=step.ws))
        # the same product added into an FP32 master gradient (D += A B^T)
        it["dwf"] = torch.zeros(N, K, dtype=torch.float32, device=it["dw"].device)
        out[f"gemm_wgrad_acc:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
            fp.row_operand(it["qdt"], it["sdt"], f), fp.row_operand(it["qxt"], it["sxt"], f), it["dwf"],
            accumulate=True))
        if n == "down":
            # the down projection's input from the gate/up output [M, 2K] in one
            # pass: SwiGLU, then both code layouts (vs a BF16 h written and read back)
            gen = torch.Generator(device=it["x"].device)
            gen.manual_seed(977)
            it["gu"] = torch.randn(M, 2 * K, generator=gen, device=it["x"].device).to(torch.bfloat16)
            out[f"quant_swiglu:{n}"] = ("quant", M * 2 * K * 2 + 2 * M * K + 2 * (K // 128) * M * sb,
                                        lambda it=it: fp.swiglu_quantize(it["gu"], f))
            # the same with h rounded once from its exact value
            out[f"quant_swiglu_exact:{n}"] = ("quant", M * 2 * K * 2 + 2 * M * K + 2 * (K // 128) * M * sb,
                                              lambda it=it: fp.swiglu_quantize(it["gu"], f, exact=True))
        if n in ("qkv", "gate_up"):
            # the projection's input from RMSNorm in one pass: rstd, h = x * rstd * gamma,
            # both code layouts (vs a BF16 h written and read back)
            it["gamma"] = (1.0 + 0.1 * torch.randn(K, device=it["x"].device)).to(torch.bfloat16)
            it["rstd"] = torch.empty(M, dtype=torch.float32, device=it["x"].device)
            out[f"quant_rmsnorm:{n}"] = ("quant", M * K * 4 + ((K // 128) * M + (M // 128) * K) * sb + 4 * M + 2 * K,
                                         lambda it=it: fp.rmsnorm_quantize(
                                             it["x"], it["gamma"], 1e-6, f,
                                             out=(it["qx"], it["sx"], it["qxt"], it["sxt"], None, it["rstd"])))
            # the same with h rounded once from its exact value (rstd in float64)
            it["rstd64"] = torch.empty(M, dtype=torch.float64, device=it["x"].device)
            out[f"quant_rmsnorm_exact:{n}"] = ("quant", M * K * 4 + ((K // 128) * M + (M // 128) * K) * sb + 8 * M
                                               + 2 * K, lambda it=it: fp.rmsnorm_quantize(
                                                   it["x"], it["gamma"], 1e-6, f, exact=True,
                                                   out=(it["qx"], it["sx"], it["qxt"], it["sxt"], None,
                                                        it["rstd64"])))
        # fused quantize-on-load: BF16 A quantized inside the GEMM
        out[f"gemm_fwd_fused:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
            fp.bf16_operand(it["x"], f), fp.block_operand(it["qw"], it["sw"], f), it["y"], workspace=step.ws))
        out[f"gemm_dgrad_fused:{n}"] = ("gemm", lin.flops, lambda it=it: fp.gemm(
            fp.bf16_operand(it["dy"], f), fp.block_operand(it["qw"], it["sw"], f, transposed=True), it["dx"],
            workspace=step.ws))
    return out


def lm_head_case(fp, fmt, dev, ws):
    """The LM head forward GEMM, [16384 x 2048] . [151936 x 2048]^T (10.2 TFLOP):
    the largest GEMM of the 28-layer sweep, timed as a single kernel."""
    from blockwise_fp8_linear_fp8bq_b200 import synth
    lin = synth.LM_HEAD
    x, w = lin.x(5000, device=dev), lin.w(5000, device=dev)
    qx, sx = fp.quantize_act(x, fmt)
    qw, sw = fp.quantize_weight(w, fmt)
    del x, w
    y = torch.empty(lin.M, lin.N, dtype=torch.bfloat16, device=dev)
    A, B = fp.row_operand(qx, sx, fmt), fp.block_operand(qw, sw, fmt)
    return {"gemm_fwd:lm_head": ("gemm", lin.flops, lambda: fp.gemm(A, B, y, workspace=ws))}


def run_case(args):
    """Time single kernels of the step (L2 flushed before every launch).
    --case all prints one line per kernel; --case NAME runs only that kernel
    (warm-up + steps launches), e.g. for an ncu capture of one kernel."""
    import blockwise_fp8_linear_fp8bq_b200 as fp
    fp.lib()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    fmt = fp.SCALE_FP32 if args.scale == "fp32" else fp.SCALE_UE8M0
    only = None if args.case == "all" else {args.case.split(":")[-1]}
    step = LayerStep(fp, fmt, seed=1000, device=dev, only=only, mx=args.scale == "mx", split=not args.no_split)
    step.run()  # produce every operand once
    torch.cuda.synchronize()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    cases = case_launchers(step, fp)
    if args.scale != "mx" and args.case in ("all", "gemm_fwd:lm_head"):
        cases.update(lm_head_case(fp, fmt, dev, step.ws))
    names = list(cases) if args.case == "all" else [args.case]
    peaks = measured_peaks()
    rows = []
    for name in names:
        if name not in cases:
            raise SystemExit(f"unknown case {name}; one of: {', '.join(cases)}")
        kind, units, fn = cases[name]
        for _ in range(args.warmup):
            fn()
        ts = []
        for _ in range(args.steps):
            l2_flush(flush)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        fp.check()
        ms = statistics.median(ts)
        if kind == "gemm":
            rate = units / (ms * 1e-3) / 1e12
            rows.append({"case": name, "us": ms * 1e3, "tflops": rate,
                         "frac_fp8_burst": rate / (peaks["bf16"] * FP8_OVER_BF16),
                         "frac_nominal_4500": rate / 4500.0})
        else:
            rate = units / (ms * 1e-3) / 1e9
            rows.append({"case": name, "us": ms * 1e3, "gbs": rate, "frac_hbm": rate / peaks["hbm_gbs"]})
    for r in rows:
        print(json.dumps(r), flush=True)


# -------------------------------------------------------------------- main --
def reduce_max(x: float, dist) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--scale", choices=["fp32", "ue8m0", "mx"], default="ue8m0",
                    help="scale format; ue8m0 = the MXFP8 route the pages take on Blackwell (1x128 groups, "
                         "128x128 weight blocks); mx = 1x32 MX blocks on every operand")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps eagerly instead of replaying a CUDA graph of the step")
    ap.add_argument("--separate-quant", action="store_true",
                    help="quantize each activation layout in its own launch instead of the dual pass")
    ap.add_argument("--no-split", action="store_true",
                    help="GEMMs without a workspace: no output tiles split along K")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the 28-layer + LM head sweep record")
    ap.add_argument("--no-group-quant", action="store_true",
                    help="quantize each linear's input and weight in separate launches instead of one grouped launch")
    ap.add_argument("--no-fp32-record", action="store_true", help="skip the FP32-scale sub-record")
    ap.add_argument("--case", default=None,
                    help="time single kernels instead of the step: 'all' or a name such as gemm_fwd:gate_up")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.case:
        run_case(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as td
        from datetime import timedelta
        backend = "gloo" if args.impl == "reference" else "nccl"
        if backend == "nccl":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        td.init_process_group(backend, timeout=timedelta(seconds=120))
        dist = td

    if args.impl == "reference":
        run_reference(args, rank, world)
        if dist is not None:
            dist.destroy_process_group()
        return

    r = run_ours(args, rank, world, dist)
    step_ms = reduce_max(r["step_ms"], dist) / args.steps
    gemm_ms = reduce_max(r["gemm_ms"], dist)
    split_ms = reduce_max(r["split_step_ms"], dist) / args.steps
    quant_ms = reduce_max(r["quant_ms"], dist)
    e2e_ms = reduce_max(r["e2e"]["ms_per_step"], dist) if r["e2e"] else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # a larger sample than each reference-arm step: seconds of CPU work
        cpu = oracle_sample(*oracle_format(args), size=16)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks = measured_peaks()
    # the timed region lasts well under a second and runs at the burst clock
    # (see `clocks`), so the denominator is the burst figure; the sustained
    # one (seconds-long loops under the power cap) is reported beside it
    fp8_peak = peaks["bf16"] * FP8_OVER_BF16
    fp8_sustained = peaks["bf16_sustained"] * FP8_OVER_BF16
    flops = r["flops"]
    value = world * flops / (step_ms * 1e-3) / 1e12
    gemm_tflops = flops * args.steps / (gemm_ms * 1e-3) / 1e12
    quant_gbs = r["qbytes"] * args.steps / (quant_ms * 1e-3) / 1e9
    traffic = load_traffic()
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": WORKLOAD, "scale_format": args.scale, "tokens": M_TOKENS,
                   "activation_quant": "separate act / act_t launches" if args.separate_quant
                   else "dual (one read of X and of dY, both code layouts)",
                   "weight_quant": "grouped with the forward input (one launch per linear)"
                   if not (args.no_group_quant or args.separate_quant or args.scale == "mx") else "own launch",
                   "launch": "eager" if args.no_graph else "CUDA graph of the timed steps",
                   "gemm_tiles": "whole tiles" if args.no_split else "last round split along K where it pays",
                   "parallelism": f"replicas{world}", "l2": "flushed between steps (write of 2x L2)"},
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / fp8_peak, "traffic": traffic,
                     "kernel": "gemm_pair_kernel (all 12 GEMM launches of the step)",
                     "peak_note": f"{peaks['source']} bf16 burst x {FP8_OVER_BF16:g} (nominal FP8/BF16)",
                     "peak_sustained": fp8_sustained, "frac_of_sustained": gemm_tflops / fp8_sustained},
        "quantizers": {"achieved_gbs": quant_gbs, "peak_gbs": peaks["hbm_gbs"],
                       "frac": quant_gbs / peaks["hbm_gbs"], "ms_per_step": quant_ms / args.steps,
                       "launches_per_step": r["quant_launches"] // args.steps},
        "gemm": {"tflops": gemm_tflops, "ms_per_step": gemm_ms / args.steps,
                 "frac_of_nominal_4500": gemm_tflops / 4500.0,
                 "launches_per_step": r["gemm_launches"] // args.steps},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
        "kernel_split": {"source": "a replay, before the timed one, of the same K steps with an event between every two launches",
                         "ms_per_step": split_ms, "clocks": r["clocks_split"]},
    }
    # the SM clock the GEMM kernels counted themselves (clock64 over
    # globaltimer, summed over CTAs) during the kernel-split replay, and the
    # tensor cores' own peak at that clock: 16384 dense FP8 FLOP per SM per
    # cycle (the nominal 4.5 PFLOP/s over 148 SMs; ncu's tensor-pipe activity
    # times the clock reproduces it on these kernels) x SMs x clock
    kmhz = r.get("gemm_kernel_mhz")
    if kmhz:
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        peak_clk = FP8_FLOP_PER_SM_CYCLE * sms * kmhz * 1e6 / 1e12
        out["roofline"]["gemm_kernel_sm_mhz"] = kmhz
        out["roofline"]["peak_at_kernel_clock"] = peak_clk
        out["roofline"]["frac_at_kernel_clock"] = gemm_tflops / peak_clk
        out["roofline"]["peak_at_kernel_clock_note"] = (
            f"{FP8_FLOP_PER_SM_CYCLE} FP8 FLOP/SM/cycle x {sms} SMs x the clock the GEMM kernels counted")
    if r.get("fp8_ceiling"):
        out["roofline"]["fp8_cublas_8192"] = r["fp8_ceiling"]
    if r.get("fp32"):
        f = r["fp32"]
        g32 = f["flops"] * args.steps / (f["gemm_ms"] * 1e-3) / 1e12
        q32 = f["qbytes"] * args.steps / (f["quant_ms"] * 1e-3) / 1e9
        out["fp32_scales"] = {
            "value": f["flops"] / (f["step_ms"] / args.steps * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": f["step_ms"] / args.steps,
            "gemm": {"tflops": g32, "frac": g32 / fp8_peak, "frac_of_nominal_4500": g32 / 4500.0,
                     "ms_per_step": f["gemm_ms"] / args.steps,
                     "sm_mhz_in_kernel": f.get("gemm_kernel_mhz")},
            "quantizers": {"achieved_gbs": q32, "frac": q32 / peaks["hbm_gbs"],
                           "ms_per_step": f["quant_ms"] / args.steps},
            "clocks": f["clocks"],
            "what": "the same step with FP32 scales (per-128-K promotion in the epilogue), same seeds and timing"}
    if r.get("sweep"):
        sw = r["sweep"]
        out["sweep"] = {"config": "28-layer Qwen3-1.7B linear sweep + untied LM head, M=16384 (end to end)",
                        "value": sw["tflops"], "unit": "TFLOP/s", "ms": sw["ms"], "ms_all": sw["ms_all"],
                        "tflop": sw["flops"] / 1e12, "frac": sw["tflops"] / fp8_peak, "launches": sw["launches"],
                        "clocks": sw["clocks"], "lm_head_check": sw["lm_head_check"], "what": sw["what"]}
    out["roofline"]["measured_peaks_keys"] = peaks.get("keys")
    if r["e2e"]:
        out["e2e"] = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "h2d_bytes_per_step": r["e2e"]["h2d_bytes_per_step"],
                      "d2h_bytes_per_step": r["e2e"]["d2h_bytes_per_step"], "ms_per_step": e2e_ms,
                      "steps": r["e2e"]["steps"], "copies": r["e2e"]["copies"]}
    if cpu is not None:
        out["cpu_baseline"] = {"value": cpu["tflops"], "unit": "TFLOP/s", "cores": cpu["cores"],
                               "kind": "oracle", "sample": cpu["sample"]}
    print(json.dumps(out), flush=True)
    if r.get("sweep") and not r["sweep"]["lm_head_check"]["ok"]:
        sys.exit("the LM head output failed its sampled check against the float64 definition")


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "blockwise_fp8_linear_fp8bq_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith("gemm") or name.endswith(".cuh"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary; null when the
    GEMM source changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        if t.get("gemm_source_hash") != kernel_source_hash():
            return None
        return t.get("gemm_bytes_per_launch")
    except Exception:
        return None


if __name__ == "__main__":
    main()
