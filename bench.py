#!/usr/bin/env python
"""Benchmark of the SageAttention forward pass on B200 (one JSON line on rank 0).

Workload: the long-sequence point the headline metric is quoted on: B=2, H=32,
N=16384, d=128, non-causal, smooth K on, P.V in FP16 (4 B H N^2 d = 8.80 T operations
per step). Inputs are seeded synthetic N(0,1) with a per-channel K offset ~ N(0,1)
(the sequence-length sweep recipe), generated once and resident in HBM; each of Q, K,
V is 268 MB, larger than the 126 MB L2, so no L2 flush is needed between steps.

A step is one pass of the whole hot path through the C ABI: K-mean + per-block INT8
quantization of Q and K (sage_quant_qk) and the fused INT8 QK^T / online softmax / FP16
P.V kernel (sage_attn_fwd_quantized); CUDA events on the launching stream time the
attention kernel inside every step for the roofline figure.

--impl reference times the CPU oracle (test infrastructure, never tuned) on the host
cores on a bounded sample of the same workload (rows of one head per step).
Multi-GPU (torchrun): every rank runs the same workload on its own GPU (weak scaling,
no collective on the data path); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TOPS (4*B*H*N^2*d/t) at N=16k d=128; % of B200 INT8/FP16 MMA peak"
WORKLOAD = dict(B=2, H=32, N=16384, d=128, causal=False, pv_mode="fp16", smooth_k=True)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _ops(B, H, N, d, causal):
    ops = 4.0 * B * H * N * N * d
    return ops / 2 if causal else ops


class ClockSampler:
    """SM clocks and throttle reasons sampled while running: through NVML every 10 ms
    (enough samples inside a timed region of a tenth of a second), else from nvidia-smi
    every 200 ms. Only reads; it changes no setting of the GPU."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []          # (time, sm MHz, max sm MHz, set of active reasons)
        self.proc = None
        self.thread = None
        self.stop = threading.Event()
        self.source = None

    def __enter__(self):
        if self._start_nvml():
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
            self.source = "nvidia-smi"
        except OSError:
            self.proc = None
        return self

    def _start_nvml(self) -> bool:
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            max_sm = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
            reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        except Exception:
            return False

        def poll():
            while not self.stop.is_set():
                try:
                    sm = float(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                    r = int(reasons_fn(handle))
                    self.samples.append((time.time(), sm, max_sm,
                                         {n for n, bit in bits.items() if r & bit}))
                except Exception:
                    pass
                self.stop.wait(0.01)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        self.source = "nvml"
        return True

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.strip().split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            self.samples.append((time.time(), sm, mx, {n for n, v in zip(self.REASONS, parts[4:8])
                                                       if v.lower() == "active"}))

    def mark(self, name):
        setattr(self, name, time.time())

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        """Samples taken between mark('t0') and mark('t1') (the timed region)."""
        pad = 0.01 if self.source == "nvml" else 0.1     # half a sampling period or so
        t0 = getattr(self, "t0", 0.0) - pad
        t1 = getattr(self, "t1", float("inf")) + pad
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": self.source}
        sm = [x[1] for x in inside]
        reasons = set().union(*(x[3] for x in inside))
        busy = [v for v in sm if v > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(x[2] for x in inside),
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


def max_over_ranks(ms: float, dist=None, device=None) -> float:
    """Largest elapsed time over all ranks (the job finishes with its slowest rank)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_tops(ops_per_step: float, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank processes the same workload in ms (max over ranks)."""
    return world * ops_per_step * steps / (ms * 1e-3) / 1e12


# A timed region shorter than this runs at the burst clock (the bf16 GEMM's "burst"
# figure, best of 10 short runs); a longer one settles under the power cap (the
# "sustained" figure, a GEMM looped for seconds).
SUSTAINED_AFTER_S = 2.0


def tensor_peaks(peaks: dict, fp8_pv: bool, timed_ms: float):
    """(mixed peak, INT8 peak, bf16 figure used, which) in TOPS. INT8 and FP8 dense run at
    2x the bf16 rate, FP16 at 1x (nominal 4.5 : 2.25 PFLOP/s); the kernel does half its
    operations in the INT8 QK^T and half in the P.V, so its bound is the harmonic mix."""
    sustained = timed_ms * 1e-3 >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in peaks
    which = "sustained" if sustained else "burst"
    bf16 = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    int8_peak = 2.0 * bf16
    pv_peak = 2.0 * bf16 if fp8_pv else bf16
    return 1.0 / (0.5 / int8_peak + 0.5 / pv_peak), int8_peak, bf16, which


def quant_bytes(B: int, H: int, Nq: int, Nk: int, d: int, fp8_pv: bool, smooth_q: bool) -> dict:
    """Bytes the quantization step must move at the least (each input read once, each
    output written once) and the bytes the two-pass form actually moves (the column-sum
    pass reads K, and V in FP8 mode, and Q with smooth Q, a second time)."""
    nq, nk = B * H * Nq * d, B * H * Nk * d
    algorithmic = 3 * nq + 3 * nk + 4 * B * H * d            # fp16 in, int8 out; the K mean
    algorithmic += 4 * B * H * (math.ceil(Nq / 128) + math.ceil(Nk / 64))   # block scales
    moved = algorithmic + 2 * nk + (2 * nq if smooth_q else 0)
    if fp8_pv:
        algorithmic += 3 * nk + 4 * B * H * d                 # V in, E4M3 out; V scales
        moved += 3 * nk + 4 * B * H * d + 2 * nk              # V statistics pass
    return {"algorithmic": algorithmic, "moved": moved}


def quant_roofline(B, H, Nq, Nk, d, fp8_pv, smooth_q, quant_ms, peaks, src) -> dict:
    """The quantization step (K column sums + Q/K codes, + V in FP8 mode) against HBM."""
    b = quant_bytes(B, H, Nq, Nk, d, fp8_pv, smooth_q)
    gbs = b["algorithmic"] / (quant_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"], "ms": quant_ms,
            "bytes_algorithmic": b["algorithmic"], "bytes_moved_two_pass": b["moved"],
            "moved_gbs": b["moved"] / (quant_ms * 1e-3) / 1e9,
            "peak_note": f"STREAM-style copy bandwidth (of {src})"}


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def torchrun_argv(n: int, script: str, argv, port: int):
    """One process per GPU on this node, rendezvous on the loopback address."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
            script, *argv]


def maybe_relaunch(gpus, script: str, argv) -> None:
    """--gpus N outside torchrun re-executes `script` under torchrun with N ranks (this
    process is replaced); inside torchrun, N must match the world size it set."""
    world = os.environ.get("WORLD_SIZE")
    if world is None:
        if gpus is not None and gpus > 1:
            cmd = torchrun_argv(gpus, script, argv, free_port())
            sys.stdout.flush()
            os.execv(cmd[0], cmd)
        return
    if gpus is not None and gpus != int(world):
        raise SystemExit(f"--gpus {gpus} but torchrun started {world} ranks")


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _oracle_case(args):
    """Host inputs and oracle layout of the workload the GPU arm times (one batch entry for
    dense workloads, every packed sequence for varlen)."""
    import oracle
    from quantized_attention_03_b200 import inputs

    W = _workload(args)
    w = W.get("gen") or inputs.sweep(W["N"], W["d"], W["causal"])
    if args.workload == "varlen":
        q, k, v, cu = inputs.make_varlen(w)
        lay = oracle.Layout.packed(cu.tolist(), w.H, w.d)
        W.update(varlen=True, lens=lay.lens)
        kvl = lay
    else:
        nq = W.get("Nq") or W["N"]
        q, k, v = inputs.make_dense(w, B=1, N=W["N"], Nq=nq)
        lay = oracle.Layout.dense(1, w.H, nq, W["d"])
        kvl = oracle.Layout.dense(1, w.H, W["N"], W["d"])
    pv = oracle.PV_FP8 if W["pv_mode"] == "fp8" else oracle.PV_FP16
    return W, q.numpy(), k.numpy(), v.numpy(), lay, pv, kvl


def _sample_ops(r0: int, r1: int, nq: int, nk: int, d: int, causal: bool) -> float:
    """Operations of query rows [r0, r1) of one head with nq queries and nk keys (4 d per
    visible key; the causal mask aligned at the bottom right)."""
    if not causal:
        return 4.0 * (r1 - r0) * nk * d
    return 4.0 * d * sum(max(0, min(r + 1 + nk - nq, nk)) for r in range(r0, r1))


def _oracle_sample(case, it: int, rows: int):
    """Run the oracle on `rows` query rows of one head; returns (seconds, ops, head)."""
    import oracle
    W, q, k, v, lay, pv, kvl = case
    s = it % lay.nseq
    h = (it // lay.nseq) % lay.H
    n = lay.lens[s]
    # row offsets spread over the sequence (golden-ratio steps), so that a causal sample
    # sees on average the workload's mean number of visible keys per row
    r0 = int(((it * 0.6180339887498949) % 1.0) * max(n - rows + 1, 1))
    r1 = min(r0 + rows, n)
    t0 = time.perf_counter()
    oracle.sage_attention(q, k, v, lay, W["causal"], W["smooth_k"], pv,
                          1.0 / math.sqrt(lay.d), heads=[(s, h)], rows=(r0, r1), kv_layout=kvl,
                          fine=W.get("fine", False), smooth_q=W.get("smooth_q", False))
    return (time.perf_counter() - t0, _sample_ops(r0, r1, n, kvl.lens[s], lay.d, W["causal"]),
            (s, h))


def run_reference(args):
    """The CPU oracle, as it stands, on rank 0: each step is a bounded sample of rows."""
    world, rank, _ = _dist()
    if rank != 0:
        return
    import oracle

    case = _oracle_case(args)
    W, lay = case[0], case[4]
    rows = args.ref_rows
    t, ops = 0.0, 0.0
    for it in range(args.warmup + args.steps):
        dt, n_ops, _ = _oracle_sample(case, it, rows)
        if it >= args.warmup:
            t += dt
            ops += n_ops
    value = ops / t / 1e12
    cores = oracle.num_threads()
    sample = (f"{rows} query rows of one head per step (heads and row offsets rotate), all "
              f"their keys, {_workload_name(W)}, quantization of that head included")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8+f16 (oracle: fp64 accumulation)"
        if W["pv_mode"] == "fp16" else "s8+f8 (oracle: fp64 accumulation)",
        "data": "synthetic",
        "config": {"workload": _workload_name(W),
                   **{k: v for k, v in W.items() if k not in ("gen",)}},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def cpu_baseline(args, seconds_target: float = 15.0):
    """Time the oracle on a bounded sample (256-row slices of heads) on the host cores."""
    import oracle

    case = _oracle_case(args)
    W = case[0]
    t_total, ops, rows, it, heads = 0.0, 0.0, 256, 0, set()
    while t_total < seconds_target and it < 64:
        dt, n_ops, head = _oracle_sample(case, it, rows)
        t_total += dt
        ops += n_ops
        heads.add(head)
        it += 1
    return {"value": ops / t_total / 1e12, "unit": "TOPS", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{it} slices of {rows} query rows x all their keys over {len(heads)} "
                      f"heads of {_workload_name(W)}, quantization of each head included "
                      f"({t_total:.1f} s of CPU work)"}


def _workload(args):
    """The workload to time: the headline point by default, one of the other target
    workloads with --workload, optionally overridden (smaller cases for profiling)."""
    from quantized_attention_03_b200 import inputs
    W = dict(WORKLOAD)
    if args.workload == "llm_prefill":
        w = inputs.llm_prefill()
    elif args.workload == "video_dit":
        w = inputs.video_dit()
    elif args.workload == "varlen":
        w = inputs.varlen()
    elif args.workload == "prefill_kv":
        w = inputs.prefill_kv()
    elif args.workload == "decode":
        w = inputs.decode()
    elif args.workload == "sweep":
        n = args.N or 16384
        w = inputs.sweep(n, args.d or 128, args.causal)
    else:
        w = None
    if w is not None:
        W.update(B=w.B, H=w.H, N=w.N, d=w.d, causal=w.causal, pv_mode=w.pv_modes[0])
        W["gen"] = w
        if w.nq:
            W["Nq"] = w.nq
    for key in ("B", "N", "d"):
        if getattr(args, key) is not None and args.workload in ("headline", "sweep"):
            W[key] = getattr(args, key)
    if args.causal:
        W["causal"] = True
    if args.pv is not None:
        W["pv_mode"] = args.pv
    W["fine"] = bool(args.fine)
    W["smooth_q"] = bool(args.smooth_q)
    return W


def _workload_name(W):
    if W.get("varlen"):
        return (f"packed varlen {len(W['lens'])} sequences (lengths {W['lens']}) H={W['H']} "
                f"d={W['d']} {'causal' if W['causal'] else 'non-causal'} PV={W['pv_mode']} "
                f"smooth_k")
    nq = f" Nq={W['Nq']} Nk={W['N']}" if W.get("Nq") else ""
    return (f"B={W['B']} H={W['H']} N={W['N']}{nq} d={W['d']} "
            f"{'causal' if W['causal'] else 'non-causal'} PV={W['pv_mode']} smooth_k"
            f"{' fine-groups' if W.get('fine') else ''}{' smooth_q' if W.get('smooth_q') else ''}")


def pipelined_e2e(steps, host_in, dev_sets, host_outs, compute, dist, dev):
    """End-to-end steps through the public API, pipelined over three streams: the
    host-to-device copy of step i+1 and the device-to-host copy of step i-1 overlap step
    i's compute (two device buffer sets, two pinned output buffers). Every step copies its
    inputs in and its result out. Returns the CUDA-event time from the first copy's start
    to the last result's arrival, max over ranks."""
    import torch
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    nb = len(dev_sets)
    ev = {k: [torch.cuda.Event() for _ in range(nb)] for k in ("in", "comp", "out")}

    def one(i):
        b = i % nb
        ins, out = dev_sets[b]
        s_in.wait_event(ev["comp"][b])              # the previous step on b has read ins
        with torch.cuda.stream(s_in):
            for d_t, h_t in zip(ins, host_in):
                d_t.copy_(h_t, non_blocking=True)
        ev["in"][b].record(s_in)
        s_comp.wait_event(ev["in"][b])
        s_comp.wait_event(ev["out"][b])             # out of the previous step on b is home
        compute(ins, out, s_comp)
        ev["comp"][b].record(s_comp)
        s_out.wait_event(ev["comp"][b])
        with torch.cuda.stream(s_out):
            host_outs[b].copy_(out, non_blocking=True)
        ev["out"][b].record(s_out)

    one(0)                                          # warm-up
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    t1.record(s_out)
    torch.cuda.synchronize()
    return max_over_ranks(max(t0.elapsed_time(t1), 1e-9), dist, dev)


def h2d_copy_ms(host_in, dev_ins, dist, dev):
    """Time of the host-to-device copy of one step's inputs alone (pinned buffers, one
    stream, CUDA events, max over ranks): with the copies overlapped with compute, the
    end-to-end step can be no shorter than this."""
    import torch
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for d_t, h_t in zip(dev_ins, host_in):      # warm-up
            d_t.copy_(h_t, non_blocking=True)
    st.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record(st)
    with torch.cuda.stream(st):
        for _ in range(reps):
            for d_t, h_t in zip(dev_ins, host_in):
                d_t.copy_(h_t, non_blocking=True)
    e1.record(st)
    st.synchronize()
    return max_over_ranks(e0.elapsed_time(e1) / reps, dist, dev)


def _e2e_bound(ops, world, h2d_bytes, copy_ms):
    """The end-to-end figure's ceiling set by the input copy alone, with its rate."""
    return {"h2d_gbs": h2d_bytes / (copy_ms * 1e-3) / 1e9,
            "h2d_bound": weak_scaling_tops(ops, 1, world, copy_ms)}


def decode_bytes(B: int, H: int, Nq: int, Nk: int, d: int) -> int:
    """Algorithmic HBM bytes of one decode step: every K code (1 byte) and V element
    (2 bytes) read once, the query codes read and the output written (2 bytes), and the
    scales."""
    return B * H * (3 * Nk * d + 3 * Nq * d + 4 * (Nq + (Nk + 63) // 64))


def run_decode(args, dist, world, rank, local):
    """A decode step (Nq = 1 new query per sequence against its 32768 quantized cached keys,
    B=8 H=32 d=128) through sage_attn_decode_quantized; the K codes and V stay resident
    between steps, as a KV cache does. The line's roofline is HBM bandwidth."""
    import torch
    import quantized_attention_03_b200 as sage
    from quantized_attention_03_b200 import inputs

    w = inputs.decode()
    B, H, Nq, Nk, d = w.B, w.H, w.nq, w.N, w.d
    qc, kc, vc = inputs.make_dense(w)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    z = sage.quant_qk(q, k, True)                  # the cache's codes, made once
    out = torch.empty_like(q)
    ws = torch.empty(sage.sage_attn_decode_workspace_size(B, H, Nq, Nk, d), dtype=torch.uint8,
                     device=q.device)
    stream = torch.cuda.current_stream()

    def step():
        rc = sage.sage_attn_decode_quantized(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v,
                                             out, B, H, Nq, Nk, d, w.causal, 0.0, 0, ws,
                                             ws.numel(), stream)
        if rc != sage.SAGE_OK:
            raise RuntimeError(sage.status_string(rc))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.__enter__()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark("t0")
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark("t1")
    clocks.__exit__(None, None, None)
    status = sage.sage_get_device_status()
    if status != sage.SAGE_OK:
        raise RuntimeError(f"device status {sage.status_string(status)}")
    ms = max_over_ranks(e0.elapsed_time(e1), dist, q.device)
    ms_step = ms / args.steps
    ops = inputs.attention_ops_kv(B, H, Nq, Nk, d, w.causal)
    nbytes = decode_bytes(B, H, Nq, Nk, d)
    gbs = nbytes / (ms_step * 1e-3) / 1e9
    peaks, peak_src = _peaks()
    line = {
        "metric": METRIC, "value": weak_scaling_tops(ops, args.steps, world, ms),
        "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8+f16", "data": "synthetic",
        "config": {"workload": f"decode B={B} H={H} Nq={Nq} Nk={Nk} d={d} causal PV=fp16 "
                               "(per GPU; K codes and V resident)",
                   "B": B, "H": H, "Nq": Nq, "Nk": Nk, "d": d, "causal": w.causal,
                   "pv_mode": "fp16", "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (K codes 1.07 GB, V 2.15 GB); no flush"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "decode_partial + decode_combine (split-K over the keys)",
                     "bytes_per_step": nbytes,
                     "peak_note": f"STREAM-style copy bandwidth (of {peak_src})"},
        "e2e": {"value": None, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0,
                "note": "a decode step's inputs are the resident K/V cache; not measured"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


def run_ours(args):
    import torch
    import quantized_attention_03_b200 as sage
    from quantized_attention_03_b200 import inputs

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))

    if args.workload == "decode":
        return run_decode(args, dist, world, rank, local)
    W = _workload(args)
    if args.workload == "varlen":
        return run_varlen(args, W, dist, world, rank, local)
    B, H, N, d = W["B"], W["H"], W["N"], W["d"]
    Nq = W.get("Nq") or N                  # queries per sequence (N keys)
    w = W.get("gen") or inputs.sweep(N, d, W["causal"])
    qc, kc, vc = inputs.make_dense(w, B=B, N=N, Nq=Nq)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    pv = sage.SAGE_PV_FP16 if W["pv_mode"] == "fp16" else sage.SAGE_PV_FP8
    vq, vscale = v, None
    if pv == sage.SAGE_PV_FP8:
        vq = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
        vscale = torch.empty((B, H, d), dtype=torch.float32, device=v.device)
    sm_scale = 1.0 / math.sqrt(d)
    dev = q.device
    fine, sq = W["fine"], W["smooth_q"]
    general = fine or sq or Nq != N          # the *_kv entry points
    nqb, nkb = (Nq, math.ceil(N / 32)) if fine else (math.ceil(Nq / 128), math.ceil(N / 64))
    qk_flags = ((sage.SAGE_SMOOTH_K if W["smooth_k"] else 0) | (sage.SAGE_QK_FINE if fine else 0)
                | (sage.SAGE_SMOOTH_Q if sq else 0))
    q_i8 = torch.empty(q.shape, dtype=torch.int8, device=dev)
    k_i8 = torch.empty(k.shape, dtype=torch.int8, device=dev)
    q_scale = torch.empty((B, H, nqb), dtype=torch.float32, device=dev)
    k_scale = torch.empty((B, H, nkb), dtype=torch.float32, device=dev)
    k_mean = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    ksum_ws = torch.empty(B * H * d * 16, dtype=torch.uint8, device=dev)  # fp64 K (and Q) sums
    q_mean = torch.empty((B, H, d), dtype=torch.float32, device=dev) if sq else None
    q_comp = (torch.empty((B, H, math.ceil(N / 128) * 128), dtype=torch.float32, device=dev)
              if sq else None)
    vstat_ws = torch.empty(B * H * d * 16, dtype=torch.uint8, device=dev)  # V column statistics

    def quant():
        if not general:
            sage.sage_quant_qk_ws(q, k, q_i8, q_scale, k_i8, k_scale, k_mean, B, H, N, d,
                                  W["smooth_k"], ksum_ws, ksum_ws.numel(), stream)
        else:
            sage.sage_quant_qk_kv(q, k, q_i8, q_scale, k_i8, k_scale, k_mean, q_mean, q_comp, B,
                                  H, Nq, N, d, qk_flags, ksum_ws, ksum_ws.numel(), stream)
        if pv == sage.SAGE_PV_FP8:
            sage.sage_quant_v_fp8_ws(v, vq, vscale, None, B, H, N, d, vstat_ws, vstat_ws.numel(),
                                     stream)

    def attend():
        if not general:
            sage.sage_attn_fwd_quantized(q_i8, q_scale, k_i8, k_scale, vq, vscale, out, B, H, N,
                                         d, W["causal"], pv, sm_scale, stream)
        else:
            sage.sage_attn_fwd_quantized_kv(q_i8, q_scale, k_i8, k_scale, vq, vscale, None, q_comp,
                                            out, B, H, Nq, N, d, W["causal"], pv, sm_scale,
                                            sage.SAGE_QK_FINE if fine else 0, stream)

    def step():
        quant()
        attend()

    clocks = ClockSampler(local)
    clocks.__enter__()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = sage.sage_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {sage.status_string(status)}")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark("t0")
    if True:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            e0, e1, e2 = ev[i]
            e0.record(stream)
            quant()
            e1.record(stream)
            attend()
            e2.record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    clocks.mark("t1")
    clocks.__exit__(None, None, None)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    status = sage.sage_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {sage.status_string(status)}")
    total_ms = t_start.elapsed_time(t_end)
    attn_ms = [e1.elapsed_time(e2) for (_, e1, e2) in ev]
    quant_ms = [e0.elapsed_time(e1) for (e0, e1, _) in ev]
    total_ms = max_over_ranks(total_ms, dist, dev)

    ops = (_ops(B, H, N, d, W["causal"]) if Nq == N
           else inputs.attention_ops_kv(B, H, Nq, N, d, W["causal"]))
    ms_per_step = total_ms / args.steps
    value = weak_scaling_tops(ops, args.steps, world, total_ms)
    attn_avg_ms = sum(attn_ms) / len(attn_ms)
    attn_tops = ops / (attn_avg_ms * 1e-3) / 1e12

    # end to end through the public API: pinned host inputs -> device -> result -> host
    # as many end-to-end steps as timed steps: the copy pipeline's fill and drain (one
    # compute and one output copy) are then a small part of the region
    e2e_steps = 0 if args.no_e2e else max(3, args.steps)
    e2e_ms = 1e-9
    if e2e_steps:
        host_in = [t.pin_memory() for t in (qc, kc, vc)]
        host_outs = [torch.empty_like(qc).pin_memory() for _ in range(2)]
        dev_sets = [([torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)],
                     torch.empty_like(q)) for _ in range(2)]

        def compute(ins, o, st):
            qd, kd, vd = ins
            if not general:
                sage.sage_attn_fwd(qd, kd, vd, o, B, H, N, d, W["causal"], W["smooth_k"], pv,
                                   sm_scale, st)
            else:
                sage.sage_attn_fwd_kv(qd, kd, vd, o, B, H, Nq, N, d, W["causal"], qk_flags, pv,
                                      sm_scale, None, 0, st)

        e2e_ms = pipelined_e2e(e2e_steps, host_in, dev_sets, host_outs, compute, dist, dev)
        copy_ms = h2d_copy_ms(host_in, dev_sets[0][0], dist, dev)
    status = sage.sage_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after e2e: {sage.status_string(status)}")
    e2e_value = weak_scaling_tops(ops, e2e_steps, world, e2e_ms) if e2e_steps else None
    elem_bytes = B * H * N * d * 2         # one K or V tensor
    q_bytes = B * H * Nq * d * 2           # Q or O

    peaks, src = _peaks()
    mixed, int8_peak, bf16, which = tensor_peaks(peaks, pv == sage.SAGE_PV_FP8, total_ms)
    quant_avg_ms = sum(quant_ms) / len(quant_ms)
    roofline = {
        "bound": "tensor", "achieved": attn_tops, "peak": mixed, "unit": "TOPS",
        "frac": attn_tops / mixed, "traffic": None,
        "kernel": f"attn_kernel<d={d}, PV={W['pv_mode']}, 2 query tiles per CTA>",
        "peak_note": (f"mixed INT8-QK/{W['pv_mode'].upper()}-PV dense peak from the {src} "
                      f"{which} bf16 GEMM ({bf16:.1f} TF/s): int8 and fp8 = 2x, fp16 = 1x, "
                      f"half the operations each (of {src})"),
        "frac_of_int8_peak": attn_tops / int8_peak,
        "attn_ms": attn_avg_ms, "quant_ms": quant_avg_ms,
        "quant": quant_roofline(B, H, Nq, N, d, pv == sage.SAGE_PV_FP8, sq, quant_avg_ms,
                                peaks, src),
    }
    traffic_file = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if os.path.exists(traffic_file):
        with open(traffic_file) as f:
            tr = json.load(f)
        if (tr.get("kernel_source_hash") == _kernel_hash() and args.workload == "headline"
                and (B, H, N, d, W["causal"], W["pv_mode"]) == (2, 32, 16384, 128, False, "fp16")):
            roofline["traffic"] = tr.get("bytes_per_launch")

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "s8+f8" if pv == sage.SAGE_PV_FP8 else "s8+f16", "data": "synthetic",
            "config": {"workload": (args.workload if args.workload != "headline" else
                                    "sequence-length sweep point") + " " + _workload_name(W) +
                                   " (per GPU)",
                       "B": B, "H": H, "N": N, "d": d, "causal": W["causal"],
                       **({"Nq": Nq, "Nk": N} if Nq != N else {}),
                       "pv_mode": W["pv_mode"], "smooth_k": W["smooth_k"],
                       "parallelism": f"replicas x{world}",
                       "l2": _l2_note(elem_bytes)},
            "roofline": roofline,
            "e2e": {"value": e2e_value, "unit": "TOPS",
                    "h2d_bytes_per_step": q_bytes + 2 * elem_bytes, "d2h_bytes_per_step": q_bytes,
                    "steps": e2e_steps,
                    **(_e2e_bound(ops, world, q_bytes + 2 * elem_bytes, copy_ms)
                       if e2e_steps else {}),
                    "pipelining": "3 streams: step i+1's inputs in and step i-1's output out "
                                  "overlap step i (sage_attn_fwd, pinned host buffers)"},
            # per step: K column sums, Q/K codes, attention; + Q column sums with smooth Q;
            # + V column statistics and V codes in FP8 mode
            "gpu_launches": (3 + (1 if sq else 0)
                             + (2 if pv == sage.SAGE_PV_FP8 else 0)) * args.steps,
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args, args.cpu_seconds)
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_varlen(args, W, dist, world, rank, local):
    """Packed varlen workload through sage_attn_varlen_fwd (quantization and attention
    in one call with caller scratch); the attention kernel is not timed separately."""
    import torch
    import quantized_attention_03_b200 as sage
    from quantized_attention_03_b200 import inputs

    w = W["gen"]
    qc, kc, vc, cu = inputs.make_varlen(w)
    lens = [int(x) for x in (cu[1:] - cu[:-1])]
    W.update(varlen=True, lens=lens)
    T, H, d = qc.shape
    nseq, maxlen = len(lens), max(lens)
    pv = sage.SAGE_PV_FP16 if W["pv_mode"] == "fp16" else sage.SAGE_PV_FP8
    q, k, v, cud = qc.cuda(), kc.cuda(), vc.cuda(), cu.cuda()
    out = torch.empty_like(q)
    need = sage.sage_workspace_size(nseq, H, maxlen, T, d, pv)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream()
    ops = inputs.varlen_ops(lens, H, d, W["causal"])

    def step(qq=q, kk=k, vv=v, oo=out, st=stream):
        flags = (sage.SAGE_SMOOTH_K | (sage.SAGE_QK_FINE if W["fine"] else 0)
                 | (sage.SAGE_SMOOTH_Q if W["smooth_q"] else 0))
        sage.sage_attn_varlen_fwd(qq, kk, vv, oo, cud, nseq, T, maxlen, H, d, W["causal"], flags,
                                  pv, 0.0, ws, need, st)

    clocks = ClockSampler(local)
    clocks.__enter__()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if sage.sage_get_device_status() != 0:
        raise RuntimeError("device status after warm-up")
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark("t0")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark("t1")
    clocks.__exit__(None, None, None)
    if sage.sage_get_device_status() != 0:
        raise RuntimeError("device status after timing")
    total_ms = max_over_ranks(e0.elapsed_time(e1), dist, q.device)
    value = weak_scaling_tops(ops, args.steps, world, total_ms)

    # as many end-to-end steps as timed steps: the copy pipeline's fill and drain (one
    # compute and one output copy) are then a small part of the region
    e2e_steps = 0 if args.no_e2e else max(3, args.steps)

    e2e_ms = 1e-9
    if e2e_steps:
        host_in = [t.pin_memory() for t in (qc, kc, vc)]
        host_outs = [torch.empty_like(qc).pin_memory() for _ in range(2)]
        dev_sets = [([torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)],
                     torch.empty_like(q)) for _ in range(2)]

        def compute(ins, o, st):
            step(ins[0], ins[1], ins[2], o, st)

        e2e_ms = pipelined_e2e(e2e_steps, host_in, dev_sets, host_outs, compute, dist, q.device)
        copy_ms = h2d_copy_ms(host_in, dev_sets[0][0], dist, q.device)
    e2e_value = weak_scaling_tops(ops, e2e_steps, world, e2e_ms) if e2e_steps else None

    peaks, src = _peaks()
    mixed, int8_peak, bf16, which = tensor_peaks(peaks, pv == sage.SAGE_PV_FP8, total_ms)
    if rank == 0:
        elem_bytes = q.numel() * 2
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "s8+f8" if pv == sage.SAGE_PV_FP8 else "s8+f16", "data": "synthetic",
            "config": {"workload": "varlen " + _workload_name(W) + " (per GPU)",
                       "H": H, "d": d, "T": T, "lens": lens, "causal": W["causal"],
                       "pv_mode": W["pv_mode"], "parallelism": f"replicas x{world}",
                       "l2": _l2_note(q.numel() * 2)},
            "roofline": {"bound": "tensor", "achieved": value / world, "peak": mixed,
                         "unit": "TOPS", "frac": value / world / mixed, "traffic": None,
                         "kernel": "whole varlen step (quantization + attention in one call; "
                                   "the attention kernel is not timed separately)",
                         "peak_note": f"mixed dense peak from the {src} {which} bf16 GEMM "
                                      f"({bf16:.1f} TF/s) (of {src})"},
            "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": 3 * elem_bytes,
                    "d2h_bytes_per_step": elem_bytes, "steps": e2e_steps,
                    **(_e2e_bound(ops, world, 3 * elem_bytes, copy_ms) if e2e_steps else {}),
                    "pipelining": "3 streams: step i+1's inputs in and step i-1's output out "
                                  "overlap step i (sage_attn_varlen_fwd, pinned host buffers)"},
            # column statistics (K and V together), quantization, attention; + Q sums
            "gpu_launches": (3 + (1 if W["smooth_q"] else 0)) * args.steps,
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args, args.cpu_seconds)
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def _l2_note(tensor_bytes: int) -> str:
    mb = tensor_bytes / 1e6
    if 3 * tensor_bytes > 126e6:
        return f"inputs larger than L2 (Q, K, V {mb:.0f} MB each); no flush"
    return f"inputs fit in L2 (Q, K, V {mb:.0f} MB each); no flush, so L2-resident"


def _kernel_hash():
    """Hash of the attention kernel's code (comments and blank lines ignored): a stored
    DRAM-traffic figure is used only for the kernel it was measured on."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in ("attn_sm100.cu", "sm100_ptx.cuh", "sage_common.cuh", "quant_codes.cuh"):
        with open(os.path.join(ROOT, "quantized_attention_03_b200", "csrc", f)) as fh:
            for line in fh:
                code = re.sub(r"//.*", "", line).strip()
                if code:
                    h.update(code.encode())
    return h.hexdigest()[:16]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=None,
                    help="ranks, one per GPU (outside torchrun, bench.py starts them itself)")
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="headline",
                    choices=["headline", "llm_prefill", "video_dit", "sweep", "varlen",
                             "prefill_kv", "decode"],
                    help="headline: B2 H32 N16384 d128 non-causal FP16 PV (the metric's point)")
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--B", type=int, default=None, help="override the batch (profiling)")
    ap.add_argument("--N", type=int, default=None, help="override the sequence length")
    ap.add_argument("--d", type=int, default=None, choices=[64, 128])
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--pv", choices=["fp16", "fp8"], default=None)
    ap.add_argument("--fine", action="store_true",
                    help="one Q scale per token and one K scale per 32 tokens")
    ap.add_argument("--smooth-q", action="store_true",
                    help="smooth Q with the mean(Q) K^T score compensation")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    maybe_relaunch(args.gpus, os.path.abspath(__file__), sys.argv[1:])
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
