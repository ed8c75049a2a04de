#!/usr/bin/env python
"""Throughput of the LSTM forward pass + BPTT (lstm_fwd + lstm_bwd) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = lstm_fwd + lstm_bwd over the whole workload (every row of the
method: input projection, forward recurrence, backward recurrence, dW, db,
dx), on synthetic seeded inputs already resident in HBM.  The default workload
is T=256, B=128, I=1024, H=1024 in bf16 (fp32 accumulate and cell state).
Rank 0 prints one JSON line.  Under torchrun (N > 1) every rank runs an
independent replica of the workload ("replicas only": the path needs no
exchange between GPUs), timed as the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload (whole sequences).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from backward_lstm_fwd_b200 import synth  # noqa: E402

METRIC = "LSTM fwd+bwd (T·B) timesteps/sec and % of bf16 tensor peak, 1×B200"
UNIT = "timesteps/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0  # dense bf16, B200 data sheet (context only)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, clk):
    """The bf16 peak a kernel timed inside this run is held to: the burst
    figure when the sampled SM clock stayed at its maximum with no throttle
    reason active (the conditions the burst figure was measured under), else
    the sustained one."""
    at_max = (clk is not None and clk.get("sm_mhz") and clk.get("sm_max_mhz")
              and clk["sm_mhz"] >= 0.98 * clk["sm_max_mhz"] and not clk.get("reasons"))
    if at_max:
        return peaks["bf16_tflops"], "burst bf16 (clocks at max, no throttle reason)"
    return peaks["bf16_tflops_sustained"], "sustained bf16 (clocks below max or throttled)"


def measured_traffic(phase: str, workload: str):
    """DRAM bytes per launch of a phase's kernel from the committed ncu record
    (profiles/traffic.json), or None when there is none for this workload or
    the kernel source changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(phase)
        if not rec or rec.get("workload") != workload or not rec.get("source_sha256"):
            return None
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
                return None
        return float(rec["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        return None


def split_by_size(items, n):
    """Split (size, key) items into n lists of keys with sizes as even as the
    greedy rule makes them: largest first, each onto the lightest list."""
    lanes, load = [[] for _ in range(n)], [0] * n
    for size, key in sorted(items, key=lambda it: -it[0]):
        j = load.index(min(load))
        lanes[j].append(key)
        load[j] += size
    return [lane for lane in lanes if lane]


def reduce_max(v: float, dist=None, device="cpu") -> float:
    """The max of `v` over the ranks of the default process group (`v` itself
    without one): a multi-GPU time is the slowest rank's."""
    if dist is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, rows: int, steps: int, ms: float) -> float:
    """Whole-job timesteps/s: every rank processes `rows` timesteps per step
    (weak scaling), and `ms` is the max over ranks of the timed region."""
    return world * rows * steps / (ms * 1e-3)


def phase_work(w: synth.Workload, phases=None):
    """Algorithmic work per phase: FLOPs for the contractions (2 * M * N * K of
    the products the method defines), bytes for the db column reduction.  With
    the measured `phases` ({name: (ms, launches)}), work moves to the phase
    that ran it: the x-part of the gate pre-activations into the forward
    recurrence when no input-projection launch ran (the fused forward kernel),
    dx into the dW phase when both share one launch."""
    TB, H, I = w.rows, w.H, w.I
    es = 4 if w.dtype == "fp32" else 2
    work = {
        "input_proj": ("flop", 2.0 * TB * 4 * H * I),
        "fwd_recur": ("flop", 2.0 * TB * 4 * H * H),
        "bwd_recur": ("flop", 2.0 * TB * 4 * H * H),
        "dW": ("flop", 2.0 * TB * 4 * H * (H + I)),
        "db": ("byte", float(TB * 4 * H * es + 4 * H * 4)),
        "dx": ("flop", 2.0 * TB * 4 * H * I),
        "other": ("byte", 0.0),
    }
    if phases is not None:
        ran = lambda k: phases.get(k, (0.0, 0))[1] > 0
        if not ran("input_proj") and ran("fwd_recur"):
            work["fwd_recur"] = ("flop", work["fwd_recur"][1] + work["input_proj"][1])
        if not ran("dx") and ran("dW"):
            work["dW"] = ("flop", work["dW"][1] + work["dx"][1])
    return work


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9 or (self.uuid and parts[0] != self.uuid):
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def cpu_baseline(w: synth.Workload, inputs, target_seconds=20.0):
    """The fp64 oracle, as it stands, on a bounded sample of whole sequences:
    waves of one sequence per thread until about `target_seconds` of wall time
    (the last wave may run past it; never more than the whole batch)."""
    import oracle
    threads = oracle.max_threads()
    per_wave = max(1, min(w.B, threads))
    done, dt = 0, 0.0
    while done < w.B and dt < target_seconds:
        n = min(per_wave, w.B - done)
        sub = synth.as_float64(synth.select_sequences(inputs, list(range(done, done + n))))
        t0 = time.perf_counter()
        oracle.lstm_fwd_bwd(**sub)
        dt += time.perf_counter() - t0
        done += n
    return {"value": w.T * done / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} of {w.B} sequences x T={w.T} steps, fwd+bwd, fp64, "
                      f"{dt:.1f} s wall on {threads} OpenMP threads"}


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    import oracle
    inputs = synth.make_inputs(w)
    threads = oracle.max_threads()
    nseq = max(1, min(w.B, threads))
    sub = synth.as_float64(synth.select_sequences(inputs, list(range(nseq))))
    for _ in range(args.warmup):
        oracle.lstm_fwd_bwd(**sub)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.lstm_fwd_bwd(**sub)
    dt = time.perf_counter() - t0
    value = w.T * nseq * args.steps / dt
    sample = (f"{nseq} of {w.B} sequences x T={w.T} steps per step, fwd+bwd, fp64, "
              f"{threads} OpenMP threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "B": w.B, "I": w.I, "H": w.H,
                   "inputs": w.dtype, "sample_sequences": nseq},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class Problem:
    """One workload resident on the device: inputs, outputs, workspaces and a
    stream, and the step (lstm_fwd + lstm_bwd) that bench times."""

    def __init__(self, L, w, dev, seq_mask=False):
        self.L, self.w, self.dev = L, w, dev
        self.inputs = synth.make_inputs(w)
        T, B, I, H = w.T, w.B, w.I, w.H
        if seq_mask:  # variable length: seeded per-sequence lengths in 0..T
            self.inputs["mask"] = synth.length_mask(
                T, B, H, synth.random_lengths(T, B, seed=w.seed), w.dtype)
        self.d = {k: v.to(dev) for k, v in self.inputs.items()}
        cd = synth.torch_dtype(w.dtype)
        self.st = L.State(T, B, I, H, cd, dev)
        self.gr = L.Grads(T, B, I, H, dev)
        self.dims = self.st.dims
        self.ws_f = L.empty_workspace(L.fwd_workspace_size(self.dims, self.d.get("mask")), dev)
        self.ws_b = L.empty_workspace(L.bwd_workspace_size(self.dims), dev)
        self.stream = torch.cuda.Stream(dev)
        self.stream.wait_stream(torch.cuda.current_stream(dev))

    def step(self, src=None, st=None, gr=None):
        L, src = self.L, src if src is not None else self.d
        st, gr = st or self.st, gr or self.gr
        L.lstm_fwd(self.dims, src["x"], src["W"], src["b"], src["h0"], src["c0"], st.y, st.hT,
                   st.cT, st.gates, st.cells, self.ws_f, stream=self.stream, mask=src.get("mask"))
        L.lstm_bwd(self.dims, src["dy"], src["dhT"], src["dcT"], src["x"], src["W"], src["h0"],
                   src["c0"], st.y, st.gates, st.cells, gr.dx, gr.dW, gr.db, gr.dh0, gr.dc0,
                   self.ws_b, stream=self.stream, mask=src.get("mask"))

    def check_status(self, where):
        for ws in (self.ws_f, self.ws_b):
            if self.L.lstm_status(ws, stream=self.stream) != self.L.LSTM_OK:
                raise RuntimeError(f"device-side status set during {where}")

    def timed(self, steps, warmup, barrier=lambda: None):
        """Device time of `steps` steps after `warmup` untimed ones: (ms,
        per-phase {name: (ms, launches)}, kernel launches)."""
        L = self.L
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                self.step()
        torch.cuda.synchronize(self.dev)
        self.check_status("warm-up")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(self.dev)
        n0 = L.launch_count()
        L.profile_begin()
        e0.record(self.stream)
        with torch.cuda.stream(self.stream):
            for _ in range(steps):
                self.step()
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        phases = L.profile_end()
        launches = L.launch_count() - n0
        barrier()
        self.check_status("the timed region")
        return e0.elapsed_time(e1), phases, launches


def config_line(w, ms, phases, steps, peak):
    """Per-workload figures of one timed run: ms and timesteps/s per step,
    TFLOP/s and its fraction of `peak`, and the device microseconds per
    recurrent step of the forward and backward recurrences."""
    step_s = ms / steps * 1e-3
    tfl = w.flops / step_s / 1e12
    us = lambda k: 1e3 * phases.get(k, (0.0, 0))[0] / steps / max(w.T, 1)
    return {"T": w.T, "B": w.B, "I": w.I, "H": w.H, "dtype": w.dtype, "steps": steps,
            "ms_per_step": ms / steps, "timesteps_per_s": w.rows / step_s, "tflops": tfl,
            "frac_bf16_peak": tfl / peak,
            "us_per_recurrent_step": {"fwd": us("fwd_recur"), "bwd": us("bwd_recur")},
            "phases_ms_per_step": {p: v[0] / steps for p, v in phases.items() if v[1] > 0}}


def run_ours(args, w, rank, world, local_rank):
    from backward_lstm_fwd_b200 import binding as L
    from backward_lstm_fwd_b200 import build as lbuild
    lbuild.build()
    L.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(v):
        return reduce_max(v, dist, dev)

    pb = Problem(L, w, dev, seq_mask=args.seq_mask)
    T, B, I, H = w.T, w.B, w.I, w.H
    inputs, stream = pb.inputs, pb.stream

    # ---------------------------------------------------------- timed region
    clocks = ClockSampler(dev) if rank == 0 else None
    if clocks:
        clocks.start()
    ms, phases, launches = pb.timed(args.steps, args.warmup, barrier)
    clk = clocks.stop() if clocks else None
    ms = max_over_ranks(ms)

    # -------------------------------------------------- end to end (host I/O)
    # Every step copies all of its inputs from pinned host memory and reads its
    # results back: the forward's outputs (y, hT, cT) and every gradient.  Two
    # device buffer sets and separate copy streams let step k+1's upload and
    # step k-1's download run under step k's compute.
    cd = synth.torch_dtype(w.dtype)
    pin_in = {k: v.pin_memory() for k, v in inputs.items()}
    dev_in = [{k: torch.empty_like(v, device=dev) for k, v in inputs.items()} for _ in range(2)]
    states = [pb.st, L.State(T, B, I, H, cd, dev)]
    grads = [pb.gr, L.Grads(T, B, I, H, dev)]
    fwd_names, grad_names = ("y", "hT", "cT"), ("dx", "dW", "db", "dh0", "dc0")
    results = [[getattr(states[i], n) for n in fwd_names] +
               [getattr(grads[i], n) for n in grad_names] for i in range(2)]
    pin_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in r] for r in results]
    h2d = sum(v.numel() * v.element_size() for v in pin_in.values())
    d2h = sum(t.numel() * t.element_size() for t in results[0])
    # two copy streams per direction, whole tensors split between them by
    # size (largest first onto the lighter stream), so that two copies of a
    # direction run at once (cutting tensors into 32 MB pieces over 2 to 4
    # streams measured slower: more, smaller copies)
    lanes_in = split_by_size([(v.numel() * v.element_size(), k) for k, v in pin_in.items()], 2)
    lanes_out = split_by_size([(t.numel() * t.element_size(), j)
                               for j, t in enumerate(results[0])], 2)
    s_h2d = [torch.cuda.Stream(dev) for _ in lanes_in]
    s_d2h = [torch.cuda.Stream(dev) for _ in lanes_out]
    ev = lambda: torch.cuda.Event()
    in_ready = [[ev() for _ in lanes_in] for _ in range(2)]
    in_free = [ev(), ev()]
    out_ready = [ev(), ev()]
    out_free = [[ev() for _ in lanes_out] for _ in range(2)]

    def e2e_step(k):
        i = k % 2
        for lane, st in enumerate(s_h2d):
            st.wait_event(in_free[i])       # step k-2's compute has read buffer i
            with torch.cuda.stream(st):
                for n in lanes_in[lane]:
                    dev_in[i][n].copy_(pin_in[n], non_blocking=True)
            in_ready[i][lane].record(st)
        for lane in range(len(s_h2d)):
            stream.wait_event(in_ready[i][lane])
        for lane in range(len(s_d2h)):
            stream.wait_event(out_free[i][lane])  # step k-2's results have been read back
        with torch.cuda.stream(stream):
            pb.step(dev_in[i], states[i], grads[i])
        in_free[i].record(stream)
        out_ready[i].record(stream)
        for lane, st in enumerate(s_d2h):
            st.wait_event(out_ready[i])
            with torch.cuda.stream(st):
                for j in lanes_out[lane]:
                    pin_out[i][j].copy_(results[i][j], non_blocking=True)
            out_free[i][lane].record(st)

    def e2e_run(nsteps):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for st in s_h2d + s_d2h:
            st.wait_event(f0)
        for k in range(nsteps):
            e2e_step(k)
        for i in range(2):
            for lane in range(len(s_d2h)):
                stream.wait_event(out_free[i][lane])
        f1.record(stream)
        torch.cuda.synchronize(dev)
        return f0, f1

    e2e_run(2)  # warm-up: allocations, pinned pages
    barrier()
    f0, f1 = e2e_run(args.steps)
    barrier()
    ms_e2e = max_over_ranks(f0.elapsed_time(f1))

    # ------------------------------------- the other workloads (figures only)
    per_config = {}
    if not args.no_per_config and args.seq_len is None and not args.seq_mask:
        for name, ow in synth.WORKLOADS.items():
            if name == w.name:
                continue
            op = Problem(L, ow, dev)
            osteps = max(3, min(args.steps, int(2000 // max(ow.T, 1))))
            oms, oph, _ = op.timed(osteps, max(3, args.warmup), barrier)
            per_config[name] = (ow, max_over_ranks(oms), oph, osteps)
            del op

    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    tpeak, tpeak_kind = tensor_peak(peaks, clk)
    work = phase_work(w, phases)
    dom = max((p for p in phases if phases[p][1] > 0), key=lambda p: phases[p][0])
    dom_ms, dom_launches = phases[dom]
    kind, amount = work[dom]
    amount *= args.steps  # work of the timed region
    if kind == "flop":
        achieved = amount / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tpeak, "unit": "TFLOP/s",
                "frac": achieved / tpeak, "traffic": measured_traffic(dom, w.name),
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS}
    else:
        achieved = amount / (dom_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": None}
    roof.update({"kernel": dom, "launches_per_step": dom_launches / args.steps,
                 "ms_per_step": dom_ms / args.steps,
                 "us_per_recurrent_step": 1e3 * dom_ms / args.steps / max(T, 1)
                 if dom in ("fwd_recur", "bwd_recur") else None,
                 "peak_source": f"{peak_src} ({tpeak_kind if kind == 'flop' else 'HBM copy'})"})
    step_s = ms / args.steps * 1e-3
    value = job_throughput(world, w.rows, args.steps, ms)
    tflops = w.flops / step_s / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded, distributions of the workload definition)",
        "config": {"workload": w.name, "T": T, "B": B, "I": I, "H": H,
                   "parallelism": f"replicas{world}" if world > 1 else "single-gpu",
                   "l2": "working set > 126 MB L2 per step (no flush needed)"},
        "tflops": tflops,
        "pct_bf16_peak": 100.0 * tflops / peaks["bf16_tflops"],
        "pct_bf16_peak_sustained": 100.0 * tflops / peaks["bf16_tflops_sustained"],
        "pct_bf16_peak_nominal": 100.0 * tflops / NOMINAL_BF16_TFLOPS,
        "roofline": roof,
        "phases_ms_per_step": {p: v[0] / args.steps for p, v in phases.items()},
        "us_per_recurrent_step": config_line(w, ms, phases, args.steps, tpeak)[
            "us_per_recurrent_step"],
        "gpu_launches": launches,
        "e2e": {"value": job_throughput(world, w.rows, args.steps, ms_e2e), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms_e2e / args.steps,
                "read_back": list(fwd_names + grad_names),
                "overlap": "uploads and read-backs on two copy streams each, two buffer sets"},
        "clocks": clk,
    }
    if per_config:
        line["per_config"] = {n: config_line(ow, oms, oph, ost, tpeak)
                              for n, (ow, oms, oph, ost) in per_config.items()}
    if args.seq_mask:
        real = float(inputs["mask"][:, :, 0].float().mean())
        line["config"]["seq_mask"] = (f"per-sequence lengths uniform in 0..T (seeded), "
                                      f"{100 * real:.0f} % of the T*B steps real; all counted")
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inputs)
    print(json.dumps(line), flush=True)
    return 0


def run_stack(args, w, rank, world, local_rank):
    """--layers L > 1: one step = lstm_stack_fwd + lstm_stack_bwd over L layers
    (layer 0 on the workload's x, layers above on H-wide inputs), inputs
    resident in HBM.  `value` counts the T*B timesteps of the stack per step;
    the roofline's FLOPs sum every layer's share of the dominant phase."""
    import dataclasses

    from backward_lstm_fwd_b200 import binding as L
    from backward_lstm_fwd_b200 import build as lbuild
    lbuild.build()
    L.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
    Lc, T, B, I, H = args.layers, w.T, w.B, w.I, w.H
    layers = [synth.make_inputs(w if l == 0 else dataclasses.replace(
        w, name=f"{w.name}_layer{l}", I=H, seed=w.seed + 7 * l)) for l in range(Lc)]
    inputs = dict(x=layers[0]["x"], dy=layers[-1]["dy"])
    for k in ("h0", "c0", "dhT", "dcT"):
        inputs[k] = torch.stack([p[k] for p in layers]).contiguous()
    Ws = [p["W"].to(dev) for p in layers]
    bs = [p["b"].to(dev) for p in layers]
    d = {k: v.to(dev) for k, v in inputs.items()}
    cd = synth.torch_dtype(w.dtype)
    st = L.StackState(Lc, T, B, I, H, cd, dev)
    gr = L.StackGrads(Lc, T, B, I, H, dev)
    ws_f = L.empty_workspace(L.stack_fwd_workspace_size(st.dims, Lc), dev)
    ws_b = L.empty_workspace(L.stack_bwd_workspace_size(st.dims, Lc), dev)
    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))

    def step(src):
        L.lstm_stack_fwd(st.dims, Lc, src["x"], Ws, bs, src["h0"], src["c0"], st.y, st.hT,
                         st.cT, st.gates, st.cells, ws_f, stream=stream)
        L.lstm_stack_bwd(st.dims, Lc, src["dy"], src["dhT"], src["dcT"], src["x"], Ws,
                         src["h0"], src["c0"], st.y, st.gates, st.cells, gr.dx, gr.dW, gr.db,
                         gr.dh0, gr.dc0, ws_b, stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(v):
        return reduce_max(v, dist, dev)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step(d)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev) if rank == 0 else None
    if clocks:
        clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    n0 = L.launch_count()
    L.profile_begin()
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            step(d)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    phases = L.profile_end()
    launches = L.launch_count() - n0
    barrier()
    clk = clocks.stop() if clocks else None
    ms = max_over_ranks(e0.elapsed_time(e1))
    for ws in (ws_f, ws_b):
        if L.lstm_status(ws, stream=stream) != L.LSTM_OK:
            raise RuntimeError("device-side status set during the timed region")

    # end to end: every step uploads its inputs from pinned host memory and
    # reads every gradient back (no overlap with the compute)
    pin_in = {k: v.pin_memory() for k, v in inputs.items()}
    outs = [gr.dx, gr.dh0, gr.dc0] + gr.dW + gr.db
    pin_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    h2d = sum(v.numel() * v.element_size() for v in pin_in.values())
    d2h = sum(t.numel() * t.element_size() for t in outs)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    f0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            for k in pin_in:
                d[k].copy_(pin_in[k], non_blocking=True)
            step(d)
            for t, p in zip(outs, pin_out):
                p.copy_(t, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms_e2e = max_over_ranks(f0.elapsed_time(f1))
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    tpeak, tpeak_kind = tensor_peak(peaks, clk)
    layer_w = [w] + [dataclasses.replace(w, I=H)] * (Lc - 1)
    works = [phase_work(lw, phases) for lw in layer_w]
    dom = max((p for p in phases if phases[p][1] > 0), key=lambda p: phases[p][0])
    dom_ms, dom_launches = phases[dom]
    kind = works[0][dom][0]
    amount = sum(wk[dom][1] for wk in works) * args.steps
    if kind == "flop":
        achieved = amount / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tpeak, "unit": "TFLOP/s",
                "frac": achieved / tpeak, "traffic": None}
    else:
        achieved = amount / (dom_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": None}
    roof.update({"kernel": dom, "launches_per_step": dom_launches / args.steps,
                 "ms_per_step": dom_ms / args.steps,
                 "peak_source": f"{peak_src} ({tpeak_kind if kind == 'flop' else 'HBM copy'})"})
    step_s = ms / args.steps * 1e-3
    tflops = sum(lw.flops for lw in layer_w) / step_s / 1e12
    line = {
        "metric": METRIC, "value": job_throughput(world, w.rows, args.steps, ms), "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded, distributions of the workload definition)",
        "config": {"workload": f"{w.name}_stack{Lc}", "T": T, "B": B, "I": I, "H": H,
                   "layers": Lc,
                   "parallelism": f"replicas{world}" if world > 1 else "single-gpu",
                   "l2": "working set > 126 MB L2 per step (no flush needed)"},
        "tflops": tflops,
        "pct_bf16_peak": 100.0 * tflops / peaks["bf16_tflops"],
        "pct_bf16_peak_sustained": 100.0 * tflops / peaks["bf16_tflops_sustained"],
        "roofline": roof,
        "phases_ms_per_step": {p: v[0] / args.steps for p, v in phases.items()},
        "gpu_launches": launches,
        "e2e": {"value": job_throughput(world, w.rows, args.steps, ms_e2e), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms_e2e / args.steps, "overlap": "none"},
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=synth.BENCH_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing the other four workloads (the per_config key)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override T (profiling aid: same per-step shape, fewer steps)")
    ap.add_argument("--dtype", choices=("bf16", "fp16"), default=None,
                    help="16-bit compute type override (fp16: the page's FLOAT16) on the "
                         "workload's shape")
    ap.add_argument("--layers", type=int, default=1,
                    help="a stack of this many LSTM layers (lstm_stack_fwd / lstm_stack_bwd)")
    ap.add_argument("--seq-mask", action="store_true",
                    help="variable length: a seq_length mask with seeded per-sequence "
                         "lengths in 0..T (every step is still computed and counted)")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.dtype is not None and args.dtype != w.dtype:
        import dataclasses
        if w.dtype == "fp32":
            ap.error("--dtype applies to the 16-bit workloads")
        w = dataclasses.replace(w, name=w.name.replace("_" + w.dtype, "_" + args.dtype),
                                dtype=args.dtype)
    if args.seq_len is not None:
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}_T{args.seq_len}", T=args.seq_len,
                                dy_last=None if w.dy_last is None else min(w.dy_last, args.seq_len))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, w, rank, world)
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.layers > 1:
            return run_stack(args, w, rank, world, local_rank)
        return run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
