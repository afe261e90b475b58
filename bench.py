"""Benchmark of the KDA operator on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl reference]

One step = one ``kda_forward`` call (varlen index + chunked prefill, every
step of the hot path) over the prefill workload ``--workload`` (default 3,
the largest prefill that fits one GPU: bf16, 8 packed sequences with
lengths drawn from U[1024, 32768], H=32, d_k=d_v=128, chunk 64; the other
two bf16 prefill workloads are timed as extra objects of the same line,
each with its own roofline).  The timed region is K
steps between a barrier + synchronize on both sides; each step's kernels
are bracketed by CUDA events on the launching stream and L2 is flushed
(256 MiB write) between steps outside those brackets.  Multi-GPU runs are
independent replicas (the operator needs no collective): each rank runs the
same workload on its own GPU and rank 0 reports the total over ranks divided
by the slowest rank's time.

The JSON line also carries: ``e2e`` (the same metric through the public
Python API from pinned host buffers, with the host<->device copies inside
the timed region), ``roofline`` (algorithmic bytes of the dominant kernel
over its measured duration against the measured HBM copy bandwidth),
``cpu_baseline`` (the fp64 CPU oracle on a bounded sample, rank 0), a
``decode`` object (64 recurrent steps of the decode workload) and the SM
clocks sampled during the timed region.

``--impl reference``: the reference arm is the fp64 CPU oracle (there is no
other implementation of this operator to run); it times K steps of a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gated_delta_rule_113_b200.inputs import WORKLOADS, decode_inputs, forward_inputs  # noqa: E402

METRIC = "KDA tokens/sec/GPU (prefill and decode) + % of tensor-pipe / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------
# accounting
# --------------------------------------------------------------------------
def _es(dtype):
    return 4 if dtype == torch.float32 else 2


def prefill_bytes(T, N, H, Dk, Dv, io_dtype, gate_dtype, has_s0):
    """Algorithmic HBM bytes of one prefill: every input read once, every output written once."""
    e, g = _es(io_dtype), _es(gate_dtype)
    per_token_head = 2 * Dk * e + Dv * e + Dk * g + g + Dv * e
    states = N * H * Dk * Dv * 4 * (2 if has_s0 else 1)
    return T * H * per_token_head + states + 4 * (N + 1)


def prefill_flops(T, H, Dk, Dv, C=64):
    """Algorithmic flops per prefill: 6*Dk*Dv + C*(3*Dk + 2*Dv) per token-head (triangles once)."""
    return T * H * (6 * Dk * Dv + C * (3 * Dk + 2 * Dv))


def decode_bytes(N, H, Dk, Dv, io_dtype):
    e = _es(io_dtype)
    return N * H * (2 * Dk * Dv * 4 + 3 * Dk * e + Dv * e + e + Dv * e)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def traffic_record(kernel, workload=None):
    """DRAM bytes per launch from a committed ncu capture (keyed by kernel, and
    workload where the traffic depends on it), if the sources are unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        recs = json.load(f)
    rec = recs.get(f"{kernel}:{workload}" if workload else kernel)
    if not rec:
        return None
    return rec["bytes_per_launch"] if sources_sha(rec) == rec.get("source_sha") else None


def sources_sha(rec):
    """Digest of every source file the recorded kernels are built from."""
    h = hashlib.sha256()
    for rel in rec.get("sources", [rec.get("source")]):
        src = os.path.join(ROOT, rel)
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, timeout=3.0):
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.02)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample
# --------------------------------------------------------------------------
def oracle_sample(w, inp, max_tokens):
    """First ``max_tokens`` tokens of every sequence, all heads (same chains, truncated)."""
    cu = inp["cu_seqlens"].numpy()
    idx, lens = [], []
    for n in range(len(cu) - 1):
        L = min(int(cu[n + 1] - cu[n]), max_tokens)
        idx.extend(range(int(cu[n]), int(cu[n]) + L))
        lens.append(L)
    idx = torch.tensor(idx, dtype=torch.long)
    sub = {k: inp[k][idx].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
    sub["S0"] = inp["S0"]
    sub["cu_seqlens"] = np.concatenate([[0], np.cumsum(lens)])
    return sub, int(sum(lens))


def run_oracle_timed(sub):
    import oracle
    t0 = time.perf_counter()
    oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], sub["S0"],
                   sub["cu_seqlens"])
    return time.perf_counter() - t0


def cpu_baseline(w, inp, max_tokens):
    import oracle
    sub, ntok = oracle_sample(w, inp, max_tokens)
    dt = run_oracle_timed(sub)
    return {"value": ntok / dt, "unit": "tokens/s", "cores": oracle.default_threads(),
            "kind": "oracle",
            "sample": f"first {max_tokens} tokens of each of the {len(inp['lengths'])} sequences, "
                      f"all {w.H} heads ({ntok} tokens, {dt:.2f} s, fp64 token-by-token)"}


# --------------------------------------------------------------------------
# distributed plumbing (replicas)
# --------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    """All ranks meet, then this rank's GPU work is finished (CPU-only runs of
    the host logic, e.g. the gloo tests, skip the device sync)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x, world):
    """Largest value over the ranks (device times are reported as the max)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, max_ms):
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (max_ms * 1e-3)


def prefill_roofline(w, inp, mean_ms, peaks, peaks_kind):
    """Roofline of one kda_forward call: algorithmic bytes over its CUDA-event
    duration against the measured HBM copy peak (the prefill is HBM-bound at
    ~109 flop/B), with the algorithmic tensor fraction beside it."""
    N, T = len(inp["lengths"]), int(inp["cu_seqlens"][-1])
    alg_bytes = prefill_bytes(T, N, w.H, w.Dk, w.Dv, w.torch_dtype, w.torch_dtype,
                              inp["S0"] is not None)
    alg_flops = prefill_flops(T, w.H, w.Dk, w.Dv)
    achieved = alg_bytes / (mean_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"],
            "traffic": traffic_record("kda_prefill", w.name),
            "peak_kind": f"{peaks_kind} HBM copy",
            "kernel": "kda_forward (varlen_index + kside + chain kernels, one call)",
            "algorithmic_bytes": alg_bytes, "algorithmic_flops": alg_flops,
            "tensor_frac_algorithmic": alg_flops / (mean_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}


def time_prefill(kda, d, out, sf, ws, flush, stream, steps):
    """CUDA-event time (ms) of each of ``steps`` kda_forward calls, L2 flushed
    between calls outside the events."""
    def step():
        kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["cu_seqlens"],
                    out=out, S_final=sf, workspace=ws)
    ev = []
    for _ in range(steps):
        flush.zero_()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        step()
        a1.record(stream)
        ev.append((a0, a1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def bench_extra_prefill(kda, dev, stream, world, wid, flush, steps, peaks, peaks_kind):
    """One more prefill workload, timed like the headline (L2 flushed between
    calls), reported with its own roofline."""
    w = WORKLOADS[wid]
    inp = forward_inputs(w)
    N, T = len(inp["lengths"]), int(inp["cu_seqlens"][-1])
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out = torch.empty((T, w.H, w.Dv), dtype=w.torch_dtype, device=dev)
    sf = torch.empty((N, w.H, w.Dk, w.Dv), dtype=torch.float32, device=dev)
    ws = torch.empty(kda.forward_workspace_size(N, T, w.H, w.Dk, w.Dv, w.torch_dtype),
                     dtype=torch.uint8, device=dev)
    time_prefill(kda, d, out, sf, ws, flush, stream, 3)
    if kda.workspace_status(ws) != 0:
        raise RuntimeError(f"device status not OK on {w.name}")
    barrier(world)
    ms = time_prefill(kda, d, out, sf, ws, flush, stream, steps)
    total = max_over_ranks(sum(ms), world)
    return {"workload": w.name, "num_seqs": N, "total_tokens": T, "H": w.H,
            "value": world * T * steps / (total * 1e-3), "unit": "tokens/s",
            "ms_per_step": total / steps, "steps": steps, "gpu_launches": 3 * steps,
            "roofline": prefill_roofline(w, inp, sum(ms) / len(ms), peaks, peaks_kind)}


# --------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------
def bench_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = WORKLOADS[args.workload]
    inp = forward_inputs(w)
    sub, ntok = oracle_sample(w, inp, args.ref_tokens)
    for _ in range(args.warmup):
        run_oracle_timed(sub)
    times = [run_oracle_timed(sub) for _ in range(args.steps)]
    total = sum(times)
    value = ntok * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "sample_tokens": ntok, "H": w.H, "Dk": w.Dk, "Dv": w.Dv},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.default_threads(),
                         "kind": "oracle",
                         "sample": f"first {args.ref_tokens} tokens of each sequence, all heads"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def bench_kda(args):
    import gated_delta_rule_113_b200 as kda
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.load_library()
    w = WORKLOADS[args.workload]
    inp = forward_inputs(w, lengths=args.lengths)
    if args.lengths:   # a reduced case of the workload (profiling): renamed accordingly
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}_lengths_{'_'.join(map(str, args.lengths))}")
    N, T, H, Dk, Dv = len(inp["lengths"]), int(inp["cu_seqlens"][-1]), w.H, w.Dk, w.Dv
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out = torch.empty((T, H, Dv), dtype=w.torch_dtype, device=dev)
    sf = torch.empty((N, H, Dk, Dv), dtype=torch.float32, device=dev)
    ws = torch.empty(kda.forward_workspace_size(N, T, H, Dk, Dv, w.torch_dtype), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["cu_seqlens"],
                    out=out, S_final=sf, workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    if kda.workspace_status(ws) != 0:
        raise RuntimeError("device status not OK after warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        # keep the GPU busy (untimed) until the sampler reports, so the clock
        # samples describe the loaded GPU around the timed region
        clk.wait_first()
        t_end = time.time() + 0.3
        while time.time() < t_end:
            flush.zero_()
            step()
            torch.cuda.synchronize()
        barrier(world)
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        barrier(world)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world)
    value = job_throughput(T * args.steps, world, total_ms)

    # ---- end to end through the public API from pinned host buffers -------
    # Every step copies its inputs in from pinned host memory, runs the
    # forward and copies the outputs (out and S_final) back.  Steps are
    # pipelined the way a serving loop would run them: step i+1's inputs copy
    # in on one copy stream while step i computes and step i-1's outputs copy
    # out on another; two device buffer sets alternate.
    names = ("q", "k", "v", "log_alpha", "beta")
    host = {k: inp[k].pin_memory() for k in names}
    host["S0"] = inp["S0"].pin_memory() if inp["S0"] is not None else None
    host_cu = inp["cu_seqlens"].pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    sf_h = [torch.empty(sf.shape, dtype=sf.dtype).pin_memory() for _ in range(2)]
    slots = []
    for _ in range(2):
        slots.append(dict(
            x={k: torch.empty_like(d[k]) for k in names},
            s0=torch.empty_like(d["S0"]) if d["S0"] is not None else None,
            cu=torch.empty_like(d["cu_seqlens"]),
            out=torch.empty_like(out), sf=torch.empty_like(sf),
            ws=torch.empty_like(ws)))
    h2d = sum(host[k].numel() * host[k].element_size() for k in names) + \
        (host["S0"].numel() * 4 if host["S0"] is not None else 0) + host_cu.numel() * 4
    d2h = out_h[0].numel() * out_h[0].element_size() + sf_h[0].numel() * 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    inputs_free, copied_in, computed, copied_out = ([ev() for _ in range(2)] for _ in range(4))

    def e2e_run(n_steps):
        for i in range(n_steps):
            b = i & 1
            sl = slots[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(inputs_free[b])
                for k in names:
                    sl["x"][k].copy_(host[k], non_blocking=True)
                if sl["s0"] is not None:
                    sl["s0"].copy_(host["S0"], non_blocking=True)
                sl["cu"].copy_(host_cu, non_blocking=True)
                copied_in[b].record(s_in)
            stream.wait_event(copied_in[b])
            if i >= 2:
                stream.wait_event(copied_out[b])     # this set's outputs have left
            kda.forward(sl["x"]["q"], sl["x"]["k"], sl["x"]["v"], sl["x"]["log_alpha"],
                        sl["x"]["beta"], sl["s0"], sl["cu"], out=sl["out"], S_final=sl["sf"],
                        workspace=sl["ws"])
            inputs_free[b].record(stream)
            computed[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[b])
                out_h[b].copy_(sl["out"], non_blocking=True)
                sf_h[b].copy_(sl["sf"], non_blocking=True)
                copied_out[b].record(s_out)

    e2e_run(max(2, args.warmup))
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    e2e_run(args.steps)
    stream.wait_stream(s_out)
    e1.record(stream)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = job_throughput(T * args.steps, world, e2e_ms)
    if not torch.equal(out_h[(args.steps - 1) & 1].to(dev), out):
        raise RuntimeError("end-to-end output differs from the device-resident run")

    # ---- prefix-cache snapshots: the same forward keeping the state every
    # 512 tokens in a slot pool (bf16, d = 128 only) ------------------------
    snap = None
    if not args.no_snapshots and w.torch_dtype == torch.bfloat16 and Dk == 128 and Dv == 128:
        every = 512
        counts = [n // every for n in inp["lengths"]]
        base = torch.tensor([sum(counts[:i]) for i in range(N)], dtype=torch.int32, device=dev)
        pool = torch.empty((max(1, sum(counts)), H, Dk, Dv), dtype=torch.float32, device=dev)

        def snap_step():
            kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                        d["cu_seqlens"], out=out, S_final=sf, workspace=ws, snapshot_pool=pool,
                        snapshot_slot_base=base, snapshot_every=every)

        for _ in range(max(3, args.warmup)):
            flush.zero_()
            snap_step()
        if kda.workspace_status(ws) != 0:
            raise RuntimeError("device status not OK with snapshots")
        sn_ms = []
        for _ in range(args.steps):
            flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            snap_step()
            a1.record(stream)
            sn_ms.append((a0, a1))
        torch.cuda.synchronize()
        sn_total = max_over_ranks(sum(a.elapsed_time(b) for a, b in sn_ms), world)
        snap = {"every_tokens": every, "snapshots_per_step": sum(counts) * H,
                "pool_bytes_written_per_step": sum(counts) * H * Dk * Dv * 4,
                "value": world * T * args.steps / (sn_total * 1e-3), "unit": "tokens/s",
                "ms_per_step": sn_total / args.steps,
                "overhead_vs_plain": sn_total / total_ms - 1.0}

    # ---- decode workload: 64 recurrent steps ------------------------------
    dec = None
    if not args.no_decode:
        dec = bench_decode(kda, dev, stream, world, args)

    # ---- roofline of the dominant kernel (prefill) -------------------------
    peaks, peaks_kind = load_peaks()
    roof = prefill_roofline(w, inp, sum(step_ms) / len(step_ms), peaks, peaks_kind)

    # ---- the other bf16 prefill workloads, each with its own roofline -----
    extra = {}
    if not args.no_extra:
        del d, out, sf, ws
        torch.cuda.empty_cache()
        for wid in (1, 2, 3):
            if wid != args.workload:
                extra[WORKLOADS[wid].name] = bench_extra_prefill(
                    kda, dev, stream, world, wid, flush, max(5, args.steps // 2), peaks,
                    peaks_kind)
                torch.cuda.empty_cache()

    # ---- backward (gradients) on the B2 T4096 H16 prefill workload ---------
    bwd = None
    if not args.no_backward:
        wb = WORKLOADS[1]
        ib = forward_inputs(wb)
        db = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in ib.items()}
        bwd = bench_backward(kda, dev, stream, world, wb, db, int(ib["cu_seqlens"][-1]),
                             len(ib["lengths"]), wb.H, wb.Dk, wb.Dv)
        del db
        torch.cuda.empty_cache()

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(w, inp, args.cpu_tokens)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.torch_dtype == torch.bfloat16 else "f32",
            "data": "synthetic (seeded generator; q,k L2-normalised, log_alpha uniform)",
            "config": {"workload": w.name, "num_seqs": N, "total_tokens": T, "H": H, "Dk": Dk,
                       "Dv": Dv, "chunk": 64, "state": "fp32",
                       "l2": "256 MiB flush between steps, outside the timed spans",
                       "parallelism": f"replicas x{world}"},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / args.steps,
                    "schedule": "pinned host buffers; step i+1 copies in while step i computes "
                                "and step i-1 copies out (two device buffer sets)"},
            # per call: varlen index, then the key-side and chain passes
            # (bf16, d = 128, full workspace) or the one CUDA-core kernel
            "gpu_launches": (3 if (w.torch_dtype == torch.bfloat16 and Dk == 128 and Dv == 128)
                             else 2) * args.steps,
            "roofline": roof,
            "cpu_baseline": cpu,
            "prefill_workloads": extra,
            "decode": dec,
            "backward": bwd,
            "snapshots": snap,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def bench_backward(kda, dev, stream, world, w, d, T, N, H, Dk, Dv, steps=3):
    """kda_backward on the prefill workload: dL/d out random, dL/dS_final and
    dL/dS0 included.  Two paths, each timed: the chunked tensor-core one (the
    default for bf16 with d = 128: the forward's two passes keeping every
    chunk's entering state, the reverse chain, the gradient assembly) and the
    fp32 CUDA-core one (token-level, 1e-4 accurate).

    Algorithmic work per token-head, counted once, is the same for both: the
    forward step 5 Dk Dv (decay, P^T k, rank-one write) and the reverse step
    16 Dk Dv flop; bytes: q, k, v, log_alpha, beta and d_out read once, dq,
    dk, dv, dlog_alpha (fp32) and dbeta written once, plus S0, dS_final and
    dS0.  At ~100 flop per byte both paths are bound by HBM under this count;
    the CUDA-core path's own roof is the fp32 FMA rate (148 SMs x 128 lanes x
    2 flop x the SM clock)."""
    g = torch.Generator(device=dev).manual_seed(5)
    d_out = torch.randn((T, H, Dv), generator=g, device=dev).to(w.torch_dtype)
    dSf = torch.randn((N, H, Dk, Dv), generator=g, device=dev)
    peaks, kind = load_peaks()
    flops = 21.0 * Dk * Dv * T * H
    io = _es(w.torch_dtype)
    moved = T * H * (3 * Dk * io + Dv * io + io + Dv * io + 3 * Dk * 4 + Dv * 4 + 4) + \
        3 * N * H * Dk * Dv * 4
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    alu_tflops = sms * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12

    def timed(force_simt, reps):
        ws = torch.empty(kda.backward_workspace_size(N, T, H, Dk, Dv, w.torch_dtype,
                                                     force_simt=force_simt),
                         dtype=torch.uint8, device=dev)

        def call():
            return kda.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                                d["cu_seqlens"], d_out=d_out, dS_final=dSf, workspace=ws,
                                force_simt=force_simt)

        for _ in range(2):
            call()
        if kda.workspace_status(ws) != 0:
            raise RuntimeError("device status not OK after the backward warm-up")
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            call()
        e1.record(stream)
        barrier(world)
        return max_over_ranks(e0.elapsed_time(e1), world) / reps

    tc = w.torch_dtype == torch.bfloat16 and Dk == 128 and Dv == 128
    ms_tc = timed(False, 10) if tc else None
    ms_f32 = timed(True, steps)
    out = {"workload": w.name,
           "grads": "dq, dk, dv, dlog_alpha, dbeta, dS0 (fp32); dS_final given",
           "algorithmic_flops": flops, "algorithmic_bytes": moved}
    if tc:
        gbs = moved / (ms_tc * 1e-3) / 1e9
        out["chunked_tc"] = {
            "value": world * T / (ms_tc * 1e-3), "unit": "tokens/s", "ms_per_call": ms_tc,
            "gpu_launches": 6 * 10,
            "kernels": "varlen_index, kside, chain (state store), rchain, assemble",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": traffic_record("kda_backward_tc"),
                         "peak_kind": f"{kind} HBM copy",
                         "tensor_frac_algorithmic": flops / (ms_tc * 1e-3) / 1e12 / peaks["bf16_tflops"]},
            "tolerance": "bf16: ||err||_F / ||oracle||_F <= 2e-2 per gradient"}
    achieved = flops / (ms_f32 * 1e-3) / 1e12
    out["fp32_cuda_cores"] = {
        "value": world * T / (ms_f32 * 1e-3), "unit": "tokens/s", "ms_per_call": ms_f32,
        "gpu_launches": 3 * steps,
        "roofline": {"bound": "alu", "achieved": achieved, "peak": alu_tflops, "unit": "TFLOP/s",
                     "frac": achieved / alu_tflops, "traffic": traffic_record("kda_backward"),
                     "peak_kind": "derived: fp32 FMA, SMs x 128 x 2 x max SM clock",
                     "hbm_frac_algorithmic": moved / (ms_f32 * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "tolerance": "fp32: relative 1e-4 per gradient"}
    return out


def bench_decode(kda, dev, stream, world, args):
    w = WORKLOADS[4]
    steps = w.decode_steps
    inp = decode_inputs(w)
    N, H, Dk, Dv = len(w.lengths), w.H, w.Dk, w.Dv
    x = {k: inp[k].to(dev) for k in ("q", "k", "v", "log_alpha", "beta")}
    S = inp["S"].to(dev)
    out = torch.empty((N, H, Dv), dtype=w.torch_dtype, device=dev)

    def run64():
        for t in range(steps):
            kda.decode_step(x["q"][t], x["k"][t], x["v"][t], x["log_alpha"][t], x["beta"][t], S,
                            out=out)

    for _ in range(3):
        run64()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record(stream)
    for _ in range(reps):
        run64()
    e1.record(stream)
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world) / (reps * steps)
    peaks, kind = load_peaks()
    b = decode_bytes(N, H, Dk, Dv, w.torch_dtype)
    gbs = b / (ms * 1e-3) / 1e9
    return {"workload": w.name, "value": world * N / (ms * 1e-3), "unit": "tokens/s",
            "us_per_step": ms * 1e3, "gpu_launches": reps * steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "frac_of_8TBs_nominal": gbs / 8000.0,
                         "traffic": traffic_record("kda_decode"), "algorithmic_bytes": b,
                         "peak_kind": f"{kind} HBM copy"},
            "state": "512 MiB fp32, larger than L2: no flush needed",
            "multi_token": bench_decode_multi(kda, dev, stream, world, x, S, w, peaks, kind)}


def bench_decode_multi(kda, dev, stream, world, x, S, w, peaks, kind, n=4):
    """Verify step of speculative decoding: n draft tokens per sequence in one
    pass over the state, the state after every token kept (kda_decode_multi)."""
    N, H, Dk, Dv = S.shape
    m = {k: x[k][:n].transpose(0, 1).contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
    out = torch.empty((N, n, H, Dv), dtype=w.torch_dtype, device=dev)
    S_tok = torch.empty((N, n, H, Dk, Dv), dtype=torch.float32, device=dev)

    def call():
        kda.decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], S, S_tokens=S_tok,
                         out=out)

    for _ in range(3):
        call()
    barrier(world)
    reps = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world) / reps
    esz = 2 if w.torch_dtype == torch.bfloat16 else 4
    # state read once, n states written, n tokens of q, k, v, log_alpha, beta, out
    b = N * H * (Dk * Dv * 4 * (1 + n) + n * esz * (3 * Dk + 2 * Dv + 1))
    gbs = b / (ms * 1e-3) / 1e9
    return {"draft_tokens": n, "value": world * N * n / (ms * 1e-3), "unit": "tokens/s",
            "us_per_call": ms * 1e3, "algorithmic_bytes": b,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "peak_kind": f"{kind} HBM copy"},
            "state": "S read once, the state after each draft token written (2.5 GiB per call)"}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=3, choices=[0, 1, 2, 3])
    ap.add_argument("--impl", default="kda", choices=["kda", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=4096,
                    help="oracle sample: first N tokens of each sequence")
    ap.add_argument("--ref-tokens", type=int, default=512,
                    help="reference arm: tokens per sequence in each timed step")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-snapshots", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lengths", type=lambda x: [int(v) for v in x.split(",")], default=None,
                    help="override the workload's sequence lengths (a reduced case, e.g. for ncu)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the extra prefill workloads (time only --workload)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return bench_reference(args)
    return bench_kda(args)


if __name__ == "__main__":
    sys.exit(main())
