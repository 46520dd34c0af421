"""Benchmark: bidirectional SSD scan throughput (tokens/s) at the DiffuMamba ~1.3B layer shape.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                    [--op fwd|bwd] [--batch B] [--dry-run]

One step is one full bidirectional scan call (forward + reverse + sum) over a
batch of synthetic seeded inputs already resident in HBM.  The default
workload is batch 4 x L 8192, 64 heads x headdim 64, d_state 128, chunk 256,
bf16 io with float32 state.  Under torchrun every rank runs its own batch of
the same size (independent sequences, no data-path collective: weak scaling);
the timed region is bracketed by a barrier and device synchronisation and the
reported time is the maximum over ranks.

The JSON line carries, besides the contract keys:
  roofline      algorithmic bytes of the dominant kernel per launch / its
                CUDA-event duration, against the measured HBM copy bandwidth
  cpu_baseline  the float64 oracle timed on this host's cores on a bounded
                sample of the same workload (rank 0, N = 1 only)
  e2e           the same metric through the public API with pinned host
                buffers, host->device inputs and device->host output copies
                inside the timed region
  clocks        SM clocks and throttle reasons sampled during the timed region
``--impl reference`` times the oracle alone (the CPU reference arm).
``--gpus N`` outside torchrun starts N rank processes itself (127.0.0.1
rendezvous); ``--dry-run`` runs only the host logic of the ranks (gloo
process group, shards, MAX reduction), without a GPU.
``--workload r2l_block_L32`` times the R2L sidecar decode: one step is 256
back-to-back denoising-step calls on fresh inputs, reported per call.
``--op bwd`` times the gradients of both directions (its own JSON line);
``--op mixer`` the whole Mamba-2 mixer layer around the scan (projections,
conv, scans, norms), against the bf16 tensor peak.  ``--batch`` replaces the batch
size, for small ncu captures.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import ssd_inputs as si  # noqa: E402

METRIC = "bidirectional SSD scan tokens/s at 1.3B shape L=8192; % of HBM/tensor roofline"
DEFAULT_WORKLOAD = "diffumamba_1p3b_L8192"
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------ accounting

def algorithmic_bytes_per_token(shape: si.Shape, directions: int = 2) -> int:
    """Bytes that must cross HBM once per token: each direction's x, dt, B, C read once, y written once."""
    e = 2 if shape.io == "bf16" else 4
    H, P, N, G = shape.nheads, shape.headdim, shape.dstate, shape.ngroups
    per_dir = e * (H * P + H + 2 * G * N)
    return directions * per_dir + e * H * P


def shard_plan(rank: int, world: int, workload: str, batch: int | None = None) -> dict:
    """Weak scaling: every rank owns one full batch of independent sequences, drawn with its own seed.

    ``batch`` replaces the workload's batch size (a smaller case of the same layer shape, for profiling)."""
    w = si.WORKLOADS[workload]
    shape = w["shape"] if batch is None else dataclasses.replace(w["shape"], batch=batch)
    return {"rank": rank, "world": world, "seed": rank, "shape": shape, "chunk": w["chunk"],
            "tokens": shape.tokens}


def max_over_ranks(value: float, dist) -> float:
    """Maximum of a per-rank float over the process group (the slowest rank sets the time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    backend = dist.get_backend()
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls NVML for SM clock and clock-event (throttle) reasons in a background thread."""
    REASONS = {0x2: "applications_clocks", 0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clocks"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop, self._th, self._h = period_s, threading.Event(), None, None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._th = threading.Thread(target=self._run, daemon=True)
            self._th.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._th is not None:
            self._th.join()

    def summary(self) -> dict:
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ peaks and profiles

def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def _kernel_source_hash() -> str:
    """Hash of the tensor-core kernels' sources and build flags: a traffic record is valid only for
    the kernel it measured.

    Comments and whitespace are left out, so that editing a comment keeps the record of an
    unchanged kernel; the nvcc architecture and flags are part of the key."""
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "bidirectional_mamba_ssd_bidir_b200")
    for f in ("ssd_tcs.cu", "ssd_tcs_seg.cu", "ssd_tc.cu", "ssd_tc.cuh", "ssd_tc_common.cuh"):
        h.update(_code_only(open(os.path.join(pkg, "csrc", f), encoding="utf-8").read()).encode())
    import importlib.util
    spec = importlib.util.spec_from_file_location("_ssd_build_flags", os.path.join(pkg, "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    h.update(" ".join(mod.ARCH + mod.FLAGS).encode())
    return h.hexdigest()[:16]


def _code_only(text: str) -> str:
    """C/CUDA source without its comments, whitespace runs collapsed to one space."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def profiled_traffic(kernel: str, workload: str, prof: str | None = None):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current kernel source."""
    prof = prof or os.path.join(ROOT, "profiles")
    if not os.path.isdir(prof):
        return None
    src_hash = _kernel_source_hash()
    for f in sorted(os.listdir(prof)):
        if not f.endswith(".md"):
            continue
        text = open(os.path.join(prof, f)).read()
        m = re.search(r"traffic-record: kernel=(\S+) workload=(\S+) source=(\S+) bytes_per_launch=(\d+)", text)
        if m and m.group(1) == kernel and m.group(2) == workload and m.group(3) == src_hash:
            return int(m.group(4))
    return None


# ------------------------------------------------------------------ CPU oracle

def oracle_sample(shape: si.Shape, seed: int, heads: int, seqlen: int | None = None):
    """Inputs for a bounded sample of the workload: batch 0, the first ``heads`` heads, the first ``seqlen`` tokens."""
    import numpy as np
    L = seqlen or shape.seqlen
    sub = si.Shape(1, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups, shape.io)
    pf, pr = si.make_bidir(sub, seed=seed)
    import oracle
    out = []
    for p in (pf, pr):
        q = oracle.params_f64(p)
        q = {"x": np.ascontiguousarray(q["x"][:, :L, :heads]), "dt": np.ascontiguousarray(q["dt"][:, :L, :heads]),
             "A": q["A"][:heads], "B": np.ascontiguousarray(q["B"][:, :L]), "C": np.ascontiguousarray(q["C"][:, :L]),
             "D": q["D"][:heads]}
        out.append(q)
    return out


def time_oracle(shape: si.Shape, seed: int, heads: int, seqlen: int | None = None, repeats: int = 1):
    import oracle
    qf, qr = oracle_sample(shape, seed, heads, seqlen)
    L = qf["x"].shape[1]
    threads = oracle.default_threads()
    oracle.bidir_f64(qf, qr, nthreads=threads)                        # warm the library
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        oracle.bidir_f64(qf, qr, nthreads=threads)
        times.append(time.perf_counter() - t0)
    # tokens/s of the whole workload: the sample covers heads/H of each of L tokens
    tok_per_s = [L * heads / shape.nheads / t for t in times]
    return tok_per_s, threads, L


def cpu_baseline(shape: si.Shape, target_s: float = 15.0) -> dict:
    """Times the oracle on a bounded sample: batch 0, all tokens, as many heads as ~target_s of CPU work allows."""
    import oracle
    cores = oracle.default_threads()
    qf, qr = oracle_sample(shape, 0, 1)
    t0 = time.perf_counter()
    oracle.bidir_f64(qf, qr, nthreads=1)
    one_head = max(time.perf_counter() - t0, 1e-4)            # CPU seconds for one head, both directions
    heads = int(min(shape.nheads, max(1, round(target_s / one_head))))
    if heads >= cores:
        heads -= heads % cores                                 # whole rounds of threads
    tps, threads, L = time_oracle(shape, 0, heads)
    return {"value": tps[0], "unit": "tokens/s", "cores": min(threads, heads), "kind": "oracle",
            "sample": f"float64 recurrence, both directions, batch 0, {heads} of {shape.nheads} heads, "
                      f"all {L} tokens (about {heads * one_head:.0f} s of CPU work); "
                      f"tokens/s scaled by heads/{shape.nheads}"}


# ------------------------------------------------------------------ our arm

def run_ours(args) -> None:
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    import bidirectional_mamba_ssd_bidir_b200 as ssd

    plan = shard_plan(rank, world, args.workload, args.batch)
    shape, chunk = plan["shape"], plan["chunk"]
    pf, pr = si.make_bidir(shape, seed=plan["seed"])
    host = {}
    for tag, p in (("f", pf), ("r", pr)):
        for k in ("x", "dt", "A", "B", "C", "D"):
            host[tag + k] = getattr(p, k).torch().pin_memory()
    devt = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    fwd = {k: devt["f" + k] for k in ("x", "dt", "A", "B", "C", "D")}
    rev = {k: devt["r" + k] for k in ("x", "dt", "A", "B", "C", "D")}
    y = torch.empty_like(fwd["x"])
    dims = (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups)
    ws = torch.zeros(max(256, ssd.workspace_bytes(dims, fwd["x"].dtype, chunk)), dtype=torch.uint8, device=dev)
    path = ssd.path_for(dims, fwd["x"].dtype, chunk)
    launches_per_step = ssd.kernel_launches(dims, fwd["x"].dtype, chunk, "bidir")
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize()

    def step():
        ssd.bidir_ssd(fwd, rev, chunk=chunk, out=y, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-timed region: inputs resident in HBM, larger than L2
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    per_launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ssd.workspace_status(ws)
    total_ms = max_over_ranks(total_ms, dist)
    ms_per_step = total_ms / args.steps
    tokens_all = plan["tokens"] * world
    value = tokens_all / (ms_per_step / 1e3)

    # ---- end to end through the public API with host buffers.  Every step copies its inputs in
    # from pinned host memory and its output back out.  Two device slots let one step's inputs
    # cross PCIe on the host-to-device copy engine while the previous step's output returns on
    # the device-to-host engine and the call in between runs; events order each slot's copy-in,
    # call and copy-out.
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y.numel() * y.element_size()
    e2e_steps = max(2, min(args.steps, 20))
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    slots = []
    for i in range(2):
        d = devt if i == 0 else {k: torch.empty_like(v) for k, v in devt.items()}
        slots.append({"dev": d, "y": y if i == 0 else torch.empty_like(y),
                      "out": torch.empty(y.shape, dtype=y.dtype).pin_memory(),
                      "in_done": torch.cuda.Event(), "cmp_done": torch.cuda.Event(), "out_done": torch.cuda.Event()})
    torch.cuda.synchronize()

    def e2e_step(i):
        sl = slots[i % 2]
        if i >= 2:
            s_in.wait_event(sl["cmp_done"])          # the call two steps back has read this slot
        with torch.cuda.stream(s_in):
            for k, v in host.items():
                sl["dev"][k].copy_(v, non_blocking=True)
            sl["in_done"].record(s_in)
        s_cmp.wait_event(sl["in_done"])
        if i >= 2:
            s_cmp.wait_event(sl["out_done"])         # this slot's previous output has left
        with torch.cuda.stream(s_cmp):
            ssd.bidir_ssd({k: sl["dev"]["f" + k] for k in ("x", "dt", "A", "B", "C", "D")},
                          {k: sl["dev"]["r" + k] for k in ("x", "dt", "A", "B", "C", "D")},
                          chunk=chunk, out=sl["y"], workspace=ws)
            sl["cmp_done"].record(s_cmp)
        s_out.wait_event(sl["cmp_done"])
        with torch.cuda.stream(s_out):
            sl["out"].copy_(sl["y"], non_blocking=True)
            sl["out_done"].record(s_out)

    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    e2.record(s_out)                                 # after the last copy-out, which follows everything
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(s2.elapsed_time(e2), dist) / e2e_steps
    e2e_value = tokens_all / (e2e_ms / 1e3)

    if rank == 0:
        peaks = measured_peaks()
        bpt = algorithmic_bytes_per_token(shape)
        alg_bytes = bpt * plan["tokens"]
        achieved = alg_bytes / (per_launch_ms / 1e3) / 1e9
        kernel = "ssd_bidir_tc" if path == 1 else "simt_call(6 kernels)"
        line = {
            "metric": METRIC if args.workload == DEFAULT_WORKLOAD else f"bidirectional SSD scan tokens/s, {args.workload}",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if shape.io == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": args.workload, "global_batch": shape.batch * world, "seq_len": shape.seqlen,
                       "nheads": shape.nheads, "headdim": shape.headdim, "dstate": shape.dstate,
                       "ngroups": shape.ngroups, "chunk": chunk, "parallelism": f"dp{world} (independent sequences)",
                       "path": "tcgen05" if path == 1 else "simt",
                       "l2": f"inputs+output {alg_bytes / 1e6:.0f} MB per step > L2 {L2_BYTES / 1e6:.0f} MB, no flush"},
            "roofline": {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": profiled_traffic(kernel, args.workload),
                         "algorithmic_bytes_per_launch": alg_bytes, "bytes_per_token": bpt,
                         "launch_ms": per_launch_ms, "peak_source": peaks["source"] + " hbm_gbs"},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "overlap": "copy-in, call and copy-out of consecutive steps overlap (two device slots)"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(shape, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_mixer(args) -> None:
    """The whole DiffuMamba mixer layer (two Mamba-2 layers around the scan), one GPU, device-timed,
    plus the same call end to end from pinned host memory."""
    import torch
    import bidirectional_mamba_ssd_bidir_b200 as ssd
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = si.WORKLOADS[args.workload]
    base = w["shape"]
    batch = base.batch if args.batch is None else args.batch
    H, P, N = base.nheads, base.headdim, base.dstate
    ms_ = si.MixerShape(batch=batch, seqlen=base.seqlen, d_model=H * P // 2, nheads=H, headdim=P, dstate=N)
    u, f, r = si.make_mixer(ms_, seed=0)
    u_h = u.torch().pin_memory()
    u_d = u_h.to(dev)
    fd = {k: v.torch(dev) for k, v in f.items()}
    rd = {k: v.torch(dev) for k, v in r.items()}
    ws = torch.zeros(ssd.mixer_workspace_bytes(ms_.batch, ms_.seqlen, ms_.d_model, H), dtype=torch.uint8, device=dev)
    out = torch.empty_like(u_d)

    def step():
        ssd.mixer_bidir(u_d, fd, rd, H, out=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    with ClockSampler(0) as clk:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize()
    ssd.workspace_status(ws)
    ms = start.elapsed_time(end) / args.steps
    tokens = ms_.tokens
    # end to end: u in from pinned host memory, the output back, every step
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_steps = max(2, min(args.steps, 10))
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(e2e_steps):
        u_d.copy_(u_h, non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
    e2.record(stream)
    torch.cuda.synchronize()
    e2e_ms = s2.elapsed_time(e2) / e2e_steps
    # tensor work per token: both layers' input projections, the output projection over both
    # layers' inner dimension, and the scan's products (16.8 MFLOP per 128 tokens and head pair
    # per direction, shared scores)
    dm, di, dinp = ms_.d_model, ms_.d_inner, ms_.d_in_proj
    fpt = 2 * 2 * dinp * dm + 2 * dm * 2 * di + 2 * (H // 2) * 16.8e6 / 128
    peaks = measured_peaks()
    achieved = fpt * tokens / (ms / 1e3) / 1e12
    line = {"metric": f"DiffuMamba bidirectional Mamba-2 mixer layer tokens/s, {args.workload} (d_model {dm})",
            "op": "mixer", "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "global_batch": batch, "seq_len": ms_.seqlen, "d_model": dm,
                       "d_inner": di, "nheads": H, "dstate": N, "d_conv": ms_.d_conv, "path": "tcgen05"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "flops_per_token": fpt,
                         "peak_source": peaks["source"] + " bf16_tflops (dense, burst)",
                         "note": "whole layer: two input projections, conv, two scans, two norms, output projection"},
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": u_h.numel() * 2, "d2h_bytes_per_step": out_h.numel() * 2,
                    "overlap": "none: copy-in, call and copy-out in order on one stream"},
            "gpu_launches": args.steps * (2 * (3 + ssd.kernel_launches(
                (batch, ms_.seqlen, H, P, N, 1), torch.bfloat16, 256 if ms_.seqlen % 256 == 0 else 128, "scan")) + 1),
            "clocks": clk.summary()}
    if not args.no_cpu_baseline:
        import oracle
        from oracle import mixer as om
        Ls = min(ms_.seqlen, 512)
        small = si.MixerShape(batch=1, seqlen=Ls, d_model=dm, nheads=H, headdim=P, dstate=N)
        uf = u.f64()[:1, :Ls]
        ff, rf = om.layer_to_f64(f), om.layer_to_f64(r)
        t0 = time.perf_counter()
        om.mixer_bidir_f64(uf, ff, rf, small)
        cpu_s = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": Ls / cpu_s, "unit": "tokens/s", "cores": oracle.default_threads(),
                                "kind": "oracle",
                                "sample": f"float64 mixer (numpy projections, C recurrence), batch 0, first {Ls} tokens"}
    print(json.dumps(line), flush=True)


def run_attention(args) -> None:
    """The DiffuMamba-H attention block (q/k/v projection, unmasked softmax attention, output
    projection), one GPU, device-timed, plus the attention kernel alone for its roofline and the
    block end to end from pinned host memory."""
    import torch
    import bidirectional_mamba_ssd_bidir_b200 as ssd
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    base = si.WORKLOADS[args.workload]["shape"]
    batch = base.batch if args.batch is None else args.batch
    dm = base.nheads * base.headdim // 2            # the layer width of the model the workload belongs to
    D = 128
    shape = si.AttnShape(batch, base.seqlen, dm // D, D, d_model=dm)
    H, L = shape.nheads, shape.seqlen
    u, wqkv, wo = si.make_attention_layer(shape, seed=0)
    u_h = u.torch().pin_memory()
    u_d, wqkv_d, wo_d = u_h.to(dev), wqkv.torch(dev), wo.torch(dev)
    ws = torch.zeros(ssd.attention_block_workspace_bytes(batch, L, H, D), dtype=torch.uint8, device=dev)
    out = torch.empty_like(u_d)

    def step():
        ssd.attention_block(u_d, wqkv_d, wo_d, H, D, out=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    with ClockSampler(0) as clk:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize()
    ssd.workspace_status(ws)
    ms = start.elapsed_time(end) / args.steps
    tokens = batch * L
    # the attention kernel alone, on the block's own q/k/v (the packed projection in the workspace)
    qkv = ws[256:256 + tokens * 3 * H * D * 2].view(torch.bfloat16).view(batch, L, 3, H, D)
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    o = torch.empty(batch, L, H, D, dtype=torch.bfloat16, device=dev)
    aws = torch.zeros(256, dtype=torch.uint8, device=dev)
    for _ in range(2):
        ssd.attention(q, k, v, out=o, workspace=aws)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        ssd.attention(q, k, v, out=o, workspace=aws)
    a1.record(stream)
    torch.cuda.synchronize()
    ssd.workspace_status(aws)
    attn_ms = a0.elapsed_time(a1) / args.steps
    # end to end: u in from pinned host memory, the output back, every step
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_steps = max(2, min(args.steps, 10))
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(e2e_steps):
        u_d.copy_(u_h, non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
    e2.record(stream)
    torch.cuda.synchronize()
    e2e_ms = s2.elapsed_time(e2) / e2e_steps
    attn_flops = 4.0 * batch * H * L * L * D          # Q K^T and P V, multiply-adds counted twice
    peaks = measured_peaks()
    achieved = attn_flops / (attn_ms / 1e3) / 1e12
    line = {"metric": f"DiffuMamba-H attention block tokens/s, {args.workload} shape (d_model {dm}, {H} heads x {D})",
            "op": "attention", "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{args.workload} attention block", "global_batch": batch, "seq_len": L,
                       "d_model": dm, "nheads": H, "headdim": D, "mask": "none (bidirectional)", "path": "tcgen05"},
            "roofline": {"bound": "tensor", "kernel": "k_attention", "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                         "flops_per_launch": attn_flops, "launch_ms": attn_ms,
                         "peak_source": peaks["source"] + " bf16_tflops (dense, burst)"},
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": u_h.numel() * 2, "d2h_bytes_per_step": out_h.numel() * 2,
                    "overlap": "none: copy-in, call and copy-out in order on one stream"},
            "gpu_launches": 3 * args.steps,
            "clocks": clk.summary()}
    if not args.no_cpu_baseline:
        import numpy as np
        import oracle
        from oracle import attention as oa
        R = 256
        uf, wq, wof = u.f64()[0], wqkv.f64(), wo.f64()
        t0 = time.perf_counter()
        kv = uf @ wq[H * D:].T                              # keys and values of all L tokens
        t1 = time.perf_counter()
        qr = (uf[:R] @ wq[:H * D].T).reshape(1, R, H, D)
        kk = kv[:, :H * D].reshape(1, L, H, D)
        vv = kv[:, H * D:].reshape(1, L, H, D)
        rows = oa.attention_rows_f64(qr, kk, vv, [(0, i, h) for i in range(R) for h in range(H)])
        np.asarray(rows).reshape(R, H * D) @ wof.T
        t2 = time.perf_counter()
        per_token = (t1 - t0) / L + (t2 - t1) / R
        line["cpu_baseline"] = {"value": 1.0 / per_token, "unit": "tokens/s", "cores": oracle.default_threads(),
                                "kind": "oracle",
                                "sample": f"float64 block on batch 0: k/v projection of all {L} tokens (cost per "
                                          f"token) + q projection, attention rows over {L} keys and output "
                                          f"projection of the first {R} tokens (cost per token)"}
    print(json.dumps(line), flush=True)


def run_r2l(args) -> None:
    """R2L sidecar decode: 256 denoising steps back to back, each a fresh block of inputs.

    One bench step is the 256 calls; the metric is microseconds per denoising-step call (lower
    is better).  Every call's inputs are generated up front and resident on the device."""
    import torch
    import torch.distributed as dist
    import bidirectional_mamba_ssd_bidir_b200 as ssd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    w = si.WORKLOADS[args.workload]
    shape, chunk, nsteps = w["shape"], w["chunk"], w["steps"]
    if args.batch is not None:
        shape = dataclasses.replace(shape, batch=args.batch)
    seed = rank
    host, dev_in, gates = [], [], []
    for st in range(nsteps):
        p = si.make_params(shape, seed=seed, offset=si.STEP_STRIDE * st + si.REV_OFFSET)
        h = {k: getattr(p, k).torch().pin_memory() for k in ("x", "dt", "A", "B", "C", "D")}
        h["res"] = si.make_residual(shape, seed=seed, step=st).torch().pin_memory()
        host.append(h)
        dev_in.append({k: v.to(dev, non_blocking=True) for k, v in h.items()})
        gates.append(si.make_gate(seed, st))
    outs = [torch.empty_like(d["res"]) for d in dev_in]
    dims = (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups)
    ws = torch.zeros(max(256, ssd.workspace_bytes(dims, torch.bfloat16, chunk)), dtype=torch.uint8, device=dev)
    path = ssd.path_for(dims, torch.bfloat16, chunk)
    per_call = ssd.kernel_launches(dims, torch.bfloat16, chunk, "r2l")
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize()

    def one_pass():
        for st in range(nsteps):
            d = dev_in[st]
            ssd.r2l_block_scan(d, gates[st], d["res"], chunk=chunk, out=outs[st], workspace=ws)

    for _ in range(args.warmup):
        one_pass()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with ClockSampler(local) as clk:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            one_pass()
        end.record(stream)
        torch.cuda.synchronize()
    ssd.workspace_status(ws)
    total_ms = max_over_ranks(start.elapsed_time(end), dist)
    us_per_call = total_ms * 1e3 / (args.steps * nsteps)

    # end to end: each call's inputs copied in from pinned host memory and its output copied back,
    # in order on one stream (a decode loop needs each step's output before the next step)
    outs_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs[:2]]
    h2d = sum(v.numel() * v.element_size() for v in host[0].values())
    d2h = outs[0].numel() * outs[0].element_size()
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for st in range(nsteps):
        d = dev_in[st]
        for k, v in host[st].items():
            d[k].copy_(v, non_blocking=True)
        ssd.r2l_block_scan(d, gates[st], d["res"], chunk=chunk, out=outs[st], workspace=ws)
        outs_h[st % 2].copy_(outs[st], non_blocking=True)
    e2.record(stream)
    torch.cuda.synchronize()
    e2e_us = max_over_ranks(s2.elapsed_time(e2), dist) * 1e3 / nsteps

    if rank == 0:
        peaks = measured_peaks()
        bpt = algorithmic_bytes_per_token(shape, directions=1) + 2 * shape.nheads * shape.headdim  # + residual
        alg_bytes = bpt * shape.tokens
        achieved = alg_bytes / (us_per_call / 1e6) / 1e9
        line = {
            "metric": "R2L sidecar block scan, microseconds per denoising step (256 steps back to back)",
            "value": us_per_call, "unit": "us", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "global_batch": shape.batch * world, "seq_len": shape.seqlen,
                       "nheads": shape.nheads, "headdim": shape.headdim, "dstate": shape.dstate, "chunk": chunk,
                       "calls_per_step": nsteps, "parallelism": f"dp{world} (independent decodes)",
                       "path": "tcgen05" if path == 1 else "simt",
                       "l2": "inputs of all 256 calls resident, no flush (a decode loop's inputs are hot)"},
            "roofline": {"bound": "hbm", "kernel": "r2l_call", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_launch": alg_bytes, "bytes_per_token": bpt,
                         "launch_us": us_per_call, "peak_source": peaks["source"] + " hbm_gbs",
                         "note": "latency-bound: a few MB per call, one launch of the single-chunk kernel per call"},
            "e2e": {"value": e2e_us, "unit": "us", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": nsteps, "overlap": "none: each call's copies and call in order on one stream"},
            "gpu_launches": per_call * nsteps * args.steps,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            cores = oracle.default_threads()
            n = 0
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < min(args.cpu_seconds, 10.0) and n < nsteps:
                p = si.make_params(shape, seed=seed, offset=si.STEP_STRIDE * n + si.REV_OFFSET)
                oracle.r2l_block_f64(oracle.params_f64(p), gates[n],
                                     si.make_residual(shape, seed=seed, step=n).f64())
                n += 1
            cpu_us = (time.perf_counter() - t0) * 1e6 / n
            line["cpu_baseline"] = {"value": cpu_us, "unit": "us", "cores": cores, "kind": "oracle",
                                    "sample": f"float64 r2l block, the first {n} of {nsteps} steps, whole block "
                                              "(input generation included)"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_dry(args) -> None:
    """Host logic of a multi-rank run, without a GPU: gloo process group, each rank's shard,
    and the MAX reduction of a per-rank time (rank r reports 1 + r: the slowest sets the line)."""
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    plan = shard_plan(rank, world, args.workload, args.batch)
    t = max_over_ranks(1.0 + rank, dist if world > 1 else None)
    mine = (rank, plan["seed"], plan["tokens"])
    ranks = [mine]
    if world > 1:
        ranks = [None] * world
        dist.all_gather_object(ranks, mine)
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_ranks": world, "ranks": ranks, "max_time": t,
                          "tokens_all": sum(r[2] for r in ranks)}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_entry(index: int, world: int, port: int, argv: list) -> None:
    os.environ.update(RANK=str(index), LOCAL_RANK=str(index), WORLD_SIZE=str(world), LOCAL_WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    main(argv)


def spawn_ranks(n: int, argv: list) -> None:
    """Start n rank processes (one per GPU), as torchrun would, and wait for them."""
    import torch.multiprocessing as mp
    mp.start_processes(_rank_entry, args=(n, _free_port(), list(argv)), nprocs=n, start_method="spawn", join=True)


# ------------------------------------------------------------------ reference arm (the oracle)

def run_bwd(args) -> None:
    """Gradients of the bidirectional mixer (both directions, the same dL/dy), one GPU, device-timed."""
    import torch
    import bidirectional_mamba_ssd_bidir_b200 as ssd
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    plan = shard_plan(0, 1, args.workload, args.batch)
    shape, chunk = plan["shape"], plan["chunk"]
    pf, pr = si.make_bidir(shape, seed=0)
    fwd = {k: getattr(pf, k).torch(dev) for k in ("x", "dt", "A", "B", "C", "D")}
    rev = {k: getattr(pr, k).torch(dev) for k in ("x", "dt", "A", "B", "C", "D")}
    gy = torch.randn(fwd["x"].shape, device=dev).to(fwd["x"].dtype)
    dims = (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups)
    s_ = ssd._Shape(*dims, ssd.SSD_BF16 if shape.io == "bf16" else ssd.SSD_F32)
    ws = torch.zeros(int(ssd.lib.ssd_bwd_workspace_bytes(ssd.ctypes.byref(s_), chunk)), dtype=torch.uint8, device=dev)

    def step():
        ssd.ssd_scan_bwd(**fwd, gy=gy, direction=1, chunk=chunk, workspace=ws)
        ssd.ssd_scan_bwd(**rev, gy=gy, direction=-1, chunk=chunk, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    with ClockSampler(0) as clk:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize()
    ms = start.elapsed_time(end) / args.steps
    e = 2 if shape.io == "bf16" else 4
    H, P, N, G = shape.nheads, shape.headdim, shape.dstate, shape.ngroups
    path = ssd.path_for(dims, fwd["x"].dtype, chunk)
    # per token and direction: read x, dt, B, C, gy; write float32 dx, ddt, dB, dC
    bpt = 2 * (e * (2 * H * P + H + 2 * G * N) + 4 * (H * P + H + 2 * G * N))
    clocks = clk.summary()
    if path == 1:
        # tensor-core chunks of Q = 128: multiply-adds per token, head and direction of the dense
        # tiles the kernels compute (the hi/lo operand halves not counted): the pair products
        # C.B^T, B.C^T (2 Q N) and x.gy^T, gy.x^T (2 Q P); the adjoint times gy and times B
        # (Q P + N P); dB and dC, in-chunk and entering parts (2 Q N + 2 P N); the chunk sums
        # (2 P N)
        Q = 128
        macs = 2 * Q * N + 2 * Q * P + Q * P + N * P + 2 * Q * N + 2 * P * N + 2 * P * N
        fpt = 2 * 2 * H * macs
        peaks = measured_peaks()
        peak_tf = peaks["bf16_tflops"]
        achieved = fpt * plan["tokens"] / (ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved / peak_tf, "flops_per_token": fpt,
                "peak_source": peaks["source"] + " bf16_tflops (dense, burst)",
                "hbm_bytes_per_token": bpt, "hbm_gbs": bpt * plan["tokens"] / (ms / 1e3) / 1e9,
                "note": "whole step: the tensor-core chunk kernels with the float32 chunk passes, "
                        "ddt sums and reductions"}
    else:
        Q = min(chunk, 64)
        # float32 multiply-adds of the chunked gradient per token, head and direction: chunk state
        # and adjoint sums 2PN; pair matrices C.B^T and x.gy^T Q(N + P); the adjoint times B,
        # entering part PN and causal in-chunk part QP/2; dB and dC, entering parts 2PN and causal
        # in-chunk parts 2 QN/2
        macs = 5 * P * N + 2 * Q * N + 1.5 * Q * P
        fpt = 2 * 2 * H * macs                       # flops per token, both directions
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        mhz = clocks.get("sm_max_mhz") or 1965
        peak_tf = sms * 128 * 2 * mhz * 1e6 / 1e12   # float32 FMA lanes per SM, 2 flops each
        achieved = fpt * plan["tokens"] / (ms / 1e3) / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved / peak_tf, "flops_per_token": fpt,
                "peak_source": f"derived: {sms} SMs x 128 float32 lanes x 2 flops x {mhz} MHz",
                "hbm_bytes_per_token": bpt, "hbm_gbs": bpt * plan["tokens"] / (ms / 1e3) / 1e9}
    line = {"metric": "bidirectional SSD scan gradients tokens/s (both directions)", "op": "bwd",
            "value": plan["tokens"] / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "f32",
            "data": "synthetic", "config": {"workload": args.workload, "global_batch": shape.batch,
                                             "seq_len": shape.seqlen, "chunk": chunk,
                                             "path": "tcgen05" if path == 1 else "simt"},
            "roofline": roof, "gpu_launches": 2 * 5 * args.steps, "clocks": clocks}
    print(json.dumps(line), flush=True)


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = si.WORKLOADS[args.workload]
    shape = w["shape"]
    import oracle
    cores = oracle.default_threads()
    if w["kind"] == "r2l":
        # the R2L decode: the float64 block per denoising step, inputs generated before the clock
        nsteps = w["steps"]
        per_step = max(1, min(nsteps, 16))
        steps_in = [(oracle.params_f64(si.make_params(shape, seed=0, offset=si.STEP_STRIDE * st + si.REV_OFFSET)),
                     si.make_gate(0, st), si.make_residual(shape, seed=0, step=st).f64()) for st in range(per_step)]
        for _ in range(args.warmup):
            oracle.r2l_block_f64(*steps_in[0])
        t0 = time.perf_counter()
        for _ in range(args.steps):
            for q, g, r in steps_in:
                oracle.r2l_block_f64(q, g, r)
        us = (time.perf_counter() - t0) * 1e6 / (args.steps * per_step)
        sample = f"float64 r2l block, the first {per_step} of {nsteps} denoising steps per bench step"
        line = {"metric": "R2L sidecar block scan, microseconds per denoising step (256 steps back to back)",
                "value": us, "unit": "us", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": us * nsteps / 1e3, "higher_is_better": False, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": args.workload, "global_batch": shape.batch, "seq_len": shape.seqlen,
                           "nheads": shape.nheads, "headdim": shape.headdim, "dstate": shape.dstate,
                           "chunk": w["chunk"], "calls_per_step": nsteps, "parallelism": "host cores"},
                "cpu_baseline": {"value": us, "unit": "us", "cores": cores, "kind": "oracle", "sample": sample},
                "e2e": {"value": us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    # size each step so that warmup + steps stay within ~args.ref_budget seconds
    per_step_budget = max(0.05, args.ref_budget / max(1, args.steps + args.warmup))
    probe, _, _ = time_oracle(shape, 0, min(cores, shape.nheads), seqlen=min(shape.seqlen, 1024))
    # probe throughput in "whole-workload tokens per second" -> seconds per token per head
    sec_per_tok_head = 1.0 / (probe[0] * shape.nheads)
    heads = min(shape.nheads, max(1, cores))
    L = int(min(shape.seqlen, max(64, per_step_budget / (sec_per_tok_head * heads))))
    qf, qr = oracle_sample(shape, 0, heads, L)
    for _ in range(args.warmup):
        oracle.bidir_f64(qf, qr, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.bidir_f64(qf, qr, nthreads=cores)
    dt = (time.perf_counter() - t0) / args.steps
    value = L * heads / shape.nheads / dt
    sample = (f"float64 recurrence, both directions, batch 0, {heads} of {shape.nheads} heads, first {L} of "
              f"{shape.seqlen} tokens per step; tokens/s scaled by heads/{shape.nheads}")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "global_batch": shape.batch, "seq_len": shape.seqlen,
                       "nheads": shape.nheads, "headdim": shape.headdim, "dstate": shape.dstate,
                       "chunk": w["chunk"], "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(si.WORKLOADS))
    ap.add_argument("--batch", type=int, default=None,
                    help="replace the workload's batch size (a smaller case of the same shape, for profiling)")
    ap.add_argument("--op", choices=["fwd", "bwd", "mixer", "attention"], default="fwd",
                    help="bwd: the gradients of both directions; mixer: the whole Mamba-2 mixer layer around the "
                         "scan; attention: the DiffuMamba-H attention block (extra lines, one GPU)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU work of the oracle baseline sample")
    ap.add_argument("--ref-budget", type=float, default=90.0, help="seconds for the reference arm's steps")
    ap.add_argument("--dry-run", action="store_true",
                    help="host logic of the ranks only (gloo group, shards, MAX reduction), no GPU")
    argv = sys.argv[1:] if argv is None else list(argv)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        spawn_ranks(args.gpus, argv)
        return
    if args.dry_run:
        run_dry(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.op == "bwd":
        run_bwd(args)
    elif args.op == "mixer":
        run_mixer(args)
    elif args.op == "attention":
        run_attention(args)
    elif si.WORKLOADS[args.workload]["kind"] == "r2l":
        run_r2l(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
