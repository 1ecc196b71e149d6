"""Benchmark of the Muon optimizer step on B200 (one JSON line on rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama7b|...] [--impl ours|reference]

Default workload: the Llama-7B-shaped layer set (32 layers x {4 x 4096x4096,
4096x14336, 14336x4096}; 71 GB of fp32 W, M, G resident in HBM), Newton-Schulz
in bf16 with T = 5, one batched step per iteration, NorMuon off for `value`
and timed on as well under `normuon_on`. Under torchrun every rank runs its
own replica of the step (the path has no cross-matrix exchange); the
reported time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only other arm) on a bounded
sample of the same workload, scaled to the whole step.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from newton_schulz_10_b200 import inputs  # noqa: E402

METRIC = "Muon optimizer step ms/step; NS GEMM TFLOP/s vs B200 bf16 peak; HBM GB/s"
COEFFS = (3.4445, -4.7750, 2.0315)

# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

WORKLOADS = {
    "single256x1024": dict(desc="single 256x1024 fp32 matrix, fp32 Newton-Schulz (T=5), one step",
                           compute="f32", gram=False, normuon=False, dion3=None),
    "gpt124m": dict(desc="GPT-124M layer set: 12 x (4 x 768x768, 768x3072, 3072x768), bf16 NS T=5",
                    compute="bf16", gram=False, normuon=False, dion3=None),
    "dion3_8192x28672": dict(desc="8192x28672, Dion3 f=1/4 (l1 rows) + NorMuon, Gram NS fp16 (restart 3), T=5",
                             compute="f16", gram=True, normuon=True, dion3=(1, 4)),
    "llama7b": dict(desc="Llama-7B layer set: 32 x (4 x 4096x4096, 4096x14336, 14336x4096), bf16 NS T=5",
                    compute="bf16", gram=False, normuon=False, dion3=None),
    "llama7b_layer": dict(desc="one layer of the Llama-7B set: 4 x 4096x4096, 4096x14336, 14336x4096, bf16 NS T=5 "
                               "(profiling case: per-launch traffic x 32 = the full set's)",
                          compute="bf16", gram=False, normuon=False, dion3=None),
    "llama_mlp_4096x14336": dict(desc="one Llama-7B MLP matrix 4096x14336, bf16 NS T=5 (profiling case)",
                                 compute="bf16", gram=False, normuon=False, dion3=None),
    "llama7b_normuon": dict(desc="Llama-7B layer set, bf16 NS T=5, NorMuon on",
                            compute="bf16", gram=False, normuon=True, dion3=None),
    "llama7b_gram": dict(desc="Llama-7B layer set, Gram NS fp16 (restart 3), T=5: the Gram reformulation on "
                              "the same 192 matrices",
                         compute="f16", gram=True, normuon=False, dion3=None),
    "llama7b_gram_layer": dict(desc="one layer of the Llama-7B set, Gram NS fp16 (restart 3), T=5 (profiling case: "
                                    "per-launch traffic x 32 = the full set's)",
                               compute="f16", gram=True, normuon=False, dion3=None),
    "spectrum4096x16384": dict(desc="one 4096x16384 bf16 matrix, singular values log-uniform in [1e-4, 1]: "
                                    "Gram NS (fp16, restart 3) vs standard NS (bf16 and fp16), T=5",
                               compute="f16", gram=True, normuon=False, dion3=None),
    "moe_alpha8_2048x16384": dict(desc="one MoE-shaped 2048x16384 bf16 matrix (aspect ratio 8, Gaussian): "
                                       "Gram NS (fp16, restart 3) vs standard NS (bf16 and fp16), T=5",
                                  compute="f16", gram=True, normuon=False, dion3=None),
}


def ns_flops(n, m, T, gram, restart_at=3):
    """The page's FLOP counts with symmetric GEMMs: standard T(3 alpha + 1) n^3,
    Gram (4T + 3 alpha - 3) n^3, plus 3(alpha - 1) n^3 per restart."""
    if not gram:
        return T * (3 * m * n * n + n ** 3)
    f = 4 * T * n ** 3 + 3 * m * n * n - 3 * n ** 3
    if restart_at and 1 < restart_at <= T:
        f += 3 * m * n * n - 3 * n ** 3
    return f


def specs_for(name: str):
    if name == "spectrum4096x16384":
        return [inputs.MatrixSpec(4096, 16384, 3000, "x")]
    if name == "moe_alpha8_2048x16384":
        return [inputs.MatrixSpec(2048, 16384, 6000, "x")]
    if name == "single256x1024":
        return [inputs.MatrixSpec(256, 1024, 1000, "x")]
    if name == "gpt124m":
        return inputs.gpt124m_layer_set()
    if name == "dion3_8192x28672":
        return [inputs.MatrixSpec(8192, 28672, 4000, "x")]
    if name == "llama_mlp_4096x14336":
        return [inputs.llama7b_layer_set()[4]]
    if name in ("llama7b_layer", "llama7b_gram_layer"):
        return inputs.llama7b_layer_set(layers=1)
    if name.startswith("llama7b"):
        return inputs.llama7b_layer_set()
    raise ValueError(name)


def host_state(spec: inputs.MatrixSpec, workload: str):
    """Seeded W, M0 = 0, G for one matrix (fp32, host)."""
    shape = (spec.rows, spec.cols)
    if workload == "single256x1024":
        W = inputs.gaussian(shape, 1.0, spec.seed, inputs.W_STREAM)
        G = inputs.gaussian(shape, 1.0, spec.seed, inputs.G_STREAM)
    elif workload == "gpt124m":
        W = inputs.gaussian(shape, 0.02, spec.seed, inputs.W_STREAM)
        G = inputs.gaussian(shape, 1e-3, spec.seed, inputs.G_STREAM)
    else:
        W = inputs.gaussian(shape, 0.02, spec.seed, inputs.W_STREAM)
        G = inputs.student_t3(shape, 1e-3, spec.seed, inputs.G_STREAM)
    return W, np.zeros(shape, np.float32), G


def device_state(spec, workload, torch, gen_on_device: bool):
    shape = (spec.rows, spec.cols)
    if not gen_on_device:
        W, M, G = host_state(spec, workload)
        return [torch.from_numpy(a).cuda() for a in (W, M, G)]
    # large sets: same distributions drawn on the device (torch Philox, seeded per matrix)
    g = torch.Generator(device="cuda")
    g.manual_seed(spec.seed)
    W = torch.randn(shape, device="cuda", generator=g) * 0.02
    z = torch.randn(shape, device="cuda", generator=g)
    chi = torch.zeros(shape, device="cuda")
    for _ in range(3):
        chi.add_(torch.randn(shape, device="cuda", generator=g).square_())
    G = z.div_(chi.div_(3.0).sqrt_()).mul_(1e-3)
    del chi
    return [W, torch.zeros(shape, device="cuda"), G]


def step_params(mu, cfg, rows_hint=None):
    comp = {"f32": mu.F32, "bf16": mu.BF16, "f16": mu.F16}[cfg["compute"]]
    ns = mu.ns_params(T=5, coeffs=COEFFS, gram=cfg["gram"], restart_at=3, compute=comp)
    return mu.step_params(mu=0.95, lr=0.02, ns=ns, normuon=cfg["normuon"], beta2=0.95, normuon_eps=1e-8,
                          dion3=cfg["dion3"] is not None, frac=cfg["dion3"] or (1, 1), select_norm=mu.NORM_L1)


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((ts, float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3][1:5]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in inside])), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside),
                "in_region": any(t0 <= r[0] <= t1 for r in rows)}


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank number over all ranks (the reported time of a
    multi-GPU run is the slowest rank's)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def source_hash(files) -> str:
    """First 16 hex digits of the SHA-256 of the named csrc/ files, in order."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "newton_schulz_10_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM read + write bytes of `kernel` on `workload` from the JSON
    sidecars of the committed ncu summaries (profiles/*.json), reported only
    while the kernel's sources hash to the value recorded with the capture.
    `per` says what the bytes cover ("launch" or "step"). A capture taken on
    a smaller case of the same kernel lists, under applies_to, the workloads
    it scales to and the factor (units one launch or step processes, relative
    to the capture). Returns (bytes, per, source) or (None, None, why)."""
    import glob
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.json"))):
        with open(path) as f:
            d = json.load(f)
        if d.get("kernel") != kernel:
            continue
        factor = d.get("applies_to", {}).get(workload)
        if factor is None:
            continue
        rel = os.path.relpath(path, ROOT)
        if source_hash(d["sources"]) != d["source_sha256_16"]:
            return None, None, f"{rel}: kernel sources changed since the capture"
        return d["dram_bytes"] * factor, d["per"], rel
    return None, None, "no capture of this kernel for this workload"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def use_graph(args, big: bool) -> bool:
    """The small layer sets (a few ms per step, tens of launches) replay the
    step as a captured CUDA graph, which takes the host out of the loop; the
    large ones run eager steps that record their own phase events, queued
    behind a short device-side sleep so the GPU runs them back to back."""
    return bool(args.graph) if args.graph >= 0 else not big


PRIME_CYCLES = 4_000_000  # ~2-3 ms of device time: the host queues the timed steps meanwhile


def prime(torch):
    """Keep the stream busy while the host queues the timed region."""
    torch.cuda._sleep(PRIME_CYCLES)


def config_for(args, specs=None) -> dict:
    """The bench line's config: identical for our arm and the reference arm."""
    cfg = WORKLOADS[args.workload]
    specs = specs if specs is not None else specs_for(args.workload)
    elems = sum(s.rows * s.cols for s in specs)
    if args.workload in ("spectrum4096x16384", "moe_alpha8_2048x16384"):
        s0 = specs[0]
        return {"workload": args.workload, "description": cfg["desc"], "step": "one gram_ns_polar call",
                "l2": f"bf16 input {2 * elems / 2**20:.0f} MiB plus working set, larger than L2",
                "parallelism": "replicas" if args.gpus > 1 else "single GPU", "rows": s0.rows, "cols": s0.cols}
    big = elems > 1_000_000_000
    return {"workload": args.workload, "description": cfg["desc"], "matrices": len(specs), "elements": elems,
            "state_bytes": 12 * elems, "l2": "inputs larger than L2 (fp32 W, M, G resident in HBM)",
            "execution": "cuda_graph" if use_graph(args, big) else "eager, queued behind a device sleep, phase events per step",
            "parallelism": "replicas" if args.gpus > 1 else "single GPU"}


def end_to_end(args, state, step, stream, elems, world):
    """The step as a training loop drives it, through the public API with
    host buffers. Every step's gradients are copied from pinned host memory
    to the device (on a copy stream, into one of two device buffers, so the
    upload of step k+1 overlaps step k); the step runs; its result, the
    updated weights W and the 4-byte device status word, is read back to
    pinned host memory. The read-back goes through a device snapshot of W
    (a device-to-device copy right after the step) on a second copy stream,
    so it overlaps the next step; the next snapshot waits for it. M and v
    stay resident, as optimizer state does in training."""
    import torch
    import torch.distributed as dist

    from newton_schulz_10_b200 import muon as mu

    h2d = 4 * elems
    d2h = 4 * elems + 4
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except ImportError:
        avail = 1 << 62
    free_dev, _ = torch.cuda.mem_get_info()
    # every rank on this node pins its own G and W copies at the same time
    ranks_here = int(os.environ.get("LOCAL_WORLD_SIZE", "1"))
    if 8 * elems * ranks_here > 0.5 * avail or 8 * elems > 0.9 * free_dev:
        return {"value": None, "unit": "ms/step", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "reason": f"needs {8 * elems / 1e9:.1f} GB pinned host memory per rank ({ranks_here} ranks on "
                          f"this node) and as much device memory ({avail / 1e9:.1f} GB host available, "
                          f"{free_dev / 1e9:.1f} GB device free)"}
    hostG = [torch.empty_like(G, device="cpu").pin_memory() for (_, _, G, _) in state]
    for hg, (_, _, G, _) in zip(hostG, state):
        hg.copy_(G)
    hostW = [torch.empty_like(W, device="cpu").pin_memory() for (W, _, _, _) in state]
    snapW = [torch.empty_like(W) for (W, _, _, _) in state]
    # second device gradient buffer and a step bound to it (same workspace)
    G2 = [torch.empty_like(G) for (_, _, G, _) in state]
    steps = [step, mu.Step([(W, M, g2, v) for (W, M, _, v), g2 in zip(state, G2)], step.params, ws=step.ws)]
    gsets = [[G for (_, _, G, _) in state], G2]
    status_host = torch.zeros(1, dtype=torch.int32).pin_memory()
    up_stream, down_stream = torch.cuda.Stream(), torch.cuda.Stream()
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]
    snapped, read = torch.cuda.Event(), torch.cuda.Event()
    # as many steps as the device-timed region (at most 50): the first
    # upload and the last read-back are not overlapped by anything, so a
    # short run charges each step with a large share of them
    e2e_steps = max(2, min(args.steps, 50))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    up_stream.wait_event(f0)
    down_stream.wait_event(f0)
    read.record(down_stream)
    for k in range(e2e_steps):
        buf = k % 2
        with torch.cuda.stream(up_stream):
            if k >= 2:
                up_stream.wait_event(done[buf])  # step k-2 has finished reading this buffer
            for hg, g in zip(hostG, gsets[buf]):
                g.copy_(hg, non_blocking=True)
            copied[buf].record(up_stream)
        stream.wait_event(copied[buf])
        steps[buf](stream)
        done[buf].record(stream)
        stream.wait_event(read)  # the previous read-back has left the snapshot
        with torch.cuda.stream(stream):
            for w, sw in zip(state, snapW):
                sw.copy_(w[0], non_blocking=True)
            status_host.copy_(steps[buf].ws[:4].view(torch.int32), non_blocking=True)
        snapped.record(stream)
        with torch.cuda.stream(down_stream):
            down_stream.wait_event(snapped)
            for hw, sw in zip(hostW, snapW):
                hw.copy_(sw, non_blocking=True)
            read.record(down_stream)
    stream.wait_event(read)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / e2e_steps, world)
    out = {"value": round(e2e_ms, 3), "unit": "ms/step", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "what": "G pinned host -> device (copy stream, double-buffered, overlapping the previous step), step, "
                   "W snapshot on the device, W and the 4-byte status word -> pinned host (second copy stream, "
                   "overlapping the next step)",
           "steps": e2e_steps, "status": mu.status_str(int(status_host.item()))}
    del hostG, hostW, snapW, G2
    return out


def phase_means(evs):
    """Mean milliseconds of each phase over the timed steps' event sets."""
    names = ("ms_prologue", "ms_ns", "ms_normuon", "ms_update")
    sums = [0.0] * 4
    for ev in evs:
        for i in range(4):
            sums[i] += ev[i].elapsed_time(ev[i + 1])
    out = {n: s / len(evs) for n, s in zip(names, sums)}
    out["ms_total"] = sum(out[n] for n in names)
    return out


def timed_eager(step, stream, steps, torch):
    """`steps` eager steps, each recording its own phase events; returns the
    event sets and the bracketing events."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for ev in evs:
        step.timed(ev, stream)
    e1.record(stream)
    return evs, e0, e1


def roofline_for(ns_flops_step, gemm_launches, ms_ns, peak, peak_src, workload, flops_exec):
    achieved = ns_flops_step / (ms_ns * 1e-3) / 1e12
    traffic, per, src = measured_traffic("gemm_kernel", workload)
    return {"bound": "tensor", "kernel": "gemm_kernel (tcgen05 NS chain)", "achieved": round(achieved, 1),
            "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "traffic": traffic, "traffic_unit": "bytes per GEMM launch (DRAM read + write, ncu)",
            "traffic_source": src, "flops_per_launch_algorithmic": ns_flops_step / max(gemm_launches, 1),
            "peak_source": peak_src, "flops_per_step_algorithmic": ns_flops_step,
            "flops_per_step_executed": flops_exec, "gemm_launches_per_step": gemm_launches,
            "achieved_executed": round(flops_exec / (ms_ns * 1e-3) / 1e12, 1)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from newton_schulz_10_b200 import muon as mu

    torch.cuda.set_device(local_rank)
    cfg = WORKLOADS[args.workload]
    specs = specs_for(args.workload)
    elems = sum(s.rows * s.cols for s in specs)
    big = elems > 1_000_000_000
    state = []
    for s in specs:
        W, M, G = device_state(s, args.workload, torch, gen_on_device=big)
        v = torch.zeros(s.rows, device="cuda")
        state.append((W, M, G, v))
    p = step_params(mu, cfg)
    step = mu.Step([tuple(x) for x in state], p)
    stream = torch.cuda.current_stream()
    graph_mode = use_graph(args, big)

    for _ in range(args.warmup):
        step(stream)
    torch.cuda.synchronize()
    status = step.device_status()
    prof = step.profiled(stream)  # FLOP and launch accounting of one step (and one more warm-up)
    graph = None
    if graph_mode:
        # capture one whole step (all its launches) in a CUDA graph, replay it
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(torch.cuda.current_stream())
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()

    # --- timed region (device-resident inputs) ------------------------------
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = mu.kernel_launch_count()
    evs = None
    with ClockSampler(local_rank) as clk:
        t0 = time.time()
        if graph is not None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        else:
            prime(torch)
            evs, e0, e1 = timed_eager(step, stream, args.steps, torch)
        torch.cuda.synchronize()
        t1 = time.time()
    launches = mu.kernel_launch_count() - n0
    if graph is not None:  # replays queue no launches from the host: count the captured ones
        launches = args.steps * prof.kernel_launches
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    clocks = clk.summary(t0, t1)
    status = step.device_status()

    # --- phases: from the timed steps' own events (eager); after graph
    # replays (which cannot be bracketed) from as many eager steps of the same
    # workload, queued behind a device sleep, right after the timed region
    if evs is None:
        if world > 1:
            dist.barrier()
        prime(torch)
        evs, _, _ = timed_eager(step, stream, args.steps, torch)
        torch.cuda.synchronize()
        phase_src = (f"CUDA events of {args.steps} eager steps (muon_step_events, queued behind a device sleep) "
                     "run after the timed graph replays, mean over steps, max over ranks")
    else:
        phase_src = "CUDA events of the timed steps (muon_step_events), mean over steps, max over ranks"
    ph = {k: max_over_ranks(v, world) for k, v in phase_means(evs).items()}

    peaks, peak_kind = measured_peaks()
    long_step = ms > 100.0
    tensor_peak = peaks["bf16_tflops_sustained" if long_step else "bf16_tflops"]
    peak_src = f"{peak_kind} {'sustained' if long_step else 'burst'} bf16 (MEASURED_PEAKS.json)"
    roof = None
    if cfg["compute"] != "f32":
        roof = roofline_for(prof.ns_flops, prof.gemm_launches, ph["ms_ns"], tensor_peak, peak_src, args.workload,
                            prof.ns_flops_executed)
        roof["time_source"] = phase_src
    hbm = peaks["hbm_gbs"]
    phases = {k: round(v, 4) for k, v in ph.items()}
    phases["source"] = phase_src
    phases["prologue_bytes_algorithmic"] = prof.bytes_prologue
    phases["update_bytes_algorithmic"] = prof.bytes_update
    phases["prologue_gbs"] = round(prof.bytes_prologue / (ph["ms_prologue"] * 1e-3) / 1e9, 1) if ph["ms_prologue"] else None
    upd_ms = ph["ms_update"] + ph["ms_normuon"]
    phases["update_gbs"] = round(prof.bytes_update / (upd_ms * 1e-3) / 1e9, 1) if upd_ms else None
    phases["hbm_peak_gbs"] = hbm
    for name, kern in (("prologue", "momentum_rows"), ("update", "update_rows")):
        tr, per, src = measured_traffic(kern, args.workload)
        phases[f"{name}_traffic"] = tr
        phases[f"{name}_traffic_source"] = src
    phases["kernel_launches_per_step"] = prof.kernel_launches

    # --- NorMuon on (Llama-7B set): the same step with Eq. (2) -------------
    normuon_on = None
    if args.workload == "llama7b" and not args.no_normuon:
        pn = step_params(mu, {**cfg, "normuon": True})
        need = mu.workspace_size([tuple(x) for x in state], pn)
        stepn = mu.Step([tuple(x) for x in state], pn, ws=step.ws if step.ws.numel() >= need else None)
        for _ in range(2):
            stepn(stream)
        torch.cuda.synchronize()
        kn = max(3, min(args.steps, 10))
        profn = stepn.profiled(stream)
        if world > 1:
            dist.barrier()
        prime(torch)
        evn, n0e, n1e = timed_eager(stepn, stream, kn, torch)
        torch.cuda.synchronize()
        msn = max_over_ranks(n0e.elapsed_time(n1e) / kn, world)
        phn = {k: max_over_ranks(v, world) for k, v in phase_means(evn).items()}
        rn = roofline_for(profn.ns_flops, profn.gemm_launches, phn["ms_ns"], tensor_peak, peak_src, args.workload,
                          profn.ns_flops_executed)
        normuon_on = {"ms_per_step": round(msn, 4), "steps": kn, "phases": {k: round(v, 4) for k, v in phn.items()},
                      "ns_achieved_tflops": rn["achieved"], "ns_frac": rn["frac"], "peak": tensor_peak,
                      "device_status": mu.status_str(stepn.device_status())}
        del stepn

    # --- end to end through host buffers ------------------------------------
    if args.no_e2e:
        e2e = None
    else:
        e2e = end_to_end(args, state, step, stream, elems, world)

    out = {
        "metric": METRIC, "value": round(ms, 4), "unit": "ms/step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg["compute"], "data": "synthetic",
        "config": config_for(args, specs),
        "roofline": roof,
        "phases": phases,
        "normuon_on": normuon_on,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "device_status": mu.status_str(status),
        "gemm": ("cta_pair" if args.cta_pair else "single_cta") + (", fused chain" if args.gemm_chain else ""),
    }
    return out


def run_spectrum(args, rank, world, local_rank):
    """Gram vs standard Newton-Schulz on one matrix: the 4096 x 16384
    spectrum matrix, or the 2048 x 16384 MoE-shaped Gaussian matrix."""
    import torch
    import torch.distributed as dist

    from newton_schulz_10_b200 import muon as mu

    torch.cuda.set_device(local_rank)
    if args.workload == "spectrum4096x16384":
        n, m = 4096, 16384
        X, _ = inputs.spectrum_matrix(n, m, -4.0, seed=3000)
    else:
        n, m = 2048, 16384
        X = inputs.gaussian((n, m), 1.0, 6000, 0)
    Xd = torch.from_numpy(X.astype(np.float32)).cuda().to(torch.bfloat16)
    del X
    variants = [("gram_f16", mu.ns_params(gram=True, restart_at=3, compute=mu.F16), True, 5),
                ("standard_bf16", mu.ns_params(compute=mu.BF16), False, 5),
                ("standard_f16", mu.ns_params(compute=mu.F16), False, 5)]
    if args.workload == "spectrum4096x16384":
        # tuned per-step schedules (minimax quintics): orthogonality error
        # against the step count, i.e. the FLOP budget
        from newton_schulz_10_b200 import schedules
        # (the Gram chain, with its single restart, is kept to the short
        # table: over ten steep steps its fp16 R drifts and overflows)
        co5, _ = schedules.minimax_schedule(5, 1e-3)
        co10, _ = schedules.minimax_schedule(10, 1e-5)
        variants += [("standard_bf16_minimax_T5", mu.ns_params(T=5, coeffs=co5, compute=mu.BF16), False, 5),
                     ("gram_f16_minimax_T5", mu.ns_params(T=5, coeffs=co5, gram=True, restart_at=3, compute=mu.F16),
                      True, 5),
                     ("standard_bf16_minimax_T10", mu.ns_params(T=10, coeffs=co10, compute=mu.BF16), False, 10),
                     ("standard_f16_minimax_T10", mu.ns_params(T=10, coeffs=co10, compute=mu.F16), False, 10)]
    stream = torch.cuda.current_stream()
    res = {}
    clocks = None
    launches = 0
    for name, p, gram, T in variants:
        O, ws = mu.ns_polar(Xd, p, out_dtype=torch.bfloat16)
        for _ in range(args.warmup):
            mu.ns_polar(Xd, p, out_dtype=torch.bfloat16, ws=ws)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        n0 = mu.kernel_launch_count()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank) as clk:
            t0 = time.time()
            prime(torch)
            e0.record(stream)
            for _ in range(args.steps):
                O, _ = mu.ns_polar(Xd, p, out_dtype=torch.bfloat16, ws=ws)
            e1.record(stream)
            torch.cuda.synchronize()
            t1 = time.time()
        ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
        if name == "gram_f16":
            clocks = clk.summary(t0, t1)
            launches = mu.kernel_launch_count() - n0
        Of = O.float()
        orth = float(torch.linalg.matrix_norm(Of @ Of.T - torch.eye(n, device="cuda")).item())
        fl = ns_flops(n, m, T, gram)
        res[name] = {"ms": round(ms, 3), "tflops_algorithmic": round(fl / (ms * 1e-3) / 1e12, 1),
                     "orthogonality_error_fro": round(orth, 4),
                     "status": mu.status_str(int(ws[:4].view(torch.int32).item()))}
        del O, ws
    peaks, kind = measured_peaks()
    g = res["gram_f16"]
    peak = peaks["bf16_tflops"]  # fp16 and bf16 share the dense tensor-core rate
    cfg = WORKLOADS[args.workload]
    return {
        "metric": METRIC, "value": g["ms"], "unit": "ms/step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": g["ms"], "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": config_for(args),
        "roofline": {"bound": "tensor", "kernel": "gemm_kernel (Gram NS chain)", "achieved": g["tflops_algorithmic"],
                     "peak": peak, "unit": "TFLOP/s", "frac": round(g["tflops_algorithmic"] / peak, 4),
                     "traffic": None, "peak_source": f"{kind} burst bf16 (fp16 has the same dense rate)"},
        "variants": res,
        "speedup_gram_vs_standard_bf16": round(res["standard_bf16"]["ms"] / g["ms"], 3),
        "flop_ratio_standard_over_gram": round(ns_flops(n, m, 5, False) / ns_flops(n, m, 5, True), 3),
        "e2e": None, "gpu_launches": launches, "clocks": clocks,
    }


# ---------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------


class OracleSampler:
    """Times the fp64 oracle on bounded samples of a layer-set workload.

    Matrices of one shape cost the oracle the same, so the whole step is
    estimated as each timed shape's mean time times that shape's count. The
    seeded inputs of every sampled matrix are kept, so later samples of the
    same matrix do not pay for drawing them again."""

    def __init__(self, workload: str):
        self.workload = workload
        self.cfg = WORKLOADS[workload]
        self.specs = specs_for(workload)
        self.count = {}
        self.first = {}
        for s in self.specs:
            key = (s.rows, s.cols)
            self.count[key] = self.count.get(key, 0) + 1
            self.first.setdefault(key, s)
        self.shapes = list(self.first)
        self.times = {}
        self.inputs = {}
        self.names = []

    def time_spec(self, s) -> float:
        import oracle
        cfg = self.cfg
        state = self.inputs.get(s.name)
        if state is None:
            state = self.inputs[s.name] = host_state(s, self.workload)
        W, M, G = state
        v = np.zeros(s.rows, np.float32)
        p = oracle.StepParams(mu=0.95, lr=0.02, coeffs=(COEFFS,) * 5, gram=cfg["gram"], normuon=cfg["normuon"])
        if cfg["dion3"] is not None:
            p = oracle.StepParams(**{**p.__dict__, "k": oracle.rows_for_fraction(s.rows, *cfg["dion3"])})
        t = time.perf_counter()
        oracle.muon_step(W, M, G, v, p)
        dt = time.perf_counter() - t
        self.times.setdefault((s.rows, s.cols), []).append(dt)
        self.names.append(s.name)
        return dt

    def time_shape(self, i: int) -> float:
        return self.time_spec(self.first[self.shapes[i % len(self.shapes)]])

    def estimate_ms(self) -> float:
        return 1e3 * sum(float(np.mean(self.times[k])) * self.count[k] for k in self.shapes)

    def describe(self, what: str) -> str:
        per = ", ".join(f"{r}x{c}: {len(self.times.get((r, c), []))} timed, x{self.count[(r, c)]}"
                        for (r, c) in self.shapes)
        return (f"oracle muon_step, {what}; the step is each shape's mean time times its count ({per}); "
                f"{len(self.specs)} matrices in the step")


def spectrum_sample(workload: str):
    """Oracle Gram NS on a scaled-down matrix of the same kind, scaled to the
    full matrix by the Gram FLOP formula; returns (ms, description)."""
    import oracle
    if workload == "moe_alpha8_2048x16384":
        X = inputs.gaussian((512, 4096), 1.0, 6000, 0).astype(np.float64)
        t = time.perf_counter()
        oracle.gram_newton_schulz(X, (COEFFS,) * 5, 1e-7, 3)
        dt = time.perf_counter() - t
        scale = ns_flops(2048, 16384, 5, True) / ns_flops(512, 4096, 5, True)
        return 1e3 * dt * scale, (f"oracle gram_newton_schulz on a 512x4096 Gaussian matrix (aspect 8), "
                                  f"{dt:.2f} s, scaled x{scale:.0f} by the Gram FLOP formula")
    X, _ = inputs.spectrum_matrix(1024, 4096, -4.0, seed=3000)
    t = time.perf_counter()
    oracle.gram_newton_schulz(X, (COEFFS,) * 5, 1e-7, 3)
    dt = time.perf_counter() - t
    scale = ns_flops(4096, 16384, 5, True) / ns_flops(1024, 4096, 5, True)
    return 1e3 * dt * scale, (f"oracle gram_newton_schulz on a 1024x4096 matrix of the same spectrum, "
                              f"{dt:.1f} s, scaled x{scale:.0f} by the Gram FLOP formula")


SPECTRUM = ("spectrum4096x16384", "moe_alpha8_2048x16384")


def oracle_baseline(workload: str, budget_s: float):
    """cpu_baseline of our arm: one matrix of every distinct shape, then more
    matrices until about budget_s of oracle time. Returns (ms, desc, cores)."""
    if workload in SPECTRUM:
        ms, desc = spectrum_sample(workload)
        return ms, desc, threads_used()
    smp = OracleSampler(workload)
    t_sum = 0.0
    for i in range(len(smp.shapes)):
        t_sum += smp.time_shape(i)
    for s in smp.specs:
        if t_sum > budget_s:
            break
        if s.name in smp.inputs:
            continue
        t_sum += smp.time_spec(s)
    return smp.estimate_ms(), smp.describe(f"{len(smp.names)} matrices timed in {t_sum:.1f} s"), threads_used()


def threads_used():
    for var in ("OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS"):
        if os.environ.get(var):
            return int(os.environ[var])
    return os.cpu_count()


def run_reference(args):
    """The reference arm: the fp64 CPU oracle as it stands. Each timed step
    times one matrix, the distinct shapes taken in turn, and reports the
    whole-step estimate from every shape's mean time so far; the warm-up
    times one matrix of every shape, so that every shape has a time before
    the first timed step."""
    vals = []
    if args.workload in SPECTRUM:
        for _ in range(args.warmup):
            spectrum_sample(args.workload)
        for _ in range(args.steps):
            ms, desc = spectrum_sample(args.workload)
            vals.append(ms)
    else:
        smp = OracleSampler(args.workload)
        k = 0
        # warm-up: one sample per distinct shape (numpy has nothing to warm;
        # these give every shape a time before the first timed step)
        for _ in range(len(smp.shapes)):
            smp.time_shape(k)
            k += 1
        for _ in range(args.steps):
            smp.time_shape(k)
            k += 1
            vals.append(smp.estimate_ms())
        desc = smp.describe(f"one matrix per step, shapes in turn, {len(smp.names)} samples")
    ms = float(np.mean(vals)) if vals else 0.0
    cfg = WORKLOADS[args.workload]
    return {"impl": "reference", "metric": METRIC, "value": round(ms, 2), "unit": "ms/step", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_for(args),
            "reference_precision": f"fp64 oracle of the {cfg['compute']} path",
            "cpu_baseline": {"value": round(ms, 2), "unit": "ms/step", "cores": threads_used(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(ms, 2), "unit": "ms/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama7b")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end arm")
    ap.add_argument("--no-normuon", action="store_true", help="skip the NorMuon-on timing of the Llama-7B set")
    ap.add_argument("--graph", type=int, default=-1,
                    help="1: replay the step as one captured CUDA graph (phases then from as many eager steps), "
                         "0: eager steps queued behind a device-side sleep, each recording its own phase events, "
                         "-1 (default): graph for the small layer sets, eager for the large ones")
    ap.add_argument("--cta-pair", type=int, default=1, help="1: CTA-pair tensor-core GEMM, 0: single-CTA")
    ap.add_argument("--gemm-chain", type=int, default=0,
                    help="1: run each Newton-Schulz chain as one fused persistent launch (completion counters "
                         "between dependent products), 0: one launch per product")
    ap.add_argument("--wait-timeout-ms", type=float, default=0.0, help="bound of device-side waits (0: default)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    from newton_schulz_10_b200 import muon as mu
    mu.set_gemm_cta_pair(bool(args.cta_pair))
    mu.set_gemm_chain(bool(args.gemm_chain))
    if args.wait_timeout_ms > 0:
        mu.set_wait_timeout_ns(int(args.wait_timeout_ms * 1e6))
    if args.workload in SPECTRUM:
        out = run_spectrum(args, rank, world, local_rank)
    else:
        out = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms, desc, cores = oracle_baseline(args.workload, args.cpu_budget)
        out["cpu_baseline"] = {"value": round(ms, 1), "unit": "ms/step", "cores": cores, "kind": "oracle",
                               "sample": desc}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
