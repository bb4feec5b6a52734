#!/usr/bin/env python
"""Throughput of the tiled, IO-aware attention path on B200.

One step = one pass of the whole hot path over one synthetic batch: the
forward (TMA-staged tiles, S = scale Q K^T, online softmax, PV, O/LSE
epilogue) followed by the backward (D = rowsum(dO * O), dK/dV and dQ with P
recomputed from LSE).  The workload is B=2, H=16, N=4096, d=128 (bf16),
non-causal; causal and forward-only legs are reported beside it.

Timing: W untimed warm-up steps, then K timed steps, each bracketed by CUDA
events on the launching stream; a 256 MiB buffer is written between timed
steps so that no step starts with its inputs in L2.  With N GPUs (torchrun,
one rank per GPU) every rank runs its own independent batch (weak scaling,
no collective on the data path); rank 0 prints the max over ranks.

--impl reference times the fp64 CPU oracle (the only other place this
script runs it) on a bounded sample of the same workload.

Other modes (each prints JSON lines and exits): --all-configs times every
named workload; --tile-sweep times every forward tile shape the kernels build
and the rescale thresholds; --ncu-case [--ncu-workload] runs a few untimed
launches for ncu.
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

_ROOT = os.path.dirname(os.path.abspath(__file__))
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

METRIC = "attention TFLOP/s fwd & fwd+bwd (bf16, N=4096, d=128) and % of BF16 tensor peak"
UNIT = "TFLOP/s"
WORKLOAD = "fwd_b2h16n4096d128"


def _peaks():
    p = os.path.join(_ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16_tflops": float(d["bf16_tflops"]), "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]),
                "hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def _flops(B, H, N, d, causal):
    fwd = 4.0 * B * H * N * N * d
    if causal:
        fwd /= 2
    return fwd, 2.5 * fwd


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region.

    NVML in a background thread every 5 ms (the timed region lasts well under
    a second); `nvidia-smi -lms 100` when NVML is not importable.  The thread
    takes its first sample before __enter__ returns."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
                   ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, device):
        self.device = device
        self.proc = None
        self.out = None
        self.samples = []      # (sm_mhz, reason bitmask)
        self.sm_max = None
        self.thread = None
        self.stop = threading.Event()

    def _nvml_handle(self, nvml):
        import torch
        p = torch.cuda.get_device_properties(self.device)
        bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        try:
            return nvml.nvmlDeviceGetHandleByPciBusId(bus)
        except nvml.NVMLError:
            return nvml.nvmlDeviceGetHandleByPciBusId(bus[4:])

    def __enter__(self):
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            h = self._nvml_handle(nvml)
            self.sm_max = float(nvml.nvmlDeviceGetMaxClockInfo(h, nvml.NVML_CLOCK_SM))
            first = threading.Event()

            def loop():
                while True:
                    try:
                        self.samples.append((float(nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM)),
                                             int(nvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except nvml.NVMLError:
                        pass
                    first.set()
                    if self.stop.wait(0.005):
                        return

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            first.wait(2.0)
            return self
        except Exception:  # no NVML: fall back to nvidia-smi
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self):
        if self.samples:
            sm = [c for c, _ in self.samples]
            mask = 0
            for _, m in self.samples:
                mask |= m
            reasons = sorted(n for n, bit in self.REASON_BITS if mask & bit)
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.sm_max, "reasons": reasons,
                    "samples": len(sm), "sm_mhz_min": min(sm), "source": "nvml, 5 ms"}
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 100 ms"}


# ---------------------------------------------------------------------------
# the CPU oracle as a baseline (bounded sample)
# ---------------------------------------------------------------------------
def oracle_sample_run(N=4096, d=128, causal=False, heads=1, seed=0):
    """fwd + bwd of `heads` heads of the workload in fp64 on the host cores.
    Returns (seconds, flops by the same convention as the GPU number)."""
    import oracle
    from io_aware_tiled_b200.inputs import attention_inputs
    q, k, v, do = attention_inputs(1, heads, N, d, seed=seed)
    args = [t.double().numpy() for t in (q, k, v, do)]
    t0 = time.perf_counter()
    oracle.backward(*args, causal, 1.0 / math.sqrt(d))
    dt = time.perf_counter() - t0
    f, b = _flops(1, heads, N, d, causal)
    return dt, f + b


def oracle_workload_samples():
    """The oracle on a bounded sample of every named workload (about 15 s in
    all): the single-head workload in full, on all cores and on one core; one
    head of the headline forward (both masks); one head of the training and
    long-sequence workloads (fwd+bwd, causal); the ragged d=64 workload in full
    (fwd+bwd, both masks).  TFLOP/s by the conventional count of the sample."""
    import oracle
    from io_aware_tiled_b200.configs import WORKLOADS
    from io_aware_tiled_b200.inputs import attention_inputs
    out = []
    plan = [("pr1_b1h1n256d64", False, "fwd", None), ("pr1_b1h1n256d64", False, "fwd", 1),
            ("fwd_b2h16n4096d128", False, "fwd", None), ("fwd_b2h16n4096d128", True, "fwd", None),
            ("train_b4h32n2048d128", True, "fwd+bwd", None), ("long_b1h16n16384d128", True, "fwd+bwd", None),
            ("ragged_b8h12n1000d64", False, "fwd+bwd", None), ("ragged_b8h12n1000d64", True, "fwd+bwd", None)]
    all_threads = oracle.num_threads()
    for name, causal, pas, threads in plan:
        w = WORKLOADS[name]
        heads = w.B * w.H if name in ("pr1_b1h1n256d64", "ragged_b8h12n1000d64") else 1
        B, H = (w.B, w.H) if heads == w.B * w.H else (1, 1)
        q, k, v, do = (t.double().numpy() if t is not None else None
                       for t in attention_inputs(B, H, w.N, w.d, seed=w.seed, sigma_qk=w.sigma_qk,
                                                 with_do=pas != "fwd"))
        if threads:
            oracle.set_num_threads(threads)
        try:
            t0 = time.perf_counter()
            if pas == "fwd":
                oracle.forward(q, k, v, causal, w.scale)
            else:
                oracle.backward(q, k, v, do, causal, w.scale)
            dt = time.perf_counter() - t0
        finally:
            if threads:
                oracle.set_num_threads(all_threads)
        f, b = _flops(B, H, w.N, w.d, causal)
        fl = f + (b if pas != "fwd" else 0.0)
        out.append({"workload": name, "causal": causal, "pass": pas,
                    "sample": "full workload" if heads == w.B * w.H else "one head",
                    "threads": threads or all_threads, "seconds": dt, "tflops": fl / dt / 1e12})
    return out


def cpu_baseline(target_s=6.0):
    import oracle
    total_t, total_f, reps = 0.0, 0.0, 0
    while total_t < target_s and reps < 8:
        dt, fl = oracle_sample_run()
        total_t += dt
        total_f += fl
        reps += 1
    return {"value": total_f / total_t / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{reps} x one head (B=1,H=1,N=4096,d=128) fwd+bwd non-causal, fp64, {total_t:.1f} s",
            "host_cpu_count": os.cpu_count(), "affinity": len(os.sched_getaffinity(0)),
            "workloads": oracle_workload_samples()}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle
    for _ in range(args.warmup):
        oracle_sample_run()
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample_run()
        times.append(dt)
        flops += fl
    total = sum(times)
    value = flops / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": 2, "H": 16, "N": 4096, "d": 128, "causal": False,
                   "step": "fwd+bwd", "sample": "one head per step (B=1,H=1,N=4096,d=128)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": "one head (B=1,H=1,N=4096,d=128) fwd+bwd non-causal per step, fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# cross-rank pieces (no GPU needed; tested with gloo ranks on the CPU)
# ---------------------------------------------------------------------------
def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's time: every rank contributes, every rank gets the max."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Weak scaling: every rank runs its own batch, so the job did world x the
    work of one rank in the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own independent batch."""
    return base_seed + rank


# ---------------------------------------------------------------------------
# DRAM traffic from ncu
# ---------------------------------------------------------------------------
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of each kernel,
# captured with `python bench.py --ncu-case fwd|bwd --ncu-batch B` and divided
# by the B*16 heads; the summaries sit in profiles/.  Each kernel reads its
# inputs once per head, so the traffic of the bench's 32-head launch is the
# per-head figure x 32.  Each entry keeps the
# sha256 of the sources the kernel is compiled from at capture time: once they
# change, the figure no longer describes the kernel and traffic is null.
NCU_TRAFFIC = {
    # profiles/fa_fwd_2sm_kernel_b2h16n4096d128_noncausal.md (32 heads)
    "fa_fwd_2sm_kernel": {"bytes_per_head": (100.750592e6 + 20.326656e6) / 32,
                          "sources": ("fa_fwd2.cuh", "fa_device.cuh"),
                          "sha256": "79c9202b8bbf5a514ac67496b988089d804e0f304b16f3a083d27b3635801ac4"},
    # B=2, H=16, N=4096, d=128 non-causal (the bench's own shape, 32 heads):
    # profiles/fa_bwd_fused_kernel_b2h16n4096d128_noncausal.md
    "fa_bwd_fused_kernel": {"bytes_per_head": (202.964992e6 + 91.349248e6) / 32,
                            "sources": ("fa_bwd_fused.cuh", "fa_device.cuh"),
                            "sha256": "9759a63692390608395b1f568300fbe91584456129788f8fa122e098c86f7282"},
}


def kernel_sources_sha(sources) -> str:
    import hashlib
    h = hashlib.sha256()
    root = os.path.join(os.path.dirname(os.path.abspath(__file__)), "io_aware_tiled_b200", "csrc")
    for name in sources:
        with open(os.path.join(root, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic_per_launch(heads: int) -> dict:
    """DRAM bytes per launch for `heads` (B*H) heads, by kernel name, for the
    kernels whose sources are unchanged since the capture."""
    return {n: e["bytes_per_head"] * heads for n, e in NCU_TRAFFIC.items()
            if kernel_sources_sha(e["sources"]) == e["sha256"]}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from io_aware_tiled_b200 import fa
    from io_aware_tiled_b200.configs import WORKLOADS
    from io_aware_tiled_b200.inputs import attention_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[WORKLOAD]
    B, H, N, d = w.B, w.H, w.N, w.d
    q, k, v, do = attention_inputs(B, H, N, d, seed=rank_seed(w.seed, rank))
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    ws = torch.empty(fa.workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd(causal):
        fa.forward(qd, kd, vd, causal, out=o, lse=lse)

    def bwd(causal, deterministic=False):
        fa.backward(qd, kd, vd, o, dod, lse, causal, workspace=ws, dq=dq, dk=dk, dv=dv, deterministic=deterministic)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    fwd_name = fa.forward_kernel_name(d, False)
    pre_name, main_bwd_name, last_bwd_name = fa.backward_kernel_names(d)

    step_times = []  # per-step ms of each timed() call, in call order

    def timed(fn, steps, per_kernel=False):
        """Run fn `steps` times, L2 flushed before each; returns total ms and
        per-kernel ms lists when per_kernel (forward + the three backward kernels)."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        kev = []
        barrier()
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(stream)
            if per_kernel:
                e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
                e[0].record(stream)
                fwd(False)
                fa.set_backward_phase_events(e[1:5])
                bwd(False)
                fa.set_backward_phase_events(None)
                kev.append(e)
            else:
                fn()
            ev[i][1].record(stream)
        barrier()
        per_step = [a.elapsed_time(b) for a, b in ev]
        total = sum(per_step)
        step_times.append(per_step)
        kern = None
        if per_kernel:
            kern = {fwd_name: [e[0].elapsed_time(e[1]) for e in kev],
                    pre_name: [e[1].elapsed_time(e[2]) for e in kev],
                    main_bwd_name: [e[2].elapsed_time(e[3]) for e in kev],
                    last_bwd_name: [e[3].elapsed_time(e[4]) for e in kev]}
        return total, kern

    # warm-up (also the status check: a kernel timeout would show here)
    for _ in range(max(args.warmup, 3)):
        fwd(False); bwd(False); fwd(True); bwd(True)
    rc = fa.sync_status(dev)
    if rc != fa.FA_OK:
        raise RuntimeError(f"library status {fa.status_string(rc)}")

    f_nc, b_nc = _flops(B, H, N, d, False)
    f_c, b_c = _flops(B, H, N, d, True)

    clocks = ClockSampler(dev)
    with clocks:
        main_ms, kern = timed(None, args.steps, per_kernel=True)
        main_steps = step_times[-1]
        fwd_ms, _ = timed(lambda: fwd(False), args.steps)
        fwd_steps = step_times[-1]
        fwdc_ms, _ = timed(lambda: fwd(True), args.steps)
        fwdc_steps = step_times[-1]
        stepc_ms, _ = timed(lambda: (fwd(True), bwd(True)), args.steps)
        stepc_steps = step_times[-1]
        # the deterministic backward form (a separate dQ kernel), for comparison
        stepd_ms, _ = timed(lambda: (fwd(False), bwd(False, True)), args.steps)
        stepd_steps = step_times[-1]
    # the standard (unfused) forward of the same batch, for the HBM-traffic
    # comparison: S and P through HBM (outside the clock sampling window)
    ws_unf = torch.empty(fa.unfused_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    for _ in range(2):
        fa.forward_unfused(qd, kd, vd, False, workspace=ws_unf, out=o, lse=lse)
    unf_steps = max(3, args.steps // 4)
    unf_ms, _ = timed(lambda: fa.forward_unfused(qd, kd, vd, False, workspace=ws_unf, out=o, lse=lse), unf_steps)
    unf_ms = max_over_ranks(unf_ms, world, dev)
    del ws_unf
    main_ms = max_over_ranks(main_ms, world, dev)
    fwd_ms = max_over_ranks(fwd_ms, world, dev)
    fwdc_ms = max_over_ranks(fwdc_ms, world, dev)
    stepc_ms = max_over_ranks(stepc_ms, world, dev)
    stepd_ms = max_over_ranks(stepd_ms, world, dev)
    rc = fa.sync_status(dev)
    if rc != fa.FA_OK:
        raise RuntimeError(f"library status {fa.status_string(rc)}")

    # end to end through the public API: pinned host inputs -> device -> fwd+bwd -> host
    hq, hk, hv, hdo = (t.pin_memory() for t in (q, k, v, do))
    ho, hdq, hdk, hdv = (torch.empty_like(hq).pin_memory() for _ in range(4))
    hl = torch.empty((B, H, N), dtype=torch.float32).pin_memory()

    def e2e_step():
        q2, k2, v2, do2 = (t.to(dev, non_blocking=True) for t in (hq, hk, hv, hdo))
        o2, l2 = fa.forward(q2, k2, v2, False)
        g = fa.backward(q2, k2, v2, o2, do2, l2, False, workspace=ws)
        for h, t in zip((ho, hl, hdq, hdk, hdv), (o2, l2, *g)):
            h.copy_(t, non_blocking=True)

    from io_aware_tiled_b200.host_pipeline import forward_backward_host

    E2E_GROUPS = 12  # head groups of the host pipeline (ceil(B*H / 12) heads each)
    ws_host = torch.empty(fa.host_workspace_bytes(B, H, N, d, E2E_GROUPS), dtype=torch.uint8, device=dev)

    def e2e_pipelined():
        # fa_fwd_bwd_host: heads in groups through the library's three streams
        # (copies in, kernels, copies out)
        forward_backward_host(hq, hk, hv, hdo, False, groups=E2E_GROUPS, out=(ho, hl, hdq, hdk, hdv), workspace=ws_host,
                              device=dev)

    e2e_steps = max(3, args.steps // 4)
    for _ in range(2):
        e2e_step()
    e2e_serial_ms, _ = timed(e2e_step, e2e_steps)
    e2e_serial_ms = max_over_ranks(e2e_serial_ms, world, dev)
    for _ in range(2):
        e2e_pipelined()
    e2e_ms, _ = timed(e2e_pipelined, e2e_steps)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    d2h = sum(t.numel() * t.element_size() for t in (ho, hl, hdq, hdk, hdv))

    # every other named workload (forward, forward + backward), median and best
    wclocks = ClockSampler(dev)
    with wclocks:
        wlines = time_workloads(args.workload_steps, max(args.warmup, 3), dev,
                                reduce_max=lambda x: max_over_ranks(x, world, dev), skip=(WORKLOAD,))

    peaks = _peaks()
    step_flops = f_nc + b_nc
    value = whole_job_tflops(world, step_flops, args.steps, main_ms)
    # per-kernel live durations (rank-local) and the dominant kernel's roofline
    kavg = {n: sum(v) / len(v) for n, v in kern.items()}
    per_kernel_flops = {  # dense MMA work each kernel performs
        fwd_name: 4.0 * B * H * N * N * d,
        main_bwd_name: 10.0 * B * H * N * N * d,         # S^T, dP^T, dV, dK, dQ^T
    }
    # bytes the memory-bound passes must move: the D pass reads O and dO,
    # writes D and zeroes the fp32 dQ accumulator; the convert pass reads the
    # accumulator and writes bf16 dQ
    per_kernel_bytes = {
        pre_name: 2.0 * B * H * N * d * 2 + 4.0 * B * H * N + 4.0 * B * H * N * d,
        last_bwd_name: 4.0 * B * H * N * d + 2.0 * B * H * N * d,
    }
    traffic = ncu_traffic_per_launch(B * H)
    dom = max(kavg, key=kavg.get)
    peak = peaks["bf16_tflops"]
    if dom in per_kernel_flops:
        ach = per_kernel_flops[dom] / (kavg[dom] * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "traffic": traffic.get(dom), "peak_kind": f"bf16 burst, {peaks['source']}"}
    else:
        ach = per_kernel_bytes[dom] / (kavg[dom] * 1e-3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": traffic.get(dom), "peak_kind": f"hbm copy, {peaks['source']}"}
    kernels = {n: {"ms": kavg[n],
                   "tflops": (per_kernel_flops[n] / (kavg[n] * 1e-3) / 1e12) if n in per_kernel_flops else None,
                   "traffic": traffic.get(n)}
               for n in kavg}
    for n, nb in per_kernel_bytes.items():
        kernels[n]["gbs"] = nb / (kavg[n] * 1e-3) / 1e9
        kernels[n]["frac_of_hbm"] = kernels[n]["gbs"] / peaks["hbm_gbs"]

    out = None
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": B, "H": H, "N": N, "d": d, "causal": False, "step": "fwd+bwd",
                       "inputs": "i.i.d. N(0,1) bf16 from seed 0 (+rank)", "l2": "256 MiB written between timed steps",
                       "parallelism": f"independent batch per GPU x{world}"},
            "frac_of_peak": value / peak,
            "median_ms_per_step": statistics.median(main_steps), "best_ms_per_step": min(main_steps),
            "value_median": world * step_flops / (statistics.median(main_steps) * 1e-3) / 1e12,
            "value_best": world * step_flops / (min(main_steps) * 1e-3) / 1e12,
            "legs": {
                "fwd_noncausal": _leg(world * f_nc, fwd_ms, args.steps, fwd_steps, peak),
                "fwd_causal": _leg(world * f_c, fwdc_ms, args.steps, fwdc_steps, peak),
                "fwd_bwd_causal": _leg(world * (f_c + b_c), stepc_ms, args.steps, stepc_steps, peak),
                # backward alone: the step minus the forward of the same mask
                "bwd_noncausal": {"tflops": world * b_nc / ((main_ms - fwd_ms) / args.steps * 1e-3) / 1e12,
                                  "ms": (main_ms - fwd_ms) / args.steps,
                                  "frac_of_measured_peak": world * b_nc / ((main_ms - fwd_ms) / args.steps * 1e-3)
                                  / 1e12 / peak, "how": "mean fwd+bwd step minus mean forward"},
                "fwd_bwd_noncausal_deterministic": _leg(world * (f_nc + b_nc), stepd_ms, args.steps, stepd_steps,
                                                        peak),
                "bwd_noncausal_deterministic": {
                    "tflops": world * b_nc / ((stepd_ms - fwd_ms) / args.steps * 1e-3) / 1e12,
                    "ms": (stepd_ms - fwd_ms) / args.steps, "how": "mean fwd+bwd step minus mean forward"},
                "bwd_causal": {"tflops": world * b_c / ((stepc_ms - fwdc_ms) / args.steps * 1e-3) / 1e12,
                               "ms": (stepc_ms - fwdc_ms) / args.steps,
                               "frac_of_measured_peak": world * b_c / ((stepc_ms - fwdc_ms) / args.steps * 1e-3)
                               / 1e12 / peak, "how": "mean fwd+bwd step minus mean forward"},
                # standard attention: S (fp16) and P (bf16) written and read
                # once each through HBM; bytes per head as in the pages'
                # table: Q, K, V, S, P read; S, P, O written
                "fwd_unfused_noncausal": {
                    "tflops": world * f_nc * unf_steps / (unf_ms * 1e-3) / 1e12, "ms": unf_ms / unf_steps,
                    "algorithmic_gbs": world * B * H * (3 * N * d * 2 + 4 * N * N * 2 + N * d * 2 + N * 4)
                    * unf_steps / (unf_ms * 1e-3) / 1e9},
            },
            "kernels": kernels,
            "roofline": roof,
            # through forward_backward_host (pinned host in, pinned host out, the
            # PCIe copies overlapped with the kernels); "serial" copies all
            # inputs, runs the kernels, then copies all outputs back
            "e2e": {"value": world * step_flops * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / e2e_steps,
                    "api": "fa_fwd_bwd_host (C ABI), called through io_aware_tiled_b200.fa.forward_backward_host",
                    "serial_value": world * step_flops * e2e_steps / (e2e_serial_ms * 1e-3) / 1e12,
                    "serial_ms_per_step": e2e_serial_ms / e2e_steps},
            "workloads": wlines,
            "workloads_clocks": wclocks.summary(),
            "gpu_launches": 4 * args.steps,
            "clocks": clocks.summary(),
            "peaks": peaks,
        }
    return out


def _leg(flops_per_step, total_ms, steps, per_step_ms, peak):
    """TFLOP/s of one timed leg: mean over the steps, plus median and best."""
    med, best = statistics.median(per_step_ms), min(per_step_ms)
    mean = total_ms / steps
    return {"tflops": flops_per_step / (mean * 1e-3) / 1e12, "ms": mean,
            "tflops_median": flops_per_step / (med * 1e-3) / 1e12, "median_ms": med,
            "tflops_best": flops_per_step / (best * 1e-3) / 1e12, "best_ms": best,
            "frac_of_measured_peak": flops_per_step / (mean * 1e-3) / 1e12 / peak}


def time_workloads(steps: int, warmup: int, dev, reduce_max=lambda x: x, skip=()):
    """Every named workload on one GPU: forward (each mask it names) and, where
    it names one, forward + backward; CUDA events around each call, the L2
    flushed before each (the small single-head workload also without the
    flush, and replayed from a CUDA graph), median and best of `steps` calls
    after `warmup`.  Returns one dict per (workload, mask, pass, timing form).
    `reduce_max` maps a local time to the max over ranks (identity on one GPU);
    every rank makes the same calls in the same order."""
    import torch

    from io_aware_tiled_b200 import fa
    from io_aware_tiled_b200.configs import WORKLOADS
    from io_aware_tiled_b200.inputs import attention_inputs
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    peak = _peaks()["bf16_tflops"]
    lines = []

    def time_calls(fn, do_flush):
        for _ in range(warmup):
            fn()
        ts = []
        for _ in range(steps):
            if do_flush:
                flush.zero_()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record()
            fn()
            b_.record()
            torch.cuda.synchronize()
            ts.append(a_.elapsed_time(b_))
        rc = fa.sync_status(dev)
        if rc != fa.FA_OK:
            raise RuntimeError(f"library status {fa.status_string(rc)}")
        return reduce_max(statistics.median(ts)), reduce_max(min(ts))

    for w in WORKLOADS.values():
        if w.name in skip:
            continue
        q, k, v, do = (t.to(dev) for t in attention_inputs(w.B, w.H, w.N, w.d, seed=w.seed, sigma_qk=w.sigma_qk))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        ws = torch.empty(fa.workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
        io_bytes = w.B * w.H * w.N * (4 * w.d * 2 + 4)  # Q, K, V read; O written; LSE written
        small = w.B * w.H * w.N <= 4096
        for causal in w.causal_modes:
            passes = [("fwd", lambda: fa.forward(q, k, v, causal, out=o, lse=lse), w.fwd_flops(causal))]
            if w.backward:
                passes.append(("fwd+bwd", lambda: (fa.forward(q, k, v, causal, out=o, lse=lse),
                                                   fa.backward(q, k, v, o, do, lse, causal, workspace=ws,
                                                               dq=dq, dk=dk, dv=dv)),
                               w.fwd_flops(causal) + w.bwd_flops(causal)))
            for name, fn, flops in passes:
                forms = [("eager", True)] + ([("eager", False)] if small else [])
                for launch, do_flush in forms:
                    med, best = time_calls(fn, do_flush)
                    line = {"workload": w.name, "causal": causal, "pass": name, "launch": launch,
                            "kernel": fa.forward_kernel_name(w.d, causal),
                            "median_us": med * 1e3, "best_us": best * 1e3,
                            "tflops_median": flops / (med * 1e-3) / 1e12, "tflops_best": flops / (best * 1e-3) / 1e12,
                            "frac_of_measured_peak_median": flops / (med * 1e-3) / 1e12 / peak,
                            "l2": "flushed before each call" if do_flush else "warm (no flush)",
                            "steps": steps, "warmup": warmup}
                    if name == "fwd":
                        line["gbs_median"] = io_bytes / (med * 1e-3) / 1e9
                        line["gbs_best"] = io_bytes / (best * 1e-3) / 1e9
                    lines.append(line)
                if small:
                    # latency-bound: `steps` eager calls back to back between two
                    # events (the host enqueues the next call while the GPU runs
                    # the current one), per call
                    for _ in range(warmup):
                        fn()
                    a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    torch.cuda.synchronize()
                    a_.record()
                    for _ in range(steps):
                        fn()
                    b_.record()
                    torch.cuda.synchronize()
                    per = reduce_max(a_.elapsed_time(b_) / steps)
                    lines.append({"workload": w.name, "causal": causal, "pass": name, "launch": "eager, back to back",
                                  "mean_us": per * 1e3, "tflops_mean": flops / (per * 1e-3) / 1e12,
                                  "gbs_mean": io_bytes / (per * 1e-3) / 1e9 if name == "fwd" else None,
                                  "l2": "warm (no flush)", "steps": steps, "warmup": warmup})
                    # the same call replayed from a CUDA graph
                    # (no host-side work between the events)
                    fn()
                    torch.cuda.synchronize()
                    graph = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
                        fn()
                    for do_flush in (True, False):
                        med, best = time_calls(graph.replay, do_flush)
                        lines.append({"workload": w.name, "causal": causal, "pass": name, "launch": "graph replay",
                                      "median_us": med * 1e3, "best_us": best * 1e3,
                                      "tflops_median": flops / (med * 1e-3) / 1e12,
                                      "tflops_best": flops / (best * 1e-3) / 1e12,
                                      "gbs_median": io_bytes / (med * 1e-3) / 1e9 if name == "fwd" else None,
                                      "gbs_best": io_bytes / (best * 1e-3) / 1e9 if name == "fwd" else None,
                                      "l2": "flushed before each call" if do_flush else "warm (no flush)",
                                      "steps": steps, "warmup": warmup})
                    del graph
        del q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    return lines


def run_all_configs(steps: int, warmup: int):
    """time_workloads on cuda:0, one JSON line per entry."""
    import torch
    for line in time_workloads(steps, warmup, torch.device("cuda", 0)):
        print(json.dumps(line), flush=True)
    return 0


def run_tile_sweep(steps: int, warmup: int):
    """Forward TFLOP/s of every tile shape the kernels build, B=2, H=16,
    N=4096, d in {64, 128}, with and without the causal mask, beside the
    working set each shape needs (the SRAM model of the first page's section
    1.2, and this layout's shared- and tensor-memory bytes per SM).  One JSON
    line per point."""
    import torch

    from io_aware_tiled_b200 import fa
    from io_aware_tiled_b200.inputs import attention_inputs
    dev = torch.device("cuda", 0)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    B, H, N = 2, 16, 4096
    # (name, FA_FWD_PAIR, FA_FWD_BN, query rows per SM, key tile, stages of K and V, S buffers)
    forms = [("one-SM", "0", "128", 256, 128, None, 2), ("one-SM", "0", "64", 256, 64, None, 2),
             ("paired", "1", "128", 128, 128, 5, 3)]
    for d in (64, 128):
        q, k, v, _ = (t.to(dev) if t is not None else None
                      for t in attention_inputs(B, H, N, d, seed=0, with_do=False))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        for name, pair, bn, tq, tk, st, ns in forms:
            if name == "paired" and d != 128:
                continue
            if st is None:
                st = ((2 if d == 128 else 4) * 128) // tk
            for causal in (False, True):
                os.environ["FA_FWD_PAIR"], os.environ["FA_FWD_BN"] = pair, bn
                try:
                    kname = fa.forward_kernel_name(d, causal)
                    for _ in range(warmup):
                        fa.forward(q, k, v, causal, out=o, lse=lse)
                    ts = []
                    for _ in range(steps):
                        flush.zero_()
                        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        a_.record()
                        fa.forward(q, k, v, causal, out=o, lse=lse)
                        b_.record()
                        torch.cuda.synchronize()
                        ts.append(a_.elapsed_time(b_))
                    rc = fa.sync_status(dev)
                finally:
                    del os.environ["FA_FWD_PAIR"], os.environ["FA_FWD_BN"]
                if rc != fa.FA_OK:
                    raise RuntimeError(f"library status {fa.status_string(rc)}")
                ms = statistics.median(ts)
                f, _ = _flops(B, H, N, d, causal)
                bq = 128  # query rows per softmax warpgroup / TMEM lane block
                q_tiles_per_sm = tq // bq
                q_bufs = 2 if (name == "one-SM" and d == 64) else 1  # d = 64 keeps two Q pairs
                smem = q_bufs * q_tiles_per_sm * bq * d * 2 + st * 2 * (tk if name == "one-SM" else tk // 2) * d * 2
                tmem_cols = ns * tk + q_tiles_per_sm * d if name == "one-SM" else ns * tk + d
                pages_sram = bq * d * 2 + 2 * tk * d * 2 + bq * tk * 2 + bq * d * 2 + bq * 8
                print(json.dumps({
                    "sweep": "forward tile shape", "kernel": kname, "form": name, "d": d, "causal": causal,
                    "T_q_per_sm": tq, "T_k": tk, "kv_stages": st,
                    "tflops": f / (ms * 1e-3) / 1e12, "ms": ms,
                    "smem_bytes_per_sm": smem, "tmem_columns": tmem_cols,
                    "pages_sram_model_bytes": pages_sram,
                    "config": {"B": B, "H": H, "N": N, "l2": "256 MiB written between timed calls"}}),
                    flush=True)
    # the online-softmax rescale threshold (default kernels)
    for d in (64, 128):
        q, k, v, _ = (t.to(dev) if t is not None else None
                      for t in attention_inputs(B, H, N, d, seed=0, with_do=False))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        for causal in (False, True):
            for thr in ("0", "8", "16"):
                os.environ["FA_FWD_RESCALE"] = thr
                try:
                    for _ in range(warmup):
                        fa.forward(q, k, v, causal, out=o, lse=lse)
                    ts = []
                    for _ in range(steps):
                        flush.zero_()
                        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        a_.record()
                        fa.forward(q, k, v, causal, out=o, lse=lse)
                        b_.record()
                        torch.cuda.synchronize()
                        ts.append(a_.elapsed_time(b_))
                    rc = fa.sync_status(dev)
                finally:
                    del os.environ["FA_FWD_RESCALE"]
                if rc != fa.FA_OK:
                    raise RuntimeError(f"library status {fa.status_string(rc)}")
                ms = statistics.median(ts)
                f, _ = _flops(B, H, N, d, causal)
                print(json.dumps({"sweep": "rescale threshold (log2)", "threshold": float(thr),
                                  "kernel": fa.forward_kernel_name(d, causal), "d": d, "causal": causal,
                                  "tflops": f / (ms * 1e-3) / 1e12, "ms": ms}), flush=True)
    # shapes that do not fit this layout (not built)
    print(json.dumps({"sweep": "forward tile shape", "not_built": [
        "T_k=256 with two 128-row Q tiles per SM: S 2x256 + O 2xd TMEM columns > 512",
        "T_q=64 per MMA: M=64 tcgen05 tiles use half the TMEM lanes and half the MMA rate",
        "T_q=256 on one SM: cta_group::1 MMAs stop at M=128; 256 rows per pair is the paired form"]}))
    return 0


def run_ncu_case(case: str, batch: int, workload: str | None = None):
    """A few launches of one kernel family, untimed, for ncu captures: the
    headline shape with B=`batch` (B=4: Q, K, V, O, dO are 67 MB each, so the
    working set exceeds the 126 MB L2), or a named workload's shape and value
    spread.  One warm-up launch, then two."""
    import torch

    from io_aware_tiled_b200 import fa
    from io_aware_tiled_b200.configs import WORKLOADS
    from io_aware_tiled_b200.inputs import attention_inputs
    dev = torch.device("cuda", 0)
    if workload:
        w = WORKLOADS[workload]
        q, k, v, do = (t.to(dev) for t in attention_inputs(w.B, w.H, w.N, w.d, seed=w.seed, sigma_qk=w.sigma_qk))
    else:
        q, k, v, do = (t.to(dev) for t in attention_inputs(batch, 16, 4096, 128, seed=0))
    causal = case.endswith("causal")
    o, lse = fa.forward(q, k, v, causal)
    ws_unf = torch.empty(fa.unfused_workspace_bytes(*q.shape), dtype=torch.uint8, device=dev) \
        if case == "fwd_unfused" else None
    for _ in range(2):
        if case == "fwd_unfused":
            fa.forward_unfused(q, k, v, False, workspace=ws_unf, out=o, lse=lse)
        elif case.startswith("fwd"):
            fa.forward(q, k, v, causal, out=o, lse=lse)
        else:
            fa.backward(q, k, v, o, do, lse, causal)
    rc = fa.sync_status(dev)
    print(f"ncu case {case} {workload or f'B={batch}'}: {fa.status_string(rc)}", flush=True)
    return 0 if rc == fa.FA_OK else 1


def launch_ranks(n: int, impl: str, argv: list) -> int:
    """`--gpus N` without a launcher: start N ranks of this script with
    torch.distributed.run on this node (rendezvous on 127.0.0.1, one rank per
    GPU), wait for them and return their exit status.  The GPU arm needs N
    visible CUDA devices; the reference arm runs on the host cores (rank 0
    only) and needs none."""
    import socket
    if impl == "ours":
        import torch
        have = torch.cuda.device_count()
        if have < n:
            print(f"bench.py: --gpus {n} needs {n} visible CUDA devices, found {have}", file=sys.stderr)
            return 2
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload-steps", type=int, default=20,
                    help="timed calls per leg of the other named workloads in the default run")
    ap.add_argument("--ncu-case", choices=["fwd", "fwd_causal", "bwd", "bwd_causal", "fwd_unfused"], default=None,
                    help="run a few untimed launches for an ncu capture and exit")
    ap.add_argument("--ncu-batch", type=int, default=4)
    ap.add_argument("--ncu-workload", default=None,
                    help="run the --ncu-case on this named workload (its B, H, N, d, spread) instead")
    ap.add_argument("--tile-sweep", action="store_true",
                    help="time the forward for every tile shape the kernels build and exit")
    ap.add_argument("--all-configs", action="store_true",
                    help="time every named workload (fwd, fwd+bwd) and exit")
    args = ap.parse_args(argv)
    if args.all_configs:
        return run_all_configs(max(args.steps, 50), max(args.warmup, 10))
    if args.tile_sweep:
        return run_tile_sweep(max(args.steps, 5), max(args.warmup, 3))
    if args.ncu_case:
        return run_ncu_case(args.ncu_case, args.ncu_batch, args.ncu_workload)

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return launch_ranks(args.gpus, args.impl, sys.argv[1:] if argv is None else list(argv))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU "
              f"(torchrun --nproc-per-node {args.gpus}) or pass --gpus {world}", file=sys.stderr)
        return 2

    if args.impl == "reference":
        return run_reference(args, rank, world)

    import datetime

    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=__import__("torch").device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline()
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
