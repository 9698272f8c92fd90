"""Throughput of the selective-scan (S6) forward on B200: one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward scan (the whole hot path: softplus, discretisation,
recurrence, readout, D skip, gate, final state) over one batch of synthetic
input.  `value` is B*D*L elements per second over all ranks, with inputs
resident in HBM; `e2e` is the same metric through the host-buffer C-ABI entry
point with the host<->device copies inside the timed region.

The scan does not shard across GPUs beyond independent replicas: with N > 1
(torchrun) every rank runs the same workload on its own GPU with no collective
on the data path (weak scaling); the only collectives are the barrier and the
max-over-ranks of the timed interval.

`--impl reference` times the fp64 CPU oracle instead (rank 0 only), on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
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

METRIC = "selective-scan Gelem/s (B*D*L/s) fwd and % of HBM/MUFU roofline on 1 B200"
UNIT = "Gelem/s"
DEFAULT_WORKLOAD = "mamba-2.8b-long"   # the largest single-GPU forward shape
L2_BYTES = 126 * 1024 * 1024
SMS = 148
EX2_PER_CLK_PER_SM = 16          # MUFU ex2 issue rate per SM per clock (sm_80 .. sm_100 family)
NOMINAL_SM_MHZ = 1965.0
HBM_NOMINAL_GBS = 8000.0          # B200 HBM3e, NVIDIA's figure; the roofline's peak is the measured copy rate
PROFILE_DIR = os.path.join(ROOT, "profiles")


def _rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


# ------------------------------------------------------------------ ranks
# One process per GPU (torchrun).  The scan shards only as independent
# replicas, so the only collectives are the barriers around the timed region
# and the max over ranks of its length; every rank takes them in the same order.

def init_ranks(backend: str, local: int, timeout_s: float = 120.0) -> int:
    """Join the process group named by the torchrun environment; returns the world size."""
    import datetime
    import torch.distributed as dist
    _, _, world = _rank_env()
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            import torch
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (the identity on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, elems_per_rank_step: int, steps: int, ms: float) -> float:
    """Whole-job Gelem/s: every rank's elements over the slowest rank's time."""
    return world * elems_per_rank_step * steps / (ms * 1e-3) / 1e9


def finish_ranks():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if dist.get_world_size() > 1:
            dist.barrier()
        dist.destroy_process_group()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", 6650.0)), float(d.get("sm_max_mhz", NOMINAL_SM_MHZ)), "measured"
    return 6650.0, NOMINAL_SM_MHZ, "fallback"


def _bf16_tflops():
    """Measured dense bf16 rate (burst: the kernel is timed in isolation), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f).get("bf16_tflops", 1590.0)), "measured"
    return 1590.0, "fallback"


SSD_Q = 128   # steps per chunk of the tensor-core (SSD) path


def _ssd_flops(d):
    """Algorithmic tensor-core flops of the chunked SSD path per call: per (batch row, head,
    chunk) G = C B^T (2 Q Q N), M X (2 Q Q P), C H (2 Q N P), B'^T X (2 N Q P).  The bf16
    hi/lo splits of M, B' and H double the executed MMAs of the last three; not counted."""
    P = d.dim // d.H
    N = d.dstate
    per = 2 * SSD_Q * (SSD_Q * N + SSD_Q * P + N * P + N * P)
    return d.batch * d.H * (d.seqlen // SSD_Q) * per


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML on a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.ok = False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ helpers

def _alg_bytes(d, with_state=True):
    """Algorithmic HBM bytes of one forward call: every input read once, every output written once."""
    e = 2 if d.dtype == "bf16" else 4
    bdl = d.batch * d.dim * d.seqlen
    b = 3 * bdl * e if d.H == d.dim else 2 * bdl * e + d.batch * d.H * d.seqlen * e   # u, z (+delta)
    b += bdl * e                                                                        # out
    b += 2 * d.batch * d.ngroups * d.dstate * d.seqlen * e                               # B, C
    b += (d.dim * d.dstate if d.H == d.dim else d.H) * 4 + d.dim * 4 + d.H * 4          # A, D, bias
    if with_state:
        b += d.batch * d.dim * d.dstate * 4                                             # last_state
    return b


def _exps(d):
    """exp count of the metric: B*D*L*N (one exp per state per step)."""
    return d.batch * d.dim * d.seqlen * d.dstate


def _kernel_hash():
    """Hash of the scan kernel's sources (the kernel and the layout choice), which the
    committed traffic figure was measured on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_30_b200", "csrc")
    for f in ("scan_kernel.cuh", "layout.h"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _src_hash(files):
    """Hash of kernel source files under csrc/ (what a committed traffic figure was measured on)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_30_b200", "csrc")
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic_from_profiles(workload, key=None, sha=None):
    """dram bytes per launch from a committed ncu summary, if it was taken on this kernel source.
    key: the entry name (default: the workload); sha: the source hash to match (default: the scan kernel's)."""
    p = os.path.join(PROFILE_DIR, "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(key or workload)
    if not ent or ent.get("kernel_src_sha") != (sha or _kernel_hash()):
        return None
    return ent.get("dram_bytes_per_launch")


def _to_dev(arr, dev):
    import torch
    if arr is None:
        return None
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(dev)


def _to_pinned(arr):
    import torch
    if arr is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16) if arr.dtype == np.uint16
                         else np.ascontiguousarray(arr))
    return t.pin_memory()


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_oracle_sample(d, recipe, seed, target_s=12.0):
    """Time the fp64 oracle (as it stands) on a bounded sample of channels of the workload."""
    import oracle
    import ssm_inputs as si
    cores = _cores()
    total = d.batch * d.dim
    rng = np.random.default_rng(7)

    def run(nch, reps=1):
        ch = sorted(int(c) for c in rng.choice(total, size=min(total, nch), replace=False))
        rows = si.make_inputs(d, recipe, seed, channels=ch)
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle.run_inputs(d, rows, channels=ch, nthreads=cores)
        return time.perf_counter() - t0, len(ch)

    # grow the sample until it takes about target_s (the whole workload, repeated,
    # when one pass over it takes less than that)
    nch, reps = min(total, cores), 1
    while True:
        dt, n = run(nch, reps)
        if dt >= target_s / 3:
            break
        grow = target_s / max(dt, 1e-3)
        if nch < total:
            nch = int(min(total, nch * min(grow, 64.0)))
        elif reps < 1000:
            reps = int(min(1000, reps * min(grow, 64.0)))
        else:
            break
    elems = n * d.seqlen * reps
    what = f"{n} of {total} channels" if n < total else f"all {total} channels" + (f", {reps} passes" if reps > 1 else "")
    return {"value": elems / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{what} x L={d.seqlen} (N={d.dstate}), fp64, {dt:.1f} s"}


def _grow_timed(run, target_s, kmax=1 << 16):
    """run(k) -> (seconds, units): grow k (up to kmax, the whole workload) until one run takes
    about target_s (at least a third of it); returns (seconds, units, k)."""
    k = 1
    while True:
        dt, units = run(k)
        if dt >= target_s / 3 or k >= kmax:
            return dt, units, k
        k = min(kmax, int(k * min(64.0, max(2.0, target_s / max(dt, 1e-3)))))


def cpu_oracle_bwd_sample(d, recipe, seed, target_s=8.0):
    """Time the fp64 oracle backward (as it stands) on a bounded sample: batch row 1 and a
    growing number of channels (whole heads in the per-head layout) of the workload's shape."""
    import oracle
    import ssm_inputs as si
    cores = _cores()
    P = d.dim // d.H if d.head_mode else 1
    maxk = d.dim // P

    def run(k):
        k = min(k, maxk)
        sub = si.Dims(1, k * P, d.seqlen, d.dstate, nheads=k if d.head_mode else 0, ngroups=1, dtype=d.dtype)
        inp = si.make_inputs(sub, recipe, seed)
        dout = si.make_grad_inputs(sub, seed + 1)["dout"]
        t0 = time.perf_counter()
        oracle.run_inputs_bwd(sub, inp, dout, nthreads=cores)
        return time.perf_counter() - t0, k * P * d.seqlen

    dt, units, k = _grow_timed(run, target_s, maxk)
    return {"value": units / dt / 1e9, "unit": "Gelem/s", "cores": cores, "kind": "oracle",
            "sample": f"{units // d.seqlen} channels x L={d.seqlen} (N={d.dstate}, batch row 1), fp64 backward, "
                      f"{dt:.1f} s"}


def cpu_oracle_decode_sample(dims, recipe, target_s=5.0):
    """Time the fp64 oracle on decode steps (a scan of one step from a state) of a growing
    number of batch rows of the decode shape."""
    import oracle
    import ssm_inputs as si
    cores = _cores()

    def run(k):
        k = min(k, dims.batch)
        sub = si.Dims(k, dims.dim, 1, dims.dstate, nheads=dims.nheads, ngroups=dims.ngroups, dtype=dims.dtype)
        inp = si.make_inputs(sub, recipe, 0)
        h0 = np.random.default_rng(1).standard_normal((k, dims.dim, dims.dstate))
        t0 = time.perf_counter()
        oracle.run_inputs(sub, inp, h0=h0, nthreads=cores)
        return time.perf_counter() - t0, k * dims.dim

    dt, units, k = _grow_timed(run, target_s, dims.batch)
    return {"value": units / dt / 1e9, "unit": "Gelem/s", "cores": cores, "kind": "oracle",
            "sample": f"{k} batch rows x {dims.dim} channels, one step (N={dims.dstate}), fp64, {dt:.1f} s"}


def cpu_oracle_conv1d_sample(sh, target_s=5.0):
    """Time the fp64 oracle convolution on a growing number of channels of one batch row."""
    import oracle
    cores = _cores()
    rng = np.random.default_rng(0)

    def run(k):
        k = min(k, sh["batch"] * sh["dim"])
        x = rng.standard_normal((1, k, sh["seqlen"]))
        w = rng.standard_normal((k, sh["width"]))
        b = rng.standard_normal(k)
        t0 = time.perf_counter()
        oracle.causal_conv1d(x, w, b, True)
        return time.perf_counter() - t0, k * sh["seqlen"]

    dt, units, k = _grow_timed(run, target_s, sh["batch"] * sh["dim"])
    return {"value": units / dt / 1e9, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
            "sample": f"{k} channels x L={sh['seqlen']} (width {sh['width']}), fp64, one thread, {dt:.1f} s"}


# ------------------------------------------------------------------ arms

def run_reference(args):
    rank, _, world = _rank_env()
    if rank != 0:
        return
    import ssm_inputs as si
    w = si.WORKLOADS[args.workload]
    d = w.dims
    per_step = []
    base = None
    for i in range(args.warmup + args.steps):
        target = max(1.0, min(20.0, 150.0 / max(1, args.warmup + args.steps)))
        r = cpu_oracle_sample(d, w.recipe, w.seed, target_s=target)
        if i >= args.warmup:
            per_step.append(r["value"])
            base = r
    v = statistics.median(per_step)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded splitmix64)",
            "config": {"workload": w.name, "batch": d.batch, "dim": d.dim, "seqlen": d.seqlen,
                       "dstate": d.dstate, "nheads": d.H, "ngroups": d.ngroups, "io_dtype": d.dtype},
            "cpu_baseline": dict(base, value=v),
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class _Nvtx:
    """An NVTX range around a timed region (seen by Nsight tools; a no-op without them)."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        import torch
        try:
            torch.cuda.nvtx.range_push(self.name)
            self.on = True
        except Exception:  # pragma: no cover - no NVTX
            self.on = False
        return self

    def __exit__(self, *a):
        import torch
        if self.on:
            torch.cuda.nvtx.range_pop()


def _probe_mufu(ssm, dev, sh, stream):
    """ex2 rate of the probe kernel in this process (G ex2/s), at whatever clock the GPU runs."""
    import torch
    sink = torch.empty(SMS * 8 * 256, device=dev)
    ssm.ssm_probe_ex2(sink, SMS * 8, 64, sh)
    torch.cuda.synchronize(dev)
    pe0, pe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pe0.record(stream)
    ssm.ssm_probe_ex2(sink, SMS * 8, 2048, sh)
    pe1.record(stream)
    torch.cuda.synchronize(dev)
    return SMS * 8 * 256 * 2048 * 16 / (pe0.elapsed_time(pe1) * 1e-3)


def _roofline(d, info, avg_launch_s, wname, probe_rate):
    """The roofline object of one forward launch: MUFU ex2 (scan kernel) or HBM / tensor (SSD)."""
    hbm_gbs, sm_max_mhz, peak_src = _peaks()
    alg_bytes = _alg_bytes(d)
    exps = _exps(d)
    mufu_peak = SMS * EX2_PER_CLK_PER_SM * sm_max_mhz * 1e6        # ex2/s at the max SM clock
    t_roof = max(alg_bytes / (hbm_gbs * 1e9), exps / mufu_peak)
    hbm_obj = {"achieved": alg_bytes / avg_launch_s / 1e9, "peak": hbm_gbs, "unit": "GB/s",
               "frac": alg_bytes / avg_launch_s / 1e9 / hbm_gbs, "peak_source": peak_src,
               "alg_bytes_per_launch": alg_bytes,
               "frac_of_nominal": alg_bytes / avg_launch_s / 1e9 / HBM_NOMINAL_GBS, "nominal_gbs": HBM_NOMINAL_GBS}
    mufu_obj = {"achieved": exps / avg_launch_s / 1e9, "peak": mufu_peak / 1e9, "unit": "Gexp/s",
                "frac": (exps / avg_launch_s) / mufu_peak,
                "what": "MUFU ex2: B*D*L*N exps per launch / mean launch time; peak = 148 SM x 16 ex2/clk x "
                        f"{sm_max_mhz:.0f} MHz (derived)",
                "mufu_probe_gexps": probe_rate / 1e9, "frac_of_probe": (exps / avg_launch_s) / probe_rate}
    if info["variant"].startswith("ssd_"):
        # the chunked tensor-core path: the bound is the slower of HBM bytes and tensor flops
        tf, tf_src = _bf16_tflops()
        flops = _ssd_flops(d)
        t_hbm, t_tc = alg_bytes / (hbm_gbs * 1e9), flops / (tf * 1e12)
        tensor_obj = {"achieved": flops / avg_launch_s / 1e12, "peak": tf, "unit": "TFLOP/s",
                      "frac": flops / avg_launch_s / 1e12 / tf, "peak_source": tf_src,
                      "flops_per_launch": flops, "what": "algorithmic SSD flops (G, M X, C H, B'^T X per chunk)"}
        main = dict(hbm_obj, bound="hbm") if t_hbm >= t_tc else dict(tensor_obj, bound="tensor")
        traffic = _traffic_from_profiles(wname, key="ssd:" + wname, sha=_src_hash(("ssd.cu", "tcgen05.cuh")))
        return dict(main, traffic=traffic, roofline_frac=max(t_hbm, t_tc) / avg_launch_s,
                    hbm=hbm_obj, tensor=tensor_obj,
                    mufu_literal=dict(mufu_obj, note="B*D*L*N exps: the SSD path takes one exp per (t, head)"))
    return {"bound": "alu", "achieved": mufu_obj["achieved"], "peak": mufu_obj["peak"], "unit": "Gexp/s",
            "frac": mufu_obj["frac"], "traffic": _traffic_from_profiles(wname), "what": mufu_obj["what"],
            "roofline_frac": t_roof / avg_launch_s, "hbm": hbm_obj,
            "mufu_probe_gexps": mufu_obj["mufu_probe_gexps"], "frac_of_probe": mufu_obj["frac_of_probe"]}


class _ScanJob:
    """One forward workload resident on the device: rotating input sets, a plan, and a step."""

    NAMES = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")

    def __init__(self, ssm, w, dev, local):
        import torch
        self.ssm, self.w, self.dev = ssm, w, dev
        d = self.d = w.dims
        io = ssm.SSM_BF16 if d.dtype == "bf16" else ssm.SSM_F32
        import ssm_inputs as si
        self.inp = si.make_inputs(d, w.recipe, w.seed)
        self.alg_bytes = _alg_bytes(d)
        # enough copies that consecutive steps never find their inputs in L2
        self.copies = max(2, int(np.ceil(3 * L2_BYTES / self.alg_bytes)))
        self.sets = []
        for _ in range(self.copies):
            t = {k: _to_dev(self.inp[k], dev) for k in self.NAMES}
            t["out"] = torch.empty_like(t["u"])
            t["last"] = torch.empty(d.batch, d.dim, d.dstate, dtype=torch.float32, device=dev)
            self.sets.append(t)
        self.dims = ssm.make_dims(d.batch, d.dim, d.seqlen, d.dstate, d.H, d.ngroups, io)
        self.plan = ssm.ssm_scan_plan(self.dims, local)
        self.info = ssm.ssm_scan_plan_info(self.plan)
        self.sched = ssm.ssm_scan_plan_schedule(self.plan)
        self.stream = torch.cuda.current_stream(dev)
        self.sh = self.stream.cuda_stream

    def step(self, i):
        t = self.sets[i % self.copies]
        self.ssm.ssm_selective_scan_fwd(self.plan, t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                        t["delta_bias"], self.w.recipe.softplus, self.dims, t["out"], t["last"],
                                        self.sh)

    def timed(self, steps, warmup, local):
        """Warm up, then time exactly `steps` launches with CUDA events on the launching stream
        (barrier + synchronize on both sides); returns per-launch ms, the max-over-ranks total ms
        and the clock record."""
        import torch
        for i in range(warmup):
            self.step(i)
        torch.cuda.synchronize(self.dev)
        barrier()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        with ClockSampler(local) as clk, _Nvtx(f"timed:{self.w.name}"):
            torch.cuda.synchronize(self.dev)
            for i in range(steps):
                starts[i].record(self.stream)
                self.step(i)
                ends[i].record(self.stream)
            torch.cuda.synchronize(self.dev)
        barrier()
        launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        total_ms = max_over_ranks(starts[0].elapsed_time(ends[-1]), self.dev)
        st = self.ssm.ssm_scan_device_status(self.plan, self.sh)
        if st != self.ssm.SSM_OK:
            raise RuntimeError(f"{self.w.name}: device status {self.ssm.ssm_status_string(st)}")
        return launch_ms, total_ms, clk.summary()

    def e2e(self, steps, world):
        """The same metric through the host-buffer entry point: pinned host inputs, copies in the timed region."""
        import torch
        d, ssm, names = self.d, self.ssm, self.NAMES
        hp = {k: _to_pinned(self.inp[k]) for k in names}
        hout = torch.empty(d.batch, d.dim, d.seqlen, dtype=torch.int16 if d.dtype == "bf16" else torch.float32,
                           pin_memory=True)
        hlast = torch.empty(d.batch, d.dim, d.dstate, dtype=torch.float32, pin_memory=True)

        def hstep():
            ssm.ssm_selective_scan_fwd_host(self.plan, hp["u"], hp["delta"], hp["A"], hp["B"], hp["C"], hp["D"],
                                            hp["z"], hp["delta_bias"], self.w.recipe.softplus, self.dims, hout,
                                            hlast, self.sh)
        for _ in range(2):
            hstep()
        torch.cuda.synchronize(self.dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with _Nvtx(f"e2e:{self.w.name}"):
            e0.record(self.stream)
            for _ in range(steps):
                hstep()
            e1.record(self.stream)
            torch.cuda.synchronize(self.dev)
        ems = max_over_ranks(e0.elapsed_time(e1), self.dev)
        h2d = sum(hp[k].numel() * hp[k].element_size() for k in names if hp[k] is not None)
        d2h = hout.numel() * hout.element_size() + hlast.numel() * hlast.element_size()
        return {"value": job_throughput(world, d.batch * d.dim * d.seqlen, steps, ems), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
                "path": "ssm_selective_scan_fwd_host (pinned host buffers)"}

    def close(self):
        import torch
        self.ssm.ssm_scan_destroy(self.plan)
        self.sets = []
        self.inp = None
        torch.cuda.synchronize(self.dev)
        torch.cuda.empty_cache()


PER_CONFIG_MIN_MS = 40.0   # each per-config line times at least this long (more launches for small shapes)


def _config_entry(job, launch_ms, total_ms, steps, clocks, probe_rate):
    d = job.d
    avg_s = statistics.mean(launch_ms) * 1e-3
    roof = _roofline(d, job.info, avg_s, job.w.name, probe_rate)
    elems = d.batch * d.dim * d.seqlen
    return {"shape": {"batch": d.batch, "dim": d.dim, "seqlen": d.seqlen, "dstate": d.dstate, "nheads": d.H,
                      "ngroups": d.ngroups, "io_dtype": d.dtype},
            "kernel": job.info["variant"], "grid": job.info["grid"], "block": job.info["block"],
            "schedule": job.sched, "steps": steps, "ms_per_call": total_ms / steps,
            "gelem_s": elems * steps / (total_ms * 1e-3) / 1e9,
            "roofline": {"bound": roof["bound"], "frac": roof["frac"], "unit": roof["unit"],
                         "achieved": roof["achieved"], "peak": roof["peak"],
                         "roofline_frac": roof["roofline_frac"], "hbm_frac": roof["hbm"]["frac"],
                         "traffic": roof["traffic"], "alg_bytes_per_launch": roof["hbm"]["alg_bytes_per_launch"]},
            "clocks": clocks}


def _bench_workload(args):
    """The named workload; with --seqlen, the same shape at a shorter sequence length (a smaller case
    of the same kernel, for profiler captures that must stay small).  The renamed workload matches no
    committed traffic figure."""
    import dataclasses
    import ssm_inputs as si
    w = si.WORKLOADS[args.workload]
    if not args.seqlen:
        return w
    return dataclasses.replace(w, name=f"{w.name}@L{args.seqlen}",
                               dims=dataclasses.replace(w.dims, seqlen=args.seqlen))


def run_ours(args):
    import torch
    import ssm_inputs as si
    import selective_state_space_30_b200 as ssm

    rank, local, world = _rank_env()
    if world > 1:
        torch.cuda.set_device(local)
    init_ranks("nccl", local)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = _bench_workload(args)
    d = w.dims
    stream = torch.cuda.current_stream(dev)
    probe_rate = _probe_mufu(ssm, dev, stream.cuda_stream, stream)

    # the headline: exactly K timed steps of the named workload
    job = _ScanJob(ssm, w, dev, local)
    if args.layout:
        # a forced kernel layout (consumer warps, states per lane, time sub-chunks, kernel: 1 = register,
        # 2 = tensor memory), to time the kernels the plan does not pick by default
        lw, ls, lk, lm = (int(x) for x in args.layout.split(","))
        for opt, val in ((ssm.SSM_OPT_TENSOR_MEMORY, lm), (ssm.SSM_OPT_CONSUMER_WARPS, lw),
                         (ssm.SSM_OPT_STATES_PER_LANE, ls), (ssm.SSM_OPT_TIME_LANES, lk)):
            ssm.ssm_scan_set_option(job.plan, opt, val)
        job.info = ssm.ssm_scan_plan_info(job.plan)
        job.sched = ssm.ssm_scan_plan_schedule(job.plan)
    launch_ms, total_ms, clocks = job.timed(args.steps, args.warmup, local)
    elems = d.batch * d.dim * d.seqlen
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, elems, args.steps, total_ms)
    roof = _roofline(d, job.info, statistics.mean(launch_ms) * 1e-3, w.name, probe_rate)
    per_config = {w.name: _config_entry(job, launch_ms, total_ms, args.steps, clocks, probe_rate)}
    e2e = None if args.no_e2e else job.e2e(max(3, min(args.steps, 50)), world)
    info, sched, copies, alg_bytes = job.info, job.sched, job.copies, job.alg_bytes
    job.close()

    # every other forward workload, one line each (the driver sees all five shapes)
    if not args.no_per_config:
        for name, wk in si.WORKLOADS.items():
            if name == args.workload:
                continue
            j = _ScanJob(ssm, wk, dev, local)
            # a short probe sizes the run so that each line times at least PER_CONFIG_MIN_MS
            pm, _, _ = j.timed(3, args.warmup, local)
            n = max(args.steps, int(np.ceil(PER_CONFIG_MIN_MS / max(statistics.mean(pm), 1e-3))))
            lm, tm, ck = j.timed(n, 2, local)
            per_config[name] = _config_entry(j, lm, tm, n, ck, probe_rate)
            j.close()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(d, w.recipe, w.seed)
        # the oracle beside every other shape too, on a shorter sample each
        for name, e in per_config.items():
            wk = si.WORKLOADS[name]
            e["cpu_baseline"] = cpu_oracle_sample(wk.dims, wk.recipe, wk.seed, target_s=3.0)

    finish_ranks()
    if rank != 0:
        return
    n_launch = args.steps * info["launches_per_call"]
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32 (bf16 I/O)" if d.dtype == "bf16" else "f32",
            "data": "synthetic (seeded splitmix64; shapes/inits of the Mamba layer)",
            "config": {"workload": w.name, "batch": d.batch, "dim": d.dim, "seqlen": d.seqlen, "dstate": d.dstate,
                       "nheads": d.H, "ngroups": d.ngroups, "io_dtype": d.dtype, "parallelism": f"replicas x{world}",
                       "l2": f"{copies} rotating input sets of {alg_bytes / 1e6:.0f} MB (> 3x 126 MB L2), no flush",
                       "kernel": info["variant"], "grid": info["grid"], "block": info["block"],
                       "schedule": sched},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clocks, "gpu_launches": n_launch,
            "per_config": per_config}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ decode step

DECODE_SHAPES = {
    # one generation step of a Mamba-1.4B layer (d_inner 4096, N 16) for 256 sequences
    "decode-mamba-1.4b-b256": dict(batch=256, dim=4096, dstate=16, nheads=4096, ngroups=1, dtype="bf16"),
    # one step of the Mamba-2-style layer (32 heads x 64, N 128) for 64 sequences
    "decode-mamba2-n128-b64": dict(batch=64, dim=2048, dstate=128, nheads=32, ngroups=1, dtype="bf16"),
}


def _decode_bytes(sh):
    """Algorithmic HBM bytes of one step: the state read and written, u, delta, z read, out written,
    B and C read, A, D, bias read."""
    e = 2 if sh["dtype"] == "bf16" else 4
    b, d, n, h, g = sh["batch"], sh["dim"], sh["dstate"], sh["nheads"], sh["ngroups"]
    return (2 * b * d * n * 4 + 3 * b * d * e + b * h * e + 2 * b * g * n * e +
            (d * n if h == d else h) * 4 + d * 4 + h * 4)


def run_decode(args):
    """ssm_selective_state_update on a decode shape: one JSON line (GB/s against the HBM roofline)."""
    import torch
    import ssm_inputs as si
    import selective_state_space_30_b200 as ssm
    rank, local, world = _rank_env()
    if world > 1:
        torch.cuda.set_device(local)
    init_ranks("nccl", local)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sh = DECODE_SHAPES[args.workload]
    dims = si.Dims(sh["batch"], sh["dim"], 1, sh["dstate"], nheads=sh["nheads"] if sh["nheads"] != sh["dim"] else 0,
                   ngroups=sh["ngroups"], dtype=sh["dtype"])
    rec = si.Recipe(a_init="neg_uniform_1_16" if dims.head_mode else "neg_n_plus_1", d_init="normal",
                    delta_init="normal_half")
    inp = si.make_inputs(dims, rec, 0)
    names = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
    alg = _decode_bytes(sh)
    copies = max(2, int(np.ceil(3 * L2_BYTES / alg)))
    sets = []
    for i in range(copies):
        t = {k: _to_dev(inp[k], dev) for k in names}
        t["state"] = torch.randn(dims.batch, dims.dim, dims.dstate, device=dev, generator=None)
        t["out"] = torch.empty_like(t["u"])
        sets.append(t)
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, 1, dims.dstate, dims.H, dims.ngroups, io)
    stream = torch.cuda.current_stream(dev)
    sh_ = stream.cuda_stream

    def step(i):
        t = sets[i % copies]
        ssm.ssm_selective_state_update(d, t["state"], t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                       t["delta_bias"], True, t["out"], sh_)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    total = max_over_ranks(e0.elapsed_time(e1), dev)
    hbm_gbs, _, src = _peaks()
    finish_ranks()
    if rank != 0:
        return
    gbs = alg / (ms * 1e-3) / 1e9
    cpu = None if (world > 1 or args.no_cpu_baseline) else cpu_oracle_decode_sample(dims, rec)
    line = {"metric": "selective-state-update (decode step) Gelem/s (batch rows x channels per second) on 1 B200",
            "op": "decode",
            "value": world * dims.batch * dims.dim * args.steps / (total * 1e-3) / 1e9, "unit": "Gelem/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 (bf16 I/O)" if dims.dtype == "bf16" else "f32", "data": "synthetic (seeded splitmix64)",
            "config": dict(sh, workload=args.workload,
                           l2=f"{copies} rotating state/input sets of {alg / 1e6:.0f} MB, no flush"),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
                         "traffic": _traffic_from_profiles(args.workload, key="decode:" + args.workload,
                                                           sha=_src_hash(("decode.cu",))),
                         "peak_source": src, "alg_bytes_per_launch": alg},
            "cpu_baseline": cpu, "clocks": clk.summary(), "gpu_launches": args.steps}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ causal conv1d

CONV_SHAPES = {
    # the x of the mamba-130m layer: batch 8, d_inner 1536, L 2048, d_conv 4, bf16
    "conv1d-mamba-130m": dict(batch=8, dim=1536, seqlen=2048, width=4, dtype="bf16"),
    # the x of the mamba-1.4b layer: batch 4, d_inner 4096, L 4096
    "conv1d-mamba-1.4b": dict(batch=4, dim=4096, seqlen=4096, width=4, dtype="bf16"),
}


def run_conv1d(args):
    """ssm_causal_conv1d_fwd on a layer's x: one JSON line (GB/s against the HBM roofline)."""
    import torch
    import ssm_inputs as si
    import selective_state_space_30_b200 as ssm
    rank, local, world = _rank_env()
    if world > 1:
        torch.cuda.set_device(local)
    init_ranks("nccl", local)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sh = CONV_SHAPES[args.workload]
    dims = si.Dims(sh["batch"], sh["dim"], sh["seqlen"], 16, dtype=sh["dtype"])
    x = si.make_inputs(dims, si.Recipe(), 0)["u"]
    e = 2 if sh["dtype"] == "bf16" else 4
    elems = sh["batch"] * sh["dim"] * sh["seqlen"]
    alg = 2 * elems * e + sh["dim"] * (sh["width"] + 1) * 4          # x read, out written, taps and bias
    copies = max(2, int(np.ceil(3 * L2_BYTES / alg)))
    rng = np.random.default_rng(0)
    w = torch.from_numpy((rng.standard_normal((sh["dim"], sh["width"])) / 2).astype(np.float32)).to(dev)
    b = torch.from_numpy((rng.standard_normal(sh["dim"]) * 0.1).astype(np.float32)).to(dev)
    sets = []
    for _ in range(copies):
        xd = _to_dev(x, dev)
        sets.append((xd, torch.empty_like(xd)))
    io = ssm.SSM_BF16 if sh["dtype"] == "bf16" else ssm.SSM_F32
    stream = torch.cuda.current_stream(dev)

    def step(i):
        xd, od = sets[i % copies]
        ssm.ssm_causal_conv1d_fwd(sh["batch"], sh["dim"], sh["seqlen"], sh["width"], io, xd, w, b, True, od,
                                  stream.cuda_stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    total = max_over_ranks(e0.elapsed_time(e1), dev)
    hbm_gbs, _, src = _peaks()
    finish_ranks()
    if rank != 0:
        return
    gbs = alg / (ms * 1e-3) / 1e9
    cpu = None if (world > 1 or args.no_cpu_baseline) else cpu_oracle_conv1d_sample(sh)
    line = {"metric": "causal conv1d (d_conv taps + SiLU) Gelem/s on 1 B200", "op": "conv1d",
            "value": job_throughput(world, elems, args.steps, total), "unit": "Gelem/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 (bf16 I/O)" if sh["dtype"] == "bf16" else "f32", "data": "synthetic (seeded splitmix64)",
            "config": dict(sh, workload=args.workload,
                           l2=f"{copies} rotating input sets of {alg / 1e6:.0f} MB, no flush"),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
                         "traffic": _traffic_from_profiles(args.workload, key="conv1d:" + args.workload,
                                                           sha=_src_hash(("conv1d.cu",))),
                         "peak_source": src, "alg_bytes_per_launch": alg},
            "cpu_baseline": cpu, "clocks": clk.summary(), "gpu_launches": args.steps}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ backward scan

BWD_WORKLOADS = ("mamba-130m", "mamba-1.4b", "mamba-2.8b-long", "mamba2-n128")


def _bwd_bytes(d):
    """Algorithmic HBM bytes of one backward call: u, delta, z, dout, B, C, A, D, bias read;
    du, ddelta, dz written in the I/O dtype, dB, dC fp32, dA, dD, dbias fp32."""
    e = 2 if d.dtype == "bf16" else 4
    elems = d.batch * d.dim * d.seqlen
    helems = d.batch * d.H * d.seqlen          # delta and ddelta rows: per channel, or per head
    bc = d.batch * d.ngroups * d.dstate * d.seqlen
    nA = d.H if d.head_mode else d.dim * d.dstate
    return 5 * elems * e + 2 * helems * e + 2 * bc * e + 2 * bc * 4 + 2 * (nA + d.dim + d.H) * 4


def run_bwd(args):
    """ssm_selective_scan_bwd on a layer shape: one JSON line (Gelem/s; roofline against the MUFU ex2 rate,
    B*D*L*N exps: each dA of the forward must be formed again at least once)."""
    import torch
    import ssm_inputs as si
    import selective_state_space_30_b200 as ssm
    rank, local, world = _rank_env()
    if world > 1:
        torch.cuda.set_device(local)
    init_ranks("nccl", local)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = _bench_workload(args)
    d = w.dims
    inp = si.make_inputs(d, w.recipe, w.seed)
    gin = si.make_grad_inputs(d, 1)
    t = {k: _to_dev(inp[k], dev) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    dout = _to_dev(gin["dout"], dev)
    io = ssm.SSM_BF16 if d.dtype == "bf16" else ssm.SSM_F32
    dims = ssm.make_dims(d.batch, d.dim, d.seqlen, d.dstate, d.H, d.ngroups, io)
    nws = ssm.ssm_selective_scan_bwd_workspace_size(dims)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"du": torch.empty_like(t["u"]), "ddelta": torch.empty_like(t["delta"]), "dA": torch.empty_like(t["A"]),
         "dB": torch.empty(t["B"].shape, **f32), "dC": torch.empty(t["C"].shape, **f32),
         "dD": torch.empty((d.dim,), **f32), "dz": torch.empty_like(t["z"]),
         "ddelta_bias": torch.empty((d.H,), **f32), "dh0": None}
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(int(x.numel() * x.element_size()) for x in list(t.values()) + [dout] if x is not None)

    # the forward's stored states (the training path: the backward then skips its recomputation),
    # where the tiled backward takes the shape; the generic backward always recomputes
    stored = ssm.bwd_covers(t["u"], t["delta"], t["A"], t["B"])
    plan = ssm.ssm_scan_plan(dims, local)
    nwin = (d.seqlen + 7) // 8
    ck = torch.empty((d.batch, d.dim, nwin, d.dstate), **f32) if stored else None
    fout = torch.empty_like(t["u"])
    fwd_args = (plan, t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"], t["delta_bias"], True, dims,
                None, fout, None)
    if stored:
        ssm.ssm_selective_scan_fwd_ckpt(*fwd_args, ck, stream.cuda_stream)

    def bwd_step(states):
        return lambda: ssm.ssm_selective_scan_bwd_ckpt(dims, t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"],
                                                       t["z"], t["delta_bias"], True, None, dout, None, states, g,
                                                       ws, nws, stream.cuda_stream)

    def timed(step, steps):
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local) as clk:
            e0.record(stream)
            for _ in range(steps):
                step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
        barrier()
        return e0.elapsed_time(e1) / steps, max_over_ranks(e0.elapsed_time(e1), dev), clk.summary()

    ms_re, total_re, clocks_re = timed(bwd_step(None), args.steps)
    if stored:
        ms, total, clocks = timed(bwd_step(ck), args.steps)
        ms_fc, _, _ = timed(lambda: ssm.ssm_selective_scan_fwd_ckpt(*fwd_args, ck, stream.cuda_stream), args.steps)
    else:
        ms, total, clocks, ms_fc = ms_re, total_re, clocks_re, None
    ms_f, _, _ = timed(lambda: ssm.ssm_selective_scan_fwd_h0(*fwd_args, stream.cuda_stream), args.steps)
    ssm.ssm_scan_destroy(plan)
    hbm_gbs, sm_max_mhz, src = _peaks()
    cpu = None if (world > 1 or args.no_cpu_baseline) else cpu_oracle_bwd_sample(d, w.recipe, w.seed)
    finish_ranks()
    if rank != 0:
        return
    elems = d.batch * d.dim * d.seqlen
    exps = _exps(d)
    mufu_peak = SMS * EX2_PER_CLK_PER_SM * sm_max_mhz * 1e6 / 1e9
    alg = _bwd_bytes(d)
    ck_bytes = int(ck.numel() * 4) if stored else 0

    def roof(ms_, traffic_key, state_bytes=0):
        # algorithmic bytes: the call's inputs read and outputs written (the stored states are
        # an input of the stored-state call)
        a = alg + state_bytes
        gexps = exps / (ms_ * 1e-3) / 1e9
        gbs = a / (ms_ * 1e-3) / 1e9
        return {"bound": "alu", "achieved": gexps, "peak": mufu_peak, "unit": "Gexp/s", "frac": gexps / mufu_peak,
                "traffic": _traffic_from_profiles(w.name, key=traffic_key,
                                                  sha=_src_hash(("bwd.cu",) if stored else ("bwd_generic.cu",))),
                "peak_source": f"148 SMs x 16 ex2/clk x {sm_max_mhz:.0f} MHz ({src} sm_max_mhz)",
                "exps_per_launch": exps,
                "hbm": {"achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
                        "alg_bytes_per_launch": a, "state_bytes_read": state_bytes, "peak_source": src}}

    line = {"metric": "selective-scan backward Gelem/s (B*D*L/s) on 1 B200", "op": "bwd",
            "value": job_throughput(world, elems, args.steps, total), "unit": "Gelem/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 (bf16 I/O)" if d.dtype == "bf16" else "f32", "data": "synthetic (seeded splitmix64)",
            "config": {"workload": w.name, "batch": d.batch, "dim": d.dim, "seqlen": d.seqlen,
                       "dstate": d.dstate, "io_dtype": d.dtype, "parallelism": f"replicas x{world}",
                       "states": (f"stored by the forward every 8 steps (ssm_selective_scan_fwd_ckpt, "
                                  f"{ck_bytes / 1e6:.0f} MB), read by ssm_selective_scan_bwd_ckpt") if stored else
                                 "recomputed (the generic backward: per-head layout or dstate other than 16)",
                       "l2": f"inputs {in_bytes / 1e6:.0f} MB and workspace {nws / 1e6:.0f} MB (> 126 MB L2), "
                             "no flush"},
            "roofline": roof(ms, ("bwd_ckpt:" if stored else "bwd:") + w.name, ck_bytes),
            "recompute": {"what": "ssm_selective_scan_bwd: the backward recomputes the states itself",
                          "ms_per_step": ms_re, "value": job_throughput(world, elems, args.steps, total_re),
                          "roofline": roof(ms_re, "bwd:" + w.name)},
            "forward": {"ms_plain": ms_f, "ms_with_states": ms_fc, "state_bytes": ck_bytes},
            "cpu_baseline": cpu, "clocks": clocks, "gpu_launches": (2 if stored else 4) * args.steps}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None,
                    help=f"the shape (default: {DEFAULT_WORKLOAD} for the scan, a per-op default otherwise)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layout", default="",
                    help="force the headline's kernel layout: warps,states_per_lane,time_lanes,kernel "
                         "(kernel 1 = register, 2 = tensor memory; 0 = automatic), e.g. 16,2,1,2")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="replace the workload's sequence length (a smaller case for profiler captures)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the named workload (default: also one line per other forward workload)")
    ap.add_argument("--op", default="scan", choices=["scan", "decode", "conv1d", "bwd"],
                    help="scan: the forward scan (the headline metric); decode: the single-step state update; "
                         "conv1d: the causal convolution in front of the scan; bwd: the backward scan")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.op == "decode":
        if args.workload is None:
            args.workload = "decode-mamba-1.4b-b256"
        run_decode(args)
        return
    if args.op == "conv1d":
        if args.workload is None:
            args.workload = "conv1d-mamba-130m"
        run_conv1d(args)
        return
    if args.op == "bwd":
        if args.workload is None:
            args.workload = "mamba-130m"
        if args.workload not in BWD_WORKLOADS:
            raise SystemExit(f"--op bwd runs on {BWD_WORKLOADS}")
        run_bwd(args)
        return
    if args.workload is None:
        args.workload = DEFAULT_WORKLOAD
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
