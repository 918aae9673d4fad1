"""Benchmark of the fused attention forward pass on B200: prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload C2] [--no-extra]

A step is one pass of the whole path over the workload: for the default workload
(B=4, H=16, Sq=Sk=1024, D=64, fp16, seed 1) a non-causal pass and a causal pass on
the same tensors, each one launch of the CUDA kernel through the C ABI.  The metric
is TFLOP/s with FLOPs = 4*B*H*Sq*Sk*D per pass, halved for causal.

Timing: inputs resident in device memory; W untimed warm-up steps; then exactly K
steps, each bracketed by CUDA events on the launching stream, with a 256 MB buffer
written between steps so every step starts with a cold L2 (the workload's 25 MB of
inputs would otherwise stay in the 126 MB L2); barrier + synchronize on both sides;
the max over ranks of the summed step time.  Multi-GPU runs (torchrun, one rank per
GPU) give every rank its own copy of the workload (weak scaling, no collective on
the data path).

Also reported: `e2e` (the same steps through attn_fwd_host from pinned host buffers,
copies included), `roofline` (the dominant kernel's achieved TFLOP/s against the
measured dense bf16 peak), `cpu_baseline` (the fp64 CPU oracle on a bounded sample
of the workload, rank 0 at N=1), `clocks` (NVML samples taken during the timed
region) and `extra` (the other large workloads, and the split-KV pass on
decode-shaped workloads, timed the same way, outside the timed region).
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs  # noqa: E402

FLUSH_BYTES = 256 << 20
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
# DRAM bytes (read + write) per launch of the dominant kernel from an ncu capture of
# the same kernel build (profiles/attn_fwd_kernel_D64_f16_B4H16S1024_bench_workload.md);
# a workload without a matching capture reports null.
NCU_TRAFFIC_BYTES = {"C2-noncausal": 25225472}


# The metric both arms report (the headline benchmark's own wording).
METRIC = "attention fwd TFLOP/s on 1 B200 (causal & non-causal), % of bf16 TC peak"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="C2", choices=sorted(WORKLOADS))
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--profile-once", action="store_true",
                    help="launch each pass of the workload once and exit (for ncu captures)")
    ap.add_argument("--profile-extra", default=None,
                    help="with --profile-once: a DEC*, SMX*, GEMM* or WD* workload instead, "
                         "optionally scaled down as NAME:n (M for GEMM*, rows for SMX*, B for "
                         "DEC*, H for WD*)")
    return ap.parse_args()


# ---------------------------------------------------------------- process group
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local) if backend == "nccl"
                                else None)
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a float over ranks (host value in, host value out)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- peaks / clocks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"bf16_tflops": FALLBACK_BF16_TFLOPS, "hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


class ClockSampler:
    """NVML samples of SM clock and clock-event reasons on a background thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        self._window = [None, None]
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than fail
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def mark(self, which):
        self._window[which] = time.perf_counter()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        t0, t1 = self._window
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = f"{len(inside)} samples inside the timed region"
        if not inside:  # region shorter than the sampling period: nearest samples
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            note = "timed region shorter than the sampling period; nearest samples"
        mask = 0
        for s in inside:
            mask |= s[2]
        reasons = [n for b, n in self.REASONS.items() if mask & b]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "note": note}


# ---------------------------------------------------------------- CUDA arm
def time_steps(launches, steps, warmup, flush, stream):
    """Run `warmup` untimed steps, then `steps` timed ones.  `launches` is a list of
    zero-argument callables, one per kernel launch of a step.  Returns per-launch
    event times (ms), shape [steps][len(launches)]."""
    for _ in range(warmup):
        for f in launches:
            f()
    n = len(launches)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.add_(1)  # write > L2 between timed steps
        ev[i][0].record(stream)
        for j, f in enumerate(launches):
            f()
            ev[i][j + 1].record(stream)
    torch.cuda.synchronize()
    return [[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(n)] for i in range(steps)]


def cuda_arm(args, world, rank, local):
    import attention_forward_18_b200 as af

    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    q, k, v = make_inputs(w)
    dq, dk, dv = q.to(dev), k.to(dev), v.to(dev)
    outs = {c: (torch.empty_like(dq), torch.empty((w.B, w.H, w.Sq), dtype=torch.float32,
                                                  device=dev)) for c in w.causal}
    dcode = af.ATTN_F16 if w.dtype == "f16" else af.ATTN_BF16

    def launcher(causal):
        o, lse = outs[causal]
        args_ = (dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), o.data_ptr(), lse.data_ptr(),
                 w.B, w.H, w.Sq, w.Sk, w.D, int(causal), w.scale, dcode, sptr)

        def f():
            rc = af.attn_fwd(*args_)
            if rc != 0:
                raise af.AttnError(rc, "attn_fwd")
        return f

    launches = [launcher(c) for c in w.causal]
    flops_step = sum(w.flops(c) for c in w.causal)
    flush = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    # bring the clocks up before the warm-up steps (untimed)
    t_end = time.perf_counter() + 0.3
    while time.perf_counter() < t_end:
        for f in launches:
            f()
        torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark(0)
    times = time_steps(launches, args.steps, args.warmup, flush, stream)
    sampler.mark(1)
    barrier(world)
    sampler.stop()
    status = af.attn_fwd_status(stream)
    if status != 0:
        raise af.AttnError(status, "device status after the timed region")

    total_ms = sum(sum(t) for t in times)
    total_ms = max_over_ranks(total_ms, world)
    value = world * flops_step * args.steps / (total_ms * 1e-3) / 1e12

    # dominant kernel: the launch slot with the largest summed time
    per_slot = [sum(t[j] for t in times) for j in range(len(launches))]
    dom = max(range(len(launches)), key=lambda j: per_slot[j])
    dom_causal = w.causal[dom]
    dom_ms = per_slot[dom] / args.steps
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))  # fp16 = bf16 nominal rate
    achieved = w.flops(dom_causal) / (dom_ms * 1e-3) / 1e12
    key = f"{w.name}-{'causal' if dom_causal else 'noncausal'}"
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": NCU_TRAFFIC_BYTES.get(key),
                "kernel": f"attn_fwd_kernel<D={w.D},{w.dtype},causal={dom_causal}>",
                "peak_source": f"{peak_kind} dense bf16 (burst; fp16 has the same nominal rate)",
                "per_launch_ms": round(dom_ms, 5),
                "hbm_gbs_at_algorithmic_bytes": round(
                    w.io_bytes() / (dom_ms * 1e-3) / 1e9, 1)}

    e2e = e2e_arm(af, w, q, k, v, dev, sptr, args, world)
    clocks = sampler.summary()

    line = {
        "metric": METRIC,
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16" if w.dtype == "f16" else "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} Sq={w.Sq} Sk={w.Sk} D={w.D} "
                               f"{w.dtype}, non-causal + causal passes per step, seed {w.seed}",
                   "B": w.B, "H": w.H, "Sq": w.Sq, "Sk": w.Sk, "D": w.D,
                   "causal_modes": list(w.causal), "accumulate": "fp32",
                   "l2": "flushed between timed steps (256 MB write)",
                   "parallelism": f"dp{world} (independent copy per GPU)"},
        "per_pass_ms": {("causal" if c else "noncausal"): round(per_slot[j] / args.steps, 5)
                        for j, c in enumerate(w.causal)},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": len(launches) * args.steps,
        "clocks": clocks,
    }
    return line


def e2e_arm(af, w, q, k, v, dev, sptr, args, world):
    """Same steps through attn_fwd_host: pinned host inputs copied in, outputs copied
    out, every step (copies inside the timed region)."""
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = {c: torch.empty_like(q).pin_memory() for c in w.causal}
    lh = {c: torch.empty((w.B, w.H, w.Sq), dtype=torch.float32).pin_memory() for c in w.causal}
    staging = (torch.empty_like(q, device=dev), torch.empty_like(k, device=dev),
               torch.empty_like(v, device=dev), torch.empty_like(q, device=dev),
               torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev))
    dcode = af.ATTN_F16 if w.dtype == "f16" else af.ATTN_BF16

    def step():
        for c in w.causal:
            rc = af.attn_fwd_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(),
                                  oh[c].data_ptr(), lh[c].data_ptr(),
                                  *(t.data_ptr() for t in staging), w.B, w.H, w.Sq, w.Sk,
                                  w.D, int(c), w.scale, dcode, sptr)
            if rc != 0:
                raise af.AttnError(rc, "attn_fwd_host")

    steps = max(3, min(args.steps, 50))
    for _ in range(max(3, args.warmup // 4)):
        step()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s = torch.cuda.current_stream(dev)
    e0.record(s)
    for _ in range(steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    flops_step = sum(w.flops(c) for c in w.causal)
    n = len(w.causal)
    return {"value": round(world * flops_step * steps / (ms * 1e-3) / 1e12, 4),
            "unit": "TFLOP/s", "steps": steps,
            "h2d_bytes_per_step": n * (q.nbytes + k.nbytes + v.nbytes),
            "d2h_bytes_per_step": n * (q.nbytes + 4 * w.B * w.H * w.Sq),
            "path": "attn_fwd_host (pinned host buffers, copies + kernel on one stream)"}


def extra_workloads(af_names, world):
    """Other workloads, timed the same way (cold L2 between launches), one line each."""
    import attention_forward_18_b200 as af
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    flush = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
    from workloads import WIDE_WORKLOADS
    res = {}
    for name in af_names:
        w = WORKLOADS[name] if name in WORKLOADS else WIDE_WORKLOADS[name]
        q, k, v = (t.to(dev) for t in make_inputs(w))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
        dcode = af.ATTN_F16 if w.dtype == "f16" else af.ATTN_BF16
        for c in w.causal:
            def f(c=c):
                rc = af.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), w.B, w.H, w.Sq, w.Sk, w.D, int(c), w.scale,
                                 dcode, stream.cuda_stream)
                if rc != 0:
                    raise af.AttnError(rc, "attn_fwd")
            t = time_steps([f], 20, 5, flush, stream)
            ms = statistics.median(x[0] for x in t)
            tf = w.flops(c) / (ms * 1e-3) / 1e12
            res[f"{name}{'-causal' if c else ''}"] = {
                "shape": f"B={w.B} H={w.H} S={w.Sq} D={w.D} {w.dtype}",
                "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                "frac_of_peak": round(tf / peak, 4),
                "hbm_gbs_at_algorithmic_bytes": round(w.io_bytes() / (ms * 1e-3) / 1e9, 1)}
        status = af.attn_fwd_status(stream)
        if status != 0:
            raise af.AttnError(status, f"device status after {name}")
        del q, k, v, o, lse
        torch.cuda.empty_cache()
    res["peak_TFLOP/s"] = f"{peak} ({peak_kind} dense bf16 burst)"
    return res


def graph_launches(names, reps=20):
    """C1 / C2 per launch inside a captured CUDA graph of `reps` back-to-back launches
    of each pass (launch overhead amortised; inputs resident and, at these sizes, warm
    in L2 after the first launch -- stated in the line)."""
    import attention_forward_18_b200 as af
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, _ = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
    res = {}
    stream = torch.cuda.Stream(dev)
    for name in names:
        w = WORKLOADS[name]
        q, k, v = (t.to(dev) for t in make_inputs(w))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
        dcode = af.ATTN_F16 if w.dtype == "f16" else af.ATTN_BF16
        for c in w.causal:
            def f(c=c):
                rc = af.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), w.B, w.H, w.Sq, w.Sk, w.D, int(c), w.scale,
                                 dcode, stream.cuda_stream)
                if rc != 0:
                    raise af.AttnError(rc, "attn_fwd")
            with torch.cuda.stream(stream):
                f()  # first call outside the capture (one-time set-up)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    f()
            times = []
            with torch.cuda.stream(stream):
                for _ in range(5):
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    g.replay()  # on the current stream: `stream`
                    e1.record(stream)
                    torch.cuda.synchronize()
                    times.append(e0.elapsed_time(e1) / reps)
            ms = statistics.median(times)
            tf = w.flops(c) / (ms * 1e-3) / 1e12
            res[f"{name}{'-causal' if c else ''}"] = {
                "ms_per_launch": round(ms, 5), "TFLOP/s": round(tf, 1),
                "frac_of_peak": round(tf / peak, 4),
                "note": f"{reps} launches per graph replay, L2 warm"}
            del g
        status = af.attn_fwd_status()
        if status != 0:
            raise af.AttnError(status, f"device status after {name}")
    return res


def decode_workloads(names):
    """The split-KV pass on decode-shaped workloads (HBM-bound: K and V are read once,
    the score work is small), timed like the rest with a cold L2; the whole pass on the
    same tensors beside it."""
    import attention_forward_18_b200 as af
    from workloads import DECODE_WORKLOADS
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    flush = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    res = {}
    for name in names:
        w = DECODE_WORKLOADS[name]
        q, k, v = (t.to(dev) for t in make_inputs(w))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
        dcode = af.ATTN_F16 if w.dtype == "f16" else af.ATTN_BF16
        Hkv = w.kv_heads
        n = af.ex_default_splits(w.B, w.H, Hkv, w.Sq, w.Sk, af.ATTN_MASK_NONE)
        nbytes = af.splitkv_workspace_bytes(w.B, w.H, w.Sq, w.D, n)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                w.B, w.H, Hkv, w.Sq, w.Sk, w.D, af.ATTN_MASK_NONE, w.scale, dcode)

        def split():
            rc = af.attn_fwd_ex(*args, n, ws.data_ptr(), nbytes, stream.cuda_stream)
            if rc != 0:
                raise af.AttnError(rc, "attn_fwd_ex")

        def whole():
            rc = af.attn_fwd_ex(*args, 0, None, 0, stream.cuda_stream)
            if rc != 0:
                raise af.AttnError(rc, "attn_fwd_ex")
        ms = statistics.median(x[0] for x in time_steps([split], 20, 5, flush, stream))
        ms_whole = statistics.median(x[0] for x in time_steps([whole], 10, 3, flush, stream))
        gbs = w.io_bytes() / (ms * 1e-3) / 1e9
        res[name] = {
            "shape": f"B={w.B} H={w.H} Hkv={Hkv} Sq={w.Sq} Sk={w.Sk} D={w.D} {w.dtype}",
            "n_splits": n, "ms": round(ms, 4), "GB/s": round(gbs, 1),
            "frac_of_hbm": round(gbs / hbm, 4),
            "TFLOP/s": round(w.flops(False) / (ms * 1e-3) / 1e12, 1),
            "whole_pass_GB/s": round(w.io_bytes() / (ms_whole * 1e-3) / 1e9, 1)}
        status = af.attn_fwd_status(stream)
        if status != 0:
            raise af.AttnError(status, f"device status after {name}")
        del q, k, v, o, lse, ws
        torch.cuda.empty_cache()
    res["peak_GB/s"] = f"{hbm} ({peak_kind} HBM copy)"
    return res


def prefill_workloads(names):
    """Grouped K/V heads with the bottom-right causal mask (attn_fwd_ex, whole pass),
    TFLOP/s at 4*D FLOPs per visible (query, key) pair."""
    import attention_forward_18_b200 as af
    from workloads import PREFILL_WORKLOADS, visible_pairs
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    flush = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
    res = {}
    for name in names:
        w = PREFILL_WORKLOADS[name]
        q, k, v = (t.to(dev) for t in make_inputs(w))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
        dcode = af.ATTN_F16 if w.dtype == "f16" else af.ATTN_BF16
        mask = af.ATTN_MASK_CAUSAL_BOTTOM_RIGHT

        def f():
            rc = af.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), w.B, w.H, w.kv_heads, w.Sq, w.Sk, w.D, mask,
                                w.scale, dcode, 0, None, 0, stream.cuda_stream)
            if rc != 0:
                raise af.AttnError(rc, "attn_fwd_ex")
        ms = statistics.median(t[0] for t in time_steps([f], 20, 5, flush, stream))
        flops = 4.0 * w.D * w.B * w.H * visible_pairs(w.Sq, w.Sk, 2)
        tf = flops / (ms * 1e-3) / 1e12
        res[name] = {"shape": f"B={w.B} H={w.H} Hkv={w.kv_heads} Sq={w.Sq} Sk={w.Sk} D={w.D} "
                              f"{w.dtype} bottom-right causal",
                     "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                     "frac_of_peak": round(tf / peak, 4)}
        status = af.attn_fwd_status(stream)
        if status != 0:
            raise af.AttnError(status, f"device status after {name}")
        del q, k, v, o, lse
        torch.cuda.empty_cache()
    res["peak_TFLOP/s"] = f"{peak} ({peak_kind} dense bf16 burst)"
    return res


def softmax_workloads(names):
    """The standalone row softmax (HBM-bound: x read once, y written once), timed like
    the rest with a cold L2, as GB/s of those algorithmic bytes."""
    import attention_forward_18_b200 as af
    from workloads import SOFTMAX_WORKLOADS, make_rows
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    flush = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    codes = {"f16": af.ATTN_F16, "bf16": af.ATTN_BF16, "f32": af.SOFTMAX_F32}
    res = {}
    for name in names:
        w = SOFTMAX_WORKLOADS[name]
        x = make_rows(w.rows, w.n, w.dtype, w.seed, w.scale).to(dev)
        y = torch.empty_like(x)

        def f():
            rc = af.row_softmax_raw(x.data_ptr(), y.data_ptr(), w.rows, w.n, codes[w.dtype],
                                    stream.cuda_stream)
            if rc != 0:
                raise af.AttnError(rc, "row_softmax")
        ms = statistics.median(t[0] for t in time_steps([f], 20, 5, flush, stream))
        gbs = w.io_bytes() / (ms * 1e-3) / 1e9
        res[name] = {"shape": f"{w.rows} x {w.n} {w.dtype}", "ms": round(ms, 4),
                     "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / hbm, 4)}
        del x, y
        torch.cuda.empty_cache()
    res["peak_GB/s"] = f"{hbm} ({peak_kind} HBM copy)"
    return res


def gemm_workloads(names):
    """The GEMM with the fused bias + activation epilogue (tensor-bound), timed like the
    rest with a cold L2, as TFLOP/s (2*M*N*K per call) against the measured bf16 peak;
    torch's cuBLAS linear + activation on the same tensors beside it for context."""
    import attention_forward_18_b200 as af
    from workloads import GEMM_WORKLOADS, make_gemm
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    flush = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
    res = {}
    for name in names:
        g = GEMM_WORKLOADS[name]
        a, w, b = (t.to(dev) for t in make_gemm(g.M, g.N, g.K, g.dtype, g.seed))
        c = torch.empty((g.M, g.N), dtype=a.dtype, device=dev)
        dcode = af.ATTN_F16 if g.dtype == "f16" else af.ATTN_BF16

        def f():
            rc = af.gemm_bias_act_raw(a.data_ptr(), w.data_ptr(), b.data_ptr(), c.data_ptr(),
                                      g.M, g.N, g.K, g.act, dcode, stream.cuda_stream)
            if rc != 0:
                raise af.AttnError(rc, "gemm_bias_act")

        def lib():
            z = torch.nn.functional.linear(a, w, b)
            if g.act == af.GEMM_ACT_GELU:
                z = torch.nn.functional.gelu(z)
            elif g.act == af.GEMM_ACT_RELU:
                z = torch.relu(z)
            return z
        ms = statistics.median(t[0] for t in time_steps([f], 20, 5, flush, stream))
        ms_lib = statistics.median(t[0] for t in time_steps([lib], 20, 5, flush, stream))
        tf = g.flops() / (ms * 1e-3) / 1e12
        res[name] = {"shape": f"M={g.M} N={g.N} K={g.K} {g.dtype} act={g.act}",
                     "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                     "frac_of_peak": round(tf / peak, 4),
                     "torch_cublas_TFLOP/s": round(g.flops() / (ms_lib * 1e-3) / 1e12, 1)}
        status = af.attn_fwd_status(stream)
        if status != 0:
            raise af.AttnError(status, f"device status after {name}")
        del a, w, b, c
        torch.cuda.empty_cache()
    res["peak_TFLOP/s"] = f"{peak} ({peak_kind} dense bf16 burst)"
    return res


# ---------------------------------------------------------------- oracle (CPU) arm
def oracle_sample(w, seconds, max_heads=None):
    """Time the fp64 CPU oracle as it stands on whole heads of the workload (every
    causal mode of the step), adding heads until `seconds` have passed or the
    workload is exhausted.  Returns (TFLOP/s, cores, description)."""
    import oracle
    q, k, v = make_inputs(w)
    qd = q.double().numpy().reshape(w.B * w.H, 1, w.Sq, w.D)
    kd = k.double().numpy().reshape(w.B * w.H, 1, w.Sk, w.D)
    vd = v.double().numpy().reshape(w.B * w.H, 1, w.Sk, w.D)
    threads = oracle.num_threads()
    total_heads = w.B * w.H if max_heads is None else min(max_heads, w.B * w.H)
    chunk = max(1, threads)
    done, flops, t_used = 0, 0.0, 0.0
    while done < total_heads and (done == 0 or t_used < seconds):
        n = min(chunk, total_heads - done)
        sl = slice(done, done + n)
        qs = qd[sl].reshape(1, n, w.Sq, w.D)
        ks = kd[sl].reshape(1, n, w.Sk, w.D)
        vs = vd[sl].reshape(1, n, w.Sk, w.D)
        t0 = time.perf_counter()
        for c in w.causal:
            oracle.attn_ref(qs, ks, vs, c, w.scale)
        t_used += time.perf_counter() - t0
        flops += sum(4.0 * n * w.Sq * w.Sk * w.D * (0.5 if c else 1.0) for c in w.causal)
        done += n
    desc = (f"{done} of {w.B * w.H} heads of {w.name} (both passes of the step), "
            f"{t_used:.1f} s of oracle time")
    return flops / t_used / 1e12, threads, desc


def reference_arm(args, world, rank):
    """The oracle as the reference implementation: K timed steps, each a bounded
    sample (whole heads) of the workload, on this host's cores."""
    w = WORKLOADS[args.workload]
    import oracle
    threads = oracle.num_threads()
    per_step_heads = max(1, threads)
    for _ in range(args.warmup):
        oracle_sample(w, 0.0, max_heads=per_step_heads)
    t_flops, t_time = 0.0, 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        tf, cores, desc = oracle_sample(w, 0.0, max_heads=per_step_heads)
        dt = time.perf_counter() - t0
        t_time += dt
        t_flops += tf * 1e12 * dt
    value = t_flops / t_time / 1e12
    sample = (f"per step: {per_step_heads} whole heads of {w.name} "
              f"(B={w.B} H={w.H} S={w.Sq} D={w.D}), non-causal + causal")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_time / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} Sq={w.Sq} Sk={w.Sk} D={w.D} "
                               f"{w.dtype} inputs upcast to fp64, non-causal + causal",
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def profile_once(args):
    """One launch per pass of the workload, nothing else on the GPU before it except
    the input copies (a short, self-ending command for ncu)."""
    import attention_forward_18_b200 as af
    if args.profile_extra:
        return profile_extra(args.profile_extra)
    w = WORKLOADS[args.workload]
    q, k, v = (t.cuda() for t in make_inputs(w))
    for c in w.causal:
        af.attention(q, k, v, causal=c, scale=w.scale)
    torch.cuda.synchronize()
    status = af.attn_fwd_status()
    if status != 0:
        raise af.AttnError(status, "device status")
    print(json.dumps({"profile_once": w.name, "passes": list(w.causal)}))


def profile_extra(spec):
    """One call of a decode, row-softmax or GEMM workload (its size optionally cut down
    along its first dimension so an ncu capture stays small)."""
    import dataclasses
    import attention_forward_18_b200 as af
    from workloads import (DECODE_WORKLOADS, GEMM_WORKLOADS, SOFTMAX_WORKLOADS, WIDE_WORKLOADS,
                           make_gemm, make_rows)
    name, _, cut = spec.partition(":")
    if name in WIDE_WORKLOADS:
        w = WIDE_WORKLOADS[name]
        if cut:
            w = dataclasses.replace(w, H=int(cut))
        q, k, v = (t.cuda() for t in make_inputs(w))
        for c in w.causal:
            af.attention(q, k, v, causal=c, scale=w.scale)
        shape = f"B={w.B} H={w.H} S={w.Sq} D={w.D} causal={list(w.causal)}"
    elif name in DECODE_WORKLOADS:
        w = DECODE_WORKLOADS[name]
        if cut:
            w = dataclasses.replace(w, B=int(cut))
        q, k, v = (t.cuda() for t in make_inputs(w))
        n = af.ex_default_splits(w.B, w.H, w.kv_heads, w.Sq, w.Sk, af.ATTN_MASK_NONE)
        af.attention_ex(q, k, v, mask=af.ATTN_MASK_NONE, scale=w.scale, n_splits=n)
        shape = f"B={w.B} H={w.H} Hkv={w.kv_heads} Sq={w.Sq} Sk={w.Sk} D={w.D} splits={n}"
    elif name in SOFTMAX_WORKLOADS:
        w = SOFTMAX_WORKLOADS[name]
        if cut:
            w = dataclasses.replace(w, rows=int(cut))
        af.row_softmax(make_rows(w.rows, w.n, w.dtype, w.seed, w.scale).cuda())
        shape = f"{w.rows} x {w.n} {w.dtype}"
    elif name in GEMM_WORKLOADS:
        g = GEMM_WORKLOADS[name]
        if cut:
            g = dataclasses.replace(g, M=int(cut))
        a, wt, b = (t.cuda() for t in make_gemm(g.M, g.N, g.K, g.dtype, g.seed))
        af.gemm_bias_act(a, wt, b, g.act)
        shape = f"M={g.M} N={g.N} K={g.K} {g.dtype} act={g.act}"
    else:
        raise SystemExit(f"unknown workload {name}")
    torch.cuda.synchronize()
    status = af.attn_fwd_status()
    if status != 0:
        raise af.AttnError(status, "device status")
    print(json.dumps({"profile_once": name, "shape": shape}))


def main():
    args = parse()
    world, rank, local = dist_setup()
    try:
        if args.profile_once:
            profile_once(args)
            return
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(reference_arm(args, 1, rank)), flush=True)
            return
        line = cuda_arm(args, world, rank, local)
        # the other workloads once, on a single-GPU run (a multi-GPU run would hold every
        # GPU while rank 0 alone works through them)
        if rank == 0 and world == 1 and not args.no_extra:
            line["extra"] = extra_workloads(["C3", "C4", "C5", "WD192", "WD256"], world)
            line["extra"]["cuda_graph"] = graph_launches(["C1", "C2"])
            line["extra"]["decode_splitkv"] = decode_workloads(
                ["DEC1", "DEC2", "DEC3", "DEC4", "DEC5", "DEC6"])
            line["extra"]["prefill_grouped_bottom_right"] = prefill_workloads(["PRE1"])
            line["extra"]["row_softmax"] = softmax_workloads(["SMX1", "SMX2", "SMX3"])
            line["extra"]["gemm_bias_act"] = gemm_workloads(["GEMM1", "GEMM2", "GEMM3"])
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            w = WORKLOADS[args.workload]
            tf, cores, desc = oracle_sample(w, args.cpu_seconds)
            line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores,
                                    "kind": "oracle", "sample": desc}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
