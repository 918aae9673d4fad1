"""Benchmark of the fused attention forward pass on B200: prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload step|C1|C2|C3|C4|C5] [--no-extra]

A step is one pass over each of the three large workloads, each pass one launch of
the CUDA kernel through the C ABI, all bf16 with head dimension 128:

    C3  B=2 H=32 Sq=Sk=4096   causal                       seed 2
    C4  B=8 H=32 Sq=Sk=2048   non-causal, K scaled by 3    seed 3
    C5  B=1 H=16 Sq=Sk=16384  causal (long context)        seed 4

The metric is TFLOP/s with FLOPs = 4*B*H*Sq*Sk*D per pass, halved for causal; `value`
is the step's FLOPs over the step's time.  `--workload C2` (or another single
workload) times that workload's passes instead.

Timing: inputs resident in device memory; W untimed warm-up steps; then exactly K
steps with CUDA events around every pass on the launching stream; barrier +
synchronize on both sides; the max over ranks of the summed step time.  Every pass of
the default step reads at least 201 MB of Q/K/V, more than the 126 MB L2, so no pass
finds its inputs in L2 (no flush is needed); a workload whose inputs fit in L2 gets a
256 MB read between steps.  Multi-GPU runs (torchrun, one rank per GPU) give every
rank its own copy of the workload (weak scaling, no collective on the data path).

Also reported: `e2e` (the same step through attn_fwd_host from pinned host buffers,
copies included), `roofline` (the dominant kernel's achieved TFLOP/s against the
measured dense bf16 peak, with its DRAM traffic from an ncu capture of the same
kernel source), `cpu_baseline` (the fp64 CPU oracle on whole query rows of every pass
of the step, rank 0 at N=1), `clocks` (NVML samples taken during the timed region),
`extra` (the small workloads, the head-dimension, decode, prefill, row-softmax and
GEMM workloads, timed the same way outside the timed region) and `runs` (the six
headline runs C1, C2 non-causal / causal, C3, C4, C5 with their fraction of the peak).
"""
import argparse
import hashlib
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
L2_BYTES = 126 * 10 ** 6
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0

# The benchmark step: the three large workloads, one pass each.
STEP = (("C3", True), ("C4", False), ("C5", True))

# Kernel sources whose DRAM traffic the ncu figures below describe; a figure is
# reported only while the hash of these files is the one it was captured with.
KERNEL_SOURCES = ("attention_forward_18_b200/csrc/attn_fwd_kernel.cuh",
                  "attention_forward_18_b200/csrc/attn_fwd.cu",
                  "attention_forward_18_b200/csrc/ptx.cuh")
# dram__bytes_read.sum + dram__bytes_write.sum of one launch (ncu, --clock-control none),
# with the kernel-source hash of the build captured
NCU_TRAFFIC = {
    "C5-causal": {"bytes": 567774720 + 49346816, "src_sha": "c7d778ee895f2184",
                  "note": "ncu --set full, one launch of C5 (read 567.8 MB, write 49.3 MB)"},
    "C4-noncausal": {"bytes": 402735872 + 111735040, "src_sha": "c7d778ee895f2184",
                     "note": "ncu --set full, one launch of C4 (read 402.7 MB, write 111.7 MB)"},
    "C3-causal": {"bytes": 525650944 + 47049728, "src_sha": "c7d778ee895f2184",
                  "note": "ncu --set full, one launch of C3 (read 525.7 MB, write 47.0 MB)"},
}

# North-star fractions of the dense bf16 peak per run (none stated for C1 and C2
# non-causal).
TARGETS = {"C2-causal": 0.50, "C3-causal": 0.50, "C4-noncausal": 0.60, "C5-causal": 0.50}

# The metric both arms report (the headline benchmark's own wording).
METRIC = "attention fwd TFLOP/s on 1 B200 (causal & non-causal), % of bf16 TC peak"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="step", choices=["step"] + sorted(WORKLOADS))
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--ref-rows", type=int, default=1024,
                    help="reference arm: query rows of each pass per step")
    ap.add_argument("--profile-once", action="store_true",
                    help="launch each pass of the workload once and exit (for ncu captures)")
    ap.add_argument("--profile-extra", default=None,
                    help="with --profile-once: a DEC*, SMX*, GEMM* or WD* workload instead, "
                         "optionally scaled down as NAME:n (M for GEMM*, rows for SMX*, B for "
                         "DEC*, H for WD*)")
    return ap.parse_args()


def step_passes(name):
    """(workload, causal) of every pass of a step."""
    if name == "step":
        return [(WORKLOADS[n], c) for n, c in STEP]
    w = WORKLOADS[name]
    return [(w, c) for c in w.causal]


def step_name(name):
    return "+".join(w.name for w, _ in step_passes(name)) if name == "step" else name


def pass_key(w, causal):
    return f"{w.name}-{'causal' if causal else 'noncausal'}"


def qkv_bytes(w):
    """Bytes of Q, K and V of a workload (16-bit)."""
    return 2 * w.B * w.D * (w.H * w.Sq + 2 * w.kv_heads * w.Sk)


def kernel_source_sha():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


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


def tensor_peak():
    """The dense bf16 peak (burst figure: every timed launch here lasts about a
    millisecond at most) and where it comes from; fp16 has the same nominal rate."""
    peaks, kind = measured_peaks()
    return float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), f"{kind} dense bf16 burst"


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
def make_flush(dev, kind):
    """A callable that evicts L2 between timed launches: "read" sums a 256 MB buffer (L2
    is left holding clean lines of it), "write" adds one to every element (L2 is left
    holding dirty lines, which drain to HBM while the next launch runs)."""
    buf = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    acc = torch.zeros((), dtype=torch.float32, device=dev)
    if kind == "read":
        return lambda: torch.sum(buf, 0, out=acc)
    return lambda: buf.add_(1)


def time_steps(launches, steps, warmup, flush, stream):
    """Run `warmup` untimed steps, then `steps` timed ones.  `launches` is a list of
    zero-argument callables, one per kernel launch of a step; `flush` (or None) runs
    before each timed step, outside the events.  Returns per-launch event times (ms),
    shape [steps][len(launches)]."""
    for _ in range(warmup):
        for f in launches:
            f()
    n = len(launches)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        if flush is not None:
            flush()
        ev[i][0].record(stream)
        for j, f in enumerate(launches):
            f()
            ev[i][j + 1].record(stream)
    torch.cuda.synchronize()
    return [[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(n)] for i in range(steps)]


def cuda_arm(args, world, rank, local):
    import attention_forward_18_b200 as af

    passes = step_passes(args.workload)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    host, devt = {}, {}
    for w, _ in passes:
        if w.name not in host:
            host[w.name] = make_inputs(w)
            devt[w.name] = tuple(t.to(dev) for t in host[w.name])
    outs = [(torch.empty_like(devt[w.name][0]),
             torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)) for w, _ in passes]

    def launcher(i):
        w, causal = passes[i]
        dq, dk, dv = devt[w.name]
        o, lse = outs[i]
        dcode = af.ATTN_F16 if w.dtype == "f16" else af.ATTN_BF16
        args_ = (dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), o.data_ptr(), lse.data_ptr(),
                 w.B, w.H, w.Sq, w.Sk, w.D, int(causal), w.scale, dcode, sptr)

        def f():
            rc = af.attn_fwd(*args_)
            if rc != 0:
                raise af.AttnError(rc, "attn_fwd")
        return f

    launches = [launcher(i) for i in range(len(passes))]
    flops_step = sum(w.flops(c) for w, c in passes)
    cold_inputs = all(qkv_bytes(w) > L2_BYTES for w, _ in passes)
    flush = None if cold_inputs else make_flush(dev, "read")

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

    peak, peak_kind = tensor_peak()
    per_slot = [sum(t[j] for t in times) / args.steps for j in range(len(launches))]
    sha = kernel_source_sha()
    per_pass = {}
    for j, (w, c) in enumerate(passes):
        tf = w.flops(c) / (per_slot[j] * 1e-3) / 1e12
        cap = NCU_TRAFFIC.get(pass_key(w, c))
        per_pass[pass_key(w, c)] = {"ms": round(per_slot[j], 5), "TFLOP/s": round(tf, 1),
                                    "frac_of_peak": round(tf / peak, 4),
                                    "algorithmic_bytes": w.io_bytes(),
                                    "traffic": cap["bytes"] if cap and cap["src_sha"] == sha
                                    else None}
    # dominant kernel: the launch slot with the largest time
    dom = max(range(len(launches)), key=lambda j: per_slot[j])
    dw, dc = passes[dom]
    dom_ms = per_slot[dom]
    achieved = dw.flops(dc) / (dom_ms * 1e-3) / 1e12
    key = pass_key(dw, dc)
    cap = NCU_TRAFFIC.get(key)
    traffic = cap["bytes"] if cap and cap["src_sha"] == sha else None
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": traffic,
                "kernel": f"attn_fwd_kernel<D={dw.D},{dw.dtype},causal={dc}> on {key}",
                "peak_source": f"{peak_kind} (fp16 has the same nominal rate)",
                "per_launch_ms": round(dom_ms, 5),
                "algorithmic_bytes": dw.io_bytes(),
                "hbm_gbs_at_algorithmic_bytes": round(dw.io_bytes() / (dom_ms * 1e-3) / 1e9, 1),
                "traffic_note": (cap["note"] if cap and traffic is not None else
                                 "no ncu capture of this kernel source"),
                "kernel_source_sha": sha,
                "per_pass": per_pass}

    e2e = e2e_arm(af, passes, host, dev, sptr, args, world)
    clocks = sampler.summary()

    line = {
        "metric": METRIC,
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16" if passes[0][0].dtype == "f16" else "bf16", "data": "synthetic",
        "config": {"workload": "; ".join(
                       f"{w.name} {'causal' if c else 'non-causal'}: B={w.B} H={w.H} Sq={w.Sq} "
                       f"Sk={w.Sk} D={w.D} {w.dtype} seed {w.seed}"
                       + (f" K x{w.k_scale:g}" if w.k_scale != 1.0 else "")
                       for w, c in passes),
                   "passes_per_step": [pass_key(w, c) for w, c in passes],
                   "accumulate": "fp32",
                   "l2": ("inputs larger than L2 (every pass reads >= 201 MB of Q/K/V); "
                          "no flush" if cold_inputs else
                          "256 MB read between timed steps (inputs fit in L2)"),
                   "parallelism": f"dp{world} (independent copy per GPU)"},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": len(launches) * args.steps,
        "clocks": clocks,
    }
    return line


def e2e_arm(af, passes, host, dev, sptr, args, world):
    """The same step through attn_fwd_host: every pass copies its workload's Q, K, V in
    from pinned host buffers and its O and LSE out, every step (copies inside the
    timed region)."""
    pinned = {name: tuple(t.pin_memory() for t in qkv) for name, qkv in host.items()}
    staging = {name: tuple(torch.empty_like(t, device=dev) for t in qkv)
               for name, qkv in host.items()}
    calls, h2d, d2h = [], 0, 0
    for w, c in passes:
        qh, kh, vh = pinned[w.name]
        oh = torch.empty_like(qh).pin_memory()
        lh = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32).pin_memory()
        qd, kd, vd = staging[w.name]
        od = torch.empty_like(qd)
        ld = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
        dcode = af.ATTN_F16 if w.dtype == "f16" else af.ATTN_BF16
        calls.append((qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), oh.data_ptr(), lh.data_ptr(),
                      qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(), ld.data_ptr(),
                      w.B, w.H, w.Sq, w.Sk, w.D, int(c), w.scale, dcode, sptr))
        h2d += qh.nbytes + kh.nbytes + vh.nbytes
        d2h += oh.nbytes + lh.nbytes
        staging.setdefault("_keep", []).extend([oh, lh, od, ld])

    def step():
        for a in calls:
            rc = af.attn_fwd_host(*a)
            if rc != 0:
                raise af.AttnError(rc, "attn_fwd_host")

    steps = max(3, min(args.steps, 20))
    for _ in range(3):
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
    flops_step = sum(w.flops(c) for w, c in passes)
    shared = len({w.name for w, _ in passes}) < len(passes)
    return {"value": round(world * flops_step * steps / (ms * 1e-3) / 1e12, 4),
            "unit": "TFLOP/s", "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "path": "attn_fwd_host per pass (pinned host buffers; a pass of 16 MB or more "
                    "of Q, K, V runs as up to 8 head chunks, copies in and out on the "
                    "library's two copy streams overlapping the kernel)" + ("; passes on the same tensors each copy them in"
                                 if shared else "")}


def extra_workloads(af_names, world):
    """Other workloads, one launch per pass timed like the step (median of 20), with a
    256 MB read between launches so a workload whose inputs fit in L2 starts cold; for
    those small workloads the same with a 256 MB write between launches (the dirty lines
    drain while the next launch runs) is reported beside it."""
    import attention_forward_18_b200 as af
    from workloads import WIDE_WORKLOADS
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    flush_read, flush_write = make_flush(dev, "read"), make_flush(dev, "write")
    peak, peak_kind = tensor_peak()
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
            ms = statistics.median(x[0] for x in time_steps([f], 20, 5, flush_read, stream))
            tf = w.flops(c) / (ms * 1e-3) / 1e12
            entry = {"shape": f"B={w.B} H={w.H} S={w.Sq} D={w.D} {w.dtype}",
                     "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                     "frac_of_peak": round(tf / peak, 4),
                     "hbm_gbs_at_algorithmic_bytes": round(w.io_bytes() / (ms * 1e-3) / 1e9, 1)}
            if qkv_bytes(w) < L2_BYTES:
                ms_w = statistics.median(
                    x[0] for x in time_steps([f], 20, 5, flush_write, stream))
                entry["ms_write_flush"] = round(ms_w, 4)
                entry["TFLOP/s_write_flush"] = round(w.flops(c) / (ms_w * 1e-3) / 1e12, 1)
            res[pass_key(w, c)] = entry
        status = af.attn_fwd_status(stream)
        if status != 0:
            raise af.AttnError(status, f"device status after {name}")
        del q, k, v, o, lse
        torch.cuda.empty_cache()
    res["peak_TFLOP/s"] = f"{peak} ({peak_kind})"
    return res


def graph_launches(names, reps=20):
    """C1 / C2 per launch inside a captured CUDA graph of `reps` back-to-back launches
    of each pass (launch overhead amortised; inputs resident and, at these sizes, warm
    in L2 after the first launch -- stated in the line)."""
    import attention_forward_18_b200 as af
    dev = torch.device("cuda", torch.cuda.current_device())
    peak, _ = tensor_peak()
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
            res[pass_key(w, c)] = {
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
    flush = make_flush(dev, "read")
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
        n = af.ex_default_splits(w.B, w.H, Hkv, w.Sq, w.Sk, af.ATTN_MASK_NONE, w.D)
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
    flush = make_flush(dev, "read")
    peak, peak_kind = tensor_peak()
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
    res["peak_TFLOP/s"] = f"{peak} ({peak_kind})"
    return res


def softmax_workloads(names):
    """The standalone row softmax (HBM-bound: x read once, y written once), timed like
    the rest with a cold L2, as GB/s of those algorithmic bytes."""
    import attention_forward_18_b200 as af
    from workloads import SOFTMAX_WORKLOADS, make_rows
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    flush = make_flush(dev, "read")
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
    flush = make_flush(dev, "read")
    peak, peak_kind = tensor_peak()
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
    res["peak_TFLOP/s"] = f"{peak} ({peak_kind})"
    return res


# ---------------------------------------------------------------- oracle (CPU) arm
def oracle_inputs(passes):
    """fp64 numpy copies of every workload's inputs (the 16-bit values upcast exactly,
    as the oracle reads them)."""
    out = {}
    for w, _ in passes:
        if w.name not in out:
            q, k, v = make_inputs(w)
            out[w.name] = (q.double().numpy(), k.double().numpy(), v.double().numpy())
    return out


def oracle_rows_timed(passes, inputs, rows_per_pass, rng):
    """One sample: `rows_per_pass` whole query rows (uniform over batch, head and row)
    of every pass through the oracle's row entry point, which materialises each row's
    Sk scores in fp64, masks them, takes the softmax and multiplies by V.  Returns the
    FLOPs the metric counts for those rows (4*Sk*D a row, halved for causal) and the
    oracle's time."""
    import numpy as np
    import oracle
    flops, secs = 0.0, 0.0
    for w, c in passes:
        qd, kd, vd = inputs[w.name]
        rows = np.stack([rng.integers(0, w.B, rows_per_pass), rng.integers(0, w.H, rows_per_pass),
                         rng.integers(0, w.Sq, rows_per_pass)], axis=1)
        rows = rows[np.lexsort((rows[:, 2], rows[:, 1], rows[:, 0]))]  # head by head
        t0 = time.perf_counter()
        oracle.attn_ref_rows(qd, kd, vd, rows, c, w.scale)
        secs += time.perf_counter() - t0
        flops += rows_per_pass * 4.0 * w.Sk * w.D * (0.5 if c else 1.0)
    return flops, secs


def oracle_sample(passes, seconds):
    """Time the fp64 CPU oracle as it stands on whole query rows of every pass of the
    step, a chunk of rows of each pass in turn, until `seconds` of oracle time have
    passed.  Returns (TFLOP/s, cores, description)."""
    import numpy as np
    import oracle
    inputs = oracle_inputs(passes)
    rng = np.random.default_rng(2024)
    threads = oracle.num_threads()
    chunk = max(64, 16 * threads)
    flops, secs, rows = 0.0, 0.0, 0
    while rows == 0 or secs < seconds:
        f, s = oracle_rows_timed(passes, inputs, chunk, rng)
        flops += f
        secs += s
        rows += chunk
    desc = (f"{rows} whole query rows of each of "
            f"{', '.join(pass_key(w, c) for w, c in passes)} (uniform over batch, head and "
            f"row; the oracle's row entry point), {secs:.1f} s of oracle time")
    return flops / secs / 1e12, threads, desc


def reference_arm(args, world, rank):
    """The oracle as the reference implementation: K timed steps, each a bounded
    sample (whole query rows of every pass of the step) on this host's cores."""
    import numpy as np
    import oracle
    passes = step_passes(args.workload)
    inputs = oracle_inputs(passes)
    rng = np.random.default_rng(2025)
    threads = oracle.num_threads()
    for _ in range(args.warmup):
        oracle_rows_timed(passes, inputs, args.ref_rows, rng)
    t_flops, t_time = 0.0, 0.0
    for _ in range(args.steps):
        f, s = oracle_rows_timed(passes, inputs, args.ref_rows, rng)
        t_flops += f
        t_time += s
    value = t_flops / t_time / 1e12
    sample = (f"per step: {args.ref_rows} whole query rows of each of "
              f"{', '.join(pass_key(w, c) for w, c in passes)} (uniform over batch, head "
              f"and row)")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_time / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{step_name(args.workload)}: "
                               + "; ".join(f"{w.name} {'causal' if c else 'non-causal'} "
                                           f"B={w.B} H={w.H} Sq={w.Sq} Sk={w.Sk} D={w.D} "
                                           f"{w.dtype}" for w, c in passes)
                               + "; inputs upcast to fp64",
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def runs_summary(line):
    """The six headline runs (C1, C2 non-causal and causal, C3, C4, C5): TFLOP/s and
    fraction of the dense bf16 peak, with the stated target where there is one."""
    out = {}
    extra = line.get("extra", {})
    found = dict(extra.items())
    found.update(line["roofline"]["per_pass"])
    for key in ("C1-noncausal", "C2-noncausal", "C2-causal", "C3-causal", "C4-noncausal",
                "C5-causal"):
        r = found.get(key)
        if not isinstance(r, dict) or "TFLOP/s" not in r:
            continue
        e = {"TFLOP/s": r["TFLOP/s"], "frac": r["frac_of_peak"]}
        if key in TARGETS:
            e["target"] = TARGETS[key]
        out[key] = e
    return out


def profile_once(args):
    """One launch per pass of the workload, nothing else on the GPU before it except
    the input copies (a short, self-ending command for ncu)."""
    import attention_forward_18_b200 as af
    if args.profile_extra:
        return profile_extra(args.profile_extra)
    passes = step_passes(args.workload)
    inputs = {}
    for w, c in passes:
        if w.name not in inputs:
            inputs[w.name] = tuple(t.cuda() for t in make_inputs(w))
        q, k, v = inputs[w.name]
        af.attention(q, k, v, causal=c, scale=w.scale)
    torch.cuda.synchronize()
    status = af.attn_fwd_status()
    if status != 0:
        raise af.AttnError(status, "device status")
    print(json.dumps({"profile_once": [pass_key(w, c) for w, c in passes]}))


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
        n = af.ex_default_splits(w.B, w.H, w.kv_heads, w.Sq, w.Sk, af.ATTN_MASK_NONE, w.D)
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
            small = [n for n in ("C1", "C2") if n != args.workload]
            line["extra"] = extra_workloads(small + ["WD192", "WD256"], world)
            line["extra"]["cuda_graph"] = graph_launches(["C1", "C2"])
            line["extra"]["decode_splitkv"] = decode_workloads(
                ["DEC1", "DEC2", "DEC3", "DEC4", "DEC5", "DEC6"])
            line["extra"]["prefill_grouped_bottom_right"] = prefill_workloads(["PRE1"])
            line["extra"]["row_softmax"] = softmax_workloads(["SMX1", "SMX2", "SMX3"])
            line["extra"]["gemm_bias_act"] = gemm_workloads(["GEMM1", "GEMM2", "GEMM3"])
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            tf, cores, desc = oracle_sample(step_passes(args.workload), args.cpu_seconds)
            line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores,
                                    "kind": "oracle", "sample": desc}
        line["runs"] = runs_summary(line)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
