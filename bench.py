"""Benchmark of the B200 block-scaled FP8 GEMM (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the GEMM (the whole hot path: TMA operand fetch, scale
fetch, tcgen05 MMA per K-block, FP32 scale promotion, split-K fix-up where the
plan uses it, BF16 epilogue) on one batch of synthetic inputs.

Default workload: the square 4096^3 NT GEMM with 128x128 block scales and 41
outlier rows of A (x50).  Other workloads (``--workload``): tiny, ffn, ffn_tn,
ffn_tt, small_m:<M>, long_k:<g>.

Timing: W warm-up launches, then K timed launches.  Inputs are resident in
HBM.  By default the launches cycle over R >= 3 copies of the inputs at
distinct addresses (R x set size >= 2x L2), so no launch finds its operands in
L2; the K launches are captured once in a CUDA graph and replayed between two
CUDA events on the launching stream (the host's per-call overhead never
starves the GPU), and the time per step is the span / K.  ``--l2 flush``
instead flushes L2 with a 512 MiB memset before each launch and brackets each
launch with its own events.  The whole-job value is total FLOPs / time, max
over ranks.  The default run also measures the HBM-bound small-M shapes
(``--hbm-points``, M x 7168 x 7168) the same way and reports them under
``hbm_bound`` with their own roofline.  ``e2e`` repeats the main workload
through the public API with the inputs in pinned host memory: host->device
copies, the GEMM and the device->host copy of the output are all inside the
timed region.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same GEMM on its
own GPU (replicas; the GEMM has no exchange step), the step time is the max
over ranks and the value sums the ranks' work ("scaling": "weak").

``--impl reference`` times the CPU oracle (the plain FP64 restatement used by
the tests) on the host cores on a bounded sample of the same workload: rank 0
only, the other ranks exit at once.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "FP8 block-scaled GEMM TFLOP/s and % of B200 FP8/HBM roofline (1 GPU)"
L2_FLUSH_BYTES = 512 << 20


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="square")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--l2", default="rotate", choices=["rotate", "flush"],
                    help="keep operands out of L2 by rotating input sets (default) or by a memset per launch")
    ap.add_argument("--quantize-a", action="store_true",
                    help="each step first quantises A from BF16 with the library's quantiser, then runs "
                         "the GEMM (NT layouts): the two-kernel activation pipeline")
    ap.add_argument("--hbm-points", default="1,128",
                    help="small-M sizes (M of M x 7168 x 7168) also measured and reported in the line; '' for none")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU seconds of the oracle sample")
    ap.add_argument("--variant", default="auto", choices=["auto", "data_parallel", "swap_ab", "cta_pair"],
                    help="override the plan's variant (default: library heuristic)")
    ap.add_argument("--bnq", type=int, default=0, help="override the tile width on the MMA N side")
    ap.add_argument("--splits", type=int, default=0, help="override the K splits per tile")
    ap.add_argument("--stream-k", type=int, default=0, choices=[-1, 0, 1],
                    help="stream-K for a ragged last wave: -1 never, 0 library heuristic, 1 always")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- workloads
def make_workload(name: str) -> workloads.Problem:
    if name == "square":
        return workloads.square()
    if name == "tiny":
        return workloads.tiny()
    if name in ("ffn", "ffn_nt"):
        return workloads.ffn(layout="nt")
    if name == "ffn_tn":
        return workloads.ffn(layout="tn")
    if name == "ffn_tt":
        return workloads.ffn(layout="tt")
    if name.startswith("small_m:"):
        return workloads.small_m(int(name.split(":")[1]))
    if name.startswith("long_k:"):
        return workloads.long_k(gran=int(name.split(":")[1]))
    raise SystemExit(f"unknown workload {name}")


def workload_config(p: workloads.Problem, name: str, l2_mode: str = "rotate") -> dict:
    return {"workload": p.name, "name": name, "M": p.M, "N": p.N, "K": p.K, "gran": p.gran,
            "layout": p.layout, "inputs": "E4M3 codes + FP32 block scales, seeded synthetic",
            "l2": l2_note(l2_mode)}


def algorithmic_bytes(p: workloads.Problem) -> int:
    kb = -(-p.K // p.gran)
    return p.M * p.K + p.N * p.K + 2 * p.M * p.N + 4 * (-(-p.M // p.gran) + -(-p.N // p.gran)) * kb


KERNEL_FILES = ("bsgemm_kernel.cuh", "bsgemm_pair.cuh", "ptx.cuh")  # the device code


def _code_only(text: str) -> str:
    """C++ source without comments and blank lines (string literals kept as they are)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = []
    for line in text.splitlines():
        i, quoted = 0, False
        while i < len(line):
            c = line[i]
            if c == '"' and (i == 0 or line[i - 1] != "\\"):
                quoted = not quoted
            elif not quoted and line.startswith("//", i):
                line = line[:i]
                break
            i += 1
        line = line.rstrip()
        if line:
            out.append(line)
    return "\n".join(out)


def kernel_source_hash() -> str:
    """Short hash of the device code of the GEMM kernels (ties ncu figures to a kernel version).

    Comments are left out, and so is host-side launch code (argument checks,
    caching of launch attributes): neither changes what a captured kernel did."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_FILES:
        path = os.path.join(ROOT, "fp8_block_scaled_bsgemm_b200", "csrc", f)
        h.update(f.encode())
        with open(path, encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary of this workload, if it
    was taken on the current kernel sources; otherwise None."""
    import glob
    want = kernel_source_hash()
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        fields = {}
        with open(path) as fh:
            for ln in fh:
                if ":" in ln and ln.split(":")[0] in ("kernel_source_sha256", "bench_workload",
                                                      "traffic_bytes_per_launch"):
                    k, v = ln.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("bench_workload") == workload and fields.get("kernel_source_sha256") == want:
            try:
                return int(fields["traffic_bytes_per_launch"])
            except (KeyError, ValueError):
                return None
    return None


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="bsgemm_clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for ln in open(self.path):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- oracle baseline
def cpu_baseline(p: workloads.Problem, seconds: float) -> dict:
    """The oracle, as it stands, on a bounded sample of whole output rows."""
    import oracle
    # a first small probe sizes the sample to about `seconds` of CPU work
    probe_rows = max(1, min(p.M, 2))
    mi, ni = _rows_sample(p, probe_rows)
    t0 = time.perf_counter()
    oracle.bsgemm_at(p.layout, p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, p.gran, mi, ni)
    dt = max(time.perf_counter() - t0, 1e-6)
    rows = int(max(1, min(p.M, probe_rows * seconds / dt)))
    mi, ni = _rows_sample(p, rows)
    t0 = time.perf_counter()
    oracle.bsgemm_at(p.layout, p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, p.gran, mi, ni)
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * p.N * p.K
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{rows} full output rows of {p.M} ({rows * p.N} outputs), {dt:.1f} s",
            "seconds": dt}


def _rows_sample(p, rows):
    step = max(1, p.M // rows)
    r = (np.arange(rows, dtype=np.int64) * step) % p.M
    mi = np.repeat(r, p.N)
    ni = np.tile(np.arange(p.N, dtype=np.int64), rows)
    return mi, ni


# ---------------------------------------------------------------- distributed plumbing
def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun sets RANK / WORLD_SIZE / LOCAL_RANK). The
    GEMM has no exchange step, so ranks are independent replicas; the process
    group serves only the barriers and the max over ranks of the step time.
    ``backend="gloo"`` runs the same plumbing on CPU (tests)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif backend == "nccl" and torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's value: the job's step time is set by its slowest replica."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput of `world` replicas that each did `flops_per_rank`
    in at most `ms_max` ms (weak scaling: per-GPU work fixed as N grows)."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


# ---------------------------------------------------------------- our arm
def input_sets(p: workloads.Problem, dev, l2_bytes: int, mode: str):
    """Device copies of the workload's inputs (and an output each).

    mode "rotate": R >= 3 copies at distinct addresses, R large enough that
    the copies together are at least twice the L2 size, so by the time a
    launch comes back to a copy the cache holds none of it.  mode "flush":
    one copy (the L2 is flushed before every launch instead)."""
    import torch
    a = torch.from_numpy(p.a).to(dev)
    b = torch.from_numpy(p.b).to(dev)
    sa = torch.from_numpy(p.sa).to(dev)
    sb = torch.from_numpy(p.sb).to(dev)
    per_set = sum(x.numel() * x.element_size() for x in (a, b, sa, sb)) + 2 * p.M * p.N
    r = 1 if mode == "flush" else max(3, -(-2 * l2_bytes // per_set))
    sets = []
    for i in range(r):
        cp = (a, b, sa, sb) if i == 0 else tuple(x.clone() for x in (a, b, sa, sb))
        sets.append(cp + (torch.empty((p.M, p.N), dtype=torch.bfloat16, device=dev),))
    return sets, per_set


def l2_note(mode: str) -> str:
    if mode == "flush":
        return "flushed (512 MiB memset) before every timed launch, outside the events"
    return "rotating input sets at distinct addresses, together >= 2x L2, launches back to back"


def time_device(call, n_sets: int, steps: int, warmup: int, stream, world: int, mode: str):
    """Device time per launch of `call(i)` (i selects the input set), in ms.

    rotate: the `steps` launches are captured once in a CUDA graph and the
    graph is replayed once between two events, so the host's call overhead
    never leaves the GPU idle between launches; per-launch time = the span /
    steps.  flush: each launch is bracketed by its own events after a 512 MiB
    memset.  Returns (mean ms, per-launch ms list or None)."""
    import torch
    for i in range(warmup):
        call(i % n_sets)
    torch.cuda.synchronize()
    if mode == "flush":
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=stream.device)
        st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(steps):
            flush.zero_()
            st[i].record(stream)
            call(i % n_sets)
            en[i].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        per = [s.elapsed_time(e) for s, e in zip(st, en)]
        return sum(per) / len(per), per
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            call((warmup + i) % n_sets)
    torch.cuda.synchronize()
    g.replay()  # the graph's own first replay uploads it; not timed
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    g.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = t0.elapsed_time(t1) / steps
    del g
    return ms, None


def roofline(p: workloads.Problem, ms: float, name: str, peaks: dict) -> dict:
    """Roofline of one launch: tensor-bound (FLOPs vs the FP8 peak) for
    M > 128, HBM-bound (algorithmic bytes vs the copy bandwidth) otherwise."""
    if p.M > 128:
        return tensor_roofline(p.flops, ms, name, peaks)
    bytes_ = algorithmic_bytes(p)
    peak = peaks["hbm_gbs"]
    achieved = bytes_ / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": profiled_traffic(name), "peak_source": f"{peaks['source']} hbm copy",
            "algorithmic_bytes_per_launch": bytes_}


def run_e2e(p, dev, stream, tuning, args, world):
    """The same GEMM end to end: every step copies its inputs from pinned host
    memory, runs the GEMM through the public binding (whose C ABI takes device
    pointers) and copies the output back to pinned host memory.  Steps are
    double-buffered the way a serving loop would run them: step i+1's
    host->device copies (on a copy stream) and step i-1's device->host copy
    (on another) overlap step i's GEMM; events order each buffer's reuse.  The
    timed region runs from before the first copy to after the last one."""
    import torch
    import fp8_block_scaled_bsgemm_b200 as bsg
    host = [tuple(torch.from_numpy(x).pin_memory() for x in (p.a, p.b, p.sa, p.sb))]
    hout = [torch.empty((p.M, p.N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dbuf = [tuple(torch.empty_like(x, device=dev) for x in host[0]) for _ in range(2)]
    dout = [torch.empty((p.M, p.N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    loaded = [ev(), ev()]       # inputs of buffer j are on the device
    computed = [ev(), ev()]     # the GEMM of buffer j is done (inputs free, output ready)
    drained = [ev(), ev()]      # output of buffer j is back on the host
    for e in computed + drained:
        e.record(stream)

    def step(i):
        j = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(computed[j])              # the GEMM that read buffer j is done
            for d, h in zip(dbuf[j], host[0]):
                d.copy_(h, non_blocking=True)
            loaded[j].record(s_in)
        stream.wait_event(loaded[j])
        stream.wait_event(drained[j])                 # dout[j] was copied out
        a, b, sa, sb = dbuf[j]
        bsg.gemm(a, b, sa, sb, out=dout[j], layout=p.layout, gran=p.gran, tuning=tuning, stream=stream)
        computed[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[j])
            hout[j].copy_(dout[j], non_blocking=True)
            drained[j].record(s_out)

    for i in range(max(1, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(s_in)
    stream.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(args.steps):
        step(i)
    s_out.wait_stream(stream)
    s_out.wait_stream(s_in)
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    e_ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
    h2d = sum(x.numel() * x.element_size() for x in host[0])
    d2h = hout[0].numel() * hout[0].element_size()

    # the link alone: the same copies, one direction at a time, nothing else running
    def copy_ms(fn, reps=5):
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        c0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(reps):
                fn()
        c1.record(stream)
        torch.cuda.synchronize()
        return c0.elapsed_time(c1) / reps

    h2d_ms = copy_ms(lambda: [d.copy_(h, non_blocking=True) for d, h in zip(dbuf[0], host[0])])
    d2h_ms = copy_ms(lambda: hout[0].copy_(dout[0], non_blocking=True))

    def both():
        # both directions at once, on the copy-in and copy-out streams
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        with torch.cuda.stream(s_in):
            for d, h in zip(dbuf[0], host[0]):
                d.copy_(h, non_blocking=True)
        with torch.cuda.stream(s_out):
            hout[1].copy_(dout[1], non_blocking=True)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    both_ms = copy_ms(both)
    return {"value": world * p.flops / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e_ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "link_alone": {"h2d_gbs": h2d / (h2d_ms * 1e-3) / 1e9, "d2h_gbs": d2h / (d2h_ms * 1e-3) / 1e9,
                           "both_directions_ms": both_ms,
                           "note": "the step's copies with no GEMM: one direction at a time (GB/s), and both "
                                   "directions at once (ms), which is the per-step floor of the e2e loop"},
            "path": "per step: pinned host -> device copies of A, B and the scales, the GEMM through the "
                    "public binding (its C ABI takes device pointers), device -> pinned host copy of out; "
                    "double-buffered over a copy-in stream, the GEMM stream and a copy-out stream"}


def clocks_under_load(call, n_sets: int, stream):
    """SM clocks and throttle reasons under this load: the sampler covers
    ~0.4 s of the same launches, eager and back to back, right after the timed
    region (which itself is far shorter than nvidia-smi's sampling interval)."""
    import torch
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_soak = time.perf_counter()
        with torch.cuda.stream(stream):
            i = 0
            while time.perf_counter() - t_soak < 0.4:
                for _ in range(20):
                    call(i % n_sets)
                    i += 1
                stream.synchronize()
    clocks = clk.summary()
    if clocks is not None:
        clocks["window"] = "0.4 s of the benchmark's own launches, back to back, after the timed region"
    return clocks


def tensor_roofline(flops: int, ms: float, name: str, peaks: dict) -> dict:
    # FP8 dense peak = measured BF16 burst x the nominal FP8/BF16 ratio (4.5 / 2.25)
    peak = peaks["bf16_tflops"] * 2.0
    achieved = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": profiled_traffic(name),
            "peak_source": f"{peaks['source']} bf16 burst x 2 (FP8/BF16 nominal ratio)",
            "frac_of_nominal_4500": achieved / 4500.0}


def run_grouped(args, dev, stream, l2_bytes, peaks, world, rank):
    """The grouped GEMM (one persistent launch over all experts) on the
    seeded mixture-of-experts workload, timed like the plain GEMM: rotating
    input sets, a CUDA graph of back-to-back launches, device events."""
    import torch
    import fp8_block_scaled_bsgemm_b200 as bsg
    gp = workloads.grouped_moe()
    rows = gp.a.shape[0]
    base = [torch.from_numpy(x).to(dev) for x in (gp.a, gp.b, gp.sa, gp.sb)]
    group_m = torch.tensor(gp.ms, dtype=torch.int32, device=dev)
    per_set = sum(x.numel() * x.element_size() for x in base) + 2 * rows * gp.N
    r = 1 if args.l2 == "flush" else max(3, -(-2 * l2_bytes // per_set))
    sets = []
    for i in range(r):
        cp = base if i == 0 else [x.clone() for x in base]
        sets.append(tuple(cp) + (torch.empty((rows, gp.N), dtype=torch.bfloat16, device=dev),))

    def call(i):
        a, b, sa, sb, out = sets[i]
        bsg.grouped_gemm(a, b, sa, sb, group_m, out=out, gran=gp.gran, stream=stream)

    with torch.cuda.stream(stream):
        ms, per = time_device(call, len(sets), args.steps, args.warmup, stream, world, args.l2)
    status = bsg.get_last_device_status(stream)
    if status != 0:
        raise SystemExit(f"device status {status} after the timed region of grouped")
    ms_max = max_over_ranks(ms, world)
    clocks = clocks_under_load(call, len(sets), stream)
    if rank != 0:
        _finish(world)
        return
    line = {
        "metric": METRIC, "value": job_tflops(gp.flops, world, ms_max), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3",
        "data": "synthetic",
        "config": {"workload": gp.name, "name": "grouped", "groups": len(gp.ms), "rows_per_group": gp.ms,
                   "N": gp.N, "K": gp.K, "gran": gp.gran, "layout": "nt",
                   "inputs": "E4M3 codes + FP32 block scales, seeded synthetic", "l2": l2_note(args.l2)},
        "parallelism": f"replicas{world}", "input_sets": len(sets), "input_set_bytes": per_set,
        "step": "grouped GEMM (one launch over all groups)",
        "roofline": tensor_roofline(gp.flops, ms, "grouped", peaks),
        "e2e": None, "gpu_launches": args.steps, "clocks": clocks, "hbm_bound": [],
    }
    if not args.no_cpu_baseline and world == 1:
        largest = max(range(len(gp.ms)), key=lambda i: gp.ms[i])
        line["cpu_baseline"] = cpu_baseline(gp.parts[largest], args.cpu_seconds)
    else:
        line["cpu_baseline"] = None
    print(json.dumps(line), flush=True)
    _finish(world)


def run_ours(args):
    import torch
    import fp8_block_scaled_bsgemm_b200 as bsg

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)   # every launch, warm-up, capture and timing on this stream
    props = torch.cuda.get_device_properties(dev)
    num_sms = props.multi_processor_count
    l2_bytes = int(getattr(props, "L2_cache_size", 126 << 20))
    tuning = None
    if args.variant != "auto" or args.bnq or args.splits or args.stream_k:
        tuning = {"variant": args.variant, "bnq": args.bnq, "splits": args.splits, "stream_k": args.stream_k}
    peaks = measured_peaks()
    if args.workload == "grouped":
        run_grouped(args, dev, stream, l2_bytes, peaks, world, rank)
        return

    def measure(name, steps, warmup, tune, quantize_a=False):
        p = make_workload(name)
        sets, per_set = input_sets(p, dev, l2_bytes, args.l2)
        plan = bsg.make_plan(p.M, p.N, p.K, p.gran, p.layout, num_sms, tune)
        if quantize_a:
            if p.layout[0] != "n":
                raise SystemExit("--quantize-a needs A stored [M, K] (nt or nn)")
            # a BF16 activation per set: the set's own A, dequantised (codes x block scales)
            xs = []
            for a, _, sa, _, _ in sets:
                deq = a.view(torch.float8_e4m3fn).float()
                sc = sa.repeat_interleave(p.gran, 0)[:p.M].repeat_interleave(p.gran, 1)[:, :p.K]
                xs.append((deq * sc).to(torch.bfloat16))
            per_set += p.M * p.K * 2

        def call(i):
            a, b, sa, sb, out = sets[i]
            if quantize_a:
                bsg.quantize(xs[i], p.gran, "e4m3", q=a, scales=sa, stream=stream)
            bsg.gemm(a, b, sa, sb, out=out, layout=p.layout, gran=p.gran, tuning=tune, stream=stream)

        with torch.cuda.stream(stream):
            ms, per = time_device(call, len(sets), steps, warmup, stream, world, args.l2)
        status = bsg.get_last_device_status(stream)
        if status != 0:
            raise SystemExit(f"device status {status} after the timed region of {name}")
        return p, sets, plan, ms, per, per_set, call

    p, sets, plan, ms, per, per_set, call = measure(args.workload, args.steps, args.warmup, tuning,
                                                    args.quantize_a)
    ms_max = max_over_ranks(ms, world)

    clocks = clocks_under_load(call, len(sets), stream)

    # ---- e2e through the public API from pinned host memory
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(p, dev, stream, tuning, args, world)

    # ---- the HBM-bound half of the metric: small-M decode shapes
    hbm_points = []
    if args.hbm_points and world == 1:
        for m in [int(x) for x in args.hbm_points.split(",") if x]:
            name = f"small_m:{m}"
            hp, hsets, hplan, hms, _, _, _ = measure(name, max(args.steps, 50), max(args.warmup, 3), None)
            hbm_points.append({"workload": name, "config": workload_config(hp, name, args.l2),
                               "ms_per_launch": hms, "tflops": hp.flops / (hms * 1e-3) / 1e12,
                               "steps": max(args.steps, 50), "plan": hplan,
                               "roofline": roofline(hp, hms, name, peaks)})
            del hsets

    if rank != 0:
        _finish(world)
        return
    line = {
        "metric": METRIC, "value": job_tflops(p.flops, world, ms_max), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3",
        "data": "synthetic", "config": workload_config(p, args.workload, args.l2),
        "parallelism": f"replicas{world}", "plan": plan, "input_sets": len(sets),
        "input_set_bytes": per_set,
        "step": ("quantise A (BF16 -> E4M3 + block scales) + GEMM" if args.quantize_a else "GEMM"),
        "roofline": roofline(p, ms, args.workload, peaks), "e2e": e2e,
        "gpu_launches": args.steps * (plan["kernels"] + (1 if args.quantize_a else 0)), "clocks": clocks,
        "hbm_bound": hbm_points,
    }
    if per:
        line["min_ms"] = min(per)
        line["median_ms"] = statistics.median(per)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(p, args.cpu_seconds)
    else:
        line["cpu_baseline"] = None
    print(json.dumps(line), flush=True)
    _finish(world)


def _finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    if args.workload == "grouped":
        # the oracle's throughput on the largest group (each group is a plain GEMM)
        gp = workloads.grouped_moe()
        p = gp.parts[max(range(len(gp.ms)), key=lambda i: gp.ms[i])]
        config = {"workload": gp.name, "name": "grouped", "sample_of": "the largest group",
                  "l2": l2_note(args.l2)}
    else:
        p = make_workload(args.workload)
        config = workload_config(p, args.workload, args.l2)
    budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))  # whole run within a few minutes
    per = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(p, min(budget, args.cpu_seconds))
        if i >= args.warmup:
            per.append(r)
    value = statistics.mean(r["value"] for r in per)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.mean(r["seconds"] for r in per) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": per[-1]["sample"] + " per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
