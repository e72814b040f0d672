"""Benchmark: causal ring attention (zigzag context parallel) forward and
forward+backward on B200, through the C ABI of libcpattn.so.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cpattn,reference}]
                    [--workload NAME]

One step = the whole hot path over one batch: cpattn_fwd (every ring step,
merged on chip) then cpattn_bwd (preprocess, recompute backward, dQ
conversion).  Inputs are resident in HBM before the timed region; q, k, v, O,
dO together are far larger than the 126 MB L2, so no flush is needed between
steps.  Timing: CUDA events on the launch stream, barrier + synchronize on
both sides, max over ranks.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the correctness reference) on the
host cores over a bounded sample of the same workload, as a baseline arm.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "causal_b1h32s32768d128_cp8_bf16"
METRIC = "causal ring-attn TFLOP/s fwd & fwd+bwd on 1 B200; % of BF16 tensor peak"


# DRAM traffic of the dominant kernel, read from a committed ncu summary.  The
# summary records a digest of the kernel's sources at capture time; when the
# sources have changed since, the figure no longer describes the kernel and
# traffic is reported as null.
TRAFFIC_FILES = {
    ("tc_dkdv", "causal_b1h32s32768d128_cp8_bf16"):
        os.path.join(ROOT, "profiles", "traffic_tc_dkdv_causal_b1h32s32768d128_cp8.txt"),
}
# the files whose contents determine the kernel's device code and its TMA boxes
# (kernels.h only declares host launchers and profiling ids)
KERNEL_SOURCES = {
    "tc_dkdv": ["tc_bwd.cu", "bwd_common.cuh", "sm100.cuh", "tmap.h", "ring.cuh"],
}


def kernel_source_digest(kernel):
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "long_sequence_context_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(kernel, workload):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch, or None."""
    path = TRAFFIC_FILES.get((kernel, workload))
    if path is None or not os.path.exists(path):
        return None
    rec = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.lstrip().startswith("#"):
                k, v = line.split(":", 1)
                rec[k.strip()] = v.strip()
    if rec.get("source_sha256") != kernel_source_digest(kernel):
        return None
    try:
        return int(rec["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# --------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = str(gpu_index)
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", self.gpu, "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        med = statistics.median(sm) if sm else None
        return {"sm_mhz": med, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ dist setup --
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def e2e_chunks(w, want):
    """Number of groups one end-to-end step is split into: a divisor of the
    heads (B == 1) or of the batch, at most `want`."""
    n = w.H if w.B == 1 else w.B
    c = max(1, min(want, n))
    while n % c:
        c -= 1
    return c


def chunk_views(t, w, c):
    """`c` contiguous views of a [B, H, S, ...] tensor: head groups when B == 1,
    batch groups otherwise."""
    dim = 1 if w.B == 1 else 0
    return list(t.chunk(c, dim=dim))


def max_over_ranks(x, world):
    """Largest value of x over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank_step, steps, ms_max, world):
    """Whole-job throughput: every rank runs its own replica of the workload."""
    return world * flops_per_rank_step * steps / (ms_max * 1e-3) / 1e12


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ CPU oracle --
def oracle_sample(w, seconds_hint=10.0):
    """fp64 oracle fwd+bwd over one head of the workload truncated to S' rows.

    Returns (TFLOP/s, description, threads).  The algorithmic FLOPs of the sample
    use the same counting as the GPU number (causal half, backward 2.5x)."""
    import numpy as np
    import torch
    from long_sequence_context_b200.inputs import make_qkv
    from oracle import oracle as orc
    S_s = min(w.S, 4096)
    q, k, v, do = make_qkv(1, 1, S_s, w.D, w.torch_dtype, seed=w.seed, qkv_scale=w.qkv_scale)
    f = lambda t: t.float().numpy().astype(np.float64)
    q, k, v, do = f(q), f(k), f(v), f(do)
    dense = 4.0 * S_s * S_s * w.D
    flops_one = (dense / 2 if w.causal else dense) * 3.5
    total, reps, t0 = 0.0, 0, time.perf_counter()
    while True:
        orc.attn_fwd(q, k, v, w.causal, w.scale)
        orc.attn_bwd(q, k, v, do, w.causal, w.scale)
        reps += 1
        total = time.perf_counter() - t0
        if total >= seconds_hint or reps >= 50:
            break
    tfl = flops_one * reps / total / 1e12
    desc = (f"fp64 oracle fwd+bwd, 1 head x S={S_s} (prefix length of the workload's shape, "
            f"same D, dtype-rounded inputs), {reps} rep(s) in {total:.1f}s")
    return tfl, desc, orc.threads()


def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    from long_sequence_context_b200.inputs import make_qkv
    from oracle import oracle as orc
    S_s = min(w.S, 2048)
    q, k, v, do = make_qkv(1, 1, S_s, w.D, w.torch_dtype, seed=w.seed, qkv_scale=w.qkv_scale)
    f = lambda t: t.float().numpy().astype(np.float64)
    q, k, v, do = f(q), f(k), f(v), f(do)
    dense = 4.0 * S_s * S_s * w.D
    flops_step = (dense / 2 if w.causal else dense) * 3.5

    def step():
        orc.attn_fwd(q, k, v, w.causal, w.scale)
        orc.attn_bwd(q, k, v, do, w.causal, w.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    val = flops_step * args.steps / dt / 1e12
    sample = (f"fp64 oracle fwd+bwd per step over 1 head x S={S_s} of the workload's shape "
              f"(dtype-rounded inputs)")
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "D": w.D,
                       "cp_size": w.cp_size, "causal": w.causal},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": orc.threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------- standalone LSE merge --
MERGE_ROWS, MERGE_D = 1 << 20, 128


def pre_bytes_per_row(D, elem=2):
    """Backward preprocess: read a row of O and of dO and its LSE, write delta
    and LSE * log2(e)."""
    return 2 * D * elem + 4 + 2 * 4


def merge_bytes_per_row(D):
    """Algorithmic bytes of one merged row: read O_acc, O_part (D fp32 each) and
    the two LSEs, write O_acc and LSE_acc."""
    return 3 * D * 4 + 3 * 4


def time_merge(cp, dev, peaks, launches=20, warmup=3, rows=MERGE_ROWS, D=MERGE_D):
    """cpattn_merge over `rows` rows of D fp32 (in place, the same buffers every
    launch; 1.6 GB of operands, far larger than L2): mean device time per launch
    from CUDA events on the launch stream, GB/s of algorithmic bytes."""
    import torch
    g = torch.Generator(device=dev).manual_seed(77)
    o_acc = torch.randn((rows, D), generator=g, device=dev)
    o_part = torch.randn((rows, D), generator=g, device=dev)
    lse_acc = torch.randn((rows,), generator=g, device=dev)
    lse_part = torch.randn((rows,), generator=g, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        cp.merge_(o_acc, lse_acc, o_part, lse_part)
    torch.cuda.synchronize(dev)
    n0 = cp.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(launches):
        cp.merge_(o_acc, lse_acc, o_part, lse_part)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    n = cp.launch_count() - n0
    ms = e0.elapsed_time(e1) / launches
    per_launch = merge_bytes_per_row(D) * rows
    gbs = per_launch / (ms * 1e-3) / 1e9
    st = cp.sync_status()
    if st != cp.OK:
        raise RuntimeError(f"merge failed: {cp.status_str(st)}")
    del o_acc, o_part, lse_acc, lse_part
    return {"kernel": "merge_kernel", "rows": rows, "D": D, "launches": n,
            "ms_per_launch": ms, "bytes_per_launch": per_launch,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"],
                         "peak_kind": f"hbm_gbs ({peaks['source']})"}}


def time_workload(cp, w, dev, peaks, steps=5, warmup=3):
    """Device time of one workload's hot path (forward, plus backward when the
    workload has one), per kernel from the library's event hooks."""
    import torch
    from long_sequence_context_b200.inputs import workload_inputs
    q, k, v, do = (t.to(dev) for t in workload_inputs(w, with_dout=True))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
    grads = [torch.empty_like(q) for _ in range(3)]
    ws = torch.empty(cp.bwd_workspace_bytes(w.B, w.H, w.S, w.D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        cp.fwd(q, k, v, w.cp_size, w.causal, w.scale, out=o, lse=lse)
        if w.backward:
            cp.bwd(q, k, v, o, lse, do, w.cp_size, w.causal, w.scale, workspace=ws,
                   dq=grads[0], dk=grads[1], dv=grads[2])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    cp.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    cp.profile(False)
    st = cp.sync_status()
    if st != cp.OK:
        raise RuntimeError(f"{w.name} failed: {cp.status_str(st)}")
    ms = e0.elapsed_time(e1) / steps
    kern = {}
    for kind, name in cp.KERNEL_KINDS.items():
        t, n = cp.profile_read(kind)
        if n:
            kern[name] = t / steps
    fwd_ms = kern.get("tc_fwd", kern.get("simt_fwd"))
    f_fwd = w.flops_fwd()
    f_bwd = w.flops_bwd() if w.backward else 0.0
    bwd_ms = (ms - fwd_ms) if (w.backward and fwd_ms) else None
    del q, k, v, do, o, lse, grads, ws
    torch.cuda.empty_cache()
    out = {"passes": "fwd+bwd" if w.backward else "fwd", "dtype": w.dtype,
           "ms_per_step": ms, "tflops": (f_fwd + f_bwd) / (ms * 1e-3) / 1e12,
           "fwd_ms": fwd_ms, "fwd_tflops": f_fwd / (fwd_ms * 1e-3) / 1e12 if fwd_ms else None,
           "kernel_ms_per_step": kern}
    if w.backward and bwd_ms:
        out["bwd_ms"] = bwd_ms
        out["bwd_tflops"] = f_bwd / (bwd_ms * 1e-3) / 1e12
    if w.dtype == "bf16":
        out["frac_of_peak"] = out["tflops"] / peaks["bf16_tflops"]
        if fwd_ms:
            out["fwd_frac_of_peak"] = out["fwd_tflops"] / peaks["bf16_tflops"]
    return out


def time_fwd_separately(cp, w, q, k, v, o, lse, peaks, local, steps=10):
    """The headline workload's forward timed on its own (K forward calls back
    to back on the resident inputs, after the warm-up and before the fwd + bwd
    region), the separate forward timing of the measurement plan.  The
    forward's time inside the fwd + bwd step is reported beside it
    (fwd_tflops), lower where the backward's power draw has lowered the clocks."""
    import torch
    stream = torch.cuda.current_stream(q.device)
    cp.fwd(q, k, v, w.cp_size, w.causal, w.scale, out=o, lse=lse)
    torch.cuda.synchronize(q.device)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        cp.fwd(q, k, v, w.cp_size, w.causal, w.scale, out=o, lse=lse)
    e1.record(stream)
    torch.cuda.synchronize(q.device)
    clk = clocks.stop()
    st = cp.sync_status()
    if st != cp.OK:
        raise RuntimeError(f"forward failed: {cp.status_str(st)}")
    ms = e0.elapsed_time(e1) / steps
    tfl = w.flops_fwd() / (ms * 1e-3) / 1e12
    return {"ms": ms, "tflops": tfl, "frac_of_peak": tfl / peaks["bf16_tflops"], "steps": steps,
            "l2": "inputs larger than L2; no flush", "clocks": clk}


def time_fp8_fwd(cp, w, q, k, v, peaks, steps=10, warmup=3):
    """The e4m3 ring forward (cpattn_fwd_fp8) on the workload's inputs, already
    quantised (K/V kept in e4m3, as a context-parallel job would hold them),
    and, separately, the quantisation of q, k, v (amax + codes, V transposed)."""
    import torch
    dev = q.device
    stream = torch.cuda.current_stream(dev)
    q8, k8, vt8, a3 = cp.quantize_qkv_e4m3(q, k, v)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    n0 = cp.launch_count()
    fwd_ms = timed(lambda: cp.fwd_fp8(q8, k8, vt8, a3, w.cp_size, w.causal, w.scale, out=o, lse=lse))
    n_fwd = (cp.launch_count() - n0) / (steps + warmup)
    quant_ms = timed(lambda: cp.quantize_qkv_e4m3(q, k, v))
    st = cp.sync_status()
    if st != cp.OK:
        raise RuntimeError(f"fp8 forward failed: {cp.status_str(st)}")
    tfl = w.flops_fwd() / (fwd_ms * 1e-3) / 1e12
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    del q8, k8, vt8, a3, o, lse
    return {"kernel": "tc_fwd_kernel<128, e4m3>", "workload": w.name, "ms": fwd_ms, "tflops": tfl,
            "launches_per_call": n_fwd,
            "roofline": {"bound": "tensor", "achieved": tfl, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": tfl / fp8_peak,
                         "peak_kind": f"2 x bf16_tflops ({peaks['source']}; nominal fp8/bf16 dense ratio 4.5/2.25)"},
            "quantize_ms": quant_ms,
            "tflops_incl_quantize": w.flops_fwd() / ((fwd_ms + quant_ms) * 1e-3) / 1e12}


# --------------------------------------------------------------- GPU arm --
def run_gpu(args, w):
    import torch
    world, rank, local = dist_setup(args.gpus)
    from long_sequence_context_b200 import cpattn as cp
    from long_sequence_context_b200.inputs import workload_inputs
    peaks = load_peaks()
    dev = torch.device("cuda", local)

    q, k, v, do = workload_inputs(w, with_dout=True)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    od = torch.empty_like(qd)
    lsed = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
    dqd, dkd, dvd = torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd)
    ws = torch.empty(cp.bwd_workspace_bytes(w.B, w.H, w.S, w.D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        cp.fwd(qd, kd, vd, w.cp_size, w.causal, w.scale, out=od, lse=lsed)
        if not args.fwd_only:
            cp.bwd(qd, kd, vd, od, lsed, dod, w.cp_size, w.causal, w.scale, workspace=ws,
                   dq=dqd, dk=dkd, dv=dvd)

    for _ in range(args.warmup):
        step()
    st = cp.sync_status()
    if st != cp.OK:
        raise RuntimeError(f"warm-up failed: {cp.status_str(st)}")

    # ---- the forward timed separately (one GPU) ----
    fwd_sep = None
    if world == 1 and not args.fwd_only and not args.no_extra:
        fwd_sep = time_fwd_separately(cp, w, qd, kd, vd, od, lsed, peaks, local, steps=args.steps)

    # ---- timed region (device events, max over ranks) ----
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    n0 = cp.launch_count()
    cp.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    cp.profile(False)
    launches = cp.launch_count() - n0
    ms_total = max_over_ranks(e0.elapsed_time(e1), world)
    clk = clocks.stop()
    st = cp.sync_status()
    if st != cp.OK:
        raise RuntimeError(f"timed region failed: {cp.status_str(st)}")

    ms_step = ms_total / args.steps
    f_fwd, f_bwd = w.flops_fwd(), (0.0 if args.fwd_only else w.flops_bwd())
    value = job_tflops(f_fwd + f_bwd, args.steps, ms_total, world)

    per_kernel = {}
    for kind, name in cp.KERNEL_KINDS.items():
        ms, n = cp.profile_read(kind)
        if n:
            per_kernel[name] = {"ms_total": ms, "launches": n, "ms_avg": ms / n}
    fwd_ms = per_kernel.get("tc_fwd", per_kernel.get("simt_fwd", {})).get("ms_avg")
    fwd_tflops = f_fwd / (fwd_ms * 1e-3) / 1e12 if fwd_ms else None

    # dominant kernel and its roofline (tensor-bound: algorithmic FLOPs per launch)
    # backward split: the dK/dV kernels own S, dP, dV, dK (4 of the 5 matrix
    # products), the dQ kernels own dQ (their S / dP recompute is not counted)
    alg_flops = {"tc_fwd": f_fwd, "simt_fwd": f_fwd, "tc_dkdv": 0.8 * f_bwd, "tc_dq": 0.2 * f_bwd,
                 "simt_dkdv": 0.8 * f_bwd, "simt_dq": 0.2 * f_bwd}
    dom = max(per_kernel, key=lambda n: per_kernel[n]["ms_total"])
    peak = peaks["bf16_tflops_sustained"]
    roof = None
    if dom in alg_flops:
        ach = alg_flops[dom] / (per_kernel[dom]["ms_avg"] * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": peak,
                "peak_kind": f"bf16_tflops_sustained ({peaks['source']})", "unit": "TFLOP/s",
                "frac": ach / peak, "frac_of_burst_peak": ach / peaks["bf16_tflops"],
                "traffic": recorded_traffic(dom, w.name), "traffic_unit": "bytes per launch"}

    # the backward preprocess (HBM-bound): O, dO read, LSE read, delta and
    # LSE*log2(e) written, per row
    pre_roof = None
    if "bwd_delta" in per_kernel:
        rows = w.B * w.H * w.S
        by = rows * pre_bytes_per_row(w.D, 2 if w.dtype == "bf16" else 4)
        gbs = by / (per_kernel["bwd_delta"]["ms_avg"] * 1e-3) / 1e9
        pre_roof = {"bound": "hbm", "kernel": "bwd_delta", "achieved": gbs, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "bytes_per_launch": by,
                    "peak_kind": f"hbm_gbs ({peaks['source']})"}

    # ---- end to end through the public API with host buffers ----
    # Every step copies its inputs (q, k, v, dO) from pinned host memory and reads
    # its results (O, LSE, dQ, dK, dV) back.  Pipelined: device tensors are
    # double-buffered, host->device copies run on one copy stream and
    # device->host reads on another, so step i+1's inputs arrive and step i's
    # results leave while step i+1 / i compute.  The serial variant (copy in,
    # compute, copy out, one after another) is reported beside it.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (t.pin_memory() for t in (q, k, v, do))
        h_in = (hq, hk, hv, hdo)
        h2d = sum(t.numel() * t.element_size() for t in h_in)

        def new_set():
            d_in = tuple(torch.empty_like(t, device=dev) for t in h_in)
            d_out = (torch.empty_like(d_in[0]), torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev),
                     torch.empty_like(d_in[0]), torch.empty_like(d_in[0]), torch.empty_like(d_in[0]))
            h_out = tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in d_out)
            return d_in, d_out, h_out

        sets = [new_set(), new_set()]
        d2h = sum(t.numel() * t.element_size() for t in sets[0][2])

        def compute(d_in, d_out):
            qq, kk, vv, dd = d_in
            oo, ll, gq, gk, gv = d_out
            cp.fwd(qq, kk, vv, w.cp_size, w.causal, w.scale, out=oo, lse=ll)
            if not args.fwd_only:
                cp.bwd(qq, kk, vv, oo, ll, dd, w.cp_size, w.causal, w.scale, workspace=ws,
                       dq=gq, dk=gk, dv=gv)

        def run_serial(n):
            for _ in range(n):
                d_in, d_out, h_out = sets[0]
                for h, d in zip(h_in, d_in):
                    d.copy_(h, non_blocking=True)
                compute(d_in, d_out)
                for d, h in zip(d_out, h_out):
                    h.copy_(d, non_blocking=True)

        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        # Each step is split into head groups (batch groups when B > 1), one
        # public-API call per group, so that the first group's compute starts
        # once its inputs are on the device and the last group's results leave
        # while nothing else is pending: only 1/C of the first copy-in and of
        # the last copy-out stay exposed.
        n_chunks = e2e_chunks(w, args.e2e_chunks)
        views = [(tuple(chunk_views(t, w, n_chunks) for t in d_in), tuple(chunk_views(t, w, n_chunks) for t in d_out),
                  tuple(chunk_views(t, w, n_chunks) for t in h_out)) for d_in, d_out, h_out in sets]
        h_in_v = tuple(chunk_views(t, w, n_chunks) for t in h_in)

        def run_pipelined(n):
            ev = lambda: torch.cuda.Event()
            in_done = [[ev() for _ in range(n_chunks)] for _ in range(2)]
            comp_done = [[ev() for _ in range(n_chunks)] for _ in range(2)]
            out_done = [[ev() for _ in range(n_chunks)] for _ in range(2)]
            for i in range(n):
                b = i % 2
                d_in, d_out, h_out = views[b]
                with torch.cuda.stream(s_in):
                    for c in range(n_chunks):
                        if i >= 2:
                            s_in.wait_event(comp_done[b][c])   # step i-2 has read this group's inputs
                        for h, d in zip(h_in_v, d_in):
                            d[c].copy_(h[c], non_blocking=True)
                        in_done[b][c].record(s_in)
                for c in range(n_chunks):
                    stream.wait_event(in_done[b][c])
                    if i >= 2:
                        stream.wait_event(out_done[b][c])      # step i-2's results of this group have left
                    compute(tuple(t[c] for t in d_in), tuple(t[c] for t in d_out))
                    comp_done[b][c].record(stream)
                    with torch.cuda.stream(s_out):
                        s_out.wait_event(comp_done[b][c])
                        for d, h in zip(d_out, h_out):
                            h[c].copy_(d[c], non_blocking=True)
                        out_done[b][c].record(s_out)
            for row in out_done:
                for e in row:
                    stream.wait_event(e)

        def timed(fn, n):
            fn(1)
            torch.cuda.synchronize(dev)
            barrier(world)
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            fn(n)
            a1.record(stream)
            torch.cuda.synchronize(dev)
            barrier(world)
            return max_over_ranks(a0.elapsed_time(a1), world)

        n_e2e = max(2, args.steps)  # as many steps as the device-timed region: fill and drain amortised alike
        ser_ms = timed(run_serial, n_e2e)
        pip_ms = timed(run_pipelined, n_e2e)
        e2e = {"value": job_tflops(f_fwd + f_bwd, n_e2e, pip_ms, world), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": pip_ms / n_e2e,
               "overlap": "double-buffered device tensors; H2D and D2H on two copy streams overlap the "
                          "neighbouring steps' compute; each step runs as `chunks` head groups, so 1/chunks of "
                          "the first copy-in and of the last copy-out stay exposed",
               "chunks": n_chunks,
               "serial": {"value": job_tflops(f_fwd + f_bwd, n_e2e, ser_ms, world),
                          "ms_per_step": ser_ms / n_e2e}}

    # ---- the other workloads and the standalone merge (device-timed, after the
    # headline region; each its own allocation) ----
    per_config, merge, fp8 = None, None, None
    if not args.no_extra and world == 1:
        if w.D == 128 and w.dtype == "bf16":
            fp8 = time_fp8_fwd(cp, w, qd, kd, vd, peaks)
        per_config = {}
        from long_sequence_context_b200.inputs import WORKLOADS
        for name, wk in WORKLOADS.items():
            if name != w.name:
                per_config[name] = time_workload(cp, wk, dev, peaks)
        merge = time_merge(cp, dev, peaks)

    # ---- CPU baseline: the oracle on this host, rank 0, N == 1 only ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tfl, desc, threads = oracle_sample(w)
        cpu = {"value": tfl, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "D": w.D,
                       "cp_size": w.cp_size, "causal": w.causal,
                       "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs (q,k,v,O,dO ~1.3 GB) larger than L2; no flush"},
            "fwd_tflops": fwd_tflops,
            "fwd_separate": fwd_sep,
            "fwd_frac_of_peak": (fwd_tflops / peaks["bf16_tflops"]) if fwd_tflops else None,
            "fwd_bwd_frac_of_peak": value / world / peaks["bf16_tflops"],
            "peaks": peaks,
            "per_kernel_ms": per_kernel,
            "roofline": roof,
            "preprocess_roofline": pre_roof,
            "per_config": per_config,
            "merge": merge,
            "fp8_fwd": fp8,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


LAYER_METRIC = "attention layer (projections + ring attention) TFLOP/s fwd+bwd on 1 B200"


def layer_oracle_sample(w, seconds_hint=10.0):
    """fp64 layer oracle (forward + backward) over the workload's layer shape
    truncated to S' = 1024 rows.  Returns (TFLOP/s, description, threads)."""
    from long_sequence_context_b200.inputs import flops_layer, make_layer_inputs
    from oracle import layer as olayer
    from oracle import oracle as orc
    S_s, E = min(w.S, 1024), w.H * w.D
    t = [a.double().numpy() for a in make_layer_inputs(1, S_s, E, seed=w.seed)]
    flops = sum(flops_layer(1, S_s, E, w.H, w.causal))
    reps, t0 = 0, time.perf_counter()
    while True:
        olayer.layer_bwd(*t, w.H, w.causal, w.scale)
        reps += 1
        total = time.perf_counter() - t0
        if total >= seconds_hint or reps >= 20:
            break
    desc = (f"fp64 layer oracle fwd+bwd, B=1 S={S_s} E={E} H={w.H} (prefix length of the "
            f"workload's shape), {reps} rep(s) in {total:.1f}s")
    return flops * reps / total / 1e12, desc, orc.threads()


def run_layer(args, w):
    """The attention layer around the ring attention, forward + backward per
    step: E = H * D of the workload, B, S, cp_size, causal as in it.  Separate
    from the headline line; prints its own JSON line."""
    import torch
    world, rank, local = dist_setup(args.gpus)
    from long_sequence_context_b200 import cpattn as cp
    from long_sequence_context_b200.inputs import flops_layer, make_layer_inputs
    peaks = load_peaks()
    dev = torch.device("cuda", local)
    B, S, H, D = w.B, w.S, w.H, w.D
    E = H * D
    x, w_qkv, b_qkv, w_o, b_o, dy = (t.to(dev) for t in make_layer_inputs(B, S, E, seed=w.seed))
    ws = torch.empty(cp.layer_workspace_bytes(B, S, E, H), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        _, saved = cp.layer_fwd(x, w_qkv, b_qkv, w_o, b_o, H, w.cp_size, w.causal, w.scale, workspace=ws)
        cp.layer_bwd(x, w_qkv, w_o, saved, dy, H, w.cp_size, w.causal, w.scale, workspace=ws)

    for _ in range(args.warmup):
        step()
    if cp.sync_status() != cp.OK:
        raise RuntimeError("layer warm-up failed")
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    n0 = cp.launch_count()
    cp.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    cp.profile(False)
    launches = cp.launch_count() - n0
    ms_total = max_over_ranks(e0.elapsed_time(e1), world)
    clk = clocks.stop()
    if cp.sync_status() != cp.OK:
        raise RuntimeError("layer timed region failed")
    f_fwd, f_bwd = flops_layer(B, S, E, H, w.causal)
    ms_step = ms_total / args.steps
    per_kernel = {}
    for kind, name in cp.KERNEL_KINDS.items():
        ms, n = cp.profile_read(kind)
        if n:
            per_kernel[name] = {"ms_total": ms, "launches": n, "ms_avg": ms / n}
    own_ms = sum(v["ms_total"] for v in per_kernel.values()) / args.steps
    # head reshapes per step: q|k|v split, O merge (fwd and bwd), dO split, dQ|dK|dV merge:
    # each reads and writes its tensor once: (3 + 1 + 1 + 1 + 3) * B*S*E bf16 elements, x2
    heads_bytes = 9 * B * S * E * 2 * 2
    hk = per_kernel.get("layer_heads")
    heads_roof = None
    if hk:
        ach = heads_bytes / (hk["ms_total"] / args.steps * 1e-3) / 1e9
        heads_roof = {"bound": "hbm", "kernel": "layer_heads", "achieved": ach, "peak": peaks["hbm_gbs"],
                      "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]}
    # projection GEMMs (tensor-bound): 8*B*S*E^2 FLOPs forward, twice that backward
    gk = per_kernel.get("gemm")
    gemm_roof = None
    if gk:
        g_flops = 24.0 * B * S * E * E
        g_ms = gk["ms_total"] / args.steps
        ach = g_flops / (g_ms * 1e-3) / 1e12
        gemm_roof = {"bound": "tensor", "kernel": "gemm", "ms_per_step": g_ms, "launches_per_step":
                     gk["launches"] / args.steps, "achieved": ach, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                     "peak_kind": f"bf16_tflops ({peaks['source']})"}
    if rank == 0:
        line = {
            "metric": LAYER_METRIC, "value": (f_fwd + f_bwd) * world / (ms_step * 1e-3) / 1e12,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (nn.Linear-range random weights)",
            "config": {"workload": f"layer_{w.name}", "B": B, "S": S, "E": E, "H": H, "D": D,
                       "cp_size": w.cp_size, "causal": w.causal},
            "flops_per_step": {"fwd": f_fwd, "bwd": f_bwd},
            "per_kernel_ms": per_kernel,
            "gemm_roofline": gemm_roof,
            "unattributed_ms_per_step": ms_step - own_ms,
            "heads_roofline": heads_roof,
            "gpu_launches": launches,
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            tfl, desc, threads = layer_oracle_sample(w)
            line["cpu_baseline"] = {"value": tfl, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": desc}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


RING_METRIC = "ring attention across ranks (one sequence, chunks per GPU) TFLOP/s fwd+bwd"


def run_ring(args, w):
    """The multi-rank ring (long_sequence_context_b200/ring.py): one sequence of
    the workload split over the N GPUs (2N zigzag chunks when causal), K/V
    exchanged between neighbours every step; strong scaling (the total work is
    the workload's).  Prints its own JSON line."""
    import torch
    world, rank, local = dist_setup(args.gpus)
    from long_sequence_context_b200 import cpattn as cp
    from long_sequence_context_b200 import ring
    from long_sequence_context_b200.inputs import workload_inputs
    dev = torch.device("cuda", local)
    q, k, v, do = workload_inputs(w, with_dout=True)
    loc = lambda x: [c.to(dev) for c in ring.local_chunks(x, rank, world, w.causal)]
    ql, kl, vl, dol = loc(q), loc(k), loc(v), loc(do)
    stream = torch.cuda.current_stream(dev)

    def step():
        o, lse = ring.ring_fwd(ql, kl, vl, w.causal, w.scale)
        ring.ring_bwd(ql, kl, vl, o, lse, dol, w.causal, w.scale)

    for _ in range(args.warmup):
        step()
    if cp.sync_status() != cp.OK:
        raise RuntimeError("ring warm-up failed")
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    n0 = cp.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    launches = cp.launch_count() - n0
    ms_total = max_over_ranks(e0.elapsed_time(e1), world)
    clk = clocks.stop()
    if cp.sync_status() != cp.OK:
        raise RuntimeError("ring timed region failed")
    flops = w.flops_fwd() + w.flops_bwd()
    if rank == 0:
        line = {"metric": RING_METRIC, "value": flops / (ms_total / args.steps * 1e-3) / 1e12,
                "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_total / args.steps, "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": f"ring_{w.name}", "B": w.B, "H": w.H, "S": w.S, "D": w.D,
                           "ring_ranks": world, "causal": w.causal,
                           "chunk_rows": w.S // (2 * world if w.causal else world)},
                "gpu_launches": launches, "clocks": clk}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


FP8_METRIC = "causal ring-attn forward on e4m3 inputs TFLOP/s on 1 B200; fraction of the fp8 tensor peak"


def run_fp8(args, w):
    """The e4m3 ring forward alone (inputs quantised before the timed region,
    as a context-parallel job keeps its K/V in e4m3).  Prints its own JSON line."""
    import torch
    world, rank, local = dist_setup(args.gpus)
    from long_sequence_context_b200 import cpattn as cp
    from long_sequence_context_b200.inputs import workload_inputs
    peaks = load_peaks()
    dev = torch.device("cuda", local)
    q, k, v, _ = workload_inputs(w, with_dout=False)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    r = time_fp8_fwd(cp, w, qd, kd, vd, peaks, steps=args.steps, warmup=args.warmup)
    clk = clocks.stop()
    ms = max_over_ranks(r["ms"], world)
    if rank == 0:
        line = {"metric": FP8_METRIC, "value": world * w.flops_fwd() / (ms * 1e-3) / 1e12,
                "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "e4m3 (fp32 accumulate, bf16 out)", "data": "synthetic",
                "config": {"workload": f"fp8_{w.name}", "B": w.B, "H": w.H, "S": w.S, "D": w.D,
                           "cp_size": w.cp_size, "causal": w.causal,
                           "l2": "inputs larger than L2; no flush"},
                "roofline": r["roofline"], "quantize_ms": r["quantize_ms"],
                "gpu_launches": int(round(r["launches_per_call"] * args.steps)), "clocks": clk}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


MERGE_METRIC = "standalone LSE merge (cpattn_merge) GB/s on 1 B200; fraction of measured HBM copy bandwidth"


def run_merge(args):
    """The standalone log-sum-exp merge of two fp32 partials over 1,048,576 rows
    of D = 128 (one S = 32K, H = 32 set of rows).  Prints its own JSON line."""
    import torch
    world, rank, local = dist_setup(args.gpus)
    from long_sequence_context_b200 import cpattn as cp
    peaks = load_peaks()
    dev = torch.device("cuda", local)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    m = time_merge(cp, dev, peaks, launches=args.steps, warmup=args.warmup)
    clk = clocks.stop()
    if rank == 0:
        line = {"metric": MERGE_METRIC, "value": m["roofline"]["achieved"], "unit": "GB/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": m["ms_per_launch"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": f"merge_rows{m['rows']}_d{m['D']}", "rows": m["rows"], "D": m["D"],
                           "l2": "operands 1.6 GB, larger than L2; no flush"},
                "roofline": m["roofline"], "gpu_launches": m["launches"], "clocks": clk}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cpattn", choices=["cpattn", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=4,
                    help="head (or batch) groups per end-to-end step, overlapping the first copy-in and last copy-out")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fwd-only", action="store_true", help="time the forward alone (profiling)")
    ap.add_argument("--ring", action="store_true",
                    help="time the multi-rank ring: one sequence split over the --gpus ranks")
    ap.add_argument("--layer", action="store_true",
                    help="time the attention layer (projections + ring attention) instead")
    ap.add_argument("--fp8", action="store_true",
                    help="time the e4m3 forward (cpattn_fwd_fp8) alone")
    ap.add_argument("--merge", action="store_true",
                    help="time the standalone LSE merge (cpattn_merge) alone")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads and the merge in the headline line")
    ap.add_argument("--shape", default=None,
                    help="B,H,S,D,cp_size,causal: a smaller case of the workload (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from long_sequence_context_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.shape:
        import dataclasses
        B, H, S, D, N, c = (int(x) for x in args.shape.split(","))
        w = dataclasses.replace(w, name=f"{w.name}@B{B}H{H}S{S}D{D}cp{N}c{c}", B=B, H=H, S=S, D=D,
                                cp_size=N, causal=bool(c))
    if args.impl == "reference":
        run_reference(args, w)
    elif args.merge:
        run_merge(args)
    elif args.fp8:
        run_fp8(args, w)
    elif args.layer:
        run_layer(args, w)
    elif args.ring:
        run_ring(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
