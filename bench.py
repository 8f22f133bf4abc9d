"""Throughput benchmark of the attention hot path (forward + backward) on B200.

One step = one pass of the whole hot path over one batch of the workload
"fwdbwd_d128": B*N = 16384 tokens, H = 16 heads of dim 128, causal, bf16, with the
sequence length N = 16384 (B = 1) by default:
    fa_fwd -> fa_bwd_preprocess -> fa_bwd_kv -> fa_bwd_dq_convert
Throughput is attention TFLOPS: 4*B*H*N^2*d (halved under the causal mask) for the
forward plus 2.5x that for the backward, over the device time of the timed steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--N 16384]

Under torchrun (N > 1) every rank runs its own copy of the workload (independent
problems, no collective on the data path: weak scaling); the step time is the max over
ranks.  Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle on
a bounded sample instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "attention fwd/bwd TFLOPS on 1 B200 vs BF16 tensor-core peak (fraction of roofline)"
UNIT = "TFLOPS"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's published dense (no 2:4 sparsity) BF16 tensor-core figure for one B200, half of
# the sparse figure it quotes per 8-GPU system (the datasheet is not reachable offline).
NOMINAL_DENSE_BF16_TFLOPS = 2250.0
KERNELS_PER_STEP = 4  # fwd, bwd_pre, bwd_main, dq_convert
# A timed region at least this long is compared with the sustained (power-capped) peak.
SUSTAINED_REGION_MS = 1000.0


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    """(rank, world_size, local_rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar (the step time) over all ranks; identity on one rank."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ measurement helpers

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["no samples"]}
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id(dev) -> str:
    """nvidia-smi selector of the device torch calls `dev` (its UUID; robust to
    CUDA_VISIBLE_DEVICES renumbering)."""
    import torch
    props = torch.cuda.get_device_properties(dev)
    u = str(getattr(props, "uuid", ""))
    if u:
        return u if u.startswith("GPU-") else "GPU-" + u
    return str(dev.index or 0)


def kernel_source_hash() -> str:
    p = os.path.join(ROOT, "exact_io_aware_88_b200", "csrc", "bwd_sm100.cu")
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of `kernel` on `workload`,
    or None when there is none or the kernel source changed since it was captured."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    if not m or not h or h.group(1) != kernel_source_hash():
        return None
    return float(m.group(1))


# ------------------------------------------------------------------ the CUDA path

def run_ours(args, rank, world, local_rank):
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = init_dist(world, "nccl")
    from exact_io_aware_88_b200 import fa

    w = workload(args.N)
    t = synthetic.draw_workload(w, with_grad=True)
    B, N, H, d = w.B, w.N, w.H, w.d
    q, k, v, dO = (t[n].to(dev) for n in ("q", "k", "v", "dO"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa.fa_bwd_workspace_bytes(B, H, N, d)
    ws = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    sc = w.scale

    def check(rc, fn):
        if rc != 0:
            raise RuntimeError(f"{fn} failed: {fa.status_string(rc)}")

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        check(fa.fa_fwd(q, k, v, o, lse, B, H, N, d, w.causal, sc, stream), "fa_fwd")
        if ev is not None:
            ev[1].record(stream)
        check(fa.fa_bwd_preprocess(o, lse, dO, B, H, N, d, ws, ws_bytes, stream), "fa_bwd_preprocess")
        if ev is not None:
            ev[2].record(stream)
        check(fa.fa_bwd_kv(q, k, v, dO, dk, dv, B, H, N, d, w.causal, sc, ws, ws_bytes, stream),
              "fa_bwd_kv")
        if ev is not None:
            ev[3].record(stream)
        check(fa.fa_bwd_dq_convert(dq, B, H, N, d, sc, ws, ws_bytes, stream), "fa_bwd_dq_convert")
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    check(fa.fa_read_device_status(None, stream), "device status")
    check(fa.fa_read_device_status(ws, stream), "backward status")

    # ---- device-resident timed region: K steps, events around each kernel.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id(dev)) as clk:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for s in range(args.steps):
            step(evs[s])
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    total_ms = max_over_ranks(start.elapsed_time(end), world, dev)
    clocks = clk.summary()
    check(fa.fa_read_device_status(None, stream), "device status")
    check(fa.fa_read_device_status(ws, stream), "backward status")
    names = ["fwd", "bwd_pre", "bwd_main", "dq_convert"]
    per_step = {nm: [e[i].elapsed_time(e[i + 1]) for e in evs] for i, nm in enumerate(names)}
    per_kernel = {nm: statistics.mean(v) for nm, v in per_step.items()}
    step_ms = [e[0].elapsed_time(e[4]) for e in evs]

    # ---- end to end through the public API with host buffers (pinned), copies included.
    # Every step copies its inputs host -> device, runs fa_fwd and fa_bwd, and copies all
    # results device -> host.  Steps are double-buffered over three streams (uploads,
    # compute, downloads) so that step i's copies overlap step i-1's kernels and the two
    # copy directions overlap each other; the timed region runs from the first upload to
    # the last download.
    hin = [{n: t[n].pin_memory() for n in ("q", "k", "v", "dO")} for _ in range(2)]
    hout = [{"o": torch.empty_like(hin[0]["q"]).pin_memory(),
             "dq": torch.empty_like(hin[0]["q"]).pin_memory(),
             "dk": torch.empty_like(hin[0]["k"]).pin_memory(),
             "dv": torch.empty_like(hin[0]["v"]).pin_memory(),
             "lse": torch.empty((B, H, N), dtype=torch.float32).pin_memory()} for _ in range(2)]
    din = [{"q": q, "k": k, "v": v, "dO": dO},
           {n: torch.empty_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("dO", dO))}]
    dout = [{"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv},
            {"o": torch.empty_like(o), "lse": torch.empty_like(lse), "dq": torch.empty_like(dq),
             "dk": torch.empty_like(dk), "dv": torch.empty_like(dv)}]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        bi = i % 2
        x, y = din[bi], dout[bi]
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(comp_done[bi])  # step i-2 has finished reading these inputs
            for n in ("q", "k", "v", "dO"):
                x[n].copy_(hin[bi][n], non_blocking=True)
            up_done[bi].record(s_up)
        stream.wait_event(up_done[bi])
        if i >= 2:
            stream.wait_event(down_done[bi])  # step i-2's results have left these buffers
        check(fa.fa_fwd(x["q"], x["k"], x["v"], y["o"], y["lse"], B, H, N, d, w.causal, sc,
                        stream), "fa_fwd")
        check(fa.fa_bwd(x["q"], x["k"], x["v"], y["o"], y["lse"], x["dO"], y["dq"], y["dk"],
                        y["dv"], B, H, N, d, w.causal, sc, ws, ws_bytes, stream), "fa_bwd")
        comp_done[bi].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[bi])
            for n in ("o", "lse", "dq", "dk", "dv"):
                hout[bi][n].copy_(y[n], non_blocking=True)
            down_done[bi].record(s_down)

    # Up to 40 steps (about 0.25 s): the pipeline's fill and drain (one upload before the
    # first kernels, one download after the last) then weigh 2 stages in 42, not 2 in 12.
    e2e_steps = max(2, min(args.steps, 40))
    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for i in range(e2e_steps):
        e2e_step(i)
    s_down.wait_event(comp_done[(e2e_steps - 1) % 2])
    e1.record(s_down)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps
    h2d = sum(x.numel() * x.element_size() for x in hin[0].values())
    d2h = sum(x.numel() * x.element_size() for x in hout[0].values())
    check(fa.fa_read_device_status(None, stream), "device status")
    check(fa.fa_read_device_status(ws, stream), "backward status")
    del din[1], dout[1]

    ms_step = total_ms / args.steps
    flops = w.fwd_flops() + w.bwd_flops()
    value = world * flops / (ms_step * 1e-3) / 1e12
    peaks, peak_src = measured_peaks()
    peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # The burst peak (a best-of-10 matmul) is the denominator for a timed region shorter than
    # a second; the sustained one (matmuls back to back for seconds, under the power cap) for
    # a longer one, whose clocks have settled.
    long_region = total_ms >= SUSTAINED_REGION_MS
    peak = peak_sus if long_region else peak_burst
    peak_kind = (f"{peak_src} bf16 {'sustained' if long_region else 'burst'} "
                 f"(timed region {total_ms:.0f} ms {'>=' if long_region else '<'} "
                 f"{SUSTAINED_REGION_MS:.0f} ms)")
    main_tflops = w.bwd_flops() / (per_kernel["bwd_main"] * 1e-3) / 1e12
    fwd_tflops = w.fwd_flops() / (per_kernel["fwd"] * 1e-3) / 1e12
    wl = f"fwdbwd_d128_N{N}"
    traffic = profiled_traffic("bwd_main", wl)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, t)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": config_of(w, world),
            "breakdown": breakdown(per_step, step_ms, w, peak_burst),
            "roofline": {"kernel": "bwd_main (fa_bwd_kv)", "bound": "tensor",
                         "achieved": round(main_tflops, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(main_tflops / peak, 4), "peak_kind": peak_kind,
                         "frac_of_burst_peak": round(main_tflops / peak_burst, 4),
                         "frac_of_sustained_peak": round(main_tflops / peak_sus, 4),
                         "frac_of_nominal_dense_bf16": round(main_tflops / NOMINAL_DENSE_BF16_TFLOPS, 4),
                         "traffic": traffic},
            "clocks": clock_record(clocks, ms_step),
            "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 3)},
            "gpu_launches": KERNELS_PER_STEP * args.steps,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _stats(v):
    return {"mean": statistics.mean(v), "median": statistics.median(v), "best": min(v)}


def breakdown(per_step, step_ms, w, peak_burst):
    """Per-kernel device times of the timed steps (mean, median, best of the K steps) and
    the forward / backward TFLOPS they imply, as fractions of the burst and nominal peaks."""
    out = {}
    for nm, v in per_step.items():
        st = _stats(v)
        out[f"{nm}_ms"] = round(st["mean"], 4)
        out[f"{nm}_ms_median"] = round(st["median"], 4)
        out[f"{nm}_ms_best"] = round(st["best"], 4)
    st = _stats(step_ms)
    out["step_ms_median"] = round(st["median"], 4)
    out["step_ms_best"] = round(st["best"], 4)
    fwd_med = w.fwd_flops() / (statistics.median(per_step["fwd"]) * 1e-3) / 1e12
    bwd_steps = [a + b + c for a, b, c in zip(per_step["bwd_pre"], per_step["bwd_main"],
                                               per_step["dq_convert"])]
    bwd_med = w.bwd_flops() / (statistics.median(bwd_steps) * 1e-3) / 1e12
    main_med = w.bwd_flops() / (statistics.median(per_step["bwd_main"]) * 1e-3) / 1e12
    out["fwd_tflops"] = round(w.fwd_flops() / (statistics.mean(per_step["fwd"]) * 1e-3) / 1e12, 1)
    out["bwd_main_tflops"] = round(w.bwd_flops() / (statistics.mean(per_step["bwd_main"]) * 1e-3) / 1e12, 1)
    out["fwd_tflops_median"] = round(fwd_med, 1)
    out["bwd_tflops_median"] = round(bwd_med, 1)
    out["bwd_main_tflops_median"] = round(main_med, 1)
    out["fwd_frac_of_burst_peak"] = round(fwd_med / peak_burst, 4)
    out["bwd_frac_of_burst_peak"] = round(bwd_med / peak_burst, 4)
    out["fwd_frac_of_nominal_dense_bf16"] = round(fwd_med / NOMINAL_DENSE_BF16_TFLOPS, 4)
    out["bwd_frac_of_nominal_dense_bf16"] = round(bwd_med / NOMINAL_DENSE_BF16_TFLOPS, 4)
    return out


def clock_record(clocks, ms_step):
    """The sampled clock summary plus step time x median SM clock (MHz * ms = kilocycles),
    which stays comparable across runs whose clocks differ."""
    c = dict(clocks)
    if c.get("sm_mhz"):
        c["step_kcycles_at_median_clock"] = round(ms_step * c["sm_mhz"], 1)
    return c


def workload(N: int):
    if N == 65536:
        return synthetic.long_context()
    return synthetic.fwdbwd(N)


def config_of(w, world: int) -> dict:
    """The JSON line's `config` for workload `w` on `world` ranks; both arms print it."""
    nbytes = 5 * w.B * w.N * w.H * w.d * 2  # q, k, v, o, dO in bf16
    return {"workload": f"{w.name}: B={w.B} N={w.N} H={w.H} d={w.d} causal bf16, "
                        f"q/k/v/dO ~ N(0,1) seed {w.seed}",
            "B": w.B, "N": w.N, "H": w.H, "d": w.d, "causal": True,
            "tokens_per_gpu": w.B * w.N,
            "parallelism": f"replicas x{world} (independent problems per GPU)",
            "l2": "no flush: inputs (q,k,v,o,dO = %d MiB) exceed the 126 MB L2" % (nbytes // 2 ** 20)}


# ------------------------------------------------------------------ the oracle on the host

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo; "unknown" elsewhere)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(t, w, b: int, h: int, n_rows: int):
    """fwd + bwd of one head of the workload, truncated to its first n_rows positions.
    Under the causal mask that prefix is itself an exact attention problem.  Returns
    (seconds, algorithmic FLOPs of the sample)."""
    import oracle
    Q, K, V, dO = (synthetic.to_f64(t[n][b, :n_rows, h]) for n in ("q", "k", "v", "dO"))
    t0 = time.perf_counter()
    oracle.forward_head(Q, K, V, w.scale, True)
    oracle.backward_head(Q, K, V, dO, w.scale, True)
    dt = time.perf_counter() - t0
    flops = 3.5 * 4.0 * n_rows * n_rows * w.d / 2
    return dt, flops


def cpu_baseline(w, t):
    n_rows = min(w.N, 16384)
    dt, flops = oracle_sample(t, w, 0, 0, n_rows)
    return {"value": round(flops / dt / 1e12, 5), "unit": UNIT, "cores": blas_threads(),
            "cpu_count": os.cpu_count(), "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"head (b=0,h=0) of the workload, first {n_rows} positions, fwd+bwd "
                      f"(fp64 numpy, S and P materialised); {dt:.1f} s",
            # Every head costs the same, and a causal prefix of n rows costs ~n^2.
            "full_workload_s_extrapolated": round(dt * w.B * w.H * (w.N / n_rows) ** 2, 1)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = workload(args.N)
    t = synthetic.draw(w.B, w.N, w.H, w.d, w.seed, "bf16", with_grad=True)
    n_rows = 4096
    for s in range(args.warmup):
        oracle_sample(t, w, 0, s % w.H, n_rows)
    secs, fl = 0.0, 0.0
    for s in range(args.steps):
        dt, f = oracle_sample(t, w, 0, s % w.H, n_rows)
        secs += dt
        fl += f
    value = fl / secs / 1e12
    cores = blas_threads()
    sample = (f"per step: one head of the workload truncated to its first {n_rows} positions "
              "(an exact causal sub-problem), fwd+bwd, fp64 numpy oracle")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * secs / args.steps, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, world),
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores,
                             "cpu_count": os.cpu_count(), "cpu_model": cpu_model(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_sweep(path: str, reps: int = 20, warmup: int = 3):
    """Times every workload of the benchmark sweep (forward-only configs: fa_fwd; forward +
    backward configs: fa_fwd, fa_bwd and fa_bwd_deterministic; decoding: fa_fwd_splitkv;
    block-sparse masks against the dense forward; the FP8 forward and its operand
    preparation) and writes one JSON line per workload to `path`.  Median of `reps`
    CUDA-event timed launches after `warmup`."""
    import numpy as np
    import torch
    from exact_io_aware_88_b200 import fa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = measured_peaks()
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts), min(ts)

    with open(path, "w") as out:
        for w in synthetic.all_workloads():
            t = synthetic.draw_workload(w, with_grad=w.backward)
            B, N, H, d = w.B, w.N, w.H, w.d
            q, k, v = (t[n].to(dev) for n in ("q", "k", "v"))
            o = torch.empty_like(q)
            lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
            f = fa.fa_fwd_f32 if w.dtype == "f32" else fa.fa_fwd
            fwd = lambda: f(q, k, v, o, lse, B, H, N, d, w.causal, w.scale, stream)
            assert fwd() == 0
            med, best = timed(fwd)
            elem = 4 if w.dtype == "f32" else 2
            # Roofline time: the slower of the tensor-core time at the burst peak and the
            # HBM time of the algorithmic bytes (read Q, K, V, write O and the LSE).
            hbm_floor = (4 * B * N * H * d * elem + 4 * B * H * N) / (hbm * 1e9) * 1e3  # ms
            roof = max(w.fwd_flops() / (burst * 1e12) * 1e3, hbm_floor)
            rec = {"workload": w.label(), "pass": "fwd", "ms": round(med, 4), "ms_best": round(best, 4),
                   "tflops": round(w.fwd_flops() / (med * 1e-3) / 1e12, 1),
                   "frac_of_burst_peak": round(w.fwd_flops() / (med * 1e-3) / 1e12 / burst, 4),
                   "hbm_floor_ms": round(hbm_floor, 4), "roofline_ms": round(roof, 4),
                   "frac_of_roofline": round(roof / med, 4), "peak_source": peak_src}
            out.write(json.dumps(rec) + "\n")
            print(json.dumps(rec), file=sys.stderr)
            if w.backward:
                dO = t["dO"].to(dev)
                dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
                nb = fa.fa_bwd_workspace_bytes(B, H, N, d)
                ws = torch.empty(nb, device=dev, dtype=torch.uint8)
                bwd = lambda: fa.fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, w.causal,
                                        w.scale, ws, nb, stream)
                assert bwd() == 0
                med, best = timed(bwd)
                # Algorithmic bytes: read Q, K, V, O, dO and the LSE, write dQ, dK, dV.
                bwd_floor = (8 * B * N * H * d * elem + 4 * B * H * N) / (hbm * 1e9) * 1e3
                roof = max(w.bwd_flops() / (burst * 1e12) * 1e3, bwd_floor)
                rec = {"workload": w.label(), "pass": "bwd", "ms": round(med, 4),
                       "ms_best": round(best, 4),
                       "tflops": round(w.bwd_flops() / (med * 1e-3) / 1e12, 1),
                       "frac_of_burst_peak": round(w.bwd_flops() / (med * 1e-3) / 1e12 / burst, 4),
                       "hbm_floor_ms": round(bwd_floor, 4), "roofline_ms": round(roof, 4),
                       "frac_of_roofline": round(roof / med, 4), "peak_source": peak_src}
                out.write(json.dumps(rec) + "\n")
                print(json.dumps(rec), file=sys.stderr)
                det = lambda: fa.fa_bwd_deterministic(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d,
                                                      w.causal, w.scale, ws, nb, stream)
                assert det() == 0
                med, best = timed(det)
                if fa.fa_read_device_status(ws, stream) != 0:
                    raise RuntimeError("backward status word reports a failure")
                rec = {"workload": w.label(), "pass": "bwd_deterministic", "ms": round(med, 4),
                       "ms_best": round(best, 4),
                       "tflops": round(w.bwd_flops() / (med * 1e-3) / 1e12, 1),
                       "frac_of_burst_peak": round(w.bwd_flops() / (med * 1e-3) / 1e12 / burst, 4),
                       "peak_source": peak_src,
                       "note": "FLOPs counted as 2.5x forward; the kernels do 3.5x (dQ recomputes S, dP)"}
                out.write(json.dumps(rec) + "\n")
                print(json.dumps(rec), file=sys.stderr)
                del dO, dq, dk, dv, ws
            del q, k, v, o, lse, t
            torch.cuda.empty_cache()
        # Decoding (split-KV): HBM-bound, reported against the measured copy bandwidth.
        for name, B, Nq, Nk, H, d, seed in synthetic.decode_workloads():
            t = synthetic.draw_decode(B, Nq, Nk, H, d, seed, "bf16")
            q, k, v = (t[n].to(dev) for n in ("q", "k", "v"))
            o = torch.empty_like(q)
            lse = torch.empty((B, H, Nq), device=dev, dtype=torch.float32)
            nb = fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d)
            ws = torch.empty(nb, device=dev, dtype=torch.uint8)
            dec = lambda: fa.fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, 1, 1.0 / math.sqrt(d),
                                            fa.FA_DTYPE_BF16, ws, nb, stream)
            assert dec() == 0
            med, best = timed(dec)
            kv_bytes = 2 * B * Nk * H * d * 2
            rec = {"workload": f"{name}:B{B}xNq{Nq}xNk{Nk}xH{H}xd{d}-causal-bf16", "pass": "fwd_splitkv",
                   "ms": round(med, 4), "ms_best": round(best, 4),
                   "kv_gbs": round(kv_bytes / (med * 1e-3) / 1e9, 1),
                   "frac_of_hbm": round(kv_bytes / (med * 1e-3) / 1e9 / hbm, 4), "peak_source": peak_src}
            out.write(json.dumps(rec) + "\n")
            print(json.dumps(rec), file=sys.stderr)
            del q, k, v, o, lse, ws, t
            torch.cuda.empty_cache()
        # Block-sparse forward: random block masks at several densities (diagonal blocks
        # always kept), timed against the dense forward of the same problem.
        B, N, H, d = 1, 16384, 16, 128
        t = synthetic.draw(B, N, H, d, 1002, "bf16")
        q, k, v = (t[n].to(dev) for n in ("q", "k", "v"))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
        nt = N // 128
        nb = fa.fa_fwd_block_sparse_workspace_bytes(B, H, N, d)
        ws = torch.empty(nb, device=dev, dtype=torch.uint8)
        rng = np.random.default_rng(7)
        for causal in (False, True):
            dense = lambda: fa.fa_fwd(q, k, v, o, lse, B, H, N, d, causal, 1.0 / math.sqrt(d), stream)
            assert dense() == 0
            dmed, _ = timed(dense)
            # Random masks at four densities, then a structured one: a band of 8 key tiles
            # ending at the diagonal plus the first key tile (local + global attention).
            band = np.zeros((nt, nt), np.uint8)
            for i in range(nt):
                band[i, max(0, i - 7):i + 1] = 1
                band[i, 0] = 1
            for dens in (1.0, 0.5, 0.25, 0.1, "band8+global"):
                if isinstance(dens, str):
                    m = band.copy()
                else:
                    m = (rng.random((nt, nt)) < dens).astype(np.uint8)
                    np.fill_diagonal(m, 1)
                if causal:
                    m = np.tril(m)
                mask = torch.from_numpy(m).to(dev)
                act = int(m.sum())
                tot = nt * (nt + 1) // 2 if causal else nt * nt
                bs = lambda: fa.fa_fwd_block_sparse(q, k, v, o, lse, B, H, N, d, causal,
                                                    1.0 / math.sqrt(d), mask, ws, nb, stream)
                assert bs() == 0
                med, best = timed(bs)
                flops = 4.0 * B * H * 128 * 128 * d * act  # active blocks, counted whole
                kind = dens if isinstance(dens, str) else "random"
                rec = {"workload": f"block_sparse:B{B}xN{N}xH{H}xd{d}" + ("-causal" if causal else "")
                       + f"-{kind}-density{act / tot:.2f}-bf16", "pass": "fwd_block_sparse",
                       "ms": round(med, 4), "ms_best": round(best, 4),
                       "tflops_active_blocks": round(flops / (med * 1e-3) / 1e12, 1),
                       "dense_fa_fwd_ms": round(dmed, 4), "speedup_vs_dense": round(dmed / med, 3),
                       "peak_source": peak_src}
                out.write(json.dumps(rec) + "\n")
                print(json.dumps(rec), file=sys.stderr)
        del q, k, v, o, lse, ws, t
        torch.cuda.empty_cache()
        # FP8 forward (E4M3 products, Hadamard-transformed Q and K): tensor-bound against the
        # bf16 measured peak x 2 (the nominal fp8 / bf16 ratio); the operand preparation
        # (fa_fp8_quantize) is timed separately and is HBM-bound.
        for name, B, N, H, d, causal, seed in synthetic.fp8_workloads():
            t = synthetic.draw(B, N, H, d, seed, "bf16")
            q, k, v = (t[n].to(dev) for n in ("q", "k", "v"))
            signs = synthetic.draw_signs(d, seed + 1).to(dev)
            npad = (N + 15) // 16 * 16
            q8 = torch.empty((B, N, H, d), device=dev, dtype=torch.uint8)
            k8 = torch.empty_like(q8)
            vt8 = torch.empty((B, H, d, npad), device=dev, dtype=torch.uint8)
            sc = torch.empty((3, B * H), device=dev, dtype=torch.float32)
            nb = fa.fa_fp8_quantize_workspace_bytes(B, H)
            ws = torch.empty(nb, device=dev, dtype=torch.uint8)
            quant = lambda: fa.fa_fp8_quantize(q, k, v, signs, q8, k8, vt8, sc, B, H, N, d, ws, nb,
                                               stream)
            assert quant() == 0
            qmed, qbest = timed(quant)
            o = torch.empty_like(q)
            lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
            f8 = lambda: fa.fa_fwd_fp8(q8, k8, vt8, sc, o, lse, B, H, N, d, causal,
                                       1.0 / math.sqrt(d), stream)
            assert f8() == 0
            med, best = timed(f8)
            flops = 4.0 * B * H * N * N * d * (0.5 if causal else 1.0)
            rec = {"workload": name + "-e4m3", "pass": "fwd_fp8", "ms": round(med, 4),
                   "ms_best": round(best, 4), "tflops": round(flops / (med * 1e-3) / 1e12, 1),
                   "frac_of_fp8_peak": round(flops / (med * 1e-3) / 1e12 / (2 * burst), 4),
                   "quantize_ms": round(qmed, 4),
                   "quantize_gbs": round(3 * B * N * H * d * (2 + 2 + 1) / (qmed * 1e-3) / 1e9, 1),
                   "peak_source": peak_src + " (fp8 peak = 2 x measured bf16 burst)"}
            out.write(json.dumps(rec) + "\n")
            print(json.dumps(rec), file=sys.stderr)
            del q, k, v, q8, k8, vt8, sc, ws, o, lse, t
            torch.cuda.empty_cache()
    if fa.fa_read_device_status(None, stream) != 0:
        raise RuntimeError("device status word reports a timeout")


KERNEL_CASES = ("fwd_d64_N4096", "fwd_fp8_N4096", "fwd_d128_N4096_causal", "bwd_N4096",
                "bwd_N16384", "bwd_det_N4096", "fp8_quant_N4096", "decode_k16384",
                "block_sparse_N16384_d50")


def run_kernel_case(name: str, launches: int = 4):
    """A few launches of one kernel on one workload, for a profiler to capture (every case
    holds well under 1 GB on the device, and its inputs exceed the 126 MB L2):
      fwd_d64_N4096          the head-dim 64 forward (B=4, N=4096, H=32, non-causal);
      fwd_fp8_N4096          the E4M3 forward (B=4, N=4096, H=16, d=128, non-causal, after
                             one fa_fp8_quantize);
      fwd_d128_N4096_causal  the head-dim 128 causal forward (B=4, N=4096, H=16);
      bwd_N4096              one forward, then `launches` backward passes (fa_bwd: its
                             three kernels) on the fwd+bwd workload at N=4096 (B=4, H=16,
                             d=128, causal);
      bwd_N16384             the same on the bench's workload (B=1, N=16384; ~0.7 GB held);
      bwd_det_N4096          the deterministic backward (its key-tile kernel without dQ, then
                             the per-query-tile dQ kernel) on the N=4096 fwd+bwd workload;
      fp8_quant_N4096        fa_fp8_quantize (amax, Q/K quantisation with the Hadamard
                             transform, V^T) on B=4, N=4096, H=16, d=128;
      decode_k16384          split-KV decoding, B=8, Nq=1, Nk=16384, H=16, d=128, causal;
      block_sparse_N16384_d50  the block-sparse forward, B=1, N=16384, H=16, d=128, non-causal,
                             a random mask of density 0.5 (diagonal kept).
    Prints one line; nothing is timed."""
    import torch
    from exact_io_aware_88_b200 import fa
    if name == "fwd_d128_N4096_causal":
        w = synthetic.fwd_sweep(128, 4096, True)
        t = synthetic.draw_workload(w)
        q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
        for _ in range(launches):
            fa.attention_forward(q, k, v, causal=True)
    elif name in ("bwd_N4096", "bwd_N16384", "bwd_det_N4096"):
        w = synthetic.fwdbwd(16384 if name == "bwd_N16384" else 4096)
        t = synthetic.draw_workload(w, with_grad=True)
        q, k, v, dO = (t[n].cuda() for n in ("q", "k", "v", "dO"))
        o, lse = fa.attention_forward(q, k, v, causal=True)
        ws = torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.H, w.N, w.d), device="cuda",
                         dtype=torch.uint8)
        for _ in range(launches):
            fa.attention_backward(q, k, v, o, lse, dO, causal=True, workspace=ws,
                                  deterministic=name == "bwd_det_N4096")
        if fa.fa_read_device_status(ws) != 0:
            raise RuntimeError("backward status word reports a failure")
    elif name == "decode_k16384":
        wl = [x for x in synthetic.decode_workloads() if x[0] == "decode_q1_k16384"][0]
        _, B, Nq, Nk, H, d, seed = wl
        t = synthetic.draw_decode(B, Nq, Nk, H, d, seed, "bf16")
        q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
        for _ in range(launches):
            fa.attention_decode(q, k, v, causal=True)
    elif name == "block_sparse_N16384_d50":
        B, N, H, d = 1, 16384, 16, 128
        t = synthetic.draw(B, N, H, d, 1002, "bf16")
        q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
        nt = N // 128
        m = (torch.rand((nt, nt), generator=torch.Generator().manual_seed(77)) < 0.5).to(torch.uint8)
        m.fill_diagonal_(1)
        mask = m.cuda()
        for _ in range(launches):
            fa.attention_block_sparse(q, k, v, mask, causal=False)
    elif name == "fwd_d64_N4096":
        w = synthetic.fwd_sweep(64, 4096, False)
        t = synthetic.draw_workload(w)
        q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
        for _ in range(launches):
            fa.attention_forward(q, k, v, causal=False)
    elif name == "fp8_quant_N4096":
        B, N, H, d = 4, 4096, 16, 128
        t = synthetic.draw(B, N, H, d, 1006, "bf16")
        q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
        signs = synthetic.draw_signs(d, 1007).cuda()
        for _ in range(launches):
            fa.fp8_quantize(q, k, v, signs)
    elif name == "fwd_fp8_N4096":
        B, N, H, d = 4, 4096, 16, 128
        t = synthetic.draw(B, N, H, d, 1006, "bf16")
        q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
        q8, k8, vt8, sc = fa.fp8_quantize(q, k, v, synthetic.draw_signs(d, 1007).cuda())
        for _ in range(launches):
            fa.attention_forward_fp8(q8, k8, vt8, sc, causal=False)
    else:
        raise ValueError(f"unknown kernel case {name}")
    torch.cuda.synchronize()
    if fa.fa_read_device_status() != 0:
        raise RuntimeError("device status word reports a timeout")
    print(json.dumps({"kernel_case": name, "launches": launches}))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=250)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--N", type=int, default=16384, choices=[1024, 2048, 4096, 8192, 16384, 65536])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-case", choices=KERNEL_CASES, default=None,
                    help="run a few launches of one kernel (for a profiler) and exit")
    ap.add_argument("--sweep", metavar="PATH", default=None,
                    help="time every workload of the benchmark sweep into PATH (JSON lines) "
                         "instead of the single-step measurement")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.kernel_case:
        run_kernel_case(args.kernel_case)
        return 0
    if args.sweep:
        run_sweep(args.sweep)
        return
    rank, world, local_rank = dist_env()
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus={args.gpus}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
