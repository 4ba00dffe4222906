"""Benchmark of the HLA hot path: permute_rope -> hla_forward (+ split combine) -> unpermute
(folded into the attention epilogue unless --unfused).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 4k|8k|1k|ragged]
                    [--impl ultragen|reference]

One step is one pass of the whole path over one layer of synthetic Q/K/V (resident in HBM).
The metric is useful TFLOP/s: 4 * head_dim FLOPs per visible (query, key) pair per head
(masked pairs and padding count for nothing), whole job over all ranks; ms per step and per
kernel are reported beside it.  Multi-GPU runs are weak scaling: every rank runs its own
independent layer (no collective on the data path); timing is the max over ranks.

--impl reference times the fp64 CPU oracle (the plain restatement the tests check against) on
a bounded row sample of the same workload, on rank 0 only.

--op warm_start measures the warm-start initialisation instead (one launch per step over a
synthetic 16-channel latent, --workload warm_8k by default): HBM GB/s of its algorithmic
bytes (noise read unless --drawn-noise, output written, low-resolution latent read), with L2
flushed between launches.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/layer and useful TFLOP/s of masked HLA at 4K/8K; % of B200 BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "hla_fwd_traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None,
                    help="4k (default), 8k, 1k, ragged; warm_8k (default for --op warm_start), warm_4k")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the workload's head count (smaller profiling captures)")
    ap.add_argument("--lr-radius", type=int, default=-1,
                    help="HR->LR scope: -1 all LR tokens (default); r >= 0 the window's anchors grown by r")
    ap.add_argument("--lr-order", type=int, default=-1, choices=[-1, 0, 1],
                    help="LR segment order with an LR-region scope: -1 automatic (default), 0 raster, 1 8x16 blocks")
    ap.add_argument("--halo", type=int, default=-1, choices=[-1, 0, 1, 2],
                    help="compact halo blocks in the K/V layout: -1 automatic (default), 0 off, "
                         "1 copied by the permute, 2 gathered by the attention")
    ap.add_argument("--qk", default="bf16", choices=["bf16", "e4m3"],
                    help="storage of the permuted Q and K: bf16 (default) or scaled e4m3 with 8-bit Q K^T")
    ap.add_argument("--q-exp", type=int, default=0, help="e4m3 Q stores x * 2^-q_exp")
    ap.add_argument("--k-exp", type=int, default=0, help="e4m3 K stores x * 2^-k_exp")
    ap.add_argument("--impl", default="ultragen", choices=["ultragen", "reference"])
    ap.add_argument("--unfused", action="store_true",
                    help="run unpermute as its own pass instead of in the attention epilogue")
    ap.add_argument("--op", default="hla", choices=["hla", "warm_start"])
    ap.add_argument("--drawn-noise", action="store_true",
                    help="warm_start: draw X_T in the kernel instead of reading a noise buffer")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-heads-per-chunk", type=int, default=2,
                    help="head slice per pipelined unit of the host-buffer (e2e) measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", default="layers", choices=["layers", "heads"],
                    help="multi-GPU: layers = an independent layer per rank (weak scaling); heads = "
                         "one layer's heads split across the ranks (strong scaling)")
    ap.add_argument("--extra-workloads", default=None,
                    help="comma list of further workloads timed after the main one and reported "
                         "under 'workloads' (default: 8k,1k,ragged for the default 4k run; "
                         "'none' to skip)")
    args = ap.parse_args()
    default_run = args.workload is None
    if args.workload is None:
        args.workload = "warm_8k" if args.op == "warm_start" else "4k"
    if args.extra_workloads is None:
        args.extra_workloads = "8k,1k,ragged" if default_run and args.op == "hla" else "none"
    return args


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """SM clock, power and throttle reasons of this process's GPU during the timed region.

    NVML (the device found by the CUDA device's UUID, so the reading is of the GPU the
    kernels run on) is polled every ~5 ms from a thread between start() and stop(); without
    NVML, nvidia-smi is polled every 20 ms.  start() is called right before the timed steps are
    enqueued and stop() right after the closing synchronize, so the samples cover the steps."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []               # (sm_mhz, power_w, reasons)
        self.smax = None
        self.stop_evt = threading.Event()
        self.thread = None
        self.proc = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.index).uuid)
        for cand in (uuid, "GPU-" + uuid):
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID(cand)
            except Exception:
                pass
        raise RuntimeError("no NVML device with the CUDA device's UUID")

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            masks = [(name, getattr(nv, attr)) for name, attr in self.REASONS]

            def poll():
                while not self.stop_evt.is_set():
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, pw, {n for n, m in masks if bits & m}))
                    except Exception:
                        pass
                    time.sleep(0.005)

            self.source = "nvml"
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for ln in self.proc.stdout:
            parts = [x.strip() for x in ln.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, self.smax, pw = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            self.samples.append((sm, pw, {n for n, v in zip(names, parts[5:9])
                                          if v.lower() in ("active", "1", "0x1")}))

    def stop(self):
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.stop_evt.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm = [x[0] for x in self.samples]
        pw = [x[1] for x in self.samples]
        reasons = set().union(*(x[2] for x in self.samples)) if self.samples else set()
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
                "sm_mhz_min": min(sm) if sm else None, "power_w_max": max(pw) if pw else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


# throttle reasons that void a timed region (sw_power_cap is kept: a 1 kW part hits it under
# dense tensor work)
SLOWDOWN_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over all ranks (the job is as slow as its slowest rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job useful TFLOP/s: every rank runs its own layer (weak scaling)."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("hla_fwd.cu", "ptx.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "diffusion_transformer_ultra_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per hla_forward launch from the committed ncu summary, only while the kernel
    source still matches the one the counters were taken on."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as f:
        d = json.load(f)
    ent = d.get(workload)
    if not ent or ent.get("kernel_sha") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


def cpu_model() -> str:
    """The host CPU's model name, from /proc/cpuinfo (empty when unavailable)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


def blas_threads():
    """Threads of the BLAS libraries NumPy uses, as threadpoolctl reports them."""
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads") or 0 for i in threadpool_info()
                    if i.get("user_api") == "blas"), default=None)
    except Exception:
        return None


def inputs_sha256(*tensors) -> str:
    """SHA-256 of the input tensors' bytes, in order (the exact bf16 values timed)."""
    h = hashlib.sha256()
    for t in tensors:
        h.update(t.contiguous().view(-1).view(__import__("torch").uint8).numpy().tobytes())
    return h.hexdigest()


def cpu_baseline(wl, q, k, v, budget_s: float = 12.0, lr_radius: int = -1, lr_block: bool = False,
                 one_core: bool = True, **fwd):
    """The oracle as it stands, timed on this host on a bounded sample: one head, rows of one
    interior window plus text and LR rows, repeated until about `budget_s` of CPU work, with
    the BLAS libraries on all cores and (one_core) again on one core.  The dense oracle costs
    the same per query row whatever its segment (every row is scored against all N_tot keys),
    so the time per sampled row, times the layer's rows, heads and batch, extrapolates to the
    whole layer (``fwd``: the oracle forward's Q/K format options)."""
    import numpy as np

    from oracle import hla_oracle as O
    g = O.Geometry(wl.H, wl.W, wl.l, wl.b, wl.rho, wl.T, lr_radius, lr_block=lr_block)
    l2 = g.l * g.l
    win = (g.nWh // 2) * g.nWw + g.nWw // 2
    rows = list(range(g.off_hr + win * l2, g.off_hr + (win + 1) * l2))
    rows += list(range(0, min(g.T, 8)))
    if g.N_lr:
        rows += list(np.linspace(g.off_lr, g.off_lr + g.N_lr - 1, 32).astype(int))
    rows = np.array(sorted(set(rows)), np.int64)
    vis_pairs = int(O.visible_rows(g, rows).sum())
    qh, kh, vh = (x[:1, :, :1, :].to(dtype=__import__("torch").float64).numpy() for x in (q, k, v))

    def timed(budget):
        t0 = time.perf_counter()
        reps = 0
        while True:
            O.forward(qh, kh, vh, g, wl.axes, rows=rows, **fwd)
            reps += 1
            if time.perf_counter() - t0 > budget:
                break
        return (time.perf_counter() - t0) / reps, reps

    dt, reps = timed(budget_s)
    threads = blas_threads()
    flops = 4.0 * wl.D * vis_pairs
    real_rows = wl.n_raster                         # every real token is one query row
    full_s = dt / len(rows) * real_rows * wl.heads * wl.batch
    out = {"value": flops / dt / 1e12, "unit": "useful TFLOP/s", "cores": os.cpu_count(),
           "blas_threads": threads, "cpu_model": cpu_model(), "kind": "oracle",
           "sample": f"1 head, {len(rows)} query rows ({vis_pairs} visible pairs), full RoPE + "
                     f"explicit mask, fp64 NumPy; {reps} rep(s), {dt:.2f} s each",
           "full_layer_s_extrapolated": full_s,
           "full_layer_note": f"extrapolated: {dt / len(rows) * 1e3:.2f} ms per sampled query row x "
                              f"{real_rows} rows x {wl.heads} heads x batch {wl.batch}"}
    if one_core:
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                dt1, reps1 = timed(budget_s / 2)
            out["one_core"] = {"value": flops / dt1 / 1e12, "unit": "useful TFLOP/s",
                               "blas_threads": 1, "s_per_rep": dt1, "reps": reps1,
                               "full_layer_s_extrapolated": dt1 / len(rows) * real_rows * wl.heads * wl.batch}
        except Exception as e:            # threadpoolctl missing: say so instead of guessing
            out["one_core"] = {"unavailable": str(e)}
    return out


def run_reference(args, rank, world):
    import torch
    if rank != 0:
        return
    import diffusion_transformer_ultra_b200 as ug
    wl = ug.WORKLOADS[args.workload]
    q, k, v = ug.make_qkv(wl)
    per_step = []
    base = None
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        r = cpu_baseline(wl, q, k, v, budget_s=0.0, one_core=False)
        if i >= args.warmup:
            per_step.append(time.perf_counter() - t0)
            base = r
    value = base["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "useful TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(per_step), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "H": wl.H, "W": wl.W, "l": wl.l, "b": wl.b, "rho": wl.rho,
                   "text_len": wl.T, "heads": wl.heads, "head_dim": wl.D, "batch": wl.batch},
        "cpu_baseline": {"kind": "oracle", "cores": base["cores"], "cpu_model": base["cpu_model"],
                         "blas_threads": base["blas_threads"], "sample": base["sample"],
                         "full_layer_s_extrapolated": base["full_layer_s_extrapolated"],
                         "value": value, "unit": "useful TFLOP/s"},
        "e2e": {"value": value, "unit": "useful TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


WARM_METRIC = "warm-start initialisation: HBM GB/s of algorithmic bytes"


def warm_bytes(wl, drawn: bool) -> int:
    n_hr = wl.batch * wl.C * wl.H * wl.W
    return 4 * n_hr * (1 if drawn else 2) + 4 * wl.batch * wl.C * wl.h * wl.w


def warm_cpu_baseline(wl, x_lr, noise, budget_s: float = 10.0):
    """The warm-start oracle on this host: whole planes, growing until about budget_s."""
    from oracle import warm_start_oracle as WO
    t0 = time.perf_counter()
    planes = 0
    while True:
        c = planes % wl.C
        WO.warm_start(x_lr[:1, c:c + 1].double().numpy(), wl.H, wl.W, wl.alpha, wl.sharpen,
                      noise=noise[:1, c:c + 1].double().numpy())
        planes += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    one = warm_bytes(type(wl)(wl.name, wl.cfg, 1, 1, wl.h, wl.w, wl.H, wl.W, wl.alpha, wl.sharpen),
                     False)
    return {"value": one * planes / dt / 1e9, "unit": "GB/s", "cores": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{planes} plane(s) of {wl.H}x{wl.W} (noise given), fp64 NumPy, "
                      f"{dt / planes:.2f} s each"}


def main_warm(args, rank, world, local):
    import torch
    import torch.distributed as dist

    import diffusion_transformer_ultra_b200 as ug
    wl = ug.WARM_WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank != 0:
            return
        x_lr, noise = ug.make_warm(wl)
        per = []
        for i in range(args.warmup + args.steps):
            r = warm_cpu_baseline(wl, x_lr, noise, budget_s=0.0)
            if i >= args.warmup:
                per.append(r)
        value = statistics.mean(r["value"] for r in per)
        print(json.dumps({
            "impl": "reference", "metric": WARM_METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * warm_bytes(wl, False) / (value * 1e9),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl.name},
            "cpu_baseline": {"kind": "oracle", "cores": per[-1]["cores"], "sample": per[-1]["sample"],
                             "value": value, "unit": "GB/s"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }), flush=True)
        return
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    x_lr, noise = ug.make_warm(wl)
    xd, nd = x_lr.cuda(), (None if args.drawn_noise else noise.cuda())
    out = torch.empty((wl.batch, wl.C, wl.H, wl.W), device="cuda")
    # L2 flush between launches: writing 256 MB evicts everything, and reading another 256 MB
    # then replaces those dirty lines with clean ones, so their write-back to HBM happens here
    # and not inside the next timed launch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.zeros(64 << 20, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        ug.warm_start(xd, out, wl.alpha, wl.sharpen, noise=nd, seed=1234, offset=0)
        return 1

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    launches = 0
    for i in range(args.steps):
        flush.zero_()
        flush_rd.sum()
        evs[i][0].record(stream)
        launches += step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    ms = max_over_ranks(ms, world, "cuda")
    nbytes = warm_bytes(wl, args.drawn_noise)
    value = nbytes * world / (ms * 1e-3) / 1e9
    pk, src = peaks()

    e2e = None
    if not args.no_e2e:
        xh = x_lr.pin_memory()
        nh = noise.pin_memory()
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        nd2 = torch.empty_like(out) if not args.drawn_noise else None

        def e2e_step():
            xd.copy_(xh, non_blocking=True)
            if nd2 is not None:
                nd2.copy_(nh, non_blocking=True)
            ug.warm_start(xd, out, wl.alpha, wl.sharpen, noise=nd2, seed=1234, offset=0)
            oh.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, args.steps // 4)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, "cuda")
        h2d = x_lr.numel() * 4 + (0 if args.drawn_noise else noise.numel() * 4)
        e2e = {"value": nbytes * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": out.numel() * 4}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = warm_cpu_baseline(wl, x_lr, noise)
    if rank == 0:
        achieved = nbytes / (ms * 1e-3) / 1e9
        peak = pk["hbm_gbs"]
        print(json.dumps({
            "metric": WARM_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded N(0,1) + smooth sinusoid latent, N(0,1) noise)",
            "config": {"workload": wl.name, "batch": wl.batch, "channels": wl.C, "h": wl.h,
                       "w": wl.w, "H": wl.H, "W": wl.W, "alpha": wl.alpha, "sharpen": wl.sharpen,
                       "noise": "drawn in the kernel (Philox4x32-10)" if args.drawn_noise else "read",
                       "l2": "flushed before every launch (256 MB written, then 256 MB read)",
                       "parallelism": f"independent latent per rank x{world}"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": f"{src} copy bandwidth",
                         "algorithmic_bytes_per_launch": nbytes},
            "e2e": e2e, "gpu_launches": launches, "clocks": clocks, "cpu_baseline": cpu,
        }), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def roofline_peak(pk, src, e4m3: bool):
    """The tensor roofline denominators: the measured burst dense-bf16 figure for `frac` (one
    denominator for every workload), the power-capped sustained one beside it."""
    burst, sust = pk["bf16_tflops"], pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    note = f"{src} bf16 dense, burst (frac); sustained under the power cap (frac_sustained)"
    if e4m3:
        # half the useful FLOPs (Q K^T) at the e4m3 rate, nominally twice the bf16 rate, half
        # (P V) at the bf16 rate: the mixed peak is 1 / (0.5 / 2P + 0.5 / P) = 4P / 3
        burst, sust = burst * 4.0 / 3.0, sust * 4.0 / 3.0
        note += "; x 4/3 (nominal ratio, not a measured e4m3 peak) for the mixed e4m3 Q K^T + bf16 P V"
    return burst, sust, note


def measure_layer(ug, args, wl, world, local, rank, heads_range=None, with_e2e=False,
                  with_cpu=False):
    """One workload: build the plan, time `args.steps` steps (permute_rope, attention with the
    unpermute in its epilogue, the split merge when there is one) after the warm-up, and return
    its record.  heads_range = (h0, h1): this rank runs those heads of the layer (split mode)."""
    import dataclasses

    import torch
    import torch.distributed as dist

    full_heads = wl.heads
    h0, h1 = heads_range if heads_range else (0, wl.heads)
    wlr = dataclasses.replace(wl, heads=h1 - h0) if heads_range else wl
    plan = ug.plan_for(wlr)
    if args.lr_radius != -1:
        plan.set_lr_scope(args.lr_radius)
    if args.lr_order != -1:
        plan.set_lr_order(args.lr_order)
    if args.halo != -1:
        plan.set_halo(args.halo)
    e4m3 = args.qk == "e4m3"
    if e4m3:
        plan.set_qk_format("e4m3", args.q_exp, args.k_exp)
    info = plan.info
    q, k, v = ug.make_qkv(wl)
    sha = inputs_sha256(q, k, v) if rank == 0 else None
    if heads_range:
        from diffusion_transformer_ultra_b200.sharding import head_slice
        q, k, v = (head_slice(x, h0, h1) for x in (q, k, v))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lay = ug.Layer(plan, wlr.batch)
    o = torch.empty((wlr.batch, info["N_raster"], wlr.heads, wlr.D), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        ug.permute_rope(qd, kd, vd, lay.qp, lay.kp, lay.vp, plan)
        n = 1
        if evs:
            evs[1].record(stream)
        if args.unfused:
            ug.hla_forward(lay.qp, lay.kp, lay.vp, lay.op, plan)
        else:
            ug.hla_forward_raster(lay.qp, lay.kp, lay.vp, o, plan)   # unpermute in the epilogue
        n += plan.last_launch_count()
        if evs:
            evs[2].record(stream)
        if args.unfused:
            ug.unpermute(lay.op, o, plan)
            n += 1
        if evs:
            evs[3].record(stream)
        return n

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if plan.sync_status() != 0:
        raise RuntimeError("device error during warm-up")

    def timed_steps():
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler = ClockSampler(local)
        # the attention kernel's own clock record (SM cycles over nanoseconds of its first CTA),
        # for the timed launches only
        plan.set_clock_record(True)
        plan.read_clock()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        sampler.start()
        launches = 0
        start.record(stream)
        for i in range(args.steps):
            launches += step(evs[i])
        end.record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop()
        kclock = plan.read_clock()
        plan.set_clock_record(False)
        return evs, start, end, clocks, kclock, launches

    evs, start, end, clocks, kclock, launches = timed_steps()
    # a hardware or thermal slowdown during the timed steps voids them: time them once more
    # (every rank together, so that all take the same collective steps)
    slowed = sorted(set(clocks.get("reasons", [])) & SLOWDOWN_REASONS)
    if max_over_ranks(1.0 if slowed else 0.0, world, "cuda") > 0:
        evs, start, end, clocks, kclock, launches = timed_steps()
        clocks["remeasured_after"] = slowed or ["another rank's slowdown"]
    clocks["kernel_sm_mhz"] = kclock["sm_mhz"]
    clocks["kernel_clock_note"] = ("hla_forward's own record: SM cycles (clock64) over nanoseconds "
                                   "(globaltimer) of its first CTA, summed over the %d timed launches"
                                   % kclock["launches"])
    if world > 1:
        dist.barrier()
    if plan.sync_status() != 0:
        raise RuntimeError("device error during the timed steps")
    ms_total = start.elapsed_time(end)
    ms_perm = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    ms_attn = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    ms_unperm = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    ms_step = max_over_ranks(ms_total, world, "cuda") / args.steps
    ms_attn_max = max_over_ranks(ms_attn, world, "cuda")

    flops_rank = 4.0 * wlr.D * info["useful_pairs"] * wlr.heads * wlr.batch
    flops_layer = 4.0 * wl.D * info["useful_pairs"] * full_heads * wl.batch
    if heads_range:   # strong scaling: the job is one layer, done when the slowest rank is
        value = flops_layer / (ms_step * 1e-3) / 1e12
    else:             # weak scaling: every rank runs its own layer
        value = job_tflops(flops_rank, world, ms_step)
    pk, src = peaks()
    attn_tflops = flops_rank / (ms_attn * 1e-3) / 1e12
    elem = wlr.batch * wlr.heads * info["N_tot"] * wlr.D
    kv_elem = wlr.batch * wlr.heads * info["kv_rows"] * wlr.D
    in_size = 2 if wl.dtype == "bf16" else 4
    qk_size = 1 if e4m3 else 2
    # permute_rope: every raster row of Q, K, V read once (copied halo blocks are written from
    # the same read), Q written over N_tot slots and K, V over kv_rows slots (pad slots as
    # zeros); gathered halo blocks cost the permute nothing
    perm_bytes = (3 * wlr.batch * info["N_raster"] * wlr.heads * wlr.D * in_size
                  + (elem + kv_elem) * qk_size + kv_elem * 2)
    perm_bytes_method = 6 * wlr.batch * info["N_raster"] * wlr.heads * wlr.D * in_size
    unperm_bytes = elem * 2 + wlr.batch * info["N_raster"] * wlr.heads * wlr.D * 2
    traffic = None if heads_range else profiled_traffic(wl.name + ("-e4m3" if e4m3 else ""))
    burst, sust, peak_note = roofline_peak(pk, src, e4m3)

    e2e = None
    if with_e2e and not args.no_e2e:
        # the public host-buffer call: page-locked Q/K/V in, O out, copies overlapped with the
        # kernels of other head slices
        qh, kh, vh = (x.to(torch.bfloat16).pin_memory() for x in (q, k, v))
        oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        runner = ug.HostRunner(plan, wlr.batch, args.e2e_heads_per_chunk)
        for _ in range(2):
            runner(qh, kh, vh, oh)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, args.steps // 4)
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(n_e2e):
            runner(qh, kh, vh, oh)
        e1.record(stream)
        torch.cuda.synchronize()
        if plan.sync_status() != 0:
            raise RuntimeError("device error during the end-to-end steps")
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, "cuda")
        e2e_value = (flops_layer / (ms_e2e * 1e-3) / 1e12 if heads_range
                     else job_tflops(flops_rank, world, ms_e2e))
        e2e = {"value": e2e_value, "unit": "useful TFLOP/s",
               "ms_per_step": ms_e2e, "api": "ultragen_host_runner_forward (host buffers)",
               "heads_per_chunk": args.e2e_heads_per_chunk,
               "h2d_bytes_per_step": 3 * qh.numel() * qh.element_size(),
               "d2h_bytes_per_step": oh.numel() * oh.element_size()}
        runner.close()

    cpu = None
    if with_cpu and rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, q, k, v, lr_radius=args.lr_radius, lr_block=bool(info["lr_block"]),
                           **({"qk_format": "e4m3", "q_exp": args.q_exp, "k_exp": args.k_exp}
                              if e4m3 else {}))

    rec = {
        "workload": wl.name + ("" if args.lr_radius < 0 else f"-lr-region-r{args.lr_radius}")
                    + ("-e4m3-qk" if e4m3 else ""),
        "value": value, "unit": "useful TFLOP/s", "ms_per_step": ms_step,
        "ms_per_layer_attention": ms_attn_max,
        "config": {"H": wl.H, "W": wl.W, "l": wl.l, "b": wl.b, "rho": wl.rho, "text_len": wl.T,
                   "lr_radius": args.lr_radius, "heads": full_heads, "head_dim": wl.D,
                   "batch": wl.batch, "N_tot": info["N_tot"],
                   "useful_pairs_per_head": info["useful_pairs"],
                   "halo_blocks": ["none", "copied", "gathered"][info["halo_copy"]],
                   "N_kv": info["N_kv"], "kv_rows": info["kv_rows"],
                   "lr_blocks": bool(info["lr_block"]), "qk_format": args.qk,
                   **({"q_exp": args.q_exp, "k_exp": args.k_exp} if e4m3 else {}),
                   "inputs_sha256": sha,
                   "l2": "inputs larger than L2 (permuted Q %.0f MB, K %.0f MB, V %.0f MB); no flush"
                         % (elem * qk_size / 1e6, kv_elem * qk_size / 1e6, kv_elem * 2 / 1e6)
                         if elem * qk_size > 126e6 else
                         "inputs smaller than L2 (permuted Q %.0f MB); steady-state layer, no flush"
                         % (elem * qk_size / 1e6)},
        "ms_per_kernel": {"permute_rope": ms_perm, "hla_forward": ms_attn,
                          "unpermute": ms_unperm if args.unfused else "in hla_forward's epilogue"},
        "path": "permute_rope + hla_forward + unpermute" if args.unfused
                else "permute_rope + hla_forward_raster (unpermute fused)",
        "hla_forward_tflops": attn_tflops,
        "permute_rope_gbs": perm_bytes / (ms_perm * 1e-3) / 1e9,
        "permute_rope_gbs_method_bytes": perm_bytes_method / (ms_perm * 1e-3) / 1e9,
        "unpermute_gbs": unperm_bytes / (ms_unperm * 1e-3) / 1e9 if args.unfused else None,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": burst, "unit": "TFLOP/s",
                     "frac": attn_tflops / burst, "frac_sustained": attn_tflops / sust,
                     "peak_sustained": sust, "traffic": traffic, "peak_source": peak_note,
                     "kernel_sm_mhz": kclock["sm_mhz"],
                     "algorithmic_flops_per_launch": flops_rank},
        "e2e": e2e, "gpu_launches": launches, "clocks": clocks, "cpu_baseline": cpu,
    }
    del qd, kd, vd, lay, o, plan
    torch.cuda.empty_cache()
    return rec


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.op == "warm_start":
        main_warm(args, rank, world, local)
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import diffusion_transformer_ultra_b200 as ug
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    def workload(name):
        wl = ug.WORKLOADS[name]
        if args.heads:
            import dataclasses
            wl = dataclasses.replace(wl, heads=args.heads)
        return wl

    def heads_of(wl):
        if args.split != "heads" or world == 1:
            return None
        from diffusion_transformer_ultra_b200.sharding import head_range
        return head_range(wl.heads, world, rank)

    wl = workload(args.workload)
    main_rec = measure_layer(ug, args, wl, world, local, rank, heads_of(wl), with_e2e=True,
                             with_cpu=True)
    extra = {}
    for name in [w for w in args.extra_workloads.split(",") if w and w != "none"]:
        if name == args.workload:
            continue
        ew = workload(name)
        extra[name] = measure_layer(ug, args, ew, world, local, rank, heads_of(ew))
    if rank == 0:
        split = heads_of(wl)
        line = {
            "metric": METRIC, "value": main_rec["value"], "unit": "useful TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": main_rec["ms_per_step"],
            "higher_is_better": True, "scaling": "strong" if split else "weak", "vs_baseline": None,
            "dtype": "e4m3 Q.K^T (fp32 acc) + bf16 P.V" if args.qk == "e4m3" else "bf16",
            "data": "synthetic (seeded N(0,1) + smooth 2D sinusoid Q/K/V; no weights needed)",
            "config": {"workload": main_rec["workload"], **main_rec["config"],
                       "parallelism": (f"heads split across {world} ranks (rank 0: heads "
                                       f"{split[0]}..{split[1] - 1}), no data exchange" if split
                                       else f"independent layer per rank x{world}")},
            **{k_: main_rec[k_] for k_ in ("ms_per_kernel", "path", "hla_forward_tflops",
                                           "permute_rope_gbs", "permute_rope_gbs_method_bytes",
                                           "unpermute_gbs", "roofline", "e2e", "gpu_launches",
                                           "clocks", "cpu_baseline")},
            "workloads": {n: {k_: r[k_] for k_ in ("value", "unit", "ms_per_step",
                                                    "ms_per_layer_attention", "hla_forward_tflops",
                                                    "ms_per_kernel", "roofline", "clocks",
                                                    "gpu_launches", "permute_rope_gbs")}
                          | {"config": r["config"]} for n, r in extra.items()},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
