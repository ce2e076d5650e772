"""Benchmark: Mpix/s per Soft Anisotropic Diagrams fitting iteration.

One step = one steady-state fitting iteration on the 2048 x 2048, N = 131,072
workload (c3 of the synthetic workloads): a propagation pass at jump 1 with
G = 2 injections, render + MSE + analytic backward, and Adam with the record
rebuild, issued through the C ABI as sad_fit_pass + sad_adam_step (the two
kernels sad_fit_iteration launches).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line.  With N > 1 (torchrun, one process per GPU) every rank
fits its own replica of the workload (the path has no data-path exchange);
value = all ranks' pixels per second over the slowest rank's device time.
``--impl reference`` times the CPU oracle (there is no other implementation
of this method to run) on the same workload and metric.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Mpix/s per fit iter (top-K prop+render+bwd+Adam), 2048² N=128K; % HBM roof"
WORKLOAD = "c3"
# the workload's own set-up before any timed or warm-up step: a full refresh
# and 50 fitting iterations, so that the timed iterations are steady-state
# ones whatever --warmup is
SETUP_ITERS = 50
ADAM_LR = dict(lr_pos=1e-3, lr_log_tau=1e-3, lr_r=1e-3, lr_color=5e-3, lr_theta=1e-3, lr_a=1e-3)

# Algorithmic DRAM bytes (compulsory traffic) per launch, per pixel and per site.
#   fit_pass: read the 8-id list 32 B + write the new list 32 B + read target
#             12 B + write image 12 B; read each 64-B record once + one 36-B
#             gradient write-back per site
#   adam    : params, m, v read+write (3 x 72 B), gradients read + zero
#             (72 B), record write 64 B
BYTES = {
    "fit_pass": (88, 100),
    "adam": (0, 352),
}
# the iteration's own compulsory traffic (fused ideal: the list is read once)
ITER_BYTES_PX, ITER_BYTES_SITE = 88, 452


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--workload", default="c3", choices=["c1", "c2", "c3", "c4", "c5", "rows"],
                    help="c3: the fitting-iteration metric (default); c1: 256x256 N=1,024 exact top-K + "
                         "render + backward + Adam; c2: 768x512 N=50,000 refresh + 200 fit iterations timed "
                         "whole; c4: full candidate refresh + render at 4096x4096, N=524,288; c5: end-to-end "
                         "768x512 fit with densify/prune (secondary measurements, each with the oracle beside)")
    ap.add_argument("--oracle-iters", type=int, default=200,
                    help="c2: fit iterations the oracle runs on all host cores (1 core: a tenth)")
    ap.add_argument("--oracle-fit", action="store_true", help="c5: also run the CPU oracle's fit (minutes)")
    ap.add_argument("--cell", type=int, default=1,
                    help="c4/c5: candidate lists on a grid of cell x cell pixel cells (1: per pixel)")
    ap.add_argument("--refresh", default="jump", choices=["jump", "jfa"],
                    help="c4: jump-flooding refresh (seed + propagation passes) or the 3x3 JFA prepass")
    ap.add_argument("--update-every", type=int, default=1,
                    help="c5: propagate the candidate lists every U iterations (cached lists between)")
    ap.add_argument("--passes-per-update", type=int, default=1, help="c5: propagation passes per update")
    ap.add_argument("--candidates", type=int, default=32, choices=[32, 16],
                    help="c4/c5: rank candidates on the float32 record (32) or the packed binary16 one (16)")
    ap.add_argument("--staging", default="loads", choices=["loads", "tma"],
                    help="c3: the fit pass loads each tile's lists per thread (default) or stages them by TMA "
                         "copies in persistent blocks")
    return ap.parse_args()


def reduce_max(x: float, device=None) -> float:
    """Max of a float over the ranks of the current process group (identity
    without one).  Uses a CPU tensor under gloo and a device tensor under
    nccl."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_mpix(world: int, pixels_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's pixels over the slowest rank's time."""
    return world * pixels_per_rank * steps / (ms_max * 1e-3) / 1e6


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"sad_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r[2] > 200.0] or rows
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in loaded:
            for n, v in zip(names, r[3][1:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded),
                "power_w_median": statistics.median(r[2] for r in loaded)}


# ---------------------------------------------------------------------------
# committed ncu traffic for the dominant kernel (null when the source changed)
# ---------------------------------------------------------------------------
def kernel_source_digest() -> str:
    """Digest of the device code the fused-pass kernel is compiled from (the
    kernel's header and the device header it includes), comments and blank
    lines removed, so that only a change of device code makes committed
    counters stale."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "soft_voronoi_render_b200", "csrc")
    for f in ("sad_device.cuh", "sad_fused_kernel.cuh"):
        txt = open(os.path.join(csrc, f)).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        lines = (re.sub(r"//.*", "", ln).rstrip() for ln in txt.splitlines())
        h.update("\n".join(ln for ln in lines if ln.strip()).encode())
    return h.hexdigest()[:16]


def committed_counter(kernel: str, key: str):
    """A per-launch counter from the committed ncu summary of the kernel, or
    None when the summary is missing or the kernel's code changed since."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_c3.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(key + r":\s*([0-9.eE+]+)", txt)
    d = re.search(r"kernel_source_digest:\s*([0-9a-f]+)", txt)
    if not m or not d or d.group(1) != kernel_source_digest():
        return None
    return float(m.group(1))


def committed_traffic(kernel: str):
    return committed_counter(kernel, "traffic_bytes_per_launch")


def issue_roofline(kernel: str, ms: float, clocks):
    """The fused pass is bound by instruction issue, not by HBM: its warp
    instructions per launch (committed ncu count) over the live launch time,
    against 148 SMs x 4 schedulers x one warp instruction per cycle at the SM
    clock sampled during the run."""
    inst = committed_counter(kernel, "inst_executed_per_launch")
    if inst is None or not clocks or not clocks.get("sm_mhz"):
        return None
    peak = 148 * 4 * clocks["sm_mhz"] * 1e6
    achieved = inst / (ms * 1e-3)
    return {"bound": "issue", "achieved": achieved, "peak": peak, "unit": "warp instructions/s",
            "frac": achieved / peak, "inst_per_launch": inst, "peak_from": "148 SMs x 4 schedulers x sampled SM clock"}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline; the oracle as it stands)
# ---------------------------------------------------------------------------
def oracle_band(tgt, prm, rows: int, r0: int):
    """A band of `rows` image rows starting at r0, as its own problem: the
    logit is translation invariant, so sites move by -r0 in y and s keeps
    1 / max(H, W) because the band keeps the full width (W = max(H, W))."""
    band_t = np.ascontiguousarray(tgt[:, r0:r0 + rows, :])
    band_p = prm.copy()
    band_p[1] = band_p[1] - np.float32(r0)
    return band_t, band_p


def time_oracle_steps(tgt, prm, H, W, G, rows, n_steps, budget_s):
    import oracle
    band_t, band_p = oracle_band(tgt, prm, rows, (H - rows) // 2)
    Hb = rows
    N = prm.shape[1]
    n_site_share = max(1, int(round(N * rows / H)))
    lr = dict(pos=1e-3, log_tau=1e-3, r=1e-3, color=5e-3, theta=1e-3, a=1e-3)
    rec = oracle.records(Hb, W, band_p)
    table = oracle.seed_table(Hb, W, band_p)
    for pas, k in enumerate(oracle.jump_schedule(Hb, W)):
        if k < Hb:
            table = oracle.propagate(Hb, W, rec, table, k, G, 1, pas)
    M = np.zeros((9, n_site_share))
    V = np.zeros((9, n_site_share))
    P64 = band_p[:, :n_site_share].astype(np.float64)
    done, t0 = 0, time.perf_counter()
    while done < n_steps:
        table = oracle.propagate(Hb, W, rec, table, 1, G, 1, 100 + done)
        L, g = oracle.loss_backward(Hb, W, band_p, table, band_t)
        P64, M, V = oracle.adam(Hb, W, P64, M, V, g[:, :n_site_share], lr, done + 1)
        band_p[:, :n_site_share] = P64.astype(np.float32)
        rec = oracle.records(Hb, W, band_p)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return done, dt, Hb * W


def cpu_baseline(tgt, prm, wl, budget_s=15.0, rows=256):
    """The oracle on all host cores (the reported baseline), and the same
    sample on one core beside it."""
    import oracle
    done, dt, px = time_oracle_steps(tgt, prm, wl.H, wl.W, wl.G, rows, 10 ** 6, budget_s)
    all_threads = oracle.num_threads()
    oracle.set_threads(1)
    try:
        done1, dt1, px1 = time_oracle_steps(tgt, prm, wl.H, wl.W, wl.G, rows // 4, 10 ** 6, budget_s / 3)
    finally:
        oracle.set_threads(all_threads)
    return {"value": px * done / dt / 1e6, "unit": "Mpix/s", "cores": all_threads, "kind": "oracle",
            "sample": f"{done} oracle fit iterations (propagate k=1 G={wl.G}, fp64 render+backward, Adam on the "
                      f"band's share of {int(round(wl.N * rows / wl.H))} sites, record rebuild) on a {rows}-row x "
                      f"{wl.W} band of the {wl.H}x{wl.W} N={wl.N} workload, {dt:.1f} s",
            "one_core": {"value": px1 * done1 / dt1 / 1e6, "cores": 1,
                         "sample": f"{done1} iterations on a {rows // 4}-row band, {dt1:.1f} s"}}


def workload_config(wl, world: int) -> dict:
    """The benchmark's config, shared by both arms."""
    return {"workload": f"{WORKLOAD}: {wl.description}", "H": wl.H, "W": wl.W, "N": wl.N, "K": 8, "G": wl.G,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "working set > L2 (two 134 MB candidate tables + 50 MB target + 50 MB image); no flush"}


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    import oracle
    import synth
    tgt, prm, wl = synth.make_workload(WORKLOAD, seed=1)
    rows = 128
    per_step_budget = 1e9
    # warm-up steps (untimed)
    time_oracle_steps(tgt, prm, wl.H, wl.W, wl.G, rows, max(args.warmup, 0), per_step_budget)
    done, dt, px = time_oracle_steps(tgt, prm, wl.H, wl.W, wl.G, rows, args.steps, 240.0)
    value = px * done / dt / 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mpix/s", "n_gpus": args.gpus,
        "steps": done, "warmup": args.warmup, "ms_per_step": dt / max(done, 1) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": "Mpix/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"each step: one oracle fit iteration on a {rows}-row band "
                                   f"of the {wl.H}x{wl.W} workload"},
        "e2e": {"value": value, "unit": "Mpix/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    import synth
    from soft_voronoi_render_b200 import Sad, _lib

    tgt, prm, wl = synth.make_workload(WORKLOAD, seed=1 + rank)
    H, W, N, G, P = wl.H, wl.W, wl.N, wl.G, wl.H * wl.W
    s = Sad(H, W, N, device=dev, seed=1 + rank)
    s.set_sites(prm)
    s.set_target(tgt)
    if args.staging == "tma":
        s.set_list_staging(_lib.SAD_STAGING_TMA)
    s.refresh(G)
    cfg = _lib.adam_cfg(**ADAM_LR)
    ctx = s.ctx
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        _lib.sad_fit_pass(ctx, G, sp)
        if ev is not None:
            ev[1].record(stream)
        _lib.sad_adam_step(ctx, cfg, sp)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(SETUP_ITERS + max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}")
    if local == 0 or world == 1:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(K):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if (local == 0 or world == 1) else None
    ms_total = t_start.elapsed_time(t_end)
    per_kernel = {n: 0.0 for n in ("fit_pass", "adam")}
    for e in evs:
        per_kernel["fit_pass"] += e[0].elapsed_time(e[1])
        per_kernel["adam"] += e[1].elapsed_time(e[2])
    ms_max = reduce_max(ms_total, dev)
    ms_step = ms_max / K
    value = aggregate_mpix(world, P, K, ms_max)

    # Cross-check with a CUDA graph: one sad_fit_iteration (the fused pass
    # and Adam, two launches) captured once, 20 warm-up replays, then 5
    # repeats of 200 timed replays; the median repeat is reported.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _lib.sad_fit_iteration(ctx, G, cfg, torch.cuda.current_stream(dev).cuda_stream)
    for _ in range(20):
        graph.replay()
    g_reps = []
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    for _ in range(5):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        g0.record(stream)
        for _ in range(200):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        g_reps.append(reduce_max(g0.elapsed_time(g1), dev) / 200)
    del graph
    graph_ms = statistics.median(g_reps)

    # end to end through the C ABI: each step's target comes from pinned host
    # memory and each step's loss goes back to pinned host memory
    E = max(1, min(args.e2e_steps, K))
    host_tgt = torch.from_numpy(np.ascontiguousarray(tgt)).pin_memory()
    from cuda.bindings import runtime as cudart
    L = _lib.load()
    h2d = cudart.cudaMemcpyKind.cudaMemcpyHostToDevice
    copy_stream = torch.cuda.Stream(dev)
    cs_h, ms_h = copy_stream.cuda_stream, stream.cuda_stream
    status = []

    def sync_all():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # Each end-to-end form runs E_REPEATS times and reports the median: a
    # window of E steps is tens of milliseconds, so one stall of the host
    # thread that issues the steps (a shared machine) moves a single run.
    E_REPEATS = 3
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    # (a) serial: set the target, one iteration, read the loss (host waits)
    def serial():
        sync_all()
        e0.record(stream)
        for _ in range(E):
            _lib.sad_set_target(ctx, host_tgt.data_ptr(), sp)
            _lib.sad_fit_iteration(ctx, G, cfg, sp)
            _lib.sad_get_loss(ctx, sp)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return reduce_max(e0.elapsed_time(e1), dev)

    e2e_serial_runs = [serial() for _ in range(E_REPEATS)]

    def pipelined(src, nbytes, bufs, per_step):
        """Each step's input copied host -> device on a copy stream into one
        of two device buffers while the previous step computes; per_step(b)
        issues the step on the compute stream; each step's loss is copied
        into its own slot of pinned host memory in stream order (no host
        wait).  Copies and stream dependencies go through the CUDA runtime
        directly: a few microseconds of host time per step."""
        no_timing = cudart.cudaEventDisableTiming
        ev_copied = [cudart.cudaEventCreateWithFlags(no_timing)[1] for _ in range(2)]
        ev_used = [cudart.cudaEventCreateWithFlags(no_timing)[1] for _ in range(2)]
        host_loss = torch.zeros(E, dtype=torch.float64).pin_memory()
        loss0 = host_loss.data_ptr()
        for ev in ev_used:
            status.append(cudart.cudaEventRecord(ev, ms_h)[0])

        def issue_copy(k):
            b = k % 2
            status.append(cudart.cudaStreamWaitEvent(cs_h, ev_used[b], 0)[0])
            status.append(cudart.cudaMemcpyAsync(bufs[b], src, nbytes, h2d, cs_h)[0])
            status.append(cudart.cudaEventRecord(ev_copied[b], cs_h)[0])

        sync_all()
        e0.record(stream)
        issue_copy(0)
        for k in range(E):
            if k + 1 < E:
                issue_copy(k + 1)
            b = k % 2
            status.append(cudart.cudaStreamWaitEvent(ms_h, ev_copied[b], 0)[0])
            per_step(b, ev_used[b])
            status.append(L.sad_copy_loss(ctx, loss0 + 8 * k, sp))
        e1.record(stream)
        torch.cuda.synchronize(dev)
        for ev in ev_copied + ev_used:
            cudart.cudaEventDestroy(ev)
        losses = host_loss.tolist()
        assert len(losses) == E and all(math.isfinite(x) and x > 0 for x in losses)
        return reduce_max(e0.elapsed_time(e1), dev)

    # (b) the workload's float32 target, bound in place (sad_bind_target)
    bufs32 = [torch.empty_like(s.target), torch.empty_like(s.target)]
    ptr32 = [b.data_ptr() for b in bufs32]

    def step32(b, ev_used):
        status.append(L.sad_bind_target(ctx, ptr32[b]))
        status.append(L.sad_fit_iteration(ctx, G, ctypes.byref(cfg), sp))
        status.append(cudart.cudaEventRecord(ev_used, ms_h)[0])

    e2e_f32_runs = [pipelined(host_tgt.data_ptr(), host_tgt.numel() * 4, ptr32, step32) for _ in range(E_REPEATS)]
    status.append(L.sad_bind_target(ctx, s.target.data_ptr()))

    # (c) the same image streamed as 8-bit RGB (the format of the photographs
    # the method fits; the image rounded to 1/255), converted on the device
    # by sad_set_target_u8 into the bound float target
    host_u8 = torch.from_numpy(np.ascontiguousarray(
        np.clip(np.rint(tgt * 255.0), 0, 255).astype(np.uint8).transpose(1, 2, 0))).pin_memory()
    bufs8 = [torch.empty(host_u8.shape, dtype=torch.uint8, device=dev) for _ in range(2)]
    ptr8 = [b.data_ptr() for b in bufs8]

    def step8(b, ev_used):
        status.append(L.sad_set_target_u8(ctx, ptr8[b], sp))
        status.append(cudart.cudaEventRecord(ev_used, ms_h)[0])
        status.append(L.sad_fit_iteration(ctx, G, ctypes.byref(cfg), sp))

    e2e_u8_runs = [pipelined(host_u8.data_ptr(), host_u8.numel(), ptr8, step8) for _ in range(E_REPEATS)]

    # the host link alone: the float32 target copied E times on the copy stream
    sync_all()
    c0 = torch.cuda.Event(enable_timing=True)
    c1 = torch.cuda.Event(enable_timing=True)
    c0.record(copy_stream)
    for k in range(E):
        status.append(cudart.cudaMemcpyAsync(ptr32[k % 2], host_tgt.data_ptr(), host_tgt.numel() * 4, h2d, cs_h)[0])
    c1.record(copy_stream)
    torch.cuda.synchronize(dev)
    h2d_ms = c0.elapsed_time(c1) / E
    bad = [x for x in status if x not in (0, cudart.cudaError_t.cudaSuccess)]
    if bad:
        raise RuntimeError(f"end-to-end loop: {len(bad)} failing calls, first {bad[0]}")
    e2e_value = aggregate_mpix(world, P, E, statistics.median(e2e_f32_runs))
    e2e_u8 = aggregate_mpix(world, P, E, statistics.median(e2e_u8_runs))
    e2e_serial = aggregate_mpix(world, P, E, statistics.median(e2e_serial_runs))
    e2e_runs = {name: [round(aggregate_mpix(world, P, E, ms), 1) for ms in runs]
                for name, runs in (("float32", e2e_f32_runs), ("u8", e2e_u8_runs), ("serial", e2e_serial_runs))}
    st = s.stats()

    if rank == 0:
        hbm, peak_kind = measured_peaks()
        avg = {k: v / K for k, v in per_kernel.items()}
        dom = max(avg, key=avg.get)
        bpx, bsite = BYTES[dom]
        alg_bytes = bpx * P + bsite * N
        achieved = alg_bytes / (avg[dom] * 1e-3) / 1e9
        traffic = committed_traffic(dom)
        iter_bytes = ITER_BYTES_PX * P + ITER_BYTES_SITE * N
        line = {
            "metric": METRIC, "value": value, "unit": "Mpix/s", "n_gpus": world, "steps": K,
            "warmup": max(args.warmup, 3), "setup_iterations": SETUP_ITERS, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(workload_config(wl, world), list_staging=args.staging),
            "hbm_roof_frac_iter": (iter_bytes / (ms_step * 1e-3) / 1e9) / hbm,
            # the same bytes over the nominal 8 TB/s of B200's HBM3e
            "hbm_roof_frac_iter_nominal_8tbs": (iter_bytes / (ms_step * 1e-3) / 1e9) / 8000.0,
            "iter_algorithmic_bytes": iter_bytes,
            "kernels_ms": {k: round(v, 5) for k, v in avg.items()},
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                         "algorithmic_bytes": alg_bytes},
            "issue_roofline": issue_roofline(dom, avg[dom], clocks),
            "e2e": {"value": e2e_value, "unit": "Mpix/s", "h2d_bytes_per_step": int(host_tgt.numel() * 4),
                    "d2h_bytes_per_step": 8, "steps": E, "repeats": E_REPEATS, "runs_mpix_s": e2e_runs,
                    "how": "per step: the step's float32 target (the workload's own), pinned host -> device on a "
                           "copy stream (double-buffered, overlapping the previous step), sad_bind_target, "
                           "sad_fit_iteration, sad_copy_loss into that step's slot of pinned host memory; the "
                           "host reads the losses after the last step; median of the repeats",
                    "h2d_ms_per_step": h2d_ms,
                    "h2d_gbs": host_tgt.numel() * 4 / (h2d_ms * 1e-3) / 1e9,
                    "bound_by": "host link" if h2d_ms > ms_step else "device",
                    "serial_value": e2e_serial,
                    "u8_value": e2e_u8, "u8_h2d_bytes_per_step": int(host_u8.numel())},
            "gpu_launches": 3 * K,  # timed region: the fused pass, its finishing launch and Adam, per step
            "graph": {"ms_per_step": graph_ms, "value": aggregate_mpix(world, P, 1, graph_ms), "unit": "Mpix/s",
                      "repeats_ms": [round(x, 5) for x in g_reps],
                      "how": "sad_fit_iteration captured once in a CUDA graph; 20 warm-up replays, 5 repeats of "
                             "200 timed replays, median"},
            "clocks": clocks,
            "device_stats": {k: st[k] for k in ("hash_overflow", "empty_pixels", "dropped_ids")},
            "loss": st["loss"],
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(tgt, prm, wl)
        print(json.dumps(line), flush=True)
    s.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_refresh(args):
    """Full candidate refresh from scratch (seed pass + jumps 2048..1 with
    G = 4, or with --refresh jfa the seed pass + 3x3 flood passes) followed
    by a render, at 4096 x 4096 with N = 524,288; with --cell the lists live
    on the downscaled candidate grid.  Also reports how often slot 0 holds
    the exact owner, on 4096 sampled cells (exact top-K on the device)."""
    import torch
    import synth
    from soft_voronoi_render_b200 import Sad, _lib

    tgt, prm, wl = synth.make_workload("c4", seed=1)
    H, W, N, G, P = wl.H, wl.W, wl.N, wl.G, wl.H * wl.W
    s = Sad(H, W, N, seed=1)
    s.set_sites(prm)
    s.set_target(tgt)
    if args.cell != 1:
        s.set_candidate_grid(args.cell)
    if args.candidates == 16:
        s.set_candidate_precision(16)
    GH, GW = (H + args.cell - 1) // args.cell, (W + args.cell - 1) // args.cell
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    def refresh():
        if args.refresh == "jfa":
            _lib.sad_jfa_prepass(s.ctx, sp)
        else:
            _lib.sad_refresh(s.ctx, G, sp)

    for _ in range(max(args.warmup, 3)):
        refresh()
        _lib.sad_render(s.ctx, None, sp)
    torch.cuda.synchronize()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for k in range(K):
        ev[k][0].record(stream)
        refresh()
        ev[k][1].record(stream)
        _lib.sad_render(s.ctx, None, sp)
        ev[k][2].record(stream)
    torch.cuda.synchronize()
    t_ref = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    t_ren = sum(e[1].elapsed_time(e[2]) for e in ev) / K
    hbm, peak_kind = measured_peaks()
    PT = GH * GW
    m = max(GH, GW)
    if args.refresh == "jfa":
        passes = max(1, (m - 1).bit_length())
    else:
        passes = max(0, m.bit_length() - 1)
    # passes: list read + write; clear; render: the cell lists + image
    alg = passes * 64 * PT + 32 * PT + 32 * PT + 12 * P
    # slot 0 against the exact owner on sampled cells
    tab = s.get_table()
    cells = np.random.default_rng(1).choice(PT, size=min(4096, PT), replace=False)
    ex = s.topk_exact(cells).cpu().numpy().view(np.uint32)
    owner_right = float(np.mean(tab[cells, 0] == ex[:, 0]))
    what = "3x3 JFA prepass (seed + flood passes)" if args.refresh == "jfa" else f"seed + {passes} passes, G={G}"
    line = {"metric": f"ms per full candidate refresh ({what}) + render, 4096x4096 N=524,288"
                      + (f", {args.cell}x{args.cell} candidate cells" if args.cell != 1 else ""),
            "value": t_ref + t_ren, "unit": "ms", "higher_is_better": False, "n_gpus": 1, "steps": K,
            "warmup": max(args.warmup, 3), "refresh_ms": t_ref, "render_ms": t_ren,
            "mpix_per_s_per_pass": PT * passes / (t_ref * 1e-3) / 1e6 if passes else None,
            "owner_right_sampled": owner_right, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"c4: {wl.description}", "H": H, "W": W, "N": N, "G": G, "cell": args.cell,
                       "refresh": args.refresh, "candidate_bits": args.candidates},
            "hbm_roof_frac": alg / ((t_ref + t_ren) * 1e-3) / 1e9 / hbm, "peak_kind": peak_kind,
            "device_stats": s.stats()}
    print(json.dumps(line), flush=True)
    s.close()
    return 0


def run_fit(args):
    """End-to-end fit of the 768 x 512 workload: 10,000 gradient-weighted
    sites growing to 50,000 (densify/prune events every 100 iterations from
    100 to 1600, +2,500 net each, 0.5 % pruned), 2000 iterations, Adam
    (lr 1e-3 positions, 5e-3 colours).  Reports time to fit and final PSNR."""
    import torch
    import synth
    from soft_voronoi_render_b200 import Sad, fit

    tgt, prm, wl = synth.make_workload("c5", seed=1)
    H, W, N_cap = wl.H, wl.W, 50_000
    sched = fit.Schedule(update_every=args.update_every, passes_per_update=args.passes_per_update)
    s = Sad(H, W, N_cap, seed=1)
    s.set_sites(prm)
    s.set_target(tgt)
    if args.cell != 1:
        s.set_candidate_grid(args.cell)
    if args.candidates == 16:
        s.set_candidate_precision(16)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    info = fit.run(s, sched)
    e1.record()
    torch.cuda.synchronize()
    t_fit = e0.elapsed_time(e1) * 1e-3
    L = s.loss()
    n_final = int((s.get_sites()[0] >= 0).sum())
    line = {"metric": "time to fit 768x512 (2000 iterations, N 10,000 -> 50,000 by densify/prune) and final PSNR",
            "value": t_fit, "unit": "s", "higher_is_better": False, "n_gpus": 1,
            "psnr_db": 10 * math.log10(3.0 / L), "final_loss": L, "n_active_final": n_final,
            "iterations": sched.iterations, "events": len(sched.events), "schedule_run": info,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"c5: {wl.description}", "H": H, "W": W, "N_start": prm.shape[1],
                       "N_cap": N_cap, "G": sched.G, "cell": args.cell, "candidate_bits": args.candidates,
                       "update_every": sched.update_every,
                       "passes_per_update": sched.passes_per_update}}
    if args.oracle_fit:
        import oracle
        lr = {k[3:] if k.startswith("lr_") else k: float(np.float32(v)) for k, v in sched.lr.items()}
        lr = {"pos": lr["pos"], "log_tau": lr["log_tau"], "r": lr["r"], "color": lr["color"],
              "theta": lr["theta"], "a": lr["a"]}
        t0 = time.perf_counter()
        if args.cell != 1:
            raise SystemExit("--oracle-fit runs the oracle's schedule on the pixel grid only")
        P, L_o, _ = oracle.fit(H, W, prm, tgt, N_cap, sched.iterations, sched.events, sched.grow, sched.prune_frac,
                               lr, sched.G, 1, update_every=sched.update_every,
                               passes_per_update=sched.passes_per_update)
        line["oracle"] = {"time_s": time.perf_counter() - t0, "psnr_db": 10 * math.log10(3.0 / L_o),
                          "final_loss": L_o, "n_active_final": int((P[0] >= 0).sum()),
                          "cores": oracle.num_threads()}
        line["psnr_diff_db"] = line["psnr_db"] - line["oracle"]["psnr_db"]
    print(json.dumps(line), flush=True)
    s.close()
    return 0


def time_oracle_c2(prm, tgt, wl, iters: int, threads: int | None):
    """The oracle's c2 pipeline (refresh, then iterations of propagate k = 1,
    render + backward in double, Adam, records) on `threads` host threads
    (None: all); returns (seconds, iterations, threads used)."""
    import oracle
    all_threads = oracle.num_threads()
    if threads is not None:
        oracle.set_threads(threads)
    try:
        lr = dict(pos=1e-3, log_tau=1e-3, r=1e-3, color=5e-3, theta=1e-3, a=1e-3)
        t0 = time.perf_counter()
        oracle.refresh(wl.H, wl.W, prm, wl.G, 1, 0)
        t_ref = time.perf_counter() - t0
        t0 = time.perf_counter()
        oracle.fit(wl.H, wl.W, prm, tgt, wl.N, iters, (), 0, 0.0, lr, wl.G, 1)
        t_fit = time.perf_counter() - t0 - t_ref  # oracle.fit refreshes first
        return t_ref, max(t_fit, 0.0), iters, oracle.num_threads()
    finally:
        oracle.set_threads(all_threads)


def run_c2(args):
    """768 x 512, N = 50,000 (the Kodak-shaped workload): seed + refresh at
    jumps 256..1 with G = 2, then 200 fitting iterations (propagation k = 1,
    G = 2, render, backward, Adam), timed whole on the GPU; the oracle runs
    the same pipeline on all host cores and on one core."""
    import torch
    import synth
    from soft_voronoi_render_b200 import Sad, _lib

    tgt, prm, wl = synth.make_workload("c2", seed=1)
    P, ITER = wl.H * wl.W, 200
    cfg = _lib.adam_cfg(**ADAM_LR)
    runs = []
    for rep in range(max(args.warmup, 1) + 3):
        s = Sad(wl.H, wl.W, wl.N, seed=1)
        s.set_sites(prm)
        s.set_target(tgt)
        stream = torch.cuda.current_stream()
        sp = stream.cuda_stream
        torch.cuda.synchronize()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        _lib.sad_refresh(s.ctx, wl.G, sp)
        e[1].record(stream)
        for _ in range(ITER):
            _lib.sad_fit_iteration(s.ctx, wl.G, cfg, sp)
        e[2].record(stream)
        torch.cuda.synchronize()
        runs.append((e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), s.loss()))
        s.close()
    timed = runs[max(args.warmup, 1):]
    ref_ms = statistics.median(r[0] for r in timed)
    fit_ms = statistics.median(r[1] for r in timed)
    line = {"metric": "768x512 N=50,000: refresh + 200 fit iterations, timed whole", "value": ref_ms + fit_ms,
            "unit": "ms", "higher_is_better": False, "n_gpus": 1, "repeats": len(timed), "refresh_ms": ref_ms,
            "fit_200_ms": fit_ms, "mpix_per_s_per_iter": P * ITER / (fit_ms * 1e-3) / 1e6,
            "final_loss": timed[-1][2], "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"c2: {wl.description}", "H": wl.H, "W": wl.W, "N": wl.N, "G": wl.G,
                       "l2": "working set (~60 MB) is L2-resident; HBM fractions are not meaningful here"}}
    if not args.no_cpu_baseline:
        oracle_runs = {}
        for label, threads, iters in (("all_cores", None, args.oracle_iters),
                                      ("one_core", 1, max(1, args.oracle_iters // 10))):
            t_ref, t_fit, n, used = time_oracle_c2(prm, tgt, wl, iters, threads)
            oracle_runs[label] = {"cores": used, "refresh_s": t_ref, "iterations": n, "fit_s": t_fit,
                                  "s_per_iter": t_fit / n, "mpix_per_s_per_iter": P * n / t_fit / 1e6,
                                  "whole_200_s_extrapolated": t_ref + t_fit / n * ITER}
        line["cpu_baseline"] = {"kind": "oracle", **oracle_runs}
    print(json.dumps(line), flush=True)
    return 0


def run_c1(args):
    """256 x 256, N = 1,024: exact brute-force top-K, render, MSE backward and
    one Adam step (lr 1e-3), each timed on the GPU with CUDA events (the
    exact top-K lists become the context's lists through sad_set_table,
    untimed); the oracle times the same four steps on all host cores and on
    one core."""
    import torch
    import synth
    from soft_voronoi_render_b200 import Sad, _lib

    tgt, prm, wl = synth.make_workload("c1", seed=1)
    P = wl.H * wl.W
    s = Sad(wl.H, wl.W, wl.N, seed=1)
    s.set_sites(prm)
    s.set_target(tgt)
    cfg = _lib.adam_cfg()
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    out = torch.empty((P, 8), dtype=torch.int32, device=s.device)
    reps = max(5, min(args.steps, 50))
    acc = {"topk_exact": [], "render": [], "backward": [], "adam": []}
    for rep in range(reps + 2):
        s.set_sites(prm)
        torch.cuda.synchronize()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        _lib.sad_topk_exact(s.ctx, None, P, out, sp)
        e[1].record(stream)
        torch.cuda.synchronize()
        s.set_table(out.cpu().numpy().view(np.uint32))
        f = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        f[0].record(stream)
        _lib.sad_render(s.ctx, None, sp)
        f[1].record(stream)
        _lib.sad_backward(s.ctx, 0, sp)
        f[2].record(stream)
        _lib.sad_adam_step(s.ctx, cfg, sp)
        f[3].record(stream)
        torch.cuda.synchronize()
        if rep >= 2:
            acc["topk_exact"].append(e[0].elapsed_time(e[1]))
            for k, (a, b) in zip(("render", "backward", "adam"), ((0, 1), (1, 2), (2, 3))):
                acc[k].append(f[a].elapsed_time(f[b]))
    ms = {k: statistics.median(v) for k, v in acc.items()}
    total = sum(ms.values())
    line = {"metric": "256x256 N=1,024: exact top-K + render + backward + one Adam step", "value": total,
            "unit": "ms", "higher_is_better": False, "n_gpus": 1, "repeats": reps, "kernels_ms": ms,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"c1: {wl.description}", "H": wl.H, "W": wl.W, "N": wl.N}}
    s.close()
    if not args.no_cpu_baseline:
        import oracle
        all_threads = oracle.num_threads()
        runs = {}
        for label, threads in (("all_cores", all_threads), ("one_core", 1)):
            oracle.set_threads(threads)
            t0 = time.perf_counter()
            rec = oracle.records(wl.H, wl.W, prm)
            table = oracle.topk_exact(wl.H, wl.W, rec)
            t1 = time.perf_counter()
            oracle.render(wl.H, wl.W, prm, table)
            t2 = time.perf_counter()
            L, g = oracle.loss_backward(wl.H, wl.W, prm, table, tgt)
            t3 = time.perf_counter()
            oracle.adam(wl.H, wl.W, prm.astype(np.float64), np.zeros((9, wl.N)), np.zeros((9, wl.N)), g,
                        dict(pos=1e-3, log_tau=1e-3, r=1e-3, color=1e-3, theta=1e-3, a=1e-3), 1)
            t4 = time.perf_counter()
            runs[label] = {"cores": oracle.num_threads(), "topk_exact_s": t1 - t0, "render_s": t2 - t1,
                           "backward_s": t3 - t2, "adam_s": t4 - t3, "total_s": t4 - t0}
        oracle.set_threads(all_threads)
        line["cpu_baseline"] = {"kind": "oracle", **runs}
    print(json.dumps(line), flush=True)
    return 0


def run_rows(args):
    """Every entry point of the path timed on its own at 2048 x 2048,
    N = 131,072 (exact top-K on the 256 x 256, N = 1,024 workload), with the
    algorithmic bytes of one call and their fraction of the measured HBM
    peak.  Secondary measurements; the headline is the default workload."""
    import torch
    import synth
    from soft_voronoi_render_b200 import SAD_DETERMINISTIC, SAD_STATS, Sad, _lib

    hbm, peak_kind = measured_peaks()
    reps = max(3, min(args.steps, 20))
    tgt, prm, wl = synth.make_workload("c3", seed=1)
    H, W, N, G, P = wl.H, wl.W, wl.N, wl.G, wl.H * wl.W
    s = Sad(H, W, N, seed=1)
    s.set_sites(prm)
    s.set_target(tgt)
    s.refresh(G)
    cfg = _lib.adam_cfg(lr_color=5e-3)
    for _ in range(5):
        s.fit_iteration(G, cfg)
    stream = torch.cuda.current_stream()

    def timed(fn, n=reps, before=None):
        for _ in range(2):
            if before:
                before()
            fn()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(n):
            if before:
                before()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        return total / n

    rows = {}

    def row(name, ms, alg_bytes, note, **extra):
        r = {"ms": ms, "alg_bytes": alg_bytes, "hbm_frac": (alg_bytes / (ms * 1e-3) / 1e9 / hbm) if alg_bytes else None,
             "what": note}
        r.update(extra)
        rows[name] = r

    row("a1_records", timed(s.prep_records), 100 * N, "records from params: 36 B read + 64 B written per site")
    row("a2_propagate_k1", timed(lambda: s.propagate(1, G)), 64 * P, "one Jacobi pass, jump 1, G = 2: lists 32 + 32 B/px")
    row("a2_propagate_k16", timed(lambda: s.propagate(16, G)), 64 * P, "one Jacobi pass, jump 16, G = 2")
    row("a4_render", timed(s.render), 44 * P, "softmax blend: list 32 + image 12 B/px")
    zero = s.grads.zero_
    row("a5_a6_backward", timed(s.backward, before=zero), 56 * P + 36 * N,
        "render + loss + backward (tile pass on the current lists): list 32 + target 12 + image 12 B/px, gradients 36 B/site")
    row("a6_backward_stats", timed(lambda: s.backward(SAD_STATS), before=zero), 56 * P + 60 * N,
        "the same with the budget statistics (+24 B/site)")
    row("a6_backward_deterministic", timed(lambda: s.backward(SAD_DETERMINISTIC), before=zero), 56 * P + 36 * N,
        "the same with 64-bit fixed-point accumulation")
    row("a2_a6_fit_pass", timed(lambda: s.fit_pass(G), before=zero), 88 * P + 100 * N,
        "fused pass: propagation k = 1 + render + loss + backward")
    row("a4_a6_fit_pass_cached", timed(s.fit_pass_cached, before=zero), 56 * P + 100 * N,
        "the tile pass on cached lists (no propagation)")
    row("a7_adam", timed(lambda: s.adam_step(cfg)), 352 * N, "Adam + records: 352 B/site")
    row("next4_tau_diffuse", timed(lambda: s.tau_diffuse(0.3)), 48 * N, "tau diffusion: list 32 + 16 B/site")
    packed = torch.empty((N, 4), dtype=torch.int32, device=s.device)
    rng = torch.empty(6, dtype=torch.float32, device=s.device)
    row("next3_pack", timed(lambda: _lib.sad_pack_sites(s.ctx, packed, rng, s.stream)), 52 * N,
        "16-byte records: 36 B read + 16 B written per site")
    row("next3_unpack", timed(lambda: _lib.sad_unpack_sites(s.ctx, packed, rng, s.stream)), 116 * N,
        "decode + records: 16 B read + 36 + 64 B written per site")
    row("a9_refresh", timed(lambda: s.refresh(G), n=3), 32 * P + 11 * 64 * P, "seed + 11 passes (jumps 1024..1)")
    row("next2_jfa_prepass", timed(s.jfa_prepass, n=3), 32 * P + 11 * 64 * P, "seed + 11 flood passes")
    s.refresh(G)
    row("next1_densify_prune", timed(lambda: s.densify_prune(_lib.densify_cfg(grow=2500, prune_frac=0.005)), n=3,
                                     before=lambda: (s.grads.zero_(), s.backward(SAD_STATS))), 0,
        "one event (statistics from a backward before each call, untimed): select, prune, split, records",
        hbm_frac=None)
    s.close()
    # a8 on the 256 x 256, N = 1,024 workload: every site scored at every pixel
    tgt1, prm1, w1 = synth.make_workload("c1", seed=1)
    s1 = Sad(w1.H, w1.W, w1.N, seed=1)
    s1.set_sites(prm1)
    ms = timed(s1.topk_exact)
    scores = w1.H * w1.W * w1.N
    row("a8_topk_exact_c1", ms, 0, "brute force over all 1,024 sites at all 65,536 pixels",
        gscores_per_s=scores / (ms * 1e-3) / 1e9, hbm_frac=None)
    s1.close()
    line = {"metric": "per-entry-point device time, 2048x2048 N=131,072 (exact top-K: 256x256 N=1,024)",
            "unit": "ms", "n_gpus": 1, "reps": reps, "peak_hbm_gbs": hbm, "peak_kind": peak_kind, "dtype": "f32",
            "data": "synthetic", "config": {"workload": f"c3: {wl.description}", "H": H, "W": W, "N": N, "G": G},
            "rows": rows}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.workload == "rows":
        return run_rows(args)
    if args.workload in ("c1", "c2") and args.impl == "ours":
        return run_c1(args) if args.workload == "c1" else run_c2(args)
    if args.workload == "c5" and args.impl == "ours":
        return run_fit(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "c4":
        return run_refresh(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
