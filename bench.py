#!/usr/bin/env python
"""Benchmark of the exact dense Sampling-VT on B200.

One step = the whole hot path over one batch: channels-last copy of the
features, fused forward gather-reduction, and the feature gradient (zero-init,
scatter, layout back).  The default workload is the largest single-GPU one,
``batched_bf16`` (B4, 6 cameras, C128 bf16 features of 32x88 from 512x1408
images, BEV 200x200x16 over +-50 m, fp32 accumulation and output);
--workload picks another (tiny, nuscenes, large, backward).  The line's
``by_workload`` block adds the forward and backward of ``large`` (B1 C80
fp32, 400x400x16) and ``nuscenes`` (B1 C64 fp32, 200x200x8), timed outside
the main timed region.

Timing: inputs resident in HBM; L2 flushed (256 MiB write) before every timed
step; the step (repack, forward, backward) captured once as a CUDA graph and
replayed between CUDA events on the launching stream; W warm-up steps, then K
timed steps between a barrier and a device synchronize; the max over ranks is
reported.  The split by stage comes from separate per-stage graph replays.  SM clocks
and throttle reasons are sampled through NVML during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank transforms its own batch (independent
calibrations and features); there is no exchange step, so no collective is
used on the data path ("scaling": "weak").

--impl reference times the CPU oracle (oracle/, plain C loop nest in fp64) on
the host cores, on a band of BEV rows per step, and prints the same JSON line
with "impl": "reference".

--op lss measures the lift-splat BEV pooling (LSS tutorial, "Lift" and
"Splat"): one step = forward + backward (depth and feature gradients) of the
``lss`` workload (6 cameras, 8x22 features, 41 depth bins, C64, 200x200).

--op ms measures the multi-scale form (FlashBEV reading notes, "Takeaway" 4):
one step = channels-last copies of four FPN levels (64x176 .. 8x22 of a
256x704 image), the fused multi-scale forward and every level's feature
gradient, on a 200x200x8 grid (``ms`` workload).

--op deform measures the deformable aggregation instead (SparseDriveV2 notes,
"Deformable Aggregation"): one step = forward + backward (feature, weight and
keypoint-offset gradients) over the queries of the ``deform`` workload (900
queries x 13 keypoints, 6 cameras, C256, 64x176 maps), timed the same way.
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
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BEV output elements/s (B·C·X·Y) and achieved HBM GB/s vs roofline, 1×B200"
UNIT = "elements/s"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None,
                    help="default: batched_bf16 (vt), deform, lss or ms (the other operators)")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--op", choices=["vt", "deform", "lss", "ms"], default="vt")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the hot-L2 and back-to-back forward timings (for launch-list profiling)")
    args = ap.parse_args()
    if args.workload is None:
        args.workload = {"vt": "batched_bf16", "deform": "deform", "lss": "lss", "ms": "ms"}[args.op]
    return args


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def workload_desc(w):
    return (f"{w.name}: B{w.B} N{w.N} C{w.C} {w.Hf}x{w.Wf} features (img {w.img_h}x{w.img_w}) -> "
            f"BEV {w.X}x{w.Y}x{w.Z} over x[{w.xr[0]},{w.xr[1]}] y[{w.yr[0]},{w.yr[1]}] "
            f"z[{w.zr[0]},{w.zr[1]}] m, {w.dtype} features, forward + feature gradient")


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = float(json.load(open(p))["hbm_gbs"])
        return v, "measured (STREAM-style copy on this pool's B200)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (earlier measurement on this pool)"


KERNEL_SOURCES = {
    "sample_forward_kernel": ["bev_forward_rows.cu", "bev_forward_rows_ms.cu", "bev_forward_rows.cuh", "bev_rows.cuh",
                              "bev_kernels.cuh", "bev_geometry.cuh"],
    "sample_backward_kernel": ["bev_backward.cu", "bev_tile.cuh", "bev_kernels.cuh", "bev_geometry.cuh"],
    "deform_forward_kernel": ["bev_deform.cu", "bev_deform.cuh", "bev_geometry.cuh"],
    "deform_backward_kernel": ["bev_deform.cu", "bev_deform.cuh", "bev_geometry.cuh"],
    "lss_forward_kernel": ["bev_lss.cu", "bev_lss.cuh"],
    "lss_backward_kernel": ["bev_lss.cu", "bev_lss.cuh"],
}


def source_digest(kernel):
    """Digest of the source files a kernel is built from."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "camera_bev_view_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the kernel's current sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        ent = json.load(open(p))[kernel][workload]
        if ent.get("source_digest") == source_digest(kernel):
            return float(ent["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """NVML sampling of the SM clock and clock-event reasons."""

    BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.err = [], set(), None
        self.stop_ev = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = f"nvml unavailable: {e}"
            self.h = None

    def _run(self):
        while not self.stop_ev.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = int(self.get_reasons(self.h))
                for b, name in self.BITS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception as e:  # pragma: no cover
                self.err = str(e)
                return
            time.sleep(0.01)

    def __enter__(self):
        if self.h is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.h is not None:
            self.stop_ev.set()
            self.t.join()

    def summary(self):
        if self.h is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err or "no samples"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, ms_per_step: float) -> float:
    """Units per second for the whole job: every rank processes its own
    batch each step, and the slowest rank sets the step time."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_step_sample(w, rows, threads):
    """One oracle forward + backward over BEV rows [i0, i0 + rows) of the
    workload (same calibrations and features); returns (seconds, elements)."""
    import oracle
    from camera_bev_view_b200 import inputs as I
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    dout = I.make_dout(w)
    dx = (w.xr[1] - w.xr[0]) / w.X
    i0 = max(0, w.X // 2 - rows // 2)
    rng = (w.xr[0] + i0 * dx, w.xr[0] + (i0 + rows) * dx) + w.ranges[2:]
    grid = oracle.Grid(rng, w.res)
    d = dout[:, :, i0:i0 + rows].contiguous()
    t0 = time.perf_counter()
    oracle.forward(F, K, E, w.img_h, w.img_w, grid, threads=threads)
    oracle.backward(d, w.N, w.Hf, w.Wf, K, E, w.img_h, w.img_w, grid, threads=threads)
    return time.perf_counter() - t0, w.B * w.C * rows * w.Y


def cpu_baseline(w, seconds):
    """The oracle as it stands, on the host cores, on slices of BEV rows at
    the grid centre (forward + backward over all batch items, cameras and
    channels of those rows) until `seconds` of CPU work (at least one)."""
    threads = cpu_cores()
    rows = max(8, w.X // 25)
    spent, elems, steps = 0.0, 0, 0
    while steps == 0 or spent < seconds:
        t, e = oracle_step_sample(w, rows, threads)
        spent += t
        elems += e
        steps += 1
    return {"value": elems / spent, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{steps} slice(s) of {rows} of the {w.X} BEV rows of the {w.name} workload, forward + "
                      f"backward ({spent:.1f} s, OpenMP over BEV rows / (batch, camera))"}


def run_reference(args):
    from camera_bev_view_b200 import inputs as I
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = I.WORKLOADS[args.workload]
    threads = cpu_cores()
    rows = 8
    for _ in range(args.warmup):
        oracle_step_sample(w, rows, threads)
    times, elems = [], 0
    for _ in range(args.steps):
        t, e = oracle_step_sample(w, rows, threads)
        times.append(t)
        elems += e
    total = sum(times)
    value = elems / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) features and 6-camera rigs; nuScenes-like shapes)",
        "config": {"workload": workload_desc(w), "sample": f"{rows} BEV rows at the grid centre per step"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{rows} of {w.X} BEV rows per step, forward + backward"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    from camera_bev_view_b200 import inputs as I
    from camera_bev_view_b200 import ops

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = I.WORKLOADS[args.workload]
    B, N, C, Hf, Wf, X, Y = w.B, w.N, w.C, w.Hf, w.Wf, w.X, w.Y
    F_h = I.make_features(w, shard=rank)
    K_h, E_h = I.make_rigs(w, shard=rank)
    dout_h = I.make_dout(w, shard=rank)
    F, K, E, dout = (t.to(dev) for t in (F_h, K_h, E_h, dout_h))
    esize = F.element_size()
    grid = ops.bev_grid_spec(w.ranges, w.res)
    Fcl = torch.empty((B, N, Hf, Wf, C), dtype=F.dtype, device=dev)
    out = torch.empty((B, C, X, Y), dtype=torch.float32, device=dev)
    dF = torch.empty((B, N, C, Hf, Wf), dtype=torch.float32, device=dev)
    ws_b = torch.empty(ops.bev_workspace_size(ops.F32, ops.NCHW, B, N, C, Hf, Wf, 1), dtype=torch.uint8,
                       device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    stages = {
        "to_channels_last": lambda: ops.bev_features_to_channels_last(F, out=Fcl),
        "forward": lambda: ops.bev_sample_forward(Fcl, K, E, w.img_h, w.img_w, grid, layout=ops.NHWC,
                                                  out=out),
        "backward": lambda: ops.bev_sample_backward(dout, K, E, w.img_h, w.img_w, grid, N, Hf, Wf, out=dF,
                                                    workspace=ws_b),
    }
    launches_per_step = {"to_channels_last": 1, "forward": 1, "backward": 2}  # + one driver memset
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    graphs = {}
    with torch.cuda.stream(stream):
        for f in stages.values():   # eager warm-up (also sets kernel attributes)
            f()
        stream.synchronize()
        for name, f in stages.items():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                f()
            graphs[name] = g
        # the step as one graph: the three stages back to back, as a training
        # step launches them
        step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(step_graph, stream=stream):
            for f in stages.values():
                f()
        for _ in range(args.warmup):
            flush.zero_()
            step_graph.replay()
            flush.zero_()
            for g in graphs.values():
                g.replay()
        stream.synchronize()

        # timed region: exactly K steps, L2 flushed before each
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(local) as clocks:
            for k in range(args.steps):
                flush.zero_()
                ev[k][0].record(stream)
                step_graph.replay()
                ev[k][1].record(stream)
            torch.cuda.synchronize(dev)
            if world > 1:
                dist.barrier()
        step_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps

        # split by stage (diagnostic, outside the timed region): each stage's
        # graph replayed between events, L2 flushed before each step
        names = list(stages)
        nsplit = min(args.steps, 300)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(nsplit)]
        for k in range(nsplit):
            flush.zero_()
            evs[k][0].record(stream)
            for s, name in enumerate(names):
                graphs[name].replay()
                evs[k][s + 1].record(stream)
        torch.cuda.synchronize(dev)
        per = {name: [evs[k][s].elapsed_time(evs[k][s + 1]) for k in range(nsplit)]
               for s, name in enumerate(names)}
    stage_ms = {name: sum(v) / len(v) for name, v in per.items()}

    # forward with a hot L2 (no flush), and as one CUDA graph of 100
    # back-to-back launches (launch overhead amortised), per launch
    fwd_hot_ms = fwd_b2b_ms = float("nan")
    if not args.no_extras:
        with torch.cuda.stream(stream):
            hot = []
            for k in range(60):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graphs["forward"].replay()
                e1.record(stream)
                e1.synchronize()
                if k >= 10:
                    hot.append(e0.elapsed_time(e1))
            g100 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g100, stream=stream):
                for _ in range(100):
                    stages["forward"]()
            g100.replay()
            reps = []
            for k in range(8):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g100.replay()
                e1.record(stream)
                e1.synchronize()
                if k >= 2:
                    reps.append(e0.elapsed_time(e1) / 100)
            g100.reset()
        fwd_hot_ms = statistics.median(hot)
        fwd_b2b_ms = statistics.median(reps)
    ms = max_over_ranks(step_ms, world, dev)
    elems = B * C * X * Y
    value = whole_job_rate(elems, world, ms)

    # roofline of the dominant kernel (by time)
    peak, peak_src = hbm_peak()
    fwd_bytes = B * N * Hf * Wf * C * esize + elems * 4
    bwd_bytes = elems * 4 + B * N * C * Hf * Wf * 4
    if stage_ms["forward"] >= stage_ms["backward"]:
        dom, dom_ms, dom_bytes, kname = "forward", stage_ms["forward"], fwd_bytes, "sample_forward_kernel"
        dom_note = "features read once + output written once; one launch"
    else:
        dom, dom_ms, dom_bytes, kname = "backward", stage_ms["backward"], bwd_bytes, "sample_backward_kernel"
        dom_note = ("dout read once + dF written once; timed over the whole backward call "
                    "(memset + scatter + layout kernel)")
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": recorded_traffic(kname, w.name), "kernel": kname, "stage": dom,
                "algorithmic_bytes_per_launch": dom_bytes, "note": dom_note, "peak_source": peak_src}
    fwd_gbs = fwd_bytes / (stage_ms["forward"] * 1e-3) / 1e9

    # end to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory, runs the forward (NCHW features, so
    # the repack is inside) and the backward, and copies out and dF back.
    # Steps are pipelined over two buffer slots and three streams (upload,
    # compute, download) -- the way a caller streaming frames runs them, with
    # host-to-device and device-to-host copies overlapping on the full-duplex
    # link -- and a step's time is the span of all steps over their number.
    pin = lambda t: t.pin_memory()
    F_p, K_p, E_p, dout_p = pin(F_h), pin(K_h), pin(E_h), pin(dout_h)
    dt_f = ops.F32 if esize == 4 else ops.BF16
    slots = []
    for _ in range(2):
        slots.append({
            "F": torch.empty_like(F), "K": torch.empty_like(K), "E": torch.empty_like(E),
            "dout": torch.empty_like(dout), "out": torch.empty_like(out), "dF": torch.empty_like(dF),
            "ws_f": torch.empty(max(256, ops.bev_workspace_size(dt_f, ops.NCHW, B, N, C, Hf, Wf, 0)),
                                dtype=torch.uint8, device=dev),
            "ws_b": torch.empty(max(256, ops.bev_workspace_size(ops.F32, ops.NCHW, B, N, C, Hf, Wf, 1)),
                                dtype=torch.uint8, device=dev),
            "out_p": torch.empty(out.shape, dtype=out.dtype).pin_memory(),
            "dF_p": torch.empty(dF.shape, dtype=dF.dtype).pin_memory(),
            "ev_in": torch.cuda.Event(), "ev_done": torch.cuda.Event(), "ev_out": torch.cuda.Event(),
        })
    s_up, s_cmp, s_dn = torch.cuda.Stream(device=dev), stream, torch.cuda.Stream(device=dev)

    def e2e_steps(n):
        for k in range(n):
            sl = slots[k % 2]
            s_up.wait_event(sl["ev_done"])      # the slot's inputs are free once its last compute ended
            with torch.cuda.stream(s_up):
                sl["F"].copy_(F_p, non_blocking=True)
                sl["K"].copy_(K_p, non_blocking=True)
                sl["E"].copy_(E_p, non_blocking=True)
                sl["dout"].copy_(dout_p, non_blocking=True)
                sl["ev_in"].record(s_up)
            s_cmp.wait_event(sl["ev_in"])
            s_cmp.wait_event(sl["ev_out"])      # and its outputs once its last download ended
            ops.bev_sample_forward(sl["F"], sl["K"], sl["E"], w.img_h, w.img_w, grid, out=sl["out"],
                                   workspace=sl["ws_f"], stream=s_cmp)
            ops.bev_sample_backward(sl["dout"], sl["K"], sl["E"], w.img_h, w.img_w, grid, N, Hf, Wf,
                                    out=sl["dF"], workspace=sl["ws_b"], stream=s_cmp)
            sl["ev_done"].record(s_cmp)
            s_dn.wait_event(sl["ev_done"])
            with torch.cuda.stream(s_dn):
                sl["out_p"].copy_(sl["out"], non_blocking=True)
                sl["dF_p"].copy_(sl["dF"], non_blocking=True)
                sl["ev_out"].record(s_dn)

    e2e_steps(4)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    s_cmp.wait_event(e0)
    s_dn.wait_event(e0)
    e2e_steps(args.e2e_steps)
    s_up.wait_stream(s_dn)
    s_up.wait_stream(s_cmp)
    e1.record(s_up)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (F_h, K_h, E_h, dout_h))
    d2h = out.numel() * 4 + dF.numel() * 4

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if esize == 4 else "bf16",
        "data": "synthetic (seeded N(0,1) features and 6-camera rigs with nuScenes-like shapes; no dataset)",
        "config": {"workload": workload_desc(w), "global_batch": B * world,
                   "parallelism": f"dp{world} (each rank its own batch, no collective)",
                   "l2": "flushed before every timed step (256 MiB write)",
                   "timing": "one CUDA graph per step (repack, forward, backward) replayed between CUDA events "
                             "on the launching stream; stages_ms from per-stage graph replays (each with its own "
                             "launch), outside the timed region"},
        "stages_ms": stage_ms,
        "forward_only": {"elements_per_s": elems / (stage_ms["forward"] * 1e-3), "GB_per_s": fwd_gbs,
                         "frac_of_hbm_peak": fwd_gbs / peak,
                         "hot_l2_us": 1e3 * fwd_hot_ms,
                         "graph_of_100_us_per_launch": 1e3 * fwd_b2b_ms,
                         "note": "L2 flushed before each timed step; hot_l2_us: no flush; graph_of_100: 100 "
                                 "back-to-back launches in one CUDA graph after one flush, per launch"},
        "roofline": roofline,
        "e2e": {"value": whole_job_rate(elems, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "pinned host -> device copies, bev_sample_forward (NCHW) + bev_sample_backward, "
                        "device -> pinned host copies; steps pipelined over two buffer slots and three "
                        "streams (upload, compute, download)"},
        "gpu_launches": args.steps * sum(launches_per_step.values()),
        "clocks": clocks.summary(),
    }
    for g in list(graphs.values()) + [step_graph]:
        g.reset()
    if not args.no_extras:
        line["by_workload"] = {name: other_workload(I, ops, I.WORKLOADS[name], dev, stream, flush, peak)
                               for name in ("large", "nuscenes") if name != w.name}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)


def other_workload(I, ops, w, dev, stream, flush, peak, reps=100):
    """Forward (channels-last features) and backward call of another dense
    workload, each captured as a CUDA graph and replayed between CUDA events
    on the launching stream with the L2 flushed before every replay; outside
    the timed region of the main workload."""
    import torch
    F = I.make_features(w, layout="nhwc").to(dev)
    K, E = (t.to(dev) for t in I.make_rigs(w))
    dout = I.make_dout(w).to(dev)
    grid = ops.bev_grid_spec(w.ranges, w.res)
    out = torch.empty((w.B, w.C, w.X, w.Y), dtype=torch.float32, device=dev)
    dF = torch.empty((w.B, w.N, w.C, w.Hf, w.Wf), dtype=torch.float32, device=dev)
    ws_b = torch.empty(ops.bev_workspace_size(ops.F32, ops.NCHW, w.B, w.N, w.C, w.Hf, w.Wf, 1), dtype=torch.uint8,
                       device=dev)
    calls = {"forward": lambda: ops.bev_sample_forward(F, K, E, w.img_h, w.img_w, grid, layout=ops.NHWC, out=out),
             "backward": lambda: ops.bev_sample_backward(dout, K, E, w.img_h, w.img_w, grid, w.N, w.Hf, w.Wf,
                                                         out=dF, workspace=ws_b)}
    res = {"workload": workload_desc(w)}
    with torch.cuda.stream(stream):
        for name, f in calls.items():
            f()
            stream.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                f()
            times = []
            for k in range(reps + 5):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                gr.replay()
                e1.record(stream)
                e1.synchronize()
                if k >= 5:
                    times.append(e0.elapsed_time(e1))
            gr.reset()
            ms = statistics.median(times)
            nbytes = (w.B * w.N * w.Hf * w.Wf * w.C * F.element_size() + w.out_elems * 4 if name == "forward"
                      else w.out_elems * 4 + w.B * w.N * w.C * w.Hf * w.Wf * 4)
            gbs = nbytes / (ms * 1e-3) / 1e9
            res[name] = {"us": 1e3 * ms, "algorithmic_bytes": nbytes, "GB_per_s": gbs, "frac_of_hbm_peak": gbs / peak,
                         "elements_per_s": w.out_elems / (ms * 1e-3)}
    res["note"] = ("median of 100 graph replays, L2 flushed before each; forward on channels-last features "
                   "(the repack is a separate call), backward = the whole call (zero-init, scatter, layout)")
    return res


DEFORM_METRIC = "deformable aggregation output elements/s (B·Q·C) and achieved HBM GB/s vs roofline, 1×B200"


def deform_oracle_step(w, threads):
    """One oracle forward + backward of the deformable aggregation over all
    queries of the workload (same seeded inputs); returns seconds."""
    import oracle
    from camera_bev_view_b200 import inputs as I
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    A, D, W = I.make_queries(w)
    g = I.make_query_dout(w)
    t0 = time.perf_counter()
    oracle.deform_forward(F, K, E, w.img_h, w.img_w, A, D, W, threads=threads)
    oracle.deform_backward(F, g, K, E, w.img_h, w.img_w, A, D, W, threads=threads)
    return time.perf_counter() - t0


def deform_cpu_baseline(w, seconds):
    """The oracle as it stands on the host cores, whole steps until `seconds`."""
    threads = cpu_cores()
    spent, steps = 0.0, 0
    while steps == 0 or spent < seconds:
        spent += deform_oracle_step(w, threads)
        steps += 1
    return {"value": w.out_elems * steps / spent, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{steps} whole forward+backward step(s) of the {w.name} workload ({spent:.1f} s, "
                      f"OpenMP over queries / (batch, camera))"}


def run_deform(args):
    import torch

    from camera_bev_view_b200 import inputs as I
    from camera_bev_view_b200 import ops

    rank, world, local = dist_env()
    w = I.DEFORM_WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank != 0:
            return
        threads = cpu_cores()
        for _ in range(args.warmup):
            deform_oracle_step(w, threads)
        times = [deform_oracle_step(w, threads) for _ in range(args.steps)]
        value = w.out_elems * len(times) / sum(times)
        line = {"impl": "reference", "metric": DEFORM_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded queries, N(0,1) features, 6-camera rig)",
                "config": {"workload": w.name},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                                 "sample": "all queries, forward + backward, per step"},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    F_h = I.make_features(w, shard=rank)
    K_h, E_h = I.make_rigs(w, shard=rank)
    A_h, D_h, W_h = I.make_queries(w, shard=rank)
    g_h = I.make_query_dout(w, shard=rank)
    F, K, E, A, D, W, g = (t.to(dev) for t in (F_h, K_h, E_h, A_h, D_h, W_h, g_h))
    B, N, C, Hf, Wf = F.shape
    Fcl = F.permute(0, 1, 3, 4, 2).contiguous()
    esize = F.element_size()
    dt = ops.BF16 if esize == 2 else ops.F32
    out = torch.empty((B, w.Q, C), device=dev)
    grads = (torch.empty((B, N, C, Hf, Wf), device=dev), torch.empty((B, w.Q, N, w.Kp), device=dev),
             torch.empty((B, w.Q, w.Kp, 3), device=dev))
    ws = torch.empty(max(256, ops.bev_deform_workspace_size(dt, ops.NHWC, B, N, C, Hf, Wf, 1)),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stages = {
        "forward": lambda: ops.bev_deform_forward(Fcl, K, E, w.img_h, w.img_w, A, D, W, layout=ops.NHWC, out=out,
                                                  workspace=ws),
        "backward": lambda: ops.bev_deform_backward(Fcl, K, E, w.img_h, w.img_w, A, D, W, g, layout=ops.NHWC,
                                                    out=grads, workspace=ws),
    }
    # texels some valid keypoint samples: the support of the feature gradient
    # for dout = 1 (weights are >= 0, so nothing cancels); measured once,
    # outside the timed region, to count the feature bytes a launch must read
    ones = torch.ones_like(g)
    dF1, _, _ = ops.bev_deform_backward(Fcl, K, E, w.img_h, w.img_w, A, D, W, ones, layout=ops.NHWC)
    touched = int(torch.count_nonzero(dF1[:, :, 0]).item())
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    graphs = {}
    with torch.cuda.stream(stream):
        for f in stages.values():
            f()
        stream.synchronize()
        for name, f in stages.items():
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                f()
            graphs[name] = gr
        step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(step_graph, stream=stream):
            for f in stages.values():
                f()
        for _ in range(args.warmup):
            flush.zero_()
            step_graph.replay()
            flush.zero_()
            for gr in graphs.values():
                gr.replay()
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        with ClockSampler(local) as clocks:
            for k in range(args.steps):
                flush.zero_()
                ev[k][0].record(stream)
                step_graph.replay()
                ev[k][1].record(stream)
            torch.cuda.synchronize(dev)
        step_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
        names = list(stages)
        nsplit = min(args.steps, 300)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(nsplit)]
        for k in range(nsplit):
            flush.zero_()
            evs[k][0].record(stream)
            for si, name in enumerate(names):
                graphs[name].replay()
                evs[k][si + 1].record(stream)
        torch.cuda.synchronize(dev)
        per = {name: [evs[k][si].elapsed_time(evs[k][si + 1]) for k in range(nsplit)]
               for si, name in enumerate(names)}
    for gr in list(graphs.values()) + [step_graph]:
        gr.reset()
    stage_ms = {name: sum(v) / len(v) for name, v in per.items()}
    ms = step_ms
    elems = w.out_elems
    peak, peak_src = hbm_peak()
    q_in = B * w.Q * (3 + w.Kp * 3 + N * w.Kp) * 4
    fwd_bytes = touched * C * esize + q_in + elems * 4
    bwd_bytes = touched * C * esize + q_in + elems * 4 + B * N * C * Hf * Wf * 4 + B * w.Q * w.Kp * (N + 3) * 4
    dom = "forward" if stage_ms["forward"] >= stage_ms["backward"] else "backward"
    dom_bytes = fwd_bytes if dom == "forward" else bwd_bytes
    kname = "deform_forward_kernel" if dom == "forward" else "deform_backward_kernel"
    achieved = dom_bytes / (stage_ms[dom] * 1e-3) / 1e9
    line = {
        "metric": DEFORM_METRIC, "value": elems / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if esize == 4 else "bf16",
        "data": "synthetic (seeded queries, N(0,1) features, 6-camera rig)",
        "config": {"workload": f"{w.name}: B{B} N{N} C{C} {Hf}x{Wf} (img {w.img_h}x{w.img_w}) Q{w.Q} K{w.Kp}",
                   "l2": "flushed before every timed step (256 MiB write)",
                   "timing": "one CUDA graph per step replayed between CUDA events on the launching stream; "
                             "stages_ms from per-stage graph replays outside the timed region"},
        "stages_ms": stage_ms,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": recorded_traffic(kname, w.name), "kernel": kname, "stage": dom,
                     "algorithmic_bytes_per_launch": dom_bytes, "touched_texels": touched,
                     "note": "texels some valid keypoint samples, read once, + query inputs + outputs "
                             "(backward: + dF written and dweights/doffsets)",
                     "peak_source": peak_src},
        "gpu_launches": args.steps * 4,
        "clocks": clocks.summary(),
    }
    if args.cpu_seconds > 0:
        line["cpu_baseline"] = deform_cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(line), flush=True)


MS_METRIC = "multi-scale BEV output elements/s (B·C·X·Y) and achieved HBM GB/s vs roofline, 1×B200"


def ms_oracle_step(w, threads):
    """One oracle forward + backward of the multi-scale operator over the
    whole workload (same seeded inputs); returns seconds."""
    import oracle
    from camera_bev_view_b200 import inputs as I
    Fs = I.make_ms_features(w)
    K, E = I.make_rigs(w)
    g = I.make_dout(w)
    grid = oracle.Grid(w.ranges, w.res)
    t0 = time.perf_counter()
    oracle.ms_forward(Fs, K, E, w.img_h, w.img_w, grid, threads=threads)
    oracle.ms_backward(g, w.N, w.levels, K, E, w.img_h, w.img_w, grid, threads=threads)
    return time.perf_counter() - t0


def run_ms(args):
    import torch

    from camera_bev_view_b200 import inputs as I
    from camera_bev_view_b200 import ops

    rank, world, local = dist_env()
    w = I.MS_WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank != 0:
            return
        threads = cpu_cores()
        for _ in range(args.warmup):
            ms_oracle_step(w, threads)
        times = [ms_oracle_step(w, threads) for _ in range(args.steps)]
        value = w.out_elems * len(times) / sum(times)
        line = {"impl": "reference", "metric": MS_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded N(0,1) pyramid levels, 6-camera rig)",
                "config": {"workload": w.name},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                                 "sample": "whole workload, forward + backward, per step"},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    Fs = [f.to(dev) for f in I.make_ms_features(w, shard=rank)]
    K_h, E_h = I.make_rigs(w, shard=rank)
    K, E = K_h.to(dev), E_h.to(dev)
    g = I.make_dout(w, shard=rank).to(dev)
    B, N, C = Fs[0].shape[:3]
    sizes = [tuple(f.shape[3:5]) for f in Fs]
    esize = Fs[0].element_size()
    grid = ops.bev_grid_spec(w.ranges, w.res)
    Fcl = [torch.empty((B, N, h, wl, C), dtype=Fs[0].dtype, device=dev) for h, wl in sizes]
    out = torch.empty((B, C, w.X, w.Y), device=dev)
    dF = [torch.empty((B, N, C, h, wl), device=dev) for h, wl in sizes]
    dt = ops.BF16 if esize == 2 else ops.F32
    ws_f = torch.empty(max(256, ops.bev_multiscale_workspace_size(dt, ops.NHWC, B, N, C, sizes, 0)),
                       dtype=torch.uint8, device=dev)
    ws_b = torch.empty(ops.bev_multiscale_workspace_size(ops.F32, ops.NCHW, B, N, C, sizes, 1),
                       dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def repack():
        for f, o in zip(Fs, Fcl):
            ops.bev_features_to_channels_last(f, out=o)

    stages = {
        "to_channels_last": repack,
        "forward": lambda: ops.bev_sample_forward_multiscale(Fcl, K, E, w.img_h, w.img_w, grid, layout=ops.NHWC,
                                                             out=out, workspace=ws_f),
        "backward": lambda: ops.bev_sample_backward_multiscale(g, K, E, w.img_h, w.img_w, grid, N, sizes, out=dF,
                                                               workspace=ws_b),
    }
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    graphs = {}
    with torch.cuda.stream(stream):
        for f in stages.values():
            f()
        stream.synchronize()
        for name, f in stages.items():
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                f()
            graphs[name] = gr
        step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(step_graph, stream=stream):
            for f in stages.values():
                f()
        for _ in range(args.warmup):
            flush.zero_()
            step_graph.replay()
            flush.zero_()
            for gr in graphs.values():
                gr.replay()
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        with ClockSampler(local) as clocks:
            for k in range(args.steps):
                flush.zero_()
                ev[k][0].record(stream)
                step_graph.replay()
                ev[k][1].record(stream)
            torch.cuda.synchronize(dev)
        step_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
        names = list(stages)
        nsplit = min(args.steps, 300)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(nsplit)]
        for k in range(nsplit):
            flush.zero_()
            evs[k][0].record(stream)
            for si, name in enumerate(names):
                graphs[name].replay()
                evs[k][si + 1].record(stream)
        torch.cuda.synchronize(dev)
        per = {name: [evs[k][si].elapsed_time(evs[k][si + 1]) for k in range(nsplit)]
               for si, name in enumerate(names)}
    for gr in list(graphs.values()) + [step_graph]:
        gr.reset()
    stage_ms = {name: sum(v) / len(v) for name, v in per.items()}
    ms_step = step_ms
    elems = w.out_elems
    rate = whole_job_rate(elems, world, max_over_ranks(ms_step, world, dev))
    peak, peak_src = hbm_peak()
    feat_bytes = sum(B * N * C * h * wl for h, wl in sizes)
    fwd_bytes = feat_bytes * esize + elems * 4
    bwd_bytes = elems * 4 + feat_bytes * 4
    dom = "forward" if stage_ms["forward"] >= stage_ms["backward"] else "backward"
    dom_bytes = fwd_bytes if dom == "forward" else bwd_bytes
    kname = "sample_forward_kernel" if dom == "forward" else "sample_backward_kernel"
    achieved = dom_bytes / (stage_ms[dom] * 1e-3) / 1e9
    lv = ",".join(f"{h}x{wl}" for h, wl in sizes)
    line = {
        "metric": MS_METRIC, "value": rate, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if esize == 4 else "bf16",
        "data": "synthetic (seeded N(0,1) pyramid levels, 6-camera rig)",
        "config": {"workload": f"{w.name}: B{B} N{N} C{C} levels {lv} (img {w.img_h}x{w.img_w}) -> "
                               f"BEV {w.X}x{w.Y}x{w.Z}",
                   "l2": "flushed before every timed step (256 MiB write)",
                   "timing": "one CUDA graph per step replayed between CUDA events on the launching stream; "
                             "stages_ms from per-stage graph replays outside the timed region"},
        "stages_ms": stage_ms,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": recorded_traffic(kname, w.name), "kernel": kname, "stage": dom,
                     "algorithmic_bytes_per_launch": dom_bytes,
                     "note": "forward: every level's features read once + out written once; backward: dout read "
                             "once + every level's dF written once (whole call timed)",
                     "peak_source": peak_src},
        "gpu_launches": args.steps * (2 * len(sizes) + 2),
        "clocks": clocks.summary(),
    }
    if args.cpu_seconds > 0 and rank == 0 and world == 1:
        threads = cpu_cores()
        spent, steps = 0.0, 0
        while steps == 0 or spent < args.cpu_seconds:
            spent += ms_oracle_step(w, threads)
            steps += 1
        line["cpu_baseline"] = {"value": elems * steps / spent, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{steps} whole forward+backward step(s) of the {w.name} workload "
                                          f"({spent:.1f} s, OpenMP over BEV rows / (batch, camera))"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


LSS_METRIC = "lift-splat BEV pooling output elements/s (B·C·X·Y) and achieved HBM GB/s vs roofline, 1×B200"


def lss_oracle_step(w):
    """One oracle forward + backward of the lift-splat pooling over the whole
    workload (same seeded inputs); returns seconds.  Single-threaded."""
    import oracle
    from camera_bev_view_b200 import inputs as I
    depth, feat = I.make_lss_inputs(w)
    K, E = I.make_rigs(w)
    dout = I.make_lss_dout(w)
    g = oracle.LssGrid(w.ranges, w.res_xy, w.dbound)
    t0 = time.perf_counter()
    oracle.lss_forward(depth, feat, K, E, w.img_h, w.img_w, g)
    oracle.lss_backward(depth, feat, dout, K, E, w.img_h, w.img_w, g)
    return time.perf_counter() - t0


def run_lss(args):
    import torch

    from camera_bev_view_b200 import inputs as I
    from camera_bev_view_b200 import ops

    rank, world, local = dist_env()
    w = I.LSS_WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank != 0:
            return
        for _ in range(args.warmup):
            lss_oracle_step(w)
        times = [lss_oracle_step(w) for _ in range(args.steps)]
        value = w.out_elems * len(times) / sum(times)
        line = {"impl": "reference", "metric": LSS_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (softmax depth, N(0,1) features, 6-camera rig)", "config": {"workload": w.name},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                                 "sample": "the whole workload, forward + backward, per step"},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    depth_h, feat_h = I.make_lss_inputs(w, shard=rank)
    K_h, E_h = I.make_rigs(w, shard=rank)
    dout_h = I.make_lss_dout(w, shard=rank)
    depth, feat, K, E, dout = (t.to(dev) for t in (depth_h, feat_h, K_h, E_h, dout_h))
    B, N, D, Hf, Wf = depth.shape
    C = feat.shape[2]
    g = ops.bev_grid_spec(w.ranges, w.res_xy + (w.zr[1] - w.zr[0],))
    dmin, _, dstep = w.dbound
    out = torch.empty((B, C, w.X, w.Y), device=dev)
    grads = (torch.empty_like(depth), torch.empty_like(feat))
    ws = torch.empty(max(ops.bev_lss_workspace_size(B, N, C, D, Hf, Wf, w.X, w.Y, 0),
                         ops.bev_lss_workspace_size(B, N, C, D, Hf, Wf, w.X, w.Y, 1)), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stages = {
        "forward": lambda: ops.bev_lss_forward(depth, feat, K, E, w.img_h, w.img_w, dmin, dstep, g, out=out,
                                               workspace=ws),
        "backward": lambda: ops.bev_lss_backward(depth, feat, dout, K, E, w.img_h, w.img_w, dmin, dstep, g,
                                                 out=grads, workspace=ws),
    }
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    graphs = {}
    with torch.cuda.stream(stream):
        for f in stages.values():
            f()
        stream.synchronize()
        for name, f in stages.items():
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                f()
            graphs[name] = gr
        step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(step_graph, stream=stream):
            for f in stages.values():
                f()
        for _ in range(args.warmup):
            flush.zero_()
            step_graph.replay()
            flush.zero_()
            for gr in graphs.values():
                gr.replay()
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        with ClockSampler(local) as clocks:
            for k in range(args.steps):
                flush.zero_()
                ev[k][0].record(stream)
                step_graph.replay()
                ev[k][1].record(stream)
            torch.cuda.synchronize(dev)
        step_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
        names = list(stages)
        nsplit = min(args.steps, 300)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(nsplit)]
        for k in range(nsplit):
            flush.zero_()
            evs[k][0].record(stream)
            for si, name in enumerate(names):
                graphs[name].replay()
                evs[k][si + 1].record(stream)
        torch.cuda.synchronize(dev)
        per = {name: [evs[k][si].elapsed_time(evs[k][si + 1]) for k in range(nsplit)]
               for si, name in enumerate(names)}
    for gr in list(graphs.values()) + [step_graph]:
        gr.reset()
    stage_ms = {name: sum(v) / len(v) for name, v in per.items()}
    ms = step_ms
    elems = w.out_elems
    peak, peak_src = hbm_peak()
    inputs_bytes = (depth.numel() + feat.numel()) * 4
    fwd_bytes = inputs_bytes + elems * 4
    bwd_bytes = inputs_bytes + elems * 4 + (depth.numel() + feat.numel()) * 4
    dom = "forward" if stage_ms["forward"] >= stage_ms["backward"] else "backward"
    dom_bytes = fwd_bytes if dom == "forward" else bwd_bytes
    kname = "lss_forward_kernel" if dom == "forward" else "lss_backward_kernel"
    achieved = dom_bytes / (stage_ms[dom] * 1e-3) / 1e9
    line = {
        "metric": LSS_METRIC, "value": elems / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (softmax depth, N(0,1) features, 6-camera rig)",
        "config": {"workload": f"{w.name}: B{B} N{N} D{D} C{C} {Hf}x{Wf} (img {w.img_h}x{w.img_w}) -> {w.X}x{w.Y}",
                   "l2": "flushed before every timed step (256 MiB write)",
                   "timing": "one CUDA graph per step replayed between CUDA events on the launching stream; "
                             "stages_ms from per-stage graph replays outside the timed region"},
        "stages_ms": stage_ms,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": recorded_traffic(kname, w.name), "kernel": kname, "stage": dom,
                     "algorithmic_bytes_per_launch": dom_bytes,
                     "note": "depth and features read once + output written once (backward: + dout read, "
                             "ddepth and dfeat written); timed over the whole call",
                     "peak_source": peak_src},
        "gpu_launches": args.steps * 6,
        "clocks": clocks.summary(),
    }
    if args.cpu_seconds > 0:
        spent, steps = 0.0, 0
        while steps == 0 or spent < args.cpu_seconds:
            spent += lss_oracle_step(w)
            steps += 1
        line["cpu_baseline"] = {"value": elems * steps / spent, "unit": UNIT, "cores": 1, "kind": "oracle",
                                "sample": f"{steps} whole forward+backward step(s) of the {w.name} workload "
                                          f"({spent:.1f} s, single-threaded)"}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.op == "lss":
        run_lss(args)
    elif args.op == "ms":
        run_ms(args)
    elif args.op == "deform":
        run_deform(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
