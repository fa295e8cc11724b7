"""Benchmark: MoE dispatch + combine (forward and backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--fwd-only] [--no-e2e] [--no-cpu-baseline]

A step is one pass of the whole path over one batch of the DeepSeek-V3-shaped
decode workload (T=4096 tokens, H=7168, E=256 experts, K=8, 8 logical EP
ranks, Zipf(0.6) routing):
    layout -> permute (bf16, with chunk-completion counters; one
    moe_dispatch call) -> combine (identity experts: y = the dispatched
    rows) -> combine backward -> dispatch backward.
value = algorithmic HBM bytes of the step / device time of the step, in GB/s
(also reported: tokens/s).  fwd_step times the forward pair alone (layout ->
permute -> combine: dispatch + combine, the metric's pair) the same way over
the same number of steps.  Inputs are resident in HBM when the timed region
starts; L2 is flushed (256 MiB write) before every timed step and the flush
is outside the timed events.  Inside the timed region the only events are
one before and one after each step; per-kernel times (phases_us: medians;
the roofline's dominant kernel: its mean) come from a separate pass right
after it with an event between every two kernels.  With N GPUs (torchrun), every rank runs its
own replica on its own data (weak scaling; no collective on the data path);
the reported time is the max over ranks.

--impl reference times the CPU oracle (single-threaded C) on a bounded sample
of the same workload and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import csv
import glob
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dispatch+combine HBM GB/s and tokens/s on 1 B200; fraction of HBM peak"
# kernels per step: layout (count + assign), permute, combine [, combine_bwd, dispatch_bwd]
LAUNCHES_PER_STEP = {False: 6, True: 4}  # layout (2), permute, combine[, combine_bwd, dispatch_bwd]
CONFIG_INDEX = 2
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="time each step as one CUDA graph replay (captured once)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the per-call timings of the other workloads")
    return ap.parse_args()


# ----------------------------------------------------------------- bytes --
def step_bytes(T, K, H, E, P, fwd_only=False):
    """Algorithmic bytes per call (what the method must move at least)."""
    TK = T * K
    b = {
        "layout": 4 * TK + 4 * TK + 4 * P + 8 * E,
        "permute": 2 * T * H + 2 * P * H,
        "combine": 2 * TK * H + 8 * TK + 2 * T * H,
    }
    if not fwd_only:
        b["combine_bwd"] = 2 * T * H + 2 * TK * H + 2 * P * H + 12 * TK
        b["dispatch_bwd"] = 2 * TK * H + 2 * T * H + 4 * TK
    return b


def groups_gbs(nbytes, phase_us):
    """Algorithmic GB/s of dispatch (layout + permute), of combine, of their
    sum (the forward pass) and, when timed, of the two backward calls, from
    the per-kernel times."""
    groups = {"dispatch": ("layout", "permute"), "combine": ("combine",),
              "dispatch_plus_combine": ("layout", "permute", "combine"),
              "backward": ("combine_bwd", "dispatch_bwd")}
    out = {}
    for g, ps in groups.items():
        if all(p in phase_us for p in ps):
            b = sum(nbytes[p] for p in ps)
            us = sum(phase_us[p] for p in ps)
            out[g] = {"GBps": round(b / (us * 1e-6) / 1e9, 1), "us": round(us, 2), "bytes": b}
    return out


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha(srcfile: str):
    """sha1[:12] of a kernel's source file followed by the shared device
    header it includes (common.cuh), or None if either is missing."""
    csrc = os.path.join(ROOT, "combine_moe_dispatch_05_b200", "csrc")
    try:
        data = open(os.path.join(csrc, srcfile), "rb").read() + \
            open(os.path.join(csrc, "common.cuh"), "rb").read()
    except OSError:
        return None
    return hashlib.sha1(data).hexdigest()[:12]


def ncu_traffic(kernel_key: str):
    """dram bytes per launch of `kernel_key` from the committed ncu summaries,
    if the kernel's sources are unchanged since the capture (else None).
    Summary lines look like:  traffic: <key> <bytes per launch> src=<sha1[:12]>
    where the sha covers the kernel's .cu file and common.cuh."""
    srcfile = {"permute": "permute.cu", "combine": "combine.cu", "combine_bwd": "combine.cu",
               "dispatch_bwd": "combine.cu", "layout": "layout.cu"}.get(kernel_key)
    if srcfile is None:
        return None
    sha = kernel_source_sha(srcfile)
    if sha is None:
        return None
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(f):
            m = re.match(r"\s*traffic:\s+(\S+)\s+(\d+)\s+src=([0-9a-f]+)", line)
            if m and m.group(1) == kernel_key and m.group(3) == sha:
                return int(m.group(2))
    return None


# ---------------------------------------------------------------- clocks --
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        for r in csv.reader(io.StringIO(self.out or "")):
            if len(r) < 9:
                continue
            try:
                rows.append((float(r[1]), float(r[2]), float(r[3]), [x.strip() for x in r[4:9]]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3][1:])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows),
                "samples": len(rows), "samples_under_load": len(loaded),
                "reasons": reasons}


def smi_id(torch, dev) -> str:
    """nvidia-smi --id for a torch device: its PCI bus id when torch exposes it
    (robust to CUDA_VISIBLE_DEVICES remapping), else the ordinal."""
    p = torch.cuda.get_device_properties(dev)
    try:
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except AttributeError:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[dev.index].strip()
        return str(dev.index)


# ------------------------------------------------------ distributed glue --
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, world: int) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_seed_offset(rank: int) -> int:
    """Each replica draws its own batch (weak scaling)."""
    return rank


# ------------------------------------------------------------- our arm --
def run_ours(args, world, rank, local):
    import torch
    from combine_moe_dispatch_05_b200 import ops
    from combine_moe_dispatch_05_b200 import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ops.lib()  # fails loudly if the CUDA library is missing
    s = W.config(CONFIG_INDEX, rank_seed_offset(rank))
    T, H, E, K, R = s.T, s.H, s.E, s.K, s.R

    ids_h = W.topk_ids(s).pin_memory()
    sc_h = W.topk_scales(s).pin_memory()
    x_h = W.tokens(s).pin_memory()
    g_h = W.grad_out(s).pin_memory()
    ids, sc, x, g = (t.to(dev) for t in (ids_h, sc_h, x_h, g_h))

    L = ops.alloc_layout(T, K, E, R, dev)
    P_cap = L.P_cap
    xp = torch.empty((P_cap, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    gy = torch.empty((P_cap, H), dtype=torch.bfloat16, device=dev)
    gs = torch.empty((T, K), dtype=torch.float32, device=dev)
    gx = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    st = ops.new_status(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(evs=None):
        # the timed steps use the one-call dispatch (layout + permute, the
        # permute's first loads overlapping the layout); the per-kernel pass
        # calls the two separately to put an event between them
        rec = (lambda i: evs[i].record(stream)) if evs else (lambda i: None)
        rec(0)
        if evs:
            ops.moe_dispatch_layout(ids, E, R, layout=L, status=st)
            rec(1)
            ops.moe_dispatch_permute(x, L, xp=xp, status=st)
        else:
            ops.moe_dispatch(ids, x, E, R, layout=L, xp=xp, status=st)
        rec(2)
        ops.moe_combine(xp, L.dst_row, sc, out=out, status=st)   # identity experts: y = xp
        rec(3)
        if not args.fwd_only:
            ops.moe_combine_bwd(g, xp, sc, L, grad_y=gy, grad_scales=gs, status=st)
            rec(4)
            ops.moe_dispatch_bwd(gy, L.dst_row, T, K, grad_x=gx, status=st)
            rec(5)

    phases = ["layout", "permute", "combine"] + ([] if args.fwd_only else
                                                 ["combine_bwd", "dispatch_bwd"])
    n_ev = len(phases) + 1
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if ops.read_status(st) != 0:
        raise RuntimeError(f"device status {ops.read_status(st)}")
    P = int(L.expert_offsets[E].item())
    nbytes = step_bytes(T, K, H, E, P, args.fwd_only)

    graph = None
    if args.graph:  # one capture of the whole step; the timed steps replay it
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            step()
        torch.cuda.synchronize()
    # Timed region: one event before and one after each step, none between
    # the kernels (an event between two kernels ends the programmatic launch
    # chain and serialises them: ~5 us per boundary).
    def timed_steps(fn):
        bounds = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            bounds[i][0].record(stream)
            fn()
            bounds[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return [a.elapsed_time(b) for a, b in bounds]

    def forward():  # dispatch + combine: the metric's pair, chained
        ops.moe_dispatch(ids, x, E, R, layout=L, xp=xp, status=st)
        ops.moe_combine(xp, L.dst_row, sc, out=out, status=st)

    def dispatch():  # layout -> permute in one call
        ops.moe_dispatch(ids, x, E, R, layout=L, xp=xp, status=st)

    with ClockSampler(smi_id(torch, dev)) as clk:
        step_ms = timed_steps(graph.replay if graph is not None else step)
        # The forward step alone (layout -> permute -> combine), timed the same
        # way over the same number of steps; with --fwd-only it is the step.
        fwd_ms = step_ms if args.fwd_only else timed_steps(forward)
        disp_ms = timed_steps(dispatch)
    if ops.read_status(st) != 0:
        raise RuntimeError(f"device status {ops.read_status(st)} in the timed steps")
    snapshot = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the last timed step's outputs, checked against the oracle's pass in
        # the cpu_baseline leg
        snapshot = {"counts": L.expert_counts, "offsets": L.expert_offsets, "scales": sc,
                    "rank_counts": L.rank_counts, "rank_offsets": L.rank_offsets,
                    "dst_row": L.dst_row, "row_src": L.row_src, "out": out.view(torch.int16)}
        if not args.fwd_only:
            snapshot.update(grad_y=gy.view(torch.int16), grad_scales=gs,
                            grad_x=gx.view(torch.int16))
        P_now = int(L.expert_offsets[E].item())
        snapshot = {k: v.cpu().numpy() for k, v in snapshot.items()}
        snapshot["xp"] = xp[:P_now].view(torch.int16).cpu().numpy()
        if "grad_y" in snapshot:
            snapshot["grad_y"] = snapshot["grad_y"][:P_now]
    # Per-kernel durations: a pass right after the timed region with an event
    # between every two kernels, which isolates each kernel's own time.
    n_phase = min(args.steps, 100)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(n_phase)]
    for i in range(n_phase):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    per_phase = {p: [] for p in phases}
    for e in evs:
        for j, p in enumerate(phases):
            per_phase[p].append(e[j].elapsed_time(e[j + 1]))
    phase_step_ms = statistics.mean(e[0].elapsed_time(e[-1]) for e in evs)
    total_ms = sum(step_ms)
    total_ms_max = max_over_ranks(total_ms, world)
    ms_per_step = total_ms_max / args.steps
    bytes_step = sum(nbytes.values())
    value = bytes_step * world / (ms_per_step * 1e-3) / 1e9
    tok_s = T * world / (ms_per_step * 1e-3)

    # per-kernel medians (a rare launch in this pass takes several times its
    # usual time, which would move a mean); the roofline uses the mean launch
    # duration of its kernel
    phase_us = {p: 1e3 * statistics.median(v) for p, v in per_phase.items()}
    phase_mean_us = {p: 1e3 * statistics.mean(v) for p, v in per_phase.items()}
    phase_gbs = {p: nbytes[p] / (phase_us[p] * 1e-6) / 1e9 for p in phases}
    dom = max((p for p in phases if p != "layout"), key=lambda p: phase_us[p])
    dom_gbs = nbytes[dom] / (phase_mean_us[dom] * 1e-6) / 1e9
    peak, peak_src = measured_peak()
    fwd_bytes = sum(nbytes[p] for p in ("layout", "permute", "combine"))
    fwd_ms_per_step = max_over_ranks(sum(fwd_ms), world) / args.steps
    fwd_gbs = fwd_bytes * world / (fwd_ms_per_step * 1e-3) / 1e9
    fwd_step = {"ms": round(fwd_ms_per_step, 5), "GBps": round(fwd_gbs, 1),
                "frac": round(fwd_gbs / world / peak, 4),
                "tokens_per_s": round(T * world / (fwd_ms_per_step * 1e-3), 1),
                "bytes": fwd_bytes, "steps": args.steps,
                "median_ms": round(statistics.median(fwd_ms), 5),
                "what": "layout -> permute (one moe_dispatch call) -> combine chained on one "
                        "stream, no events between the kernels, L2 flushed before each step "
                        "(outside the events); max over ranks"}
    disp_bytes = nbytes["layout"] + nbytes["permute"]
    disp_ms_per_step = max_over_ranks(sum(disp_ms), world) / args.steps
    disp_gbs = disp_bytes * world / (disp_ms_per_step * 1e-3) / 1e9
    dispatch_step = {"ms": round(disp_ms_per_step, 5), "GBps": round(disp_gbs, 1),
                     "frac": round(disp_gbs / world / peak, 4), "bytes": disp_bytes,
                     "what": "layout -> permute in one moe_dispatch call, timed like fwd_step"}
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(dom_gbs, 1),
                "peak": peak, "unit": "GB/s", "frac": round(dom_gbs / peak, 4),
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src ==
                "measured" else "fallback 6.65 TB/s",
                "traffic": ncu_traffic(dom),
                "algorithmic_bytes_per_launch": nbytes[dom],
                "duration_source": f"mean of {n_phase} launches in the per-kernel pass after "
                                   "the timed region (events on the launching stream on both "
                                   "sides of each kernel, L2 flushed before each step)",
                "step_frac": round(bytes_step / (ms_per_step * 1e-3) / 1e9 / peak, 4),
                "fwd_step_frac": fwd_step["frac"]}

    res = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s",
           "tokens_per_s": round(tok_s, 1), "n_gpus": world, "steps": args.steps,
           "warmup": max(args.warmup, 3), "ms_per_step": round(ms_per_step, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded Zipf routing, N(0,1) activations; identity experts)",
           "config": {"workload": f"{s.name}: T={T} H={H} E={E} K={K} R={R} Zipf(s={s.zipf_s})"
                                  f" {'fwd' if args.fwd_only else 'fwd+bwd'}",
                      "P": P, "P_cap": P_cap, "bytes_per_step": bytes_step,
                      "l2": "flushed before every timed step (256 MiB write, outside the events)",
                      "launch": "CUDA graph replay per step" if graph is not None else
                                "eager launches (programmatic dependent launch)",
                      "parallelism": f"replicas x{world}"},
           "phases_us": {p: round(v, 2) for p, v in phase_us.items()},
           "phases_us_mean_max": {p: [round(phase_mean_us[p], 2), round(1e3 * max(v), 2)]
                                  for p, v in per_phase.items()},
           "phases_note": f"medians of a per-kernel pass of {n_phase} steps with an event between "
                          f"every two kernels (which serialises them): {phase_step_ms:.4f} ms "
                          "per step there, against ms_per_step in the timed region",
           "phases_gbs": {p: round(v, 1) for p, v in phase_gbs.items()},
           "groups_gbs": groups_gbs(nbytes, phase_us),
           "roofline": roofline,
           "fwd_step": fwd_step,
           "dispatch_step": dispatch_step,
           "gpu_launches": LAUNCHES_PER_STEP[args.fwd_only] * args.steps +
           (0 if args.fwd_only else LAUNCHES_PER_STEP[True] * args.steps) + 3 * args.steps,
           "clocks": clk.summary()}
    if snapshot is not None:
        res["_timed_outputs"] = snapshot
    q = statistics.quantiles(step_ms, n=10) if len(step_ms) >= 2 else step_ms * 9
    res["step_ms_distribution"] = {"median": round(statistics.median(step_ms), 5),
                                   "p10": round(q[0], 5), "p90": round(q[-1], 5),
                                   "note": "this rank's per-step event times, L2 flushed"}
    if world == 1 and graph is None:
        # the same step back to back without the flush: part of each step's
        # inputs is still in L2 from the step before
        warm = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(min(args.steps, 100))]
        for a, b in warm:
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        warm_ms = statistics.median(a.elapsed_time(b) for a, b in warm)
        res["warm_l2"] = {"ms_per_step_median": round(warm_ms, 5),
                          "value": round(bytes_step / (warm_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                          "note": "L2 not flushed between steps; not the headline value"}
        if ops.read_status(st) != 0:
            raise RuntimeError(f"device status {ops.read_status(st)} in the warm runs")

    if not args.no_extra and world == 1:
        cs = torch.zeros(((P_cap + 127) // 128,), dtype=torch.int32, device=dev)
        st2 = ops.new_status(dev)
        # the layout call resets the counters, so it leads both variants
        t = time_calls(torch, [
            ("layout_permute_then_consumer",
             lambda: (ops.moe_dispatch_layout(ids, E, R, layout=L, status=st2),
                      ops.moe_dispatch_permute(x, L, xp=xp, status=st2),
                      ops.moe_wait_tiles_checksum(L, xp, checksums=cs, status=st2))),
            ("layout_permute_with_concurrent_consumer",
             lambda: (ops.moe_dispatch_layout(ids, E, R, layout=L, status=st2),
                      ops.moe_dispatch_permute_consume(x, L, xp=xp, checksums=cs, status=st2))),
        ], flush, 20, stream)
        if ops.read_status(st2) != 0:
            raise RuntimeError(f"device status {ops.read_status(st2)} in the overlap runs")
        res["overlap"] = {"workload": res["config"]["workload"].replace(" fwd+bwd", ""),
                          "what": "permute + a consumer that acquires each 128-row tile and "
                                  "reads all of it (checksum): separate launches vs one "
                                  "cooperative launch with consumers working while the copy runs",
                          "us": {k: round(v, 1) for k, v in t.items()},
                          "gain": round(1 - t["layout_permute_with_concurrent_consumer"] /
                                        t["layout_permute_then_consumer"], 3)}
        res["shared_expert_overlap"] = shared_expert_overlap(ops, torch, dev, flush, stream, ids,
                                                             sc, x, L, xp, E, R)
        res["l2_writeback"] = l2_writeback(torch, dev, flush, stream, [
            ("combine", lambda: ops.moe_combine(xp, L.dst_row, sc, out=out, status=st2)),
            ("combine_bwd", lambda: ops.moe_combine_bwd(g, xp, sc, L, grad_y=gy, grad_scales=gs,
                                                        status=st2)),
            ("dispatch_bwd", lambda: ops.moe_dispatch_bwd(gy, L.dst_row, T, K, grad_x=gx,
                                                          status=st2)),
        ])
        if ops.read_status(st2) != 0:
            raise RuntimeError(f"device status {ops.read_status(st2)} in the L2 runs")
        res["other_workloads"] = extra_workloads(args, dev, flush, stream)
        res["planner"] = plan_on(L, E, R, ops)

    if not args.no_e2e:
        res["e2e"] = e2e(args, ops, torch, dev, stream, L, (ids_h, sc_h, x_h, g_h),
                         (ids, sc, x, g), (xp, out, gy, gs, gx, st), flush, T, K, E, R,
                         bytes_step, world)
    return res


def e2e(args, ops, torch, dev, stream, L, host_in, dev_in, bufs, flush, T, K, E, R, bytes_step,
        world):
    """The same step through the public API with host buffers: every step
    copies its inputs (ids, scales, x, grad_out) from pinned host memory and
    its results (out, grad_x, grad_scales) back, inside the timed region.
    Copies run on their own streams (host->device and device->host engines)
    and overlap the kernels of the same and of the neighbouring step; two
    sets of device buffers alternate so no step overwrites data another one
    still uses.  Timed as one region over all steps (events), max over ranks."""
    ids_h, sc_h, x_h, g_h = host_in
    h2d_s = torch.cuda.Stream(device=dev)
    d2h_s = torch.cuda.Stream(device=dev)
    comp = stream

    def new_set(first):
        if first:
            ids, sc, x, g = dev_in
            xp, out, gy, gs, gx, st = bufs
            Ls = L
        else:
            ids, sc, x, g = (torch.empty_like(t) for t in dev_in)
            xp, out, gy, gs, gx = (torch.empty_like(t) for t in bufs[:5])
            st = ops.new_status(dev)
            Ls = ops.alloc_layout(T, K, E, R, dev)
        return dict(ids=ids, sc=sc, x=x, g=g, xp=xp, out=out, gy=gy, gs=gs, gx=gx, st=st, L=Ls,
                    out_h=torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
                    gx_h=torch.empty(gx.shape, dtype=gx.dtype, pin_memory=True),
                    gs_h=torch.empty(gs.shape, dtype=gs.dtype, pin_memory=True),
                    free=None)

    sets = [new_set(True), new_set(False)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = T * sets[0]["out"].shape[1] * 2 + (0 if args.fwd_only else
                                             T * sets[0]["out"].shape[1] * 2 + T * K * 4)

    def one(i):
        b = sets[i % 2]
        ev = {k: torch.cuda.Event() for k in ("a", "x", "g", "out", "bwd", "done")}
        if b["free"] is not None:            # results of this set's previous step are on the host
            h2d_s.wait_event(b["free"])
            comp.wait_event(b["free"])
        with torch.cuda.stream(h2d_s):
            b["ids"].copy_(ids_h, non_blocking=True)
            b["sc"].copy_(sc_h, non_blocking=True)
            ev["a"].record(h2d_s)
            b["x"].copy_(x_h, non_blocking=True)
            ev["x"].record(h2d_s)
            if not args.fwd_only:
                b["g"].copy_(g_h, non_blocking=True)
                ev["g"].record(h2d_s)
        comp.wait_event(ev["a"])
        ops.moe_dispatch_layout(b["ids"], E, R, layout=b["L"], status=b["st"], stream=comp)
        comp.wait_event(ev["x"])
        ops.moe_dispatch_permute(b["x"], b["L"], xp=b["xp"], status=b["st"], stream=comp)
        ops.moe_combine(b["xp"], b["L"].dst_row, b["sc"], out=b["out"], status=b["st"],
                        stream=comp)
        ev["out"].record(comp)
        if not args.fwd_only:
            comp.wait_event(ev["g"])
            ops.moe_combine_bwd(b["g"], b["xp"], b["sc"], b["L"], grad_y=b["gy"],
                                grad_scales=b["gs"], status=b["st"], stream=comp)
            ops.moe_dispatch_bwd(b["gy"], b["L"].dst_row, T, K, grad_x=b["gx"], status=b["st"],
                                 stream=comp)
            ev["bwd"].record(comp)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev["out"])
            b["out_h"].copy_(b["out"], non_blocking=True)
            if not args.fwd_only:
                d2h_s.wait_event(ev["bwd"])
                b["gx_h"].copy_(b["gx"], non_blocking=True)
                b["gs_h"].copy_(b["gs"], non_blocking=True)
            ev["done"].record(d2h_s)
        b["free"] = ev["done"]

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    for b in sets:
        if ops.read_status(b["st"]) != 0:
            raise RuntimeError("device status set during the end-to-end run")
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    h2d_s.wait_stream(comp)
    for i in range(args.steps):
        one(i)
    comp.wait_stream(h2d_s)
    comp.wait_stream(d2h_s)
    end.record(comp)
    end.synchronize()
    tot = max_over_ranks(start.elapsed_time(end), world)
    ms = tot / args.steps
    res = {"value": round(bytes_step * world / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
           "ms_per_step": round(ms, 4), "tokens_per_s": round(T * world / (ms * 1e-3), 1),
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "overlap": "copies on separate streams, two alternating buffer sets",
           "l2": "not flushed: each step moves ~3.2 GB through HBM, far beyond L2"}
    if world == 1:
        # the copies alone, both directions at once on the same streams: the
        # PCIe bound of this end-to-end step (no kernels)
        b = sets[0]
        pairs_in = [(b["ids"], ids_h), (b["sc"], sc_h), (b["x"], x_h)] + \
            ([] if args.fwd_only else [(b["g"], g_h)])
        pairs_out = [(b["out_h"], b["out"])] + \
            ([] if args.fwd_only else [(b["gx_h"], b["gx"]), (b["gs_h"], b["gs"])])

        def copies():
            with torch.cuda.stream(h2d_s):
                for d, h in pairs_in:
                    d.copy_(h, non_blocking=True)
            with torch.cuda.stream(d2h_s):
                for h, d in pairs_out:
                    h.copy_(d, non_blocking=True)
        copies()
        torch.cuda.synchronize()
        n = min(args.steps, 20)
        start.record(comp)
        h2d_s.wait_stream(comp)
        d2h_s.wait_stream(comp)
        for _ in range(n):
            copies()
        comp.wait_stream(h2d_s)
        comp.wait_stream(d2h_s)
        end.record(comp)
        end.synchronize()
        copy_ms = start.elapsed_time(end) / n
        res["copies_only_ms_per_step"] = round(copy_ms, 4)
        res["pcie_gbps_per_direction"] = round(max(h2d, d2h) / (copy_ms * 1e-3) / 1e9, 1)
        res["frac_of_copy_bound"] = round(copy_ms / ms, 4)
    return res


# ------------------------------------------------------ other workloads --
def time_calls(torch, calls, flush, steps, stream):
    """Median device time (us) of each call, L2 flushed before each."""
    out = {}
    for name, fn in calls:
        for _ in range(3):
            flush.zero_()
            fn()
        ts = []
        for _ in range(steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        out[name] = statistics.median(ts)
    return out


def l2_writeback(torch, dev, flush, stream, calls):
    """Each gather kernel timed after two kinds of L2 flush: the standard one
    (a 256 MiB write, which leaves L2 full of dirty lines that the kernel then
    has to write back to HBM, as it would the previous layer's output) and the
    same write followed by a 256 MiB read (L2 left holding clean lines).  The
    difference is the write-back of what earlier work left in L2, traffic that
    is not the kernel's own; every headline number keeps the standard flush."""
    rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    acc = torch.empty((), dtype=torch.float32, device=dev)

    class CleanFlush:
        @staticmethod
        def zero_():
            flush.zero_()
            torch.sum(rd, dim=0, out=acc)

    dirty = time_calls(torch, calls, flush, 30, stream)
    clean = time_calls(torch, calls, CleanFlush, 30, stream)
    out = {"what": "medians of 30 launches after a 256 MiB write (dirty L2, the standard "
                   "flush) and after the same write plus a 256 MiB read (clean L2). After the "
                   "clean flush a kernel's own last writes (up to its output size, at most L2) "
                   "also stay in L2 unpaid, so clean_us is a lower bound, not a throughput",
}
    for name, _ in calls:
        out[name] = {"dirty_us": round(dirty[name], 1), "clean_us": round(clean[name], 1),
                     "difference_us": round(dirty[name] - clean[name], 1)}
    return out


def shared_expert_overlap(ops, torch, dev, flush, stream, ids, sc, x, L, xp, E, R):
    """Shared-expert work on a second stream while the dispatch runs.

    Stand-in for the shared expert: a dense MLP on every token,
    shared_x = silu(x @ W1) @ W2 with DeepSeek-V3's shared-expert width
    (2048), done by torch matmuls (cuBLAS); it is not part of this library.
    Sequential: layout, permute, shared MLP, combine(+shared_x) on one stream.
    Overlapped: the shared MLP runs on a second stream from the start of the
    step; combine waits for both.  Medians of 20 runs, L2 flushed before
    each; the two combine outputs must be identical."""
    T, H = x.shape
    g = torch.Generator(device=dev).manual_seed(20260100)
    w1 = (torch.randn((H, 2048), generator=g, device=dev) * H ** -0.5).to(torch.bfloat16)
    w2 = (torch.randn((2048, H), generator=g, device=dev) * 2048 ** -0.5).to(torch.bfloat16)
    sh = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    hid = torch.empty((T, 2048), dtype=torch.bfloat16, device=dev)
    outs = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    st = ops.new_status(dev)
    side = torch.cuda.Stream(device=dev)

    def mlp():
        torch.matmul(x, w1, out=hid)
        torch.nn.functional.silu(hid, inplace=True)
        torch.matmul(hid, w2, out=sh)

    def sequential():
        ops.moe_dispatch_layout(ids, E, R, layout=L, status=st)
        ops.moe_dispatch_permute(x, L, xp=xp, status=st)
        mlp()
        ops.moe_combine(xp, L.dst_row, sc, shared_x=sh, out=outs[0], status=st)

    def overlapped():
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            mlp()
        ops.moe_dispatch_layout(ids, E, R, layout=L, status=st)
        ops.moe_dispatch_permute(x, L, xp=xp, status=st)
        stream.wait_stream(side)
        ops.moe_combine(xp, L.dst_row, sc, shared_x=sh, out=outs[1], status=st)

    t = time_calls(torch, [("mlp_alone", mlp), ("layout_permute", lambda: (
        ops.moe_dispatch_layout(ids, E, R, layout=L, status=st),
        ops.moe_dispatch_permute(x, L, xp=xp, status=st))),
        ("sequential", sequential), ("overlapped", overlapped)], flush, 20, stream)
    torch.cuda.synchronize()
    if ops.read_status(st) != 0:
        raise RuntimeError(f"device status {ops.read_status(st)} in the shared-expert runs")
    flops = 2 * 2 * T * H * 2048
    return {"what": "layout + permute with a shared-expert MLP stand-in (x @ W1 -> silu -> @ W2, "
                    "width 2048, torch/cuBLAS bf16) on a second stream, then combine with "
                    "shared_x",
            "us": {k: round(v, 1) for k, v in t.items()},
            "mlp_tflops": round(flops / (t["mlp_alone"] * 1e-6) / 1e12, 1),
            "gain": round(1 - t["overlapped"] / t["sequential"], 3),
            "outputs_identical": bool(torch.equal(outs[0], outs[1]))}


def extra_workloads(args, dev, flush, stream):
    """Per-call device times on the other workloads (prefill FP8 dispatch,
    shared-expert combine, skewed backward), reported beside the step."""
    import torch
    from combine_moe_dispatch_05_b200 import ops
    from combine_moe_dispatch_05_b200 import workloads as W
    steps = 10
    res = {}

    # prefill: FP8 dispatch (quantise then permute, and the fused call), bf16 combine
    s = W.config(3)
    T, H, E, K, R = s.T, s.H, s.E, s.K, s.R
    ids = W.topk_ids(s).to(dev)
    x = W.tokens(s, device=dev)
    L = ops.moe_dispatch_layout(ids, E, R)
    q, qs = ops.moe_quantize_e4m3(x)
    xp, xps = ops.moe_dispatch_permute(q, L, x_scales=qs)
    y = W.expert_out(s, L.P_cap, device=dev)
    sc = W.topk_scales(s).to(dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    P = int(L.expert_offsets[E])
    nb = H // 128
    t = time_calls(torch, [
        ("layout", lambda: ops.moe_dispatch_layout(ids, E, R, layout=L)),
        ("quantize", lambda: ops.moe_quantize_e4m3(x, q=q, q_scales=qs)),
        ("permute_e4m3", lambda: ops.moe_dispatch_permute(q, L, xp=xp, x_scales=qs,
                                                          xp_scales=xps)),
        ("permute_quant_fused", lambda: ops.moe_dispatch_permute_quant(x, L, xp=xp,
                                                                       xp_scales=xps)),
        ("combine", lambda: ops.moe_combine(y, L.dst_row, sc, out=out)),
        # the forward pass as one chained step: layout, fused FP8 dispatch, combine
        ("fwd_step", lambda: (ops.moe_dispatch_layout(ids, E, R, layout=L),
                              ops.moe_dispatch_permute_quant(x, L, xp=xp, xp_scales=xps),
                              ops.moe_combine(y, L.dst_row, sc, out=out))),
    ], flush, steps, stream)
    b = {"layout": 8 * T * K + 4 * P, "quantize": 2 * T * H + T * H + 4 * T * nb,
         "permute_e4m3": T * H + 4 * T * nb + P * H + 4 * P * nb,
         "permute_quant_fused": 2 * T * H + P * H + 4 * P * nb,
         "combine": 2 * T * K * H + 8 * T * K + 2 * T * H}
    b["fwd_step"] = b["layout"] + b["permute_quant_fused"] + b["combine"]
    res[s.name] = {"T": T, "H": H, "E": E, "K": K, "P": P,
                   "us": {k: round(v, 1) for k, v in t.items()},
                   "GBps": {k: round(b[k] / (t[k] * 1e-6) / 1e9, 1) for k in t},
                   "dispatch_unfused_us": round(t["quantize"] + t["permute_e4m3"], 1),
                   "dispatch_fused_us": round(t["permute_quant_fused"], 1),
                   "fwd_step_tokens_per_s": round(T / (t["fwd_step"] * 1e-6), 1)}
    del x, q, qs, xp, xps, y, out, L
    torch.cuda.empty_cache()

    # shared expert: bf16 dispatch + combine with the unweighted shared term
    s = W.config(4)
    T, H, E, K, R = s.T, s.H, s.E, s.K, s.R
    ids = W.topk_ids(s).to(dev)
    x = W.tokens(s, device=dev)
    L = ops.moe_dispatch_layout(ids, E, R)
    xp = ops.moe_dispatch_permute(x, L)
    y = W.expert_out(s, L.P_cap, device=dev)
    sh = W.shared_out(s, device=dev)
    sc = W.topk_scales(s).to(dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    P = int(L.expert_offsets[E])
    t = time_calls(torch, [
        ("layout", lambda: ops.moe_dispatch_layout(ids, E, R, layout=L)),
        ("permute", lambda: ops.moe_dispatch_permute(x, L, xp=xp)),
        ("combine_shared", lambda: ops.moe_combine(y, L.dst_row, sc, shared_x=sh, out=out)),
        ("fwd_step", lambda: (ops.moe_dispatch_layout(ids, E, R, layout=L),
                              ops.moe_dispatch_permute(x, L, xp=xp),
                              ops.moe_combine(y, L.dst_row, sc, shared_x=sh, out=out))),
    ], flush, steps, stream)
    b = {"layout": 8 * T * K + 4 * P, "permute": 2 * T * H + 2 * P * H,
         "combine_shared": 2 * T * K * H + 8 * T * K + 4 * T * H}
    b["fwd_step"] = b["layout"] + b["permute"] + b["combine_shared"]
    res[s.name] = {"T": T, "H": H, "E": E, "K": K, "P": P,
                   "us": {k: round(v, 1) for k, v in t.items()},
                   "GBps": {k: round(b[k] / (t[k] * 1e-6) / 1e9, 1) for k in t}}
    if not args.no_cpu_baseline:
        # the last timed combine's output and its inputs, for the check of its
        # elements against the exact sum (done on the host after the GPU work)
        res[s.name]["_combine_snapshot"] = {
            "out": W.as_u16(out.cpu()), "y": W.as_u16(y.cpu()), "dst_row": L.dst_row.cpu().numpy(),
            "scales": sc.cpu().numpy(), "shared": W.as_u16(sh.cpu())}
    del x, xp, y, sh, out, L
    torch.cuda.empty_cache()

    # backward under skew: the hot expert in 60% of the rows, and the stress
    # variant with it in every row
    for name, spec in (("bwd_skew", W.config(5)),
                       ("bwd_skew_hot100", W.config(5).with_(hot_p=1.0))):
        s = spec
        T, H, E, K, R = s.T, s.H, s.E, s.K, s.R
        ids = W.topk_ids(s).to(dev)
        L = ops.moe_dispatch_layout(ids, E, R)
        y = W.expert_out(s, L.P_cap, device=dev)
        g = W.grad_out(s, device=dev)
        sc = W.topk_scales(s).to(dev)
        gy = torch.empty_like(y)
        gs = torch.empty((T, K), dtype=torch.float32, device=dev)
        gx = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        P = int(L.expert_offsets[E])
        t = time_calls(torch, [
            ("layout", lambda: ops.moe_dispatch_layout(ids, E, R, layout=L)),
            ("combine_bwd", lambda: ops.moe_combine_bwd(g, y, sc, L, grad_y=gy, grad_scales=gs)),
            ("dispatch_bwd", lambda: ops.moe_dispatch_bwd(gy, L.dst_row, T, K, grad_x=gx)),
            ("bwd_step", lambda: (ops.moe_combine_bwd(g, y, sc, L, grad_y=gy, grad_scales=gs),
                                  ops.moe_dispatch_bwd(gy, L.dst_row, T, K, grad_x=gx))),
        ], flush, steps, stream)
        b = {"layout": 8 * T * K + 4 * P,
             "combine_bwd": 2 * T * H + 2 * T * K * H + 2 * P * H + 12 * T * K,
             "dispatch_bwd": 2 * T * K * H + 2 * T * H + 4 * T * K}
        b["bwd_step"] = b["combine_bwd"] + b["dispatch_bwd"]
        res[name] = {"T": T, "H": H, "E": E, "K": K, "P": P, "hot_p": s.hot_p,
                     "us": {k: round(v, 1) for k, v in t.items()},
                     "GBps": {k: round(b[k] / (t[k] * 1e-6) / 1e9, 1) for k in t}}
    return res


def plan_on(L, E, R, ops):
    """Host balance planner on this step's per-expert counts (token-bound cost
    model: beta * N dominates b * G)."""
    counts = L.expert_counts.cpu().tolist()
    cost = dict(a=0.0, b=5.0, b2=1.0, c=0.0, beta=1.0, mig=0.01)
    t0 = time.perf_counter()
    moves, before, after = ops.moe_plan_balance(counts, R, max_moves=128, **cost)
    us = (time.perf_counter() - t0) * 1e6
    G = sum(1 for n in counts if n > 0)
    N = sum(counts)
    ideal = max(cost["a"] + cost["b"] * G / R, cost["c"] + cost["beta"] * N / R)
    return {"cost_model": cost, "moves": len(moves), "makespan_before": before,
            "makespan_after": after, "ideal_lower_bound": ideal,
            "ideal_over_after": round(ideal / after, 4), "host_us": round(us, 1)}


# --------------------------------------------------------- oracle timing --
def oracle_step_sample(T_sample: int, fwd_only: bool):
    """One pass of the oracle over the first T_sample tokens of the workload.
    Returns (seconds, algorithmic bytes of the sample)."""
    import numpy as np
    import torch

    import oracle
    from combine_moe_dispatch_05_b200 import workloads as W

    s = W.config(CONFIG_INDEX)
    ids = W.topk_ids(s)[:T_sample].numpy()
    sc = W.topk_scales(s)[:T_sample].numpy()
    x = W.as_u16(W.tokens(s.with_(T=T_sample)))
    g = W.as_u16(W.grad_out(s.with_(T=T_sample)))
    t0 = time.perf_counter()
    L = oracle.layout(ids, s.E, s.R)
    xp = np.zeros((L.P_cap, s.H), np.uint16)
    oracle.permute_rows(x, L.dst_row, s.K, L.counts, L.offsets, xp)
    oracle.combine(xp, L.dst_row, sc, None)
    if not fwd_only:
        gy = np.zeros_like(xp)
        oracle.combine_bwd(g, xp, sc, L.dst_row, L.counts, L.offsets, gy)
        oracle.dispatch_bwd(gy, L.dst_row, T_sample, s.K)
    dt = time.perf_counter() - t0
    b = sum(step_bytes(T_sample, s.K, s.H, s.E, L.P, fwd_only).values())
    return dt, b, s


def host_cpu():
    """(threads this process may run on, CPU model name)."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return n, model


def oracle_pass_partitioned(s, ids, sc, x, g, fwd_only, threads):
    """One pass of the oracle over all s.T tokens with the tokens split into
    `threads` contiguous ranges, one per host thread; the layout stays
    serial.  The oracle's C loops run unchanged on each range (ctypes drops
    the GIL for the call), and only the first range writes the padding rows.
    Returns (seconds, outputs)."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle

    K = s.K
    cuts = [s.T * i // threads for i in range(threads + 1)]
    parts = [(i, cuts[i], cuts[i + 1]) for i in range(threads) if cuts[i + 1] > cuts[i]]
    with ThreadPoolExecutor(max_workers=max(len(parts), 1)) as pool:
        def each(fn):
            list(pool.map(lambda p: fn(*p), parts))

        t0 = time.perf_counter()
        L = oracle.layout(ids, s.E, s.R)
        no_pad = np.diff(L.offsets).astype(np.int32)  # counts that leave no padding row
        xp = np.zeros((L.P_cap, s.H), np.uint16)
        out = np.empty((s.T, s.H), np.uint16)
        each(lambda i, a, b: oracle.permute_rows(x[a:b], L.dst_row[a * K:b * K], K,
                                                 L.counts if i == 0 else no_pad, L.offsets, xp))

        def comb(i, a, b):
            out[a:b] = oracle.combine(xp, L.dst_row[a * K:b * K], sc[a:b], None)
        each(comb)
        res = {"layout": L, "xp": xp, "out": out}
        if not fwd_only:
            gy = np.zeros_like(xp)
            gs = np.empty((s.T, K), np.float32)
            gx = np.empty((s.T, s.H), np.uint16)

            def cbwd(i, a, b):
                gs[a:b] = oracle.combine_bwd(g[a:b], xp, sc[a:b], L.dst_row[a * K:b * K],
                                             L.counts if i == 0 else no_pad, L.offsets, gy)
            each(cbwd)

            def dbwd(i, a, b):
                gx[a:b] = oracle.dispatch_bwd(gy, L.dst_row[a * K:b * K], b - a, K)
            each(dbwd)
            res.update(grad_y=gy, grad_scales=gs, grad_x=gx)
        dt = time.perf_counter() - t0
    return dt, res


def bf16_max_ulp(gpu_bits, ref_bits):
    """Largest |gpu - ref| over all elements, in units of one bf16 ulp of ref
    (ulp of a normal r = 2^(floor(log2|r|) - 7); of zero, the smallest
    subnormal)."""
    import numpy as np

    def f(b):
        return (np.asarray(b).view(np.uint16).astype(np.uint32) << 16).view(np.float32) \
            .astype(np.float64)
    g, r = f(gpu_bits), f(ref_bits)
    a = np.abs(r)
    ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 7), 2.0 ** -133)
    return float(np.max(np.abs(g - r) / ulp)) if g.size else 0.0


def combine_exceptions(out_bits, y_bits, dst_row, scales, shared_bits=None, chunk=256):
    """Elements of a combine output farther than one bf16 ulp (2^-7 |exact|)
    from the exact sum (fp64), and how many of those are NOT cancellation
    cases.  An fp32 running sum of n terms is within gamma_n * sum|terms| of
    the exact sum, and rounding it once to bf16 adds at most 2^-8 of its
    magnitude, so an element can pass one ulp only where
    |exact| < 257 * gamma_n * sum|terms| (n = K, plus one with a shared
    term): those are the cancellation cases; any other exception is a bug."""
    import numpy as np

    def f(b):
        return (np.asarray(b).view(np.uint16).astype(np.uint32) << 16).view(np.float32) \
            .astype(np.float64)
    T, K = scales.shape
    n = K + (0 if shared_bits is None else 1)
    gam = n * 2.0 ** -24 / (1 - n * 2.0 ** -24)
    rows = np.asarray(dst_row)[:T * K].reshape(T, K)
    over = not_cancel = 0
    for a in range(0, T, chunk):
        b = min(T, a + chunk)
        yv = f(y_bits[rows[a:b]])                              # [c, K, H]
        sv = scales[a:b].astype(np.float64)
        exact = np.einsum("tk,tkh->th", sv, yv)
        mag = np.einsum("tk,tkh->th", np.abs(sv), np.abs(yv))
        if shared_bits is not None:
            sh = f(shared_bits[a:b])
            exact += sh
            mag += np.abs(sh)
        o = np.abs(f(out_bits[a:b]) - exact) > 2.0 ** -7 * np.abs(exact)
        over += int(o.sum())
        not_cancel += int((o & (np.abs(exact) >= 257 * gam * mag + 2.0 ** -126)).sum())
    return {"elements": int(T * y_bits.shape[1]), "over_one_ulp_of_exact": over,
            "over_one_ulp_not_cancellation": not_cancel}


def check_timed_outputs(s, res, gpu, x, g, fwd_only):
    """The last timed GPU step against the oracle's pass over the same inputs:
    integers and the permuted bytes must be identical; the bf16 outputs are
    reported as their largest error in bf16 ulps, grad_scales as its largest
    error relative to |g_t|*|y_row| (which bounds the sum of |terms|)."""
    import numpy as np

    L = res["layout"]
    K = s.K
    chk = {"layout_bit_exact": bool(
        np.array_equal(gpu["counts"], L.counts) and np.array_equal(gpu["offsets"], L.offsets)
        and np.array_equal(gpu["dst_row"][:s.T * K], L.dst_row)
        and np.array_equal(gpu["row_src"][:L.P_cap], L.row_src[:L.P_cap])
        and np.array_equal(gpu["rank_counts"], L.rank_counts)
        and np.array_equal(gpu["rank_offsets"], L.rank_offsets))}
    P = L.P
    chk["permute_bytes_exact"] = bool(gpu["xp"].shape[0] == P and np.array_equal(
        gpu["xp"].view(np.uint16), res["xp"][:P]))
    chk["combine_max_ulp"] = round(bf16_max_ulp(gpu["out"], res["out"]), 3)
    chk["combine_vs_exact_sum"] = combine_exceptions(gpu["out"], res["xp"], L.dst_row,
                                                     gpu["scales"])
    if not fwd_only:
        chk["combine_bwd_grad_y_max_ulp"] = round(
            bf16_max_ulp(gpu["grad_y"], res["grad_y"][:P]), 3)
        chk["combine_bwd_grad_y_bit_exact"] = bool(np.array_equal(
            gpu["grad_y"].view(np.uint16), res["grad_y"][:P]))
        chk["dispatch_bwd_max_ulp"] = round(bf16_max_ulp(gpu["grad_x"], res["grad_x"]), 3)

        def f(b):
            return (b.view(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        gn = np.linalg.norm(f(g), axis=1)                        # [T]
        yn = np.linalg.norm(f(res["xp"]), axis=1)                # [P_cap]
        rows = L.dst_row.reshape(s.T, K)
        scale = np.maximum(gn[:, None] * yn[rows], 1e-30)
        err = np.abs(gpu["grad_scales"].astype(np.float64) - res["grad_scales"].astype(np.float64))
        chk["grad_scales_max_err_over_norms"] = float(np.max(err / scale))
    chk["what"] = ("outputs of the last timed step against the oracle's pass over the same "
                   "inputs (identity experts)")
    return chk


def cpu_baseline_all_cores(fwd_only, timed_outputs=None):
    """The whole workload (every token of one step) through the oracle on all
    host threads, token-partitioned.  Returns (baseline, check of the timed
    GPU outputs against this pass, or None)."""
    from combine_moe_dispatch_05_b200 import workloads as W

    n, model = host_cpu()
    s = W.config(CONFIG_INDEX)
    ids = W.topk_ids(s).numpy()
    sc = W.topk_scales(s).numpy()
    x = W.as_u16(W.tokens(s))
    g = W.as_u16(W.grad_out(s))
    dt, res = oracle_pass_partitioned(s, ids, sc, x, g, fwd_only, n)
    b = sum(step_bytes(s.T, s.K, s.H, s.E, res["layout"].P, fwd_only).values())
    base = {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": n, "kind": "oracle",
            "cpu_model": model, "seconds": round(dt, 3), "tokens_per_s": round(s.T / dt, 1),
            "sample": f"all {s.T} tokens of one {'fwd' if fwd_only else 'fwd+bwd'} step, the "
                      f"C oracle's loops run on {n} contiguous token ranges in parallel "
                      f"(layout serial)"}
    chk = None if timed_outputs is None else check_timed_outputs(s, res, timed_outputs, x, g,
                                                                  fwd_only)
    return base, chk


ORACLE_SAMPLE_TOKENS = 1024


def cpu_baseline(fwd_only):
    dt, b, s = oracle_step_sample(ORACLE_SAMPLE_TOKENS, fwd_only)
    return {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "cpu_model": host_cpu()[1], "host_threads": host_cpu()[0], "seconds": round(dt, 3),
            "tokens_per_s": round(ORACLE_SAMPLE_TOKENS / dt, 1),
            "sample": f"first {ORACLE_SAMPLE_TOKENS} of the {s.T} tokens of the same workload, "
                      f"one full {'fwd' if fwd_only else 'fwd+bwd'} pass of the single-threaded "
                      f"C oracle"}


REFERENCE_BUDGET_S = 150.0


def run_reference(args):
    """The oracle, as it stands, on the host: each step is one pass over a
    token sample of the workload, sized so the whole run stays within about
    REFERENCE_BUDGET_S seconds."""
    from combine_moe_dispatch_05_b200 import workloads as W
    s = W.config(CONFIG_INDEX)
    probe_tokens = 64
    dt, _, _ = oracle_step_sample(probe_tokens, args.fwd_only)      # untimed probe
    per_token = dt / probe_tokens
    n_steps = args.steps + max(0, args.warmup - 1)
    sample = int(REFERENCE_BUDGET_S / max(n_steps, 1) / per_token)
    sample = max(16, min(ORACLE_SAMPLE_TOKENS, sample))
    for _ in range(max(0, args.warmup - 1)):
        oracle_step_sample(sample, args.fwd_only)
    tot, tot_b = 0.0, 0
    for _ in range(args.steps):
        dt, b, _ = oracle_step_sample(sample, args.fwd_only)
        tot += dt
        tot_b += b
    v = tot_b / tot / 1e9
    ms = 1e3 * tot / args.steps
    desc = (f"first {sample} of the {s.T} tokens per step, single-threaded C oracle, "
            f"{'fwd' if args.fwd_only else 'fwd+bwd'}")
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "GB/s",
            "tokens_per_s": round(sample / (ms * 1e-3), 1), "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"{s.name}: T={s.T} H={s.H} E={s.E} K={s.K} R={s.R} "
                                   f"Zipf(s={s.zipf_s}) {'fwd' if args.fwd_only else 'fwd+bwd'}",
                       "sample_tokens": sample},
            "cpu_baseline": {"value": round(v, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(v, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world, rank, local = dist_env()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        res = run_ours(args, world, rank, local)
        timed = res.pop("_timed_outputs", None)
        shared_snap = res.get("other_workloads", {}).get("shared_expert", {}).pop(
            "_combine_snapshot", None)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args.fwd_only)
            res["cpu_baseline_all_cores"], res["timed_run_check"] = \
                cpu_baseline_all_cores(args.fwd_only, timed)
            if shared_snap is not None:
                res["timed_run_check"]["shared_expert_combine_vs_exact_sum"] = \
                    combine_exceptions(shared_snap["out"], shared_snap["y"],
                                       shared_snap["dst_row"], shared_snap["scales"],
                                       shared_snap["shared"])
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
