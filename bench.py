#!/usr/bin/env python
"""Throughput of the balanced expert-parallel hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
mep_plan (T_e, maxvio, offsets, stable scatter, segments, replicas) ->
mep_dispatch -> mep_combine -> mep_reduce_replica_grads, all through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mep|reference]

* value: tokens per second of the whole job (tokens of all ranks / max-over-ranks
  device time), inputs resident in HBM, L2 flushed between steps outside the
  timed events (a 512 MB write, then a 512 MB read that writes the fill's
  dirty lines back, so no timed kernel pays for the flush's write-back).  The
  step is captured once in a CUDA graph and replayed (``eager`` keeps the
  launch-by-launch timing, whose per-kernel events give the roofline
  breakdown).
* e2e: the same metric through the public API with pinned host buffers: every
  step copies that step's inputs host->device and its outputs (combine
  output, home gradients, plan scalars) back; consecutive steps overlap on
  separate copy and compute streams.
* roofline: the step's dominant kernel, algorithmic bytes / its mean event
  time, against the measured HBM copy peak.
* cpu_baseline / --impl reference: the CPU oracle, single-threaded, on a
  bounded sample of the same workload, scaled to tokens per second.
Multi-GPU (torchrun): every rank runs an independent replica of the
single-device problem ("replicas only"); timing is the max over ranks.
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

import workloads  # noqa: E402

METRIC = "plan+dispatch+combine tokens/sec and HBM GB/s (% of roofline), 1 B200"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # the nominal HBM3e figure (8 TB/s), reported beside the measured one
FLUSH_BYTES = 512 << 20
KERNEL_SOURCES = {"plan": "plan.cu", "dispatch": "dispatch.cu", "combine": "combine.cu",
                  "reduce": "reduce.cu"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mep", "reference"], default="mep")
    ap.add_argument("--workload", default=workloads.BENCH_WORKLOAD,
                    choices=list(workloads.WORKLOADS))
    ap.add_argument("--S", type=int, default=None,
                    help="tokens per rank (default: the workload's); for small profiling cases")
    ap.add_argument("--P", type=int, default=None,
                    help="gradient row length (default: the workload's); for small profiling cases")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the CUDA-graph replay timing of the step")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the separately timed backward kernels")
    ap.add_argument("--no-exchange", action="store_true",
                    help="skip the timing of the per-rank (rank-addressed) exchange calls")
    ap.add_argument("--dispatch-form", choices=["register", "bulk"], default="register",
                    help="dispatch through registers (mep_dispatch) or the bulk-copy engine "
                         "(mep_dispatch_bulk, the staged form kept for comparison)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_sha(name: str) -> str:
    p = os.path.join(ROOT, "token_dispatch_mep_b200", "csrc", KERNEL_SOURCES[name])
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:12]


def dram_traffic(name: str, workload: str):
    """Per-launch DRAM bytes of `name` on `workload` from the committed ncu
    summary, or None if absent or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = kernel_sha(name)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == name \
                    and parts[1] == workload and parts[3] == sha:
                return float(parts[2])
    return None


def host_pin_budget(ranks_on_node: int) -> int:
    """Bytes of pinned host memory one rank may take for the end-to-end
    inputs: half the node's available memory, shared by its ranks."""
    import psutil
    return int(0.5 * psutil.virtual_memory().available / max(1, ranks_on_node))


def pinned_sources(tensors: dict, budget: int, pin: bool = True):
    """Pinned host copies of the device tensors in `tensors` (None entries
    pass through): whole while they fit `budget` bytes together, otherwise
    each holds its first rows only, in proportion.  Returns the copies in
    order and a description of each source."""
    import torch
    big = {k: t for k, t in tensors.items() if t is not None}
    total = sum(t.numel() * t.element_size() for t in big.values())
    frac = 1.0 if total <= budget else max(budget, 0) / total
    out, desc = [], {}
    for k, t in tensors.items():
        if t is None:
            out.append(None)
            continue
        n = t.shape[0]
        m = n if frac >= 1.0 else max(1, min(n, int(n * frac)))
        h = torch.empty((m,) + tuple(t.shape[1:]), dtype=t.dtype, pin_memory=pin).copy_(t[:m])
        out.append(h)
        desc[k] = ("pinned whole" if m == n else
                   f"first {m} of {n} rows pinned, copied {(n + m - 1) // m} times per step")
    return out[0], out[1], desc


def copy_rows(dst, src):
    """dst[:] = src repeated over dst's rows (host -> device, on the current
    stream, asynchronous)."""
    n, m = dst.shape[0], src.shape[0]
    for r0 in range(0, n, m):
        r1 = min(n, r0 + m)
        dst[r0:r1].copy_(src[:r1 - r0], non_blocking=True)


# ------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples the SM clock and the clock-event reasons with NVML every
    ~10 ms in a background thread (reads only; changes no setting)."""

    BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            try:
                props = torch.cuda.get_device_properties(device_index)
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = get_reasons(self._h)
                for bit, name in self.BITS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def start(self):
        if self._h is not None:
            self._t.start()
        return self

    def stop(self):
        self._stop.set()
        if self._h is not None:
            self._t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------- multi-rank

def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (the step time of the slowest
    replica); a no-op for one rank."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_replicas_max(plan_host: dict, experts_per_rank: int, R: int) -> int:
    """Most replica segments on one rank, from a host copy of a plan."""
    seg = np.asarray(plan_host["seg"])[:plan_host["num_seg"]]
    rep = seg[seg[:, 1] != seg[:, 0] // experts_per_rank]
    return int(np.bincount(rep[:, 1], minlength=R).max()) if len(rep) else 0


def whole_job_rate(tokens_per_rank: int, world: int, ms: float) -> float:
    """Tokens per second of all replicas together, timed by the slowest."""
    return tokens_per_rank * world / (ms * 1e-3)


# ------------------------------------------------------------ config

L2_NOTE = ("flushed between steps, outside the events: a 512 MB write, then a 512 MB read "
           "that writes the fill's dirty lines back")


def bench_config(wl, world: int) -> dict:
    """The workload's `config`, identical in both arms' lines."""
    return {"workload": wl.name, "R": wl.R, "S": wl.S, "E": wl.E, "K": wl.K, "H": wl.H,
            "P": wl.P,
            "step": "plan+dispatch+combine" + ("+replica-grad reduce" if wl.P else ""),
            "l2": L2_NOTE, "parallelism": f"replicas x{world}"}


# ------------------------------------------------------------ CPU oracle leg

# Host bytes above which the combine sample reads a folded copy of the
# expert outputs (see oracle_throughput).
Y_HOST_LIMIT = 2 << 30


def oracle_throughput(wl, target_seconds: float, host=None):
    """Time the oracle, as it stands, on a bounded sample of the workload:
    the whole plan; dispatch of the first n slots and combine of the first n
    tokens, both through the plan's own src_pair / slot (so rows are read
    and written in the plan's scattered order); the reduction of the first c
    gradient columns; scaled to tokens per second of the full step.
    Single-threaded C.  Where the expert outputs would exceed Y_HOST_LIMIT
    bytes of host memory, the combine reads them from M rows (M*H*2 bytes
    just under the limit, far larger than the host's caches) at slot mod M."""
    import oracle
    import torch
    ora = oracle.get()
    R, S, E, K, H, P, N, NK = wl.R, wl.S, wl.E, wl.K, wl.H, wl.P, wl.N, wl.NK
    if host is None:
        idx, w = workloads.routing(wl)
        host = dict(idx=idx, w=w)
    idx, w = host["idx"], host["w"]
    # size the samples from the budget (about 12 ns per combine term, 3 ns per
    # reduced element on this kind of host core)
    per_tok = K * H * 12.5e-9
    n_tok = int(max(1, min(N, (0.5 * target_seconds) / per_tok)))
    n_slot = min(NK, n_tok * K)
    n_col = int(max(1, min(P, (0.4 * target_seconds) / (3.2e-9 * (wl.seg_rows + E))))) if P else 0
    m_rows = int(min(NK, max(1, Y_HOST_LIMIT // (2 * H))))
    # the synthetic inputs are generated once per workload and kept in `host`
    # (untimed); a later call with a larger sample regenerates the gradients
    u16 = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    if "plan" not in host:
        host["plan"] = ora.plan(R, S, E, K, idx)
        host["x"] = u16(workloads.hidden(N, H, seed=1))
        host["y"] = u16(workloads.expert_outputs(m_rows, H, seed=2))
    if P and host.get("G_cols", 0) < n_col:
        host["G"] = workloads.seg_grads(wl.seg_rows, n_col, seed=3).numpy()
        host["G_cols"] = n_col
    pl, x, y = host["plan"], host["x"], host["y"]
    src = np.ascontiguousarray(pl["src_pair"][:n_slot])
    slot = np.ascontiguousarray(pl["slot"][:n_tok] % m_rows).astype(np.int32)
    G = np.ascontiguousarray(host["G"][:, :n_col]) if P else None
    # Where the sample is the whole workload and takes less than the budget,
    # it is repeated (at most 8 times) and the median repetition is reported.
    reps, measured = [], 0.0
    while not reps or (measured < 0.8 * target_seconds and len(reps) < 8):
        t0 = time.perf_counter()
        pl = ora.plan(R, S, E, K, idx)
        t_plan = time.perf_counter() - t0
        t0 = time.perf_counter()
        ora.dispatch(K, src, x)
        t_disp = time.perf_counter() - t0
        t0 = time.perf_counter()
        ora.combine(slot, w[:n_tok], y)
        t_comb = time.perf_counter() - t0
        t_red = 0.0
        if P:
            t0 = time.perf_counter()
            ora.reduce(pl["expert_seg_ptr"], G)
            t_red = time.perf_counter() - t0
        t_step = (t_plan + t_disp * (NK / n_slot) + t_comb * (N / n_tok)
                  + (t_red * (P / n_col) if P else 0.0))
        reps.append((t_step, dict(plan=t_plan, dispatch=t_disp, combine=t_comb, reduce=t_red)))
        measured += t_plan + t_disp + t_comb + t_red
    reps.sort(key=lambda r: r[0])
    t_step, parts = reps[len(reps) // 2]
    fold = "" if m_rows == NK else f" (expert outputs folded to {m_rows} rows: slot mod {m_rows})"
    sample = (f"whole plan; dispatch of {n_slot}/{NK} slots via the plan's src_pair; "
              f"combine of {n_tok}/{N} tokens via the plan's slots{fold}; "
              + (f"reduce of {n_col}/{P} gradient columns; " if P else "")
              + f"scaled to the full step; median of {len(reps)} repetition(s)")
    return dict(value=N / t_step, t_step=t_step, sample=sample, measured_s=measured,
                repetitions=len(reps), parts=parts)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workloads.WORKLOADS[args.workload]
    idx, w = workloads.routing(wl)
    host = dict(idx=idx, w=w)
    budget = max(0.5, min(4.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_throughput(wl, budget, host)
    vals = [oracle_throughput(wl, budget, host) for _ in range(max(1, args.steps))]
    t = statistics.mean(v["t_step"] for v in vals)
    value = wl.N / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, args.gpus),
        "timing": "host wall clock (time.perf_counter) around each oracle call",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": vals[0]["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- GPU arm

def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    import token_dispatch_mep_b200 as mep

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = workloads.WORKLOADS[args.workload]
    if args.S is not None or args.P is not None:
        wl = workloads.reduced(wl, S=args.S or wl.S, P=args.P if args.P is not None else wl.P)
    R, S, E, K, H, P, N, NK = wl.R, wl.S, wl.E, wl.K, wl.H, wl.P, wl.N, wl.NK
    s = mep.Shape(R, S, E, K)
    idx_h, w_h = workloads.routing(wl, seed=0)
    idx = torch.from_numpy(idx_h).to(dev)
    w = torch.from_numpy(w_h).to(dev)
    x = workloads.hidden(N, H, seed=1, device=dev)
    y = workloads.expert_outputs(NK, H, seed=2, device=dev)
    G = workloads.seg_grads(wl.seg_rows, P, seed=3, device=dev) if P else None
    plan = mep.Plan(s, dev)
    buf = torch.empty((R, S * K, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    home = torch.empty((E, P), dtype=torch.float32, device=dev) if P else None
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)

    def flush_l2():
        # A write larger than L2 evicts every line of the step's inputs and
        # outputs; the read of a second buffer larger than L2 then writes back
        # the fill's own dirty lines, so the timed kernels start from a cold,
        # clean L2 and pay for no one else's write-back.
        flush.zero_()
        clean.sum()

    dispatch = mep.mep_dispatch_bulk if args.dispatch_form == "bulk" else mep.mep_dispatch

    def step(evs=None):
        if evs:
            evs[0].record()
        mep.mep_plan(s, idx, plan)
        if evs:
            evs[1].record()
        dispatch(s, H, plan, x, buf)
        if evs:
            evs[2].record()
        mep.mep_combine(s, H, plan, y, w, out)
        if evs:
            evs[3].record()
        if P:
            mep.mep_reduce_replica_grads(s, plan, P, G, home)
        if evs:
            evs[4].record()

    launches_per_step = 4 if P else 3
    for _ in range(max(3, args.warmup)):
        flush_l2()
        step()
    torch.cuda.synchronize()
    if mep.mep_read_status(plan) != 0:
        raise RuntimeError("device status not OK after warm-up")
    num_seg = plan.host()["num_seg"]

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local).start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2()
        step(evs[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    st = mep.mep_read_status(plan)
    if st != 0:
        raise RuntimeError(f"device status {mep.mep_status_string(st)}")

    stage = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)]
                      for i in range(args.steps)])          # ms
    ms_step = max_over_ranks(float(stage.sum(axis=1).mean()), world, dev)
    value = whole_job_rate(N, world, ms_step)

    stage_ms = dict(zip(["plan", "dispatch", "combine", "reduce"], stage.mean(axis=0).tolist()))
    # plan + dispatch + combine alone (the rate the metric names), slowest rank
    pdc_ms = max_over_ranks(stage_ms["plan"] + stage_ms["dispatch"] + stage_ms["combine"], world, dev)
    algo = {
        "plan": 3 * NK * 4,
        "dispatch": N * H * 2 + NK * H * 2 + NK * 4,
        "combine": NK * H * 2 + NK * 4 + NK * 4 + N * H * 2,
        "reduce": (num_seg + E) * P * 4,
    }
    peak, peak_kind = measured_peak()
    kernels = {}
    for k in ("plan", "dispatch", "combine", "reduce"):
        if k == "reduce" and not P:
            continue
        gbs = algo[k] / (stage_ms[k] * 1e-3) / 1e9
        kernels[k] = {"ms": stage_ms[k], "bytes": algo[k], "gbs": gbs, "frac": gbs / peak,
                      "frac_nominal": gbs / NOMINAL_HBM_GBS}
    dom = max((k for k in kernels if k != "plan"), key=lambda k: kernels[k]["ms"])
    roofline = {"bound": "hbm", "achieved": kernels[dom]["gbs"], "peak": peak, "unit": "GB/s",
                "frac": kernels[dom]["gbs"] / peak, "traffic": dram_traffic(dom, wl.name),
                "kernel": dom, "peak_source": f"{peak_kind} hbm_gbs (copy)"}

    # ---- the home-first (low-replica) plan: latency and replica count
    home_first = None
    capped = None
    if not args.no_backward:
        hf = mep.Plan(s, dev)
        hts = []
        for it in range(3 + 20):
            flush_l2()
            h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            h0.record()
            mep.mep_plan_home_first(s, idx, hf)
            h1.record()
            if it >= 3:
                hts.append((h0, h1))
        torch.cuda.synchronize()
        if mep.mep_read_status(hf) != 0:
            raise RuntimeError("device status not OK after the home-first plan")
        hh = hf.host()
        home_first = {"plan_us": float(np.median([a.elapsed_time(b) for a, b in hts])) * 1e3,
                      "num_replicas": hh["num_replicas"], "num_seg": hh["num_seg"],
                      "num_replicas_contiguous": plan.host()["num_replicas"]}
        # the capped plan at the pages' two values of B (training E/R,
        # inference 4): latency, replicas, and the most replicas on one rank
        capped = {}
        for B in (E // R, 4):
            mr = torch.zeros(1, dtype=torch.int32, device=dev)
            cts = []
            for it in range(3 + 20):
                flush_l2()
                h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                h0.record()
                mep.mep_plan_capped(s, B, idx, hf, mr)
                h1.record()
                if it >= 3:
                    cts.append((h0, h1))
            torch.cuda.synchronize()
            if mep.mep_read_status(hf) != 0:
                raise RuntimeError("device status not OK after the capped plan")
            hc = hf.host()
            capped[f"B={B}"] = {"plan_us": float(np.median([a.elapsed_time(b) for a, b in cts])) * 1e3,
                                "num_replicas": hc["num_replicas"], "num_seg": hc["num_seg"],
                                "max_rank_replicas": int(mr.item())}
        home_first["max_rank_replicas"] = rank_replicas_max(hh, E // R, R)
        home_first["max_rank_replicas_contiguous"] = rank_replicas_max(plan.host(), E // R, R)
        del hf

    # ---- the same step captured once in a CUDA graph and replayed
    graph = None
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg):
            step()
        gts = []
        for it in range(3 + args.steps):
            flush_l2()
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record()
            cg.replay()
            g1.record()
            if it >= 3:
                gts.append((g0, g1))
        torch.cuda.synchronize()
        gms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in gts])), world, dev)
        if mep.mep_read_status(plan) != 0:
            raise RuntimeError("device status not OK after graph replays")
        graph = {"ms_per_step": gms, "value": whole_job_rate(N, world, gms), "unit": "tokens/s"}
        del cg
    # the clock record spans both timed loops (eager and graph replay)
    clocks = sampler.stop()

    # ---- backward of combine and dispatch and the replica weight prefetch
    # (each timed alone, not part of the step)
    backward = None
    if not args.no_backward:
        grad_y = torch.empty_like(buf)
        grad_w = torch.empty((N, K), dtype=torch.float32, device=dev)
        grad_x = torch.empty_like(x)
        bwd = {"combine_backward": (lambda: mep.mep_combine_backward(s, H, plan, out, w, y, grad_y, grad_w),
                                    N * H * 2 + 2 * NK * H * 2 + NK * 8),
               "dispatch_backward": (lambda: mep.mep_dispatch_backward(s, H, plan, buf, grad_x),
                                     NK * H * 2 + N * H * 2 + NK * 4)}
        if P:   # replica weight prefetch of expert weights the size of a gradient row
            nrep = plan.host()["num_replicas"]
            w_rep = torch.empty_like(G)
            bwd["prefetch_replica_weights"] = (
                lambda: mep.mep_prefetch_replica_weights(s, plan, home, w_rep), 2 * nrep * P * 4)
        backward = {}
        for name, (fn, nbytes) in bwd.items():
            ts = []
            for it in range(3 + 20):
                flush_l2()
                b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                b0.record()
                fn()
                b1.record()
                if it >= 3:
                    torch.cuda.synchronize()
                    ts.append(b0.elapsed_time(b1))
            ms = float(np.median(ts))
            gbs = nbytes / (ms * 1e-3) / 1e9
            backward[name] = {"ms": ms, "bytes": nbytes, "gbs": gbs, "frac": gbs / peak,
                              "frac_nominal": gbs / NOMINAL_HBM_GBS}
        if mep.mep_read_status(plan) != 0:
            raise RuntimeError("device status not OK after the backward kernels")
        del grad_y, grad_w, grad_x

    # ---- the exchange's per-rank calls on this one GPU: rank r dispatches its
    # own S tokens into the R rank buffers and combines them back from the R
    # expert-output buffers (here slices of the single buffers, reached
    # through the rank pointer tables, as peer buffers would be).  All R
    # ranks' calls run back to back; the bytes are those of the whole calls.
    # The whole-range rank-addressed calls (one launch each) are timed beside
    # them.
    exchange = None
    if not args.no_exchange:
        SK = S * K
        btab = mep.rank_pointer_table([buf.view(NK, H)[r * SK:(r + 1) * SK] for r in range(R)], s, H, dev)
        ytab = mep.rank_pointer_table([y[r * SK:(r + 1) * SK] for r in range(R)], s, H, dev)
        legs = {"dispatch_ranked_tokens": (lambda: [mep.mep_dispatch_ranked_tokens(
                    s, H, plan, r * S, x[r * S:(r + 1) * S], btab) for r in range(R)], algo["dispatch"], R),
                "combine_ranked_tokens": (lambda: [mep.mep_combine_ranked_tokens(
                    s, H, plan, r * S, ytab, w[r * S:(r + 1) * S], out[r * S:(r + 1) * S]) for r in range(R)],
                    algo["combine"], R),
                # the same kernels over the whole token range in one call each
                "dispatch_ranked": (lambda: mep.mep_dispatch_ranked(s, H, plan, x, btab), algo["dispatch"], 1),
                "combine_ranked": (lambda: mep.mep_combine_ranked(s, H, plan, ytab, w, out), algo["combine"], 1)}
        grads = None
        if P:
            # each rank's segment gradients in its own buffer (row j = the
            # rank's j-th segment in slot order); every home rank reduces its
            # experts, reading the rows from the buffers that hold them
            from token_dispatch_mep_b200 import ep
            ph = plan.host()
            grads = []
            for q in range(R):
                segs = ep.local_segments(ph, q)
                gq = torch.empty((max(1, len(segs)), P), dtype=torch.float32, device=dev)
                for j, seg in enumerate(segs):
                    gq[j] = G[seg[0]]
                grads.append(gq)
            rows = max(gq.shape[0] for gq in grads)
            gtab = mep.pointer_table([gq.data_ptr() for gq in grads], dev)
            Bx = E // R
            homes = [home[q * Bx:(q + 1) * Bx] for q in range(R)]
            legs["reduce_ranked_per_home_rank"] = (lambda: [mep.mep_reduce_replica_grads_ranked(
                s, plan, P, q, gtab, rows, homes[q]) for q in range(R)], algo["reduce"], R)
        exchange = {}
        for name, (fn, nbytes, calls) in legs.items():
            ts = []
            for it in range(3 + 10):
                flush_l2()
                b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                b0.record()
                fn()
                b1.record()
                if it >= 3:
                    ts.append((b0, b1))
            torch.cuda.synchronize()
            ms = float(np.median([a.elapsed_time(b) for a, b in ts]))
            gbs = nbytes / (ms * 1e-3) / 1e9
            exchange[name] = {"ms_all_ranks": ms, "calls": calls, "us_per_call": ms * 1e3 / calls,
                              "bytes": nbytes, "gbs": gbs, "frac": gbs / peak}
        if mep.mep_read_status(plan) != 0:
            raise RuntimeError("device status not OK after the exchange calls")
        del grads

    # ---- e2e: host buffers through the public API, as a user would pipeline
    # it: two device buffer sets, inputs copied host->device on one stream,
    # the path on another, outputs copied back on a third, so the two copy
    # directions and the kernels overlap across consecutive steps.
    e2e = None
    if args.e2e_steps > 0:
        pin = dict(pin_memory=True)
        hi = torch.from_numpy(idx_h).pin_memory()
        hw = torch.from_numpy(w_h).pin_memory()
        hx = torch.empty(x.shape, dtype=x.dtype, **pin).copy_(x)
        # The large inputs (expert outputs, segment gradients) are pinned whole
        # when the node's available memory, shared by its ranks, holds them;
        # otherwise each rank pins their first rows and copies those rows
        # repeatedly into the device buffer: the same bytes cross PCIe every
        # step, from a smaller pinned source.
        local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
        budget = host_pin_budget(local_world) - hx.numel() * hx.element_size()
        hy, hG, sources = pinned_sources({"y": y, "G": G if P else None}, budget)
        hG = hG if P else None
        sets = []
        for b in range(2):
            d = dict(idx=idx if b == 0 else torch.empty_like(idx), w=w if b == 0 else torch.empty_like(w),
                     x=x if b == 0 else torch.empty_like(x), y=y if b == 0 else torch.empty_like(y),
                     G=(G if b == 0 else torch.empty_like(G)) if P else None,
                     plan=plan if b == 0 else mep.Plan(s, dev),
                     buf=buf if b == 0 else torch.empty_like(buf),
                     out=out if b == 0 else torch.empty_like(out),
                     home=(home if b == 0 else torch.empty_like(home)) if P else None,
                     ho=torch.empty(out.shape, dtype=out.dtype, **pin),
                     hh=torch.empty(home.shape, dtype=home.dtype, **pin) if P else None,
                     hsc=torch.empty(4, dtype=torch.int32, **pin),
                     hmv=torch.empty(1, dtype=torch.float64, **pin))
            d["ev_in"], d["ev_cmp"], d["ev_out"] = (torch.cuda.Event() for _ in range(3))
            sets.append(d)
        h2d = sum(t.numel() * t.element_size() for t in (hi, hw, hx, y) + ((G,) if P else ()))
        d2h = sum(t.numel() * t.element_size()
                  for t in (sets[0]["ho"], sets[0]["hsc"], sets[0]["hmv"]) + ((sets[0]["hh"],) if P else ()))
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_step(i):
            d = sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(d["ev_cmp"])      # step i-2 has finished reading these inputs
                d["idx"].copy_(hi, non_blocking=True)
                d["w"].copy_(hw, non_blocking=True)
                d["x"].copy_(hx, non_blocking=True)
                copy_rows(d["y"], hy)
                if P:
                    copy_rows(d["G"], hG)
                d["ev_in"].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(d["ev_in"])
                if i >= 2:
                    s_cmp.wait_event(d["ev_out"])     # step i-2's outputs are on the host
                pl = d["plan"]
                mep.mep_plan(s, d["idx"], pl)
                mep.mep_dispatch(s, H, pl, d["x"], d["buf"])
                mep.mep_combine(s, H, pl, d["y"], d["w"], d["out"])
                if P:
                    mep.mep_reduce_replica_grads(s, pl, P, d["G"], d["home"])
                d["ev_cmp"].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(d["ev_cmp"])
                d["ho"].copy_(d["out"], non_blocking=True)
                if P:
                    d["hh"].copy_(d["home"], non_blocking=True)
                d["hsc"].copy_(d["plan"].scalars, non_blocking=True)
                d["hmv"].copy_(d["plan"].maxvio_t, non_blocking=True)
                d["ev_out"].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(s_in)
        for i in range(2, 2 + args.e2e_steps):
            e2e_step(i)
        e1.record(s_out)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
        if any(int(d["hsc"][3].item()) != 0 for d in sets):
            raise RuntimeError("device status not OK after e2e steps")
        e2e = {"value": whole_job_rate(N, world, ms_e2e), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "pipeline": "2 buffer sets; H2D, kernels, D2H on 3 streams",
               "host_sources": sources}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_throughput(wl, args.cpu_seconds, dict(idx=idx_h, w=w_h))
        cpu = {"value": r["value"], "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": r["sample"], "measured_s": r["measured_s"]}

    eager = {"ms_per_step": ms_step, "value": value, "unit": "tokens/s"}
    if graph is not None:   # headline: the step as a user runs it, one graph replay per step
        ms_step, value = graph["ms_per_step"], graph["value"]
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(bench_config(wl, world), **(
                {"dispatch_form": "bulk copy (mep_dispatch_bulk)"} if args.dispatch_form == "bulk" else {})),
            "timing": ("CUDA-graph replay of the captured step, events around each replay"
                       if graph is not None else "eager launches, events around each kernel"),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clocks,
            "gpu_launches": launches_per_step * args.steps,
            "stages_ms": stage_ms,
            "backward_kernels": backward,
            "exchange_kernels": exchange,
            "graph_replay": graph,
            "home_first_plan": home_first,
            "capped_plan": capped,
            "eager": eager,
            "kernels": kernels,
            "plan_us": stage_ms["plan"] * 1e3,
            "pdc_tokens_per_s": whole_job_rate(N, world, pdc_ms),
            "num_seg": num_seg,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
