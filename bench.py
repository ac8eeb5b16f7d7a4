"""Benchmark: verified draft-tree nodes per second through a gated-delta linear-attention
layer on B200, and the achieved fraction of the HBM roofline.

One step = the whole hot path over one batch: tree_verify (metadata, S_root products,
tree solve, outputs) followed by tree_commit of every sequence's accepted path.  The
workload is 32 sequences x 32 heads of 64-node draft trees (depth <= 8, branching 1..4),
dk = dv = 128, bf16 q/k/v, fp32 S_root and gates.  One node = one tree node of one
sequence processed for all heads.  Inputs are rotated over three seeded sets (3 x 185 MB
of verify traffic, larger than the 126 MB L2), so every step reads cold HBM.  Outputs o
and U are fp32.

Timing: the step rate comes from K steps between two CUDA events with nothing between the
kernels, so each kernel's CTAs can become resident while the previous kernel drains (both
are launched with programmatic stream serialisation).  Per-kernel durations, used for the
roofline figures, come from a second timed pass with an event before and after every
kernel; those events keep the kernels apart, so that pass is slower than the step rate.
Also reported: verify alone launched back to back, the ragged (B=128, 8..48 nodes) and
wide (B=8, 256 nodes) workloads timed per launch, and the float64 oracle on this host's
cores, whose values for the whole workload are compared with this run's GPU outputs
(the run fails if any element is off by more than 2e-2 of the tensor's RMS).

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
Multi-GPU (one process per GPU under torchrun): each rank runs an independent replica
of the workload on its own GPU; no collective touches the data path, only a barrier and
a max-reduction of the timings.  value = nodes processed by all ranks / max rank time.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified tree nodes/sec (GDN, dk=dv=128) at 1 B200; % of HBM roofline"
WORKLOAD_IDX = 3
WORKLOAD = ("gdn draft trees B=32 H=32 nodes=64 depth<=8 branching<=4 dk=dv=128, "
            "bf16 q/k/v, fp32 state, gates and outputs")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
N_SETS = 3


# ----------------------------------------------------------------------------- byte counts
def verify_bytes(w) -> int:
    """Algorithmic bytes of one tree_verify: inputs read once, outputs written once."""
    in_b = 2 if w.in_dtype == "bf16" else 4
    out_b = 2 if w.out_dtype == "bf16" else 4
    T, H, B = w.T, w.H, w.B
    return (B * H * w.dk * w.dv * 4 + T * H * (2 * w.dk + w.dv) * in_b + T * H * 8 +
            4 * T + 4 * (B + 1) + T * H * w.dv * out_b + T * H * w.dv * 4)


def commit_bytes(w) -> int:
    """Algorithmic bytes of one tree_commit: S_root read + S_new written + path rows."""
    in_b = 2 if w.in_dtype == "bf16" else 4
    m = int((w.accepted_path >= 0).sum())
    return (2 * w.B * w.H * w.dk * w.dv * 4 + m * w.H * (w.dv * 4 + w.dk * in_b + 4) +
            w.accepted_path.size * 4 + 4 * (w.B + 1) + 4 * m)


# ---------------------------------------------------------------------------- distributed
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity on one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(nodes_per_rank_step: int, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: every rank's nodes over the slowest rank's time."""
    return nodes_per_rank_step * steps * world / max_seconds


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._stop = threading.Event()
        self._thread = None

    def _one(self):
        try:
            out = subprocess.run(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                  "--format=csv,noheader,nounits"], capture_output=True,
                                 text=True, timeout=5).stdout.strip()
            if out:
                self.samples.append([x.strip() for x in out.split(",")])
        except Exception:
            pass

    def _loop(self):
        while not self._stop.is_set():
            self._one()
            self._stop.wait(0.2)

    def start(self):
        self._thread = threading.Thread(target=self._loop, daemon=True)
        self._thread.start()

    def stop(self) -> dict:
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=10)
        if not self.samples:
            self._one()
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4)
                          if len(s) > 5 + i and s[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples)}


# --------------------------------------------------------------------------------- peaks
def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def traffic_record(kernel_file: str, kernel_name: str):
    """Per-launch DRAM bytes from a committed ncu summary, if taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    src = os.path.join(ROOT, "linear_attention_tree_b200", "csrc", kernel_file)
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_name)
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
        if rec and rec.get("source_sha") == sha:
            return rec.get("bytes_per_launch")
    except Exception:
        pass
    return None


# ------------------------------------------------------------------------------ oracle leg
def oracle_nodes(w, rows):
    """Time the float64 oracle on global node rows (every head of each row), plus the
    commit of every sequence whose last node is among them.  Returns (nodes, seconds)."""
    from threadpoolctl import threadpool_limits
    from oracle import oracle as O
    seq_of = np.searchsorted(w.node_offsets, np.asarray(rows), side="right") - 1
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for row, s in zip(rows, seq_of):
            n = int(row - w.node_offsets[s])
            for h in range(w.H):
                O.verify_node(w, int(s), n, h)
            if row == w.node_offsets[s + 1] - 1:
                for h in range(w.H):
                    O.commit_sequence(w, int(s), h, w.accepted_path[s])
        dt = time.perf_counter() - t0
    return len(rows), dt


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from oracle.pool import oracle_rows, start_pool
    cores = _cores()
    pool = start_pool(cores)
    try:
        # about two minutes of oracle work for the whole run on the host's cores, at least
        # one node per step
        per_node_s = 0.035 / cores
        k = int(min(w.T, max(1, 120.0 / ((args.steps + args.warmup) * per_node_s))))
        for i in range(args.warmup):
            oracle_rows(WORKLOAD_IDX, 0, [(i * k + j) % w.T for j in range(k)], pool)
        total_nodes, total_t = 0, 0.0
        for i in range(args.steps):
            t0 = time.perf_counter()
            total_nodes += oracle_rows(WORKLOAD_IDX, 0,
                                       [((args.warmup + i) * k + j) % w.T for j in range(k)], pool)
            total_t += time.perf_counter() - t0
    finally:
        pool.close()
        pool.join()
    value = total_nodes / total_t
    sample = (f"{args.steps} step(s) of {k} consecutive node(s) x {w.H} heads of the workload "
              f"(verify of each node, commit of each sequence completed), fp64 numpy, "
              f"{cores} worker processes of one BLAS thread each")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "nodes/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "nodes_per_tree": 64,
                   "dk": w.dk, "dv": w.dv, "seed": 0},
        "cpu_baseline": {"value": value, "unit": "nodes/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "nodes/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _cores() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def cpu_baseline_and_self_check(w, got, tol=2e-2):
    """The float64 oracle timed on this host (one core on a sample, then every core on the
    whole workload), and the whole workload's oracle values compared with this run's GPU
    outputs for the same inputs (o, U and S_new, element by element, max|err| <= tol * RMS).
    ``got`` = (o, U, S_new) as float64 arrays.  Raises if the outputs are off."""
    from oracle.pool import oracle_config, start_pool
    n1, dt1 = oracle_nodes(w, list(range(10 * 64)))
    cores = _cores()
    pool = start_pool(cores)
    try:
        t0 = time.perf_counter()
        _, o, U, S_new = oracle_config(WORKLOAD_IDX, 0, pool=pool)
        dt = time.perf_counter() - t0
    finally:
        pool.close()
        pool.join()
    check = {}
    for name, g, want in (("o", got[0], o), ("U", got[1], U), ("S_new", got[2], S_new)):
        rms = float(np.sqrt(np.mean(want ** 2)))
        err = float(np.max(np.abs(g - want)))
        check[name] = {"max_err_over_rms": err / rms, "elements": int(want.size)}
        if not err <= tol * rms:
            raise RuntimeError(f"self-check failed: {name} max|err| {err:.3e} > {tol} * RMS {rms:.3e}")
    return {
        "value": w.T / dt, "unit": "nodes/s", "cores": cores, "kind": "oracle",
        "sample": (f"the whole workload (seed 0: {w.T} nodes x {w.H} heads, verify, and the "
                   f"commit of all {w.B} sequences), fp64 numpy, {cores} worker processes of "
                   "one BLAS thread each"),
        "seconds": dt,
        "single_core": {"value": n1 / dt1, "unit": "nodes/s", "cores": 1, "seconds": dt1,
                        "sample": "sequences 0-9 (10 x 64 nodes x 32 heads), verify + commit"},
        "self_check": dict(check, tolerance=f"max|err| <= {tol} * RMS(oracle), every element",
                           outputs="this run's GPU outputs for input set 0"),
    }


# --------------------------------------------------------------------------------- GPU leg
def run_b200(args, workloads):
    import torch
    import linear_attention_tree_b200 as L
    from linear_attention_tree_b200.tensors import to_device

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    w0 = workloads[0]
    sets = [to_device(w, dev) for w in workloads]
    B, H, T = w0.B, w0.H, w0.T
    prob = L.make_problem(B, H, w0.dk, w0.dv, T, w0.max_nodes, max(w.max_path for w in workloads))
    ws = L.new_workspace(prob, dev)
    odt = torch.float32 if w0.out_dtype == "f32" else torch.bfloat16
    outs = [(torch.empty((T, H, w0.dv), dtype=odt, device=dev),
             torch.empty((T, H, w0.dv), dtype=torch.float32, device=dev),
             torch.empty_like(d["S_root"])) for d in sets]
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        d, (o, U, S_new) = sets[i % N_SETS], outs[i % N_SETS]
        if ev is not None:
            ev[0].record(stream)
        L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                      d["node_offsets"], d["S_root"], max_nodes=w0.max_nodes, out=o, U=U,
                      workspace=ws, kernel=args.kernel)
        if ev is not None:
            ev[1].record(stream)
        L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"],
                      d["accepted_path"], max_nodes=w0.max_nodes, S_new=S_new, workspace=ws)
        if ev is not None:
            ev[2].record(stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    st = L.get_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    k_steps = min(args.steps, 2000)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(k_steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    clocks = ClockSampler(int(visible[local]) if len(visible) > local and
                          visible[local].strip().isdigit() else local)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start.record(stream)
    for i in range(args.steps):
        step(i)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    # per-kernel durations: a second timed pass with events around every kernel
    for i in range(k_steps):
        step(i, evs[i])
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier()
    elapsed_s = t_start.elapsed_time(t_end) / 1e3
    verify_ms = [e[0].elapsed_time(e[1]) for e in evs]
    commit_ms = [e[1].elapsed_time(e[2]) for e in evs]
    max_s = max_over_ranks(elapsed_s, world, dev)
    value = aggregate(T, args.steps, world, max_s)
    st = L.get_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed region")

    # ---- verify alone, launched back to back (rotating inputs), one event pair around all
    n_b2b = min(max(args.steps, 20), 2000)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for i in range(n_b2b):
        d, (o, U, S_new) = sets[i % N_SETS], outs[i % N_SETS]
        L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                      d["node_offsets"], d["S_root"], max_nodes=w0.max_nodes, out=o, U=U,
                      workspace=ws, kernel=args.kernel)
    b1.record(stream)
    torch.cuda.synchronize(dev)
    b2b_s = b0.elapsed_time(b1) / 1e3 / n_b2b

    # ---- decode steps through the fused entry point: the previous set's commit and this
    # set's verify in one launch, the state updated in place
    S_run = sets[0]["S_root"].clone()
    n_fused = min(max(args.steps, 20), 2000)

    def fused_step(i):
        dp, dn = sets[(i - 1) % N_SETS], sets[i % N_SETS]
        L.tree_commit_verify(outs[(i - 1) % N_SETS][1], dp["k"], dp["log_a"], dp["node_offsets"],
                             dp["accepted_path"], S_run, dn["q"], dn["k"], dn["v"], dn["log_a"],
                             dn["b"], dn["parent"], dn["node_offsets"],
                             max_nodes_prev=w0.max_nodes, max_nodes=w0.max_nodes, S_new=S_run,
                             out=outs[i % N_SETS][0], U=outs[i % N_SETS][1], workspace=ws,
                             kernel=args.kernel)
    for i in range(1, 6):
        fused_step(i)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(6, 6 + n_fused):
        fused_step(i)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    fused_s = f0.elapsed_time(f1) / 1e3 / n_fused
    if L.get_status(ws) != 0:
        raise RuntimeError("device status after the fused decode steps")

    # ---- end to end through the public API: pinned host inputs in, results out
    host = [to_device(w, "cpu", pin=True) for w in workloads]
    h_out = [torch.empty((T, H, w0.dv), dtype=odt).pin_memory() for _ in range(N_SETS)]
    h_S = [torch.empty_like(h["S_root"]).pin_memory() for h in host]
    names = ["q", "k", "v", "log_a", "b", "parent", "node_offsets", "S_root", "accepted_path"]
    h2d = sum(host[0][n].numel() * host[0][n].element_size() for n in names)
    d2h = h_out[0].numel() * h_out[0].element_size() + h_S[0].numel() * 4
    e2e_steps = max(3, min(args.steps, 50))

    # pipelined over the three buffer sets: inputs go up on one stream, the step runs on
    # the launching stream, results come down on a third, so that copies in both
    # directions overlap other steps' kernels
    copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(N_SETS)]
    done = [torch.cuda.Event() for _ in range(N_SETS)]
    out_read = [torch.cuda.Event() for _ in range(N_SETS)]
    used = [False] * N_SETS

    def e2e_step(i):
        slot = i % N_SETS
        h, d = host[slot], sets[slot]
        o, U, S_new = outs[slot]
        if used[slot]:
            copy_in.wait_event(done[slot])          # the last step on this slot has read it
        with torch.cuda.stream(copy_in):
            for n in names:
                d[n].copy_(h[n], non_blocking=True)
            in_ready[slot].record(copy_in)
        stream.wait_event(in_ready[slot])
        if used[slot]:
            stream.wait_event(out_read[slot])       # its previous results have been copied out
        L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                      d["node_offsets"], d["S_root"], max_nodes=w0.max_nodes, out=o, U=U,
                      workspace=ws, kernel=args.kernel)
        L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"],
                      d["accepted_path"], max_nodes=w0.max_nodes, S_new=S_new, workspace=ws)
        done[slot].record(stream)
        copy_out.wait_event(done[slot])
        with torch.cuda.stream(copy_out):
            h_out[slot].copy_(o, non_blocking=True)
            h_S[slot].copy_(S_new, non_blocking=True)
            out_read[slot].record(copy_out)
        used[slot] = True

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_in.wait_event(e0)
    copy_out.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(copy_out)
    stream.wait_stream(copy_in)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    e2e_value = aggregate(T, e2e_steps, world, e2e_s)

    if rank == 0:
        peak, peak_src = hbm_peak()
        vb, cb = verify_bytes(w0), commit_bytes(w0)
        v_avg = statistics.mean(verify_ms) / 1e3
        c_avg = statistics.mean(commit_ms) / 1e3
        tc = args.kernel != "simt"
        kfile, kname = ((("verify_tc.cu", "verify_tc") if w0.max_nodes <= 64 else
                         ("verify_tcw.cu", "verify_tcw")) if tc else ("verify_simt.cu", "verify_simt"))
        achieved = vb / v_avg / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "nodes/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * max_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16/tf32 tensor, f32 accumulate" if tc else "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": B, "H": H, "nodes_per_tree": 64,
                       "dk": w0.dk, "dv": w0.dv, "seeds": list(range(N_SETS)),
                       "l2": f"{N_SETS} rotating input sets, {N_SETS}x{vb / 1e6:.0f} MB > 126 MB L2",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "kernel": kname},
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "peak_source": peak_src,
                         "traffic": traffic_record(kfile, kname),
                         "algorithmic_bytes_per_launch": vb,
                         "frac_of_8TBps": achieved / NOMINAL_HBM_GBS},
            "verify_us": 1e6 * v_avg, "commit_us": 1e6 * c_avg,
            "verify_us_p10_p50_p90": [1e3 * float(np.percentile(verify_ms, q)) for q in (10, 50, 90)],
            "commit_us_p10_p50_p90": [1e3 * float(np.percentile(commit_ms, q)) for q in (10, 50, 90)],
            "kernel_timing": f"events around each kernel, second timed pass of {k_steps} steps",
            "verify_nodes_per_s": T / v_avg,
            "commit_roofline": {"achieved": cb / c_avg / 1e9, "unit": "GB/s",
                                "frac": cb / c_avg / 1e9 / peak,
                                "algorithmic_bytes_per_launch": cb},
            "step_bytes_per_s": (vb + cb) * args.steps / max_s / 1e9,
            "e2e": {"value": e2e_value, "unit": "nodes/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": 2 * args.steps,
            "clocks": clk,
        }
        line["roofline"]["region"] = ("tv_tree_verify alone: CUDA events around each launch in "
                                      "the per-kernel pass (the figure the 60% bar applies to); "
                                      "value is the verify + commit step rate")
        line["verify_back_to_back"] = {
            "us_per_launch": 1e6 * b2b_s, "nodes_per_s": T / b2b_s,
            "frac_of_measured": vb / b2b_s / 1e9 / peak, "frac_of_8TBps": vb / b2b_s / 1e9 / NOMINAL_HBM_GBS,
            "how": f"{n_b2b} verify launches back to back over the rotating sets, one event pair"}
        line["roofline"]["sustained"] = {
            "achieved": vb / b2b_s / 1e9, "frac": vb / b2b_s / 1e9 / peak,
            "frac_of_8TBps": vb / b2b_s / 1e9 / NOMINAL_HBM_GBS,
            "how": "the same bytes over the per-launch time of verify_back_to_back (a sustained "
                   "stream of launches); achieved / frac above are per launch with events around each"}
        fb = vb + cb - w0.B * w0.H * w0.dk * w0.dv * 4      # S_root read once, not twice
        line["fused_decode_step"] = {
            "us_per_step": 1e6 * fused_s, "nodes_per_s": T / fused_s,
            "algorithmic_bytes_per_step": fb, "achieved_GBps": fb / fused_s / 1e9,
            "frac_of_measured": fb / fused_s / 1e9 / peak,
            "how": (f"{n_fused} calls of tv_tree_commit_verify back to back (commit of the "
                    "previous set's accepted paths + verify of this set, one launch, state in "
                    "place), one event pair; compare ms_per_step (two launches per step)")}
        if world == 1 and not args.no_snapshot_baseline:
            line["snapshot_baseline"] = snapshot_baseline(args, L, sets, w0, ws, 1e6 * v_avg,
                                                          1e6 * c_avg, 1e6 * max_s / args.steps)
        if world == 1 and not args.other_configs_off:
            line["other_workloads"] = other_workloads(args, L, dev, peak)
        if world == 1 and not args.no_budget:
            try:
                line["batch_budget"] = batch_budget(line, 1e6 * c_avg)
            except Exception as e:   # an auxiliary figure: report it, keep the line
                line["batch_budget"] = {"error": f"{type(e).__name__}: {e}"}
        if world == 1 and not args.no_cpu_baseline:
            got = tuple(t.float().cpu().numpy().astype(np.float64) for t in outs[0])
            line["cpu_baseline"] = cpu_baseline_and_self_check(workloads[0], got)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def snapshot_baseline(args, L, sets, w0, ws, verify_us, commit_us, step_us) -> dict:
    """The pages' baseline on this GPU and workload: every node's full state materialised
    (tv_snapshot_verify), the accepted state copied out of its snapshot (tv_snapshot_commit).
    Timed per launch with CUDA events over the rotating input sets."""
    import torch
    T, H, dk, dv = w0.T, w0.H, w0.dk, w0.dv
    dev = sets[0]["q"].device
    snap = torch.empty((T, H, dv, dk), dtype=torch.float32, device=dev)
    out = torch.empty((T, H, dv), dtype=torch.float32, device=dev)
    U = torch.empty_like(out)
    S_new = torch.empty_like(sets[0]["S_root"])

    def run(i, ev):
        d = sets[i % N_SETS]
        ev[0].record()
        L.snapshot_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                          d["node_offsets"], d["S_root"], max_nodes=w0.max_nodes,
                          snapshots=snap, out=out, U=U, workspace=ws)
        ev[1].record()
        L.snapshot_commit(snap, d["S_root"], d["node_offsets"], d["accepted_path"],
                          max_nodes=w0.max_nodes, S_new=S_new, workspace=ws)
        ev[2].record()
    n = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n + 2)]
    for i in range(n + 2):
        run(i, evs[i])
    torch.cuda.synchronize(dev)
    if L.get_status(ws) != 0:
        raise RuntimeError("device status after the snapshot baseline")
    sv = statistics.mean(e[0].elapsed_time(e[1]) for e in evs[2:]) * 1e3
    sc = statistics.mean(e[1].elapsed_time(e[2]) for e in evs[2:]) * 1e3
    snap_bytes = T * H * dv * dk * 4
    ours_bytes = T * H * dv * 4 + L.workspace_size(L.make_problem(w0.B, H, dk, dv, T, w0.max_nodes))
    del snap
    torch.cuda.empty_cache()
    return {
        "verify_us": sv, "commit_us": sc, "step_us": sv + sc,
        "speedup_verify": sv / verify_us, "speedup_step": (sv + sc) / step_us,
        "transient_bytes": snap_bytes, "ours_transient_bytes": ours_bytes,
        "transient_memory_ratio": snap_bytes / ours_bytes,
        "how": (f"CUDA events around each of {n} launches after 2 warm-up launches; the "
                "baseline visits nodes in index order from the parent's snapshot, one CTA per "
                "(sequence, head); ours = fp32 U plus the workspace"),
        "pages": ("context only, not re-measured: 3.4-7.7x faster linear-attention tree "
                  "verification and 82-99x less transient state memory than per-node snapshots "
                  "(two GPU platforms, four hybrid models)")}


def other_workloads(args, L, dev, peak) -> dict:
    """Per-launch verify timing of the ragged (config 4) and wide-tree (config 5) workloads:
    rotating input sets, CUDA events around each launch."""
    import torch
    from linear_attention_tree_b200 import workloads as W
    from linear_attention_tree_b200.tensors import to_device
    res = {}
    for idx, label in ((4, "gdn ragged trees B=128 H=32, 8..48 nodes, budget 3072, depth<=7"),
                       (5, "gdn wide trees B=8 H=32, 256 nodes, depth<=10, branching<=8")):
        ws_ = [W.config(idx, s) for s in range(N_SETS)]
        ds = [to_device(x, dev) for x in ws_]
        w = ws_[0]
        odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
        outs = [(torch.empty((x.T, x.H, x.dv), dtype=odt, device=dev),
                 torch.empty((x.T, x.H, x.dv), dtype=torch.float32, device=dev)) for x in ws_]
        ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, w.max_path), dev)

        def one(i, kernel):
            d, (o, U), x = ds[i % N_SETS], outs[i % N_SETS], ws_[i % N_SETS]
            L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                          d["node_offsets"], d["S_root"], max_nodes=x.max_nodes, out=o, U=U,
                          workspace=ws, kernel=kernel)

        def timed(kernel, n):
            for i in range(10 if n > 20 else 3):
                one(i, kernel)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(n)]
            for i, (e0, e1) in enumerate(ev):
                e0.record()
                one(i, kernel)
                e1.record()
            torch.cuda.synchronize(dev)
            if L.get_status(ws) != 0:
                raise RuntimeError(f"device status after workload {idx}")
            return statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev) / 1e3
        n = 60
        t = timed(args.kernel, n)
        # the CUDA-core kernel on the same batches, for comparison
        t_simt = timed("simt", 12) if args.kernel != "simt" else t
        vb = statistics.mean(verify_bytes(x) for x in ws_)
        T = statistics.mean(x.T for x in ws_)
        kname = ("verify_tc" if w.max_nodes <= 64 else "verify_tcw") if args.kernel != "simt" \
            else "verify_simt"
        res[f"config{idx}"] = {
            "workload": label, "kernel": kname, "verify_us": 1e6 * t,
            "verify_nodes_per_s": T / t, "algorithmic_bytes_per_launch": int(vb),
            "achieved_GBps": vb / t / 1e9, "frac_of_measured": vb / t / 1e9 / peak,
            "frac_of_8TBps": vb / t / 1e9 / NOMINAL_HBM_GBS,
            "timing": f"CUDA events around each of {n} launches, {N_SETS} rotating input sets",
            "verify_simt_us": 1e6 * t_simt, "speedup_vs_simt": t_simt / t}
        del ds, outs
        torch.cuda.empty_cache()
    return res


def batch_budget(line: dict, commit_us: float) -> dict:
    """The batch-wide verification budget on this GPU: fit the verify cost model, check its
    predictions against this run's measured launches, and let it choose the budget for a
    synthetic draft batch (128 trees of 64 nodes with acceptance estimates), the step being
    this layer's verify plus its measured commit."""
    import numpy as np
    from linear_attention_tree_b200 import budget as Bd
    from linear_attention_tree_b200 import workloads as W
    model, samples = Bd.calibrate(launches=8)
    fit_err = max(abs(model.predict_us(z, h) / us - 1) for z, h, us in samples)
    checks = {}
    measured = {"config3": line["verify_us"]}
    for name, rec in line.get("other_workloads", {}).items():
        measured[name] = rec["verify_us"]
    for name, us in measured.items():
        w = W.config(int(name[-1]), 0)
        pred = model.predict_us([int(x) for x in np.diff(w.node_offsets)], w.H)
        checks[name] = {"predicted_us": pred, "measured_us": us, "rel_err": pred / us - 1}
    parents = [W.frontier_tree(900 + s, 64, 8, 4)[0] for s in range(128)]
    trees = [(par, W.acceptance_estimates(par, 900 + s)) for s, par in enumerate(parents)]
    pick = Bd.choose_budget(trees, 32, model, fixed_us=commit_us)
    def rate(keeps):
        sizes = [len(k) for k in keeps]
        return Bd.expected_tokens(trees, keeps) / (commit_us + model.predict_us(sizes, 32))
    all_nodes = [np.arange(64) for _ in trees]
    raw = np.random.Generator(np.random.PCG64(4000)).integers(8, 49, size=128)
    capped = [np.arange(int(n)) for n in Bd.cap_largest(np.minimum(raw, 64), 3072)]
    greedy_3072 = Bd.select_nodes(trees, 3072, min_nodes=1)
    return {
        "model_us": {"tc": model.tc, "wide": model.wide,
                     "features": "tc: 1, B*H, T*H; wide: 1, B*H, T*H, H*sum(ceil(n/64))"},
        "fit_samples": len(samples), "fit_max_rel_err": fit_err,
        "prediction_vs_this_run": checks,
        "example": {
            "batch": "128 frontier trees of 64 nodes, depth<=8, acceptance Beta(4,2)*0.6^rank",
            "step": f"verify + this run's commit ({commit_us:.1f} us), one layer",
            "chosen_budget_nodes": pick["budget"], "predicted_verify_us": pick["us"] - commit_us,
            "expected_tokens": pick["tokens"], "tokens_per_us": pick["tokens_per_us"],
            "verify_everything_tokens_per_us": rate(all_nodes),
            "greedy_3072_tokens_per_us": rate(greedy_3072),
            "index_prefix_cap_largest_3072_tokens_per_us": rate(capped)},
    }


CASES = {
    "verify3": (3, "verify"), "verify4": (4, "verify"), "verify5": (5, "verify"),
    "commit3": (3, "commit"), "fused3": (3, "fused"), "snapshot3": (3, "snapshot"),
}


def run_case(args) -> int:
    """A few launches of one operation on one named workload and nothing else (no timing,
    no output): the command a profiler wraps.  Input set 0; the state is not updated."""
    import torch
    import linear_attention_tree_b200 as L
    from linear_attention_tree_b200 import workloads as W
    from linear_attention_tree_b200.tensors import to_device
    idx, op = CASES[args.case]
    w = W.config(idx, 0)
    d = to_device(w, "cuda")
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, w.max_path))
    out = torch.empty((w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    U = torch.empty_like(out)
    U2 = torch.empty_like(out)
    S = d["S_root"].clone()
    S_new = torch.empty_like(S)
    L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"], d["node_offsets"],
                  S, max_nodes=w.max_nodes, out=out, U=U, workspace=ws, kernel=args.kernel)
    snap = (torch.empty((w.T, w.H, w.dv, w.dk), dtype=torch.float32, device="cuda")
            if op == "snapshot" else None)
    for _ in range(args.launches):
        if op == "verify":
            L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                          d["node_offsets"], S, max_nodes=w.max_nodes, out=out, U=U,
                          workspace=ws, kernel=args.kernel)
        elif op == "commit":
            L.tree_commit(U, d["k"], d["log_a"], S, d["node_offsets"], d["accepted_path"],
                          max_nodes=w.max_nodes, S_new=S_new, workspace=ws)
        elif op == "fused":
            L.tree_commit_verify(U, d["k"], d["log_a"], d["node_offsets"], d["accepted_path"],
                                 S, d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                                 d["node_offsets"], max_nodes_prev=w.max_nodes,
                                 max_nodes=w.max_nodes, S_new=S_new, out=out, U=U2,
                                 workspace=ws, kernel=args.kernel)
        else:
            L.snapshot_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                              d["node_offsets"], S, max_nodes=w.max_nodes, snapshots=snap,
                              out=out, U=U2, workspace=ws)
    torch.cuda.synchronize()
    if L.get_status(ws) != 0:
        raise RuntimeError("device status after the case")
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--kernel", choices=["auto", "tc", "simt"], default="auto")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-snapshot-baseline", action="store_true",
                    help="skip the per-node-snapshot baseline (4.3 GB of snapshots)")
    ap.add_argument("--other-configs-off", action="store_true",
                    help="skip the per-launch timing of the ragged and wide-tree workloads")
    ap.add_argument("--no-budget", action="store_true",
                    help="skip the cost-model calibration and the batch-budget example")
    ap.add_argument("--case", choices=sorted(CASES),
                    help="only launch one operation --launches times on one workload (for a "
                         "profiler): verifyN = tv_tree_verify on workload N, commit3, fused3 = "
                         "tv_tree_commit_verify, snapshot3 = the per-node-snapshot baseline")
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args(argv)
    if args.case:
        return run_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from linear_attention_tree_b200 import workloads as W
    if args.impl == "reference":
        return run_reference(args, W.config(WORKLOAD_IDX, 0))
    workloads = [W.config(WORKLOAD_IDX, s) for s in range(N_SETS)]
    return run_b200(args, workloads)


if __name__ == "__main__":
    sys.exit(main())
