#!/usr/bin/env python
"""Throughput benchmark of the streaming semi-CRF hot path on B200.

One step = the whole hot path over one batch: prefix sums + forward rings
(semicrf_forward), checkpoint-parallel posteriors and gradients
(semicrf_backward) and Viterbi decoding (semicrf_viterbi), all through the
C ABI.  The workload is the speech-scale batch (B=32, lengths uniform in
[300, 800], padded T=800, K=30, C=39, seeded synthetic emissions standing in
for TIMIT).  Metric: edge evaluations per second, edges = sum_b L_b * K * C^2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) each rank runs its own batch
(seeded per rank: weak scaling) and the batch-summed parameter gradients
(grad_trans, grad_dur) are all-reduced over NCCL every step, as a
data-parallel training step needs.  Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle (the only other
implementation here) on the host cores on a bounded sample of the same
workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

WORKLOAD = "speech"
METRIC = "semi-CRF fwd+bwd edge evals/s (B·T·K·C²), positions/s, peak HBM, % roofline"
UNIT = "edge evals/s"
MUFU_PER_SM_PER_CLK = 16          # ex2/lg2 results per SM per clock (SFU)
FP32_PER_SM_PER_CLK = 128         # fp32 lanes per SM per clock (4 partitions x 32)
L2_BYTES = 126 * 1024 * 1024
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "semi_markov_crf_b200", "csrc")


# ----------------------------------------------------------------------------- helpers
def shard_seed(base_seed: int, rank: int) -> int:
    """Rank r draws its own batch from seed base + r (rank 0 = the canonical one)."""
    return base_seed + rank


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without torch.distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_param_grads(tensors):
    """Sum the batch-summed parameter gradients over ranks (data parallel)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)


def edges_of(lengths, K, C) -> int:
    return int(np.sum(lengths, dtype=np.int64)) * K * C * C


def edge_ops_per_position(kernel: str, K: int, C: int) -> tuple[int, str] | None:
    """The method's algorithmic work per sequence position and the unit it
    runs on, counted per edge (k, c', c) as the hot-path table does: one
    exponential per edge for each of the forward ring, the backward ring and
    the edge posteriors (3 K C^2 per position for forward + backward), one add
    and one max per edge for Viterbi.  The kernels compute the same sums with
    fewer operations (the label fan-in is grouped once per boundary), so a
    fraction against this count credits the algorithm's work, not the
    instructions issued; mufu_ops_per_position gives the latter."""
    kc2 = K * C * C
    if kernel in ("chain_kernel", "chain_exp_kernel"):
        return 2 * kc2, "mufu"      # forward and backward rings
    if kernel in ("posterior_kernel", "segment_kernel"):
        return kc2, "mufu"          # the edge posteriors
    if kernel in ("viterbi_kernel", "viterbi_pipe_kernel"):
        return 2 * kc2, "fp32"      # an add and a max per edge
    return None


def mufu_ops_per_position(kernel: str, K: int, C: int) -> int:
    """MUFU (ex2/lg2) operations the kernels issue per sequence position.

    Per boundary the k fan-in needs K*C exponentials (one log-sum-exp over K
    durations for each of C labels) plus C logarithms; the label fan-in runs
    in the exponential domain: C exponentials and C logarithms.  The forward
    and backward rings run in the same launch (2 x), the posterior kernel
    recomputes both over its segment and adds 2C exponentials for the start
    and end marginals.  Viterbi uses no MUFU."""
    one_ring = K * C + 3 * C
    if kernel in ("chain_kernel", "chain_exp_kernel"):
        return 2 * one_ring
    if kernel == "segment_kernel":
        return 2 * one_ring + 2 * C
    if kernel == "posterior_kernel":
        # one exponential per (start, duration, label) term and per boundary
        return K * C + 1
    return 0


def alu_ops_per_position(kernel: str, K: int, C: int) -> int:
    """Algorithmic fp32 operations per position of the max-semiring kernel:
    one add and one max per (duration, label) term of the k fan-in and per
    (label, label) term of the label fan-in."""
    if kernel in ("viterbi_kernel", "viterbi_pipe_kernel"):
        return 2 * (K * C + C * C)
    return 0


def csrc_digest() -> str:
    """sha256 over the kernel sources, to tie a stored ncu traffic figure to
    the build it was measured on."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def stored_traffic(kernel: str):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    summary, or None when it was taken on other kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("csrc_sha256") != csrc_digest() or t.get("workload") != WORKLOAD:
        return None
    return t.get("kernels", {}).get(kernel)


def kernel_roofline(name: str, info: dict, K: int, C: int, positions: int, steps: int,
                    sm_count: int, sm_max_mhz: float, issued: bool = False) -> dict | None:
    """Roofline entry of one kernel: algorithmic ops per launch (the per-edge
    count of edge_ops_per_position; with issued=True the operations the
    kernel issues) over its mean launch time, against the unit that bounds
    it (MUFU for the log-semiring kernels, fp32 lanes for Viterbi).  None for
    the O(T C) HBM kernels."""
    if positions <= 0:
        return None
    if issued:
        mufu, alu = mufu_ops_per_position(name, K, C), alu_ops_per_position(name, K, C)
    else:
        e = edge_ops_per_position(name, K, C)
        mufu, alu = (e[0], 0) if e and e[1] == "mufu" else (0, e[0] if e else 0)
    if mufu:
        per_clk, ops_pos, what = MUFU_PER_SM_PER_CLK, mufu, "MUFU ops/clk"
    elif alu:
        per_clk, ops_pos, what = FP32_PER_SM_PER_CLK, alu, "fp32 lanes/clk"
    else:
        return None
    peak = sm_count * per_clk * sm_max_mhz * 1e6
    per_launch = ops_pos * positions / (info["launches"] / steps)
    achieved = per_launch / (info["ms_per_launch"] * 1e-3)
    return {"bound": "alu", "kernel": name, "achieved": achieved / 1e9, "peak": peak / 1e9,
            "unit": "Gop/s", "frac": achieved / peak, "traffic": stored_traffic(name),
            "peak_source": f"derived: {sm_count} SMs x {per_clk} {what} x {sm_max_mhz:.0f} MHz "
                           f"(sm_max_mhz of MEASURED_PEAKS.json)",
            "ops_per_launch": per_launch,
            "count": "issued by the kernel" if issued else "per edge (hot-path table)"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(r["power"] for r in rows)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return {}


# ----------------------------------------------------------------------------- CPU oracle arm
def oracle_sample_time(w, n_seq: int, threads: int):
    """Time the float64 oracle (forward-backward + Viterbi) on the first n_seq
    sequences of workload w.  Returns (seconds, edges, positions)."""
    import oracle
    sel = slice(0, n_seq)
    K = w["dur"].shape[0]
    C = w["em"].shape[2]
    t0 = time.perf_counter()
    oracle.forward_backward(w["em"][sel], w["lengths"][sel], w["trans"], w["dur"], K, threads=threads)
    oracle.viterbi(w["em"][sel], w["lengths"][sel], w["trans"], w["dur"], K, threads=threads)
    dt = time.perf_counter() - t0
    return dt, edges_of(w["lengths"][sel], K, C), int(np.sum(w["lengths"][sel]))


def cpu_baseline(w, n_seq: int = 16):
    threads = min(os.cpu_count() or 1, n_seq)
    dt, edges, pos = oracle_sample_time(w, n_seq, threads)
    return {"value": edges / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"first {n_seq} of {len(w['lengths'])} sequences of the {WORKLOAD} batch "
                      f"({pos} positions), forward-backward + Viterbi, float64, "
                      f"{threads} threads, {dt:.2f} s",
            "positions_per_s": pos / dt}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from semi_markov_crf_b200 import synth
    w = synth.make(WORKLOAD)
    n_seq = 4
    threads = min(os.cpu_count() or 1, n_seq)
    for _ in range(args.warmup):
        oracle_sample_time(w, n_seq, threads)
    times, edges = [], 0
    for _ in range(args.steps):
        dt, edges, pos = oracle_sample_time(w, n_seq, threads)
        times.append(dt)
    total = sum(times)
    value = edges * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": 32, "T": 800, "K": 30, "C": 39,
                   "sample_sequences_per_step": n_seq},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"first {n_seq} sequences of the {WORKLOAD} batch per step, "
                                   f"forward-backward + Viterbi in float64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from semi_markov_crf_b200 import semicrf, synth
    base = synth.CONFIGS[WORKLOAD]
    w = synth.make(WORKLOAD, seed=shard_seed(base.seed, rank))
    B, T, C = w["em"].shape
    K = w["dur"].shape[0]
    em = torch.from_numpy(w["em"]).to(dev)
    lengths = torch.from_numpy(w["lengths"]).to(dev)
    trans = torch.from_numpy(w["trans"]).to(dev)
    dur = torch.from_numpy(w["dur"]).to(dev)
    edges = edges_of(w["lengths"], K, C)
    positions = int(w["lengths"].sum())

    ws = semicrf.Workspace(B, T, C, K, 0, dev)
    logZ = torch.empty(B, dtype=torch.float64, device=dev)
    out = {}
    vws = semicrf.Workspace(B, T, C, K, 0, dev)

    vout = (torch.empty(B, dtype=torch.float64, device=dev),
            torch.empty((B, T), dtype=torch.int32, device=dev),
            torch.empty((B, T), dtype=torch.uint8, device=dev))
    side = torch.cuda.Stream(dev)

    def lib_step(em_, lengths_, trans_, dur_):
        # Viterbi does not depend on the forward-backward pass and the two use
        # 3B of the 148 SMs between them: decode on a side stream, join at the end.
        main = torch.cuda.current_stream(dev)
        side.wait_stream(main)
        with torch.cuda.stream(side):
            res = semicrf.viterbi(em_, lengths_, trans_, dur_, ws=vws, out=vout)
        semicrf.forward(em_, lengths_, trans_, dur_, ws=ws, logZ=logZ)
        semicrf.backward(ws, lengths_, trans_, dur_, out=out)
        main.wait_stream(side)
        return res

    def step(em_, lengths_, trans_, dur_):
        res = lib_step(em_, lengths_, trans_, dur_)
        allreduce_param_grads([out["grad_trans"], out["grad_dur"]])
        return res

    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(max(args.warmup, 3)):
        step(em, lengths, trans, dur)
    torch.cuda.synchronize(dev)
    if semicrf.get_status(ws) != 0:
        raise RuntimeError(f"device status {semicrf.get_status(ws)}")
    # which kernel ran each ring (both ring kernels launch every step; each
    # takes its own sequences): positions per ring kernel, both directions
    dom = semicrf.ring_domains(ws)
    lens = [int(x) for x in w["lengths"]]
    kept = [dom[b] == 1 and dom[B + b] == 1 for b in range(B)]
    ring_pos = {"chain_exp_kernel": sum(lens[i % B] for i, m in enumerate(dom) if m == 1) / 2,
                "chain_kernel": sum(lens[i % B] for i, m in enumerate(dom) if m == 2) / 2,
                # the posterior pass takes the sequences both of whose rings
                # kept their values, the checkpoint walk the others
                "posterior_kernel": sum(l for l, k in zip(lens, kept) if k),
                "segment_kernel": sum(l for l, k in zip(lens, kept) if not k)}

    stream = torch.cuda.current_stream(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    semicrf.profile_enable(True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()                       # evict L2 between timed steps (outside the events)
        starts[i].record(stream)
        step(em, lengths, trans, dur)
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    semicrf.profile_enable(False)
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms = reduce_max(ms, dev)
    ms_eager = ms / args.steps

    # The same step captured once into a CUDA graph and replayed: the library
    # allocates nothing and never synchronises inside a call, so the whole
    # step (both streams, the library's own side stream) is capturable; the
    # replay removes the host launch latency and the gaps between dependent
    # launches.  The gradient all-reduce (N > 1) stays outside the graph.
    # Per-kernel times and the roofline come from the eager loop above.
    graph, launch_mode = None, "eager"
    if not args.no_graph:
        try:
            # rank-local outputs of the last eager step (grad_trans / grad_dur
            # are all-reduced across ranks, the replay below is not)
            ref_logz, ref_gem = logZ.clone(), out["grad_em"].clone()
            torch.cuda.synchronize(dev)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, capture_error_mode="relaxed"):
                lib_step(em, lengths, trans, dur)
            graph.replay()
            torch.cuda.synchronize(dev)
            if semicrf.get_status(ws) != 0 or not torch.equal(logZ, ref_logz) \
                    or not torch.equal(out["grad_em"], ref_gem):
                raise RuntimeError("graph replay differs from the eager step")
            launch_mode = "cuda graph (the step captured once, replayed)"
        except Exception as exc:  # keep the eager number
            graph = None
            launch_mode = f"eager (graph capture failed: {str(exc).splitlines()[0][:120]})"
    if world > 1:
        # every rank times the same way: the graph only if all captured it
        ok = torch.tensor([1 if graph is not None else 0], dtype=torch.int32, device=dev)
        dist.all_reduce(ok, op=dist.ReduceOp.MIN)
        if graph is not None and int(ok.item()) == 0:
            graph, launch_mode = None, "eager (graph capture failed on another rank)"
    if graph is not None:
        g_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        g_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.zero_()
            g_s[i].record(stream)
            graph.replay()
            allreduce_param_grads([out["grad_trans"], out["grad_dur"]])
            g_e[i].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        ms_step = reduce_max(sum(a.elapsed_time(b) for a, b in zip(g_s, g_e)), dev) / args.steps
    else:
        ms_step = ms_eager
    clocks = sampler.stop()
    kern = {}
    for name in semicrf.KERNELS:
        tot, n = semicrf.profile_read(name)
        if n:
            kern[name] = {"ms_total": tot, "launches": n, "ms_per_launch": tot / n}
    launches_per_step = sum(v["launches"] for v in kern.values()) / args.steps
    peak_mem = torch.cuda.max_memory_allocated(dev)

    # --- the loss: log Z - score(gold) with its gradient (the gold-path part
    # subtracted from the step's gradients), timed on its own: it is not part
    # of the fwd+bwd metric
    gold = torch.from_numpy(w["gold"]).to(dev)
    gold_start = torch.from_numpy(w["gold_start"]).to(dev)
    nll_grads = {k: torch.zeros_like(out[k]) for k in ("grad_em", "grad_trans", "grad_dur")}
    gscore = torch.empty(B, dtype=torch.float64, device=dev)

    def nll_step():
        semicrf.path_score(em, lengths, trans, dur, gold, gold_start, ws=ws, negate=True,
                           grads=nll_grads, score=gscore)

    for _ in range(max(args.warmup, 3)):
        nll_step()
    torch.cuda.synchronize(dev)
    n_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    n_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    semicrf.profile_enable(True)
    for i in range(args.steps):
        flush.zero_()
        n_s[i].record(stream)
        nll_step()
        n_e[i].record(stream)
    torch.cuda.synchronize(dev)
    semicrf.profile_enable(False)
    nll_ms = reduce_max(sum(a.elapsed_time(b) for a, b in zip(n_s, n_e)), dev) / args.steps
    nll_kern = {}
    for name in ("path_terms_kernel", "path_grad_kernel"):
        tot, n = semicrf.profile_read(name)
        if n:
            nll_kern[name] = {"ms_total": tot, "launches": n, "ms_per_launch": tot / n}
    nll_ok = bool(torch.isfinite(gscore).all().item()) and semicrf.get_status(ws) == 0

    # --- end to end: host (pinned) inputs -> device -> results back to host
    h_em = torch.from_numpy(w["em"]).pin_memory()
    h_len = torch.from_numpy(w["lengths"]).pin_memory()
    h_tr = torch.from_numpy(w["trans"]).pin_memory()
    h_du = torch.from_numpy(w["dur"]).pin_memory()
    d_em, d_len, d_tr, d_du = (torch.empty_like(x, device=dev) for x in (h_em, h_len, h_tr, h_du))
    h_out = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in
             (("logZ", logZ), ("grad_em", out["grad_em"]), ("grad_trans", out["grad_trans"]),
              ("grad_dur", out["grad_dur"]))}
    h_score = torch.empty(B, dtype=torch.float64).pin_memory()
    h_lab = torch.empty((B, T), dtype=torch.int32).pin_memory()
    h_seg = torch.empty((B, T), dtype=torch.uint8).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (h_em, h_len, h_tr, h_du))
    d2h = sum(x.numel() * x.element_size() for x in list(h_out.values()) + [h_score, h_lab, h_seg])

    def e2e_step():
        if graph is not None:
            for h, d in ((h_em, em), (h_len, lengths), (h_tr, trans), (h_du, dur)):
                d.copy_(h, non_blocking=True)
            graph.replay()
            allreduce_param_grads([out["grad_trans"], out["grad_dur"]])
            score, lab, seg = vout
        else:
            for h, d in ((h_em, d_em), (h_len, d_len), (h_tr, d_tr), (h_du, d_du)):
                d.copy_(h, non_blocking=True)
            score, lab, seg = step(d_em, d_len, d_tr, d_du)
        h_out["logZ"].copy_(logZ, non_blocking=True)
        for k in ("grad_em", "grad_trans", "grad_dur"):
            h_out[k].copy_(out[k], non_blocking=True)
        h_score.copy_(score, non_blocking=True)
        h_lab.copy_(lab, non_blocking=True)
        h_seg.copy_(seg, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()
        e_s[i].record(stream)
        e2e_step()
        e_e[i].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(sum(a.elapsed_time(b) for a, b in zip(e_s, e_e)), dev) / args.steps
    ok = bool(np.allclose(h_out["logZ"].numpy(), logZ.cpu().numpy()))

    line = None
    if rank == 0:
        peaks = measured_peaks()
        sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
        sm_max = float(peaks.get("sm_max_mhz", 1965.0))
        mufu_peak = sm_count * MUFU_PER_SM_PER_CLK * sm_max * 1e6      # ops/s
        roofs = {k: kernel_roofline(k, v, K, C, ring_pos.get(k, positions), args.steps,
                                    sm_count, sm_max)
                 for k, v in kern.items()}
        roofs = {k: v for k, v in roofs.items() if v}
        roofs_issued = {k: kernel_roofline(k, v, K, C, ring_pos.get(k, positions), args.steps,
                                           sm_count, sm_max, issued=True)
                        for k, v in kern.items()}
        roofs_issued = {k: v for k, v in roofs_issued.items() if v}
        # the dominant kernel: the largest share of device time
        dom = max(kern, key=lambda k: kern[k]["ms_total"]) if kern else None
        roof = roofs.get(dom)
        step_ops = 3 * K * C * C * positions  # forward + backward, per edge
        value = edges * world / (ms_step * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "ms_per_step_eager": ms_eager,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": B, "T": T, "K": K, "C": C,
                       "sum_lengths": positions, "edges_per_step_per_gpu": edges,
                       "padded_edges_per_step_per_gpu": B * T * K * C * C,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": "flushed between timed steps (256 MB write outside the events)",
                       "step": "forward + backward (marginals, grads) + viterbi (side stream)",
                       "launch": launch_mode},
            "positions_per_s": positions * world / (ms_step * 1e-3),
            "padded_edge_evals_per_s": B * T * K * C * C * world / (ms_step * 1e-3),
            "peak_hbm_bytes": peak_mem,
            "kernels": kern,
            "gpu_launches": int(round(launches_per_step * args.steps)),
            "step_mufu_frac": step_ops / (ms_step * 1e-3) / mufu_peak,
            "roofline": roof,
            "roofline_issued": roofs_issued.get(dom),
            "roofline_all": {k: {"frac": v["frac"], "achieved": v["achieved"], "peak": v["peak"],
                                 "frac_issued": roofs_issued[k]["frac"] if k in roofs_issued else None}
                             for k, v in roofs.items()},
            "e2e": {"value": edges * world / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "results_checked": bool(ok)},
            "clocks": clocks,
        }
        # algorithmic bytes per position: the terms pass reads the emission
        # row (4C, for nu), the label (4) and the start flag (1); the
        # gradient pass reads and writes the emission-gradient row (8C) and
        # reads the label (4); the count tables are O(C^2 + KC) per sequence
        nll_bytes = {"path_terms_kernel": (4 * C + 5) * positions,
                     "path_grad_kernel": (8 * C + 4) * positions}
        nll_roofs = {}
        for k, nb in nll_bytes.items():
            if k in nll_kern:
                per = nll_kern[k]["ms_per_launch"]
                nll_roofs[k] = {"bound": "hbm", "achieved": nb / (per * 1e-3) / 1e9,
                                "peak": peaks.get("hbm_gbs"), "unit": "GB/s",
                                "frac": (nb / (per * 1e-3) / 1e9) / peaks["hbm_gbs"]
                                if peaks.get("hbm_gbs") else None,
                                "bytes_per_launch": nb, "traffic": stored_traffic(k)}
        line["nll"] = {
            "what": "loss log Z - score(gold) and its gradient: semicrf_path_score with "
                    "SEMICRF_FLAG_NEGATE_GRAD on the gradient buffers (gold = the generating "
                    "segmentation), timed alone with L2 flushed between steps",
            "ms_per_step": nll_ms, "kernels": nll_kern, "roofline": nll_roofs,
            "gpu_launches_per_step": sum(v["launches"] for v in nll_kern.values()) / args.steps,
            "scores_finite": nll_ok,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the eager step only (no CUDA graph replay)")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
