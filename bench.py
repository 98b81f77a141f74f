#!/usr/bin/env python
"""Throughput benchmark of the streaming semi-CRF hot path on B200.

One step = the whole hot path over one batch, through the C ABI: prefix sums
and both rings (semicrf_forward), the posteriors with every output -- log Z,
position / start / end marginals, grad_em, grad_trans, grad_dur --
(semicrf_backward), and Viterbi decoding (semicrf_viterbi, on a side stream).
Metric: edge evaluations per second, edges = sum_b L_b * K * C^2 per step.

The headline workload is the largest single-GPU configuration, the
large-label batch (B=8, T=10,000, K=64, C=128: 8.4e10 edges per pass).  The
same line carries one entry per other workload under "workloads" (speech,
genomic, ultra, tiny), each timed the same way with its own roofline,
itemised peak memory and a sampled CPU-oracle baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--extras a,b,...|none]

With N > 1 (launched by torch.distributed.run) each rank runs its own batch
of the headline workload (seeded per rank: weak scaling) and the
batch-summed parameter gradients (grad_trans, grad_dur) are all-reduced over
NCCL every step, as a data-parallel training step needs; the extra
workloads run only at N = 1.  Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle (the only other
implementation here) on the host cores, on a bounded sample of the headline
workload per step.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

HEADLINE = "large"
EXTRAS = ("speech", "genomic", "ultra", "tiny")
METRIC = "semi-CRF fwd+bwd edge evals/s (B·T·K·C²), positions/s, peak HBM, % roofline"
UNIT = "edge evals/s"
MUFU_PER_SM_PER_CLK = 16          # ex2/lg2 results per SM per clock (SFU)
FP32_PER_SM_PER_CLK = 128         # fp32 lanes per SM per clock (4 partitions x 32)
L2_BYTES = 126 * 1024 * 1024
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "semi_markov_crf_b200", "csrc")

# kernels of the forward + backward pass (the metric); the decoder's are the rest
FWD_BWD_KERNELS = ("prefix_reduce_kernel", "prefix_scan_kernel", "chain_exp_kernel",
                   "chain_kernel", "cut_grid_kernel", "posterior_kernel", "segment_kernel",
                   "finalize_positions_kernel", "reduce_partials_kernel")

# Bounded samples of each workload for the float64 oracle on the host cores:
# (sequences, positions per sequence).  Sized for roughly 5-15 s of CPU time
# at the oracle's explicit-edge cost (K C^2 fp64 exponentials per position
# and pass).
CPU_SAMPLE = {"tiny": (1, 64), "speech": (32, 800), "genomic": (4, 16000),
              "ultra": (1, 24000), "large": (8, 200)}
# per step of the reference arm (it runs warm-up + steps samples)
REF_SAMPLE = {"tiny": (1, 64), "speech": (8, 800), "genomic": (4, 2000), "ultra": (1, 4000),
              "large": (8, 48)}


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


def algorithmic_ops_per_position(kernel: str, K: int, C: int):
    """Algorithmic work per sequence position of the factored recursion the
    kernels run, and the unit it occupies; None for kernels without such a
    count.

    The label fan-in is taken once per boundary (gamma = LSE over c' of
    alpha + trans), then the duration fan-in per label: K*C exponentials per
    boundary and direction (one per (k, c) term), C^2 multiply-adds for the
    label fan-in in the exponential domain.  MUFU binds (K*C / 16 per clock
    against C^2 / 128 per clock on the fp32 lanes at every configuration).
      rings (forward + backward in one launch):   2 K C exponentials
      posterior pass from the kept ring values:   K C   (one per (start, k, c) term)
      checkpoint walk (log-domain sequences):     2 K C (alpha recompute + beta walk)
      Viterbi recursion:                          2 (K C + C^2) fp32 add / max
    The nominal per-edge count K C^2 is the metric's unit of work, never a
    roofline numerator: the kernels do not execute it."""
    kc = K * C
    if kernel in ("chain_exp_kernel", "chain_kernel"):
        return 2 * kc, "mufu"
    if kernel == "posterior_kernel":
        return kc, "mufu"
    if kernel == "segment_kernel":
        return 2 * kc, "mufu"
    if kernel in ("viterbi_kernel", "viterbi_pipe_kernel"):
        return 2 * (kc + C * C), "fp32"
    return None


def hbm_bytes_per_position(kernel: str, C: int):
    """Algorithmic DRAM bytes per position of the O(T C) streaming kernels:
    the prefix-sum pass reads the emission row (4C) and writes the split
    prefix sums (8C); the reduction reads the emission row once (4C)."""
    if kernel == "prefix_scan_kernel":
        return 12 * C
    if kernel == "prefix_reduce_kernel":
        return 4 * C
    return None


def csrc_digest() -> str:
    """sha256 over the kernel sources, to tie a stored ncu traffic figure to
    the build it was measured on (the digest the library compiles in)."""
    from semi_markov_crf_b200.build import source_digest
    return source_digest()


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the
    committed ncu summary, or None when it was taken on other kernel
    sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("csrc_sha256") != csrc_digest():
        return None
    return t.get("workloads", {}).get(workload, {}).get(kernel)


def kernel_roofline(name: str, info: dict, K: int, C: int, positions: int, steps: int,
                    sm_count: int, sm_max_mhz: float, hbm_gbs: float | None = None,
                    workload: str | None = None) -> dict | None:
    """Roofline entry of one kernel: the algorithmic work of
    algorithmic_ops_per_position (or the bytes of hbm_bytes_per_position)
    times the positions one launch processes, over the kernel's mean launch
    time, against the unit that bounds it.  None for kernels without a
    count."""
    if positions <= 0 or not info.get("launches"):
        return None
    per_launch_positions = positions / (info["launches"] / steps)
    sec = info["ms_per_launch"] * 1e-3
    e = algorithmic_ops_per_position(name, K, C)
    if e is not None:
        ops_pos, unit = e
        per_clk, what = ((MUFU_PER_SM_PER_CLK, "MUFU ops/clk") if unit == "mufu"
                         else (FP32_PER_SM_PER_CLK, "fp32 lanes/clk"))
        peak = sm_count * per_clk * sm_max_mhz * 1e6
        per_launch = ops_pos * per_launch_positions
        achieved = per_launch / sec
        return {"bound": "alu", "kernel": name, "achieved": achieved / 1e9, "peak": peak / 1e9,
                "unit": "Gop/s", "frac": achieved / peak,
                "traffic": stored_traffic(name, workload) if workload else None,
                "peak_source": f"derived: {sm_count} SMs x {per_clk} {what} x {sm_max_mhz:.0f} MHz "
                               f"(sm_max_mhz of MEASURED_PEAKS.json)",
                "ops_per_launch": per_launch, "ops_per_position": ops_pos,
                "count": "factored fan-in: " + ("K*C exponentials per boundary and pass"
                                                if unit == "mufu" else
                                                "(K*C + C^2) add/max pairs per boundary")}
    nb = hbm_bytes_per_position(name, C)
    if nb is not None and hbm_gbs:
        per_launch = nb * per_launch_positions
        achieved = per_launch / sec / 1e9
        return {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": hbm_gbs,
                "unit": "GB/s", "frac": achieved / hbm_gbs,
                "traffic": stored_traffic(name, workload) if workload else None,
                "peak_source": "hbm_gbs of MEASURED_PEAKS.json (measured copy)",
                "bytes_per_launch": per_launch}
    return None


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


# ----------------------------------------------------------------------------- CPU oracle
def sample_of(w, n_seq: int, n_pos: int):
    """The first n_pos positions of the first n_seq sequences of workload w
    (a bounded sample with the workload's K, C and value distributions)."""
    n_seq = min(n_seq, w["em"].shape[0])
    n_pos = min(n_pos, w["em"].shape[1])
    em = np.ascontiguousarray(w["em"][:n_seq, :n_pos])
    lengths = np.minimum(w["lengths"][:n_seq], n_pos).astype(np.int32)
    return em, lengths


def oracle_sample_time(w, n_seq: int, n_pos: int, threads: int):
    """Time the float64 oracle (forward-backward + Viterbi) on a sample of
    workload w.  Returns (seconds, edges, positions)."""
    import oracle
    em, lengths = sample_of(w, n_seq, n_pos)
    K = w["dur"].shape[0]
    C = w["em"].shape[2]
    t0 = time.perf_counter()
    oracle.forward_backward(em, lengths, w["trans"], w["dur"], K, threads=threads)
    oracle.viterbi(em, lengths, w["trans"], w["dur"], K, threads=threads)
    dt = time.perf_counter() - t0
    return dt, edges_of(lengths, K, C), int(np.sum(lengths))


def cpu_baseline(name: str, w):
    n_seq, n_pos = CPU_SAMPLE[name]
    n_seq = min(n_seq, w["em"].shape[0])
    threads = min(os.cpu_count() or 1, n_seq)
    dt, edges, pos = oracle_sample_time(w, n_seq, n_pos, threads)
    reps = 1
    while dt * reps < 2.0 and reps < 256:   # tiny samples: repeat to a measurable time
        dt2, _, _ = oracle_sample_time(w, n_seq, n_pos, threads)
        dt += dt2
        reps += 1
    return {"value": edges * reps / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"first {min(n_pos, w['em'].shape[1])} positions of the first {n_seq} "
                      f"sequences of the {name} batch ({pos} positions), forward-backward + "
                      f"Viterbi in float64 with explicit edges, {threads} threads, "
                      f"{reps} run(s), {dt:.2f} s",
            "positions_per_s": pos * reps / dt}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from semi_markov_crf_b200 import synth
    name = args.workload
    w = synth.make(name)
    n_seq, n_pos = REF_SAMPLE[name]
    n_seq = min(n_seq, w["em"].shape[0])
    threads = min(os.cpu_count() or 1, n_seq)
    for _ in range(args.warmup):
        oracle_sample_time(w, n_seq, n_pos, threads)
    times, edges, pos = [], 0, 0
    for _ in range(args.steps):
        dt, edges, pos = oracle_sample_time(w, n_seq, n_pos, threads)
        times.append(dt)
    total = sum(times)
    value = edges * args.steps / total
    B, T, C = w["em"].shape
    K = w["dur"].shape[0]
    sample = (f"first {min(n_pos, T)} positions of the first {n_seq} sequences of the {name} "
              f"batch per step ({pos} positions), forward-backward + Viterbi in float64")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": name, "B": B, "T": T, "K": K, "C": C,
                   "sample_sequences_per_step": n_seq, "sample_positions_per_sequence": n_pos},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm
def _nbytes(*ts):
    return int(sum(t.numel() * t.element_size() for t in ts))


class Workload:
    """Inputs, workspaces, outputs and the step of one workload on one GPU."""

    def __init__(self, name: str, seed: int, dev):
        import torch
        from semi_markov_crf_b200 import semicrf, synth
        self.name = name
        self.dev = dev
        self.semicrf = semicrf
        self.w = w = synth.make(name, seed=seed)
        self.B, self.T, self.C = w["em"].shape
        self.K = w["dur"].shape[0]
        B, T, C, K = self.B, self.T, self.C, self.K
        self.mem0 = torch.cuda.memory_allocated(dev)
        self.em = torch.from_numpy(w["em"]).to(dev)
        self.lengths = torch.from_numpy(w["lengths"]).to(dev)
        self.trans = torch.from_numpy(w["trans"]).to(dev)
        self.dur = torch.from_numpy(w["dur"]).to(dev)
        self.edges = edges_of(w["lengths"], K, C)
        self.positions = int(w["lengths"].sum())
        self.ws = semicrf.Workspace(B, T, C, K, 0, dev)
        self.vws = semicrf.Workspace(B, T, C, K, 0, dev)
        self.logZ = torch.empty(B, dtype=torch.float64, device=dev)
        self.out = {"grad_em": torch.empty((B, T, C), dtype=torch.float32, device=dev),
                    "grad_trans": torch.empty((C, C), dtype=torch.float32, device=dev),
                    "grad_dur": torch.empty((K, C), dtype=torch.float32, device=dev),
                    "pos_marg": torch.empty((B, T, C), dtype=torch.float32, device=dev),
                    "start_marg": torch.empty((B, T + 1, C), dtype=torch.float32, device=dev),
                    "end_marg": torch.empty((B, T + 1, C), dtype=torch.float32, device=dev)}
        self.vout = (torch.empty(B, dtype=torch.float64, device=dev),
                     torch.empty((B, T), dtype=torch.int32, device=dev),
                     torch.empty((B, T), dtype=torch.uint8, device=dev))
        self.side = torch.cuda.Stream(dev)

    def lib_step(self, em_, lengths_, trans_, dur_):
        """One pass of the hot path.  Viterbi does not depend on the
        forward-backward pass and the two leave most SMs free between them:
        decode on a side stream, join at the end."""
        import torch
        s = self.semicrf
        main = torch.cuda.current_stream(self.dev)
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            res = s.viterbi(em_, lengths_, trans_, dur_, ws=self.vws, out=self.vout)
        s.forward(em_, lengths_, trans_, dur_, ws=self.ws, logZ=self.logZ)
        s.backward(self.ws, lengths_, trans_, dur_, marginals=True, out=self.out)
        main.wait_stream(self.side)
        return res

    def step(self):
        res = self.lib_step(self.em, self.lengths, self.trans, self.dur)
        allreduce_param_grads([self.out["grad_trans"], self.out["grad_dur"]])
        return res

    def memory(self, peak_alloc: int) -> dict:
        """Peak device memory of the step, itemised: inputs, the two
        workspaces (forward-backward and decoder) by group, outputs."""
        s = self.semicrf
        B, T, C, K = self.B, self.T, self.C, self.K
        inputs = _nbytes(self.em, self.lengths, self.trans, self.dur)
        outputs = _nbytes(self.logZ, *self.out.values(), *self.vout)
        ws_fb = s.workspace_itemize(B, T, C, K, 0)
        ws_v = s.workspace_itemize(B, T, C, K, 0)
        items = {"inputs": inputs, "outputs": outputs,
                 "workspace_fwd_bwd": ws_fb, "workspace_fwd_bwd_bytes": self.ws.nbytes,
                 "workspace_viterbi_bytes": self.vws.nbytes,
                 "workspace_viterbi_used": {k: ws_v[k] for k in ("other", "prefix_sums", "viterbi")}}
        return {"peak_bytes": int(peak_alloc - self.mem0),
                "itemised_sum": inputs + outputs + self.ws.nbytes + self.vws.nbytes,
                "items": items,
                "explicit_edge_tensor_bytes": B * T * K * C * C * 4,
                "note": "peak = torch.cuda.max_memory_allocated over the warm-up steps minus what "
                        "was allocated before this workload (the L2-flush buffer included); the "
                        "decoder's workspace is a second one of the same size, since it runs "
                        "concurrently, and uses only its prefix-sum and decoder groups"}


def time_steps(fn, steps, stream, flush, dev):
    import torch
    s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i in range(steps):
        flush.zero_()                       # evict L2 between timed steps (outside the events)
        s[i].record(stream)
        fn()
        e[i].record(stream)
    torch.cuda.synchronize(dev)
    return sum(a.elapsed_time(b) for a, b in zip(s, e))


def measure(wl: Workload, steps: int, warmup: int, flush, world: int, local: int,
            use_graph: bool, peaks: dict, sm_count: int):
    """Device time of `steps` steps of wl (eager with per-kernel timing, then
    the same step replayed as a CUDA graph), clocks, roofline and memory."""
    import torch
    import torch.distributed as dist
    s = wl.semicrf
    dev = wl.dev
    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(max(warmup, 3)):
        wl.step()
    torch.cuda.synchronize(dev)
    if s.get_status(wl.ws) != 0:
        raise RuntimeError(f"{wl.name}: device status {s.get_status(wl.ws)}")
    peak_alloc = torch.cuda.max_memory_allocated(dev)
    B, T, C, K = wl.B, wl.T, wl.C, wl.K
    # which kernel ran each ring: positions per ring kernel, both directions
    dom = s.ring_domains(wl.ws)
    lens = [int(x) for x in wl.w["lengths"]]
    kept = [dom[b] == 1 and dom[B + b] == 1 for b in range(B)]
    ring_pos = {"chain_exp_kernel": sum(lens[i % B] for i, m in enumerate(dom) if m == 1) / 2,
                "chain_kernel": sum(lens[i % B] for i, m in enumerate(dom) if m == 2) / 2,
                "posterior_kernel": sum(l for l, k in zip(lens, kept) if k),
                "segment_kernel": sum(l for l, k in zip(lens, kept) if not k)}

    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    s.profile_enable(True)
    if world > 1:
        dist.barrier()
    ms_eager = reduce_max(time_steps(wl.step, steps, stream, flush, dev), dev) / steps
    if world > 1:
        dist.barrier()
    s.profile_enable(False)
    kern = {}
    for name in s.KERNELS:
        tot, n = s.profile_read(name)
        if n:
            kern[name] = {"ms_total": tot, "launches": n, "ms_per_launch": tot / n}

    # The same step captured once into a CUDA graph and replayed: the library
    # allocates nothing and never synchronises inside a call, so the whole
    # step (both streams, the library's own side stream) is capturable; the
    # replay removes the host launch latency and the gaps between dependent
    # launches.  The gradient all-reduce (N > 1) stays outside the graph.
    graph, launch_mode = None, "eager"
    if use_graph:
        try:
            ref_logz, ref_gem = wl.logZ.clone(), wl.out["grad_em"].clone()
            ref_lab = wl.vout[1].clone()
            torch.cuda.synchronize(dev)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, capture_error_mode="relaxed"):
                wl.lib_step(wl.em, wl.lengths, wl.trans, wl.dur)
            graph.replay()
            torch.cuda.synchronize(dev)
            if s.get_status(wl.ws) != 0 or not torch.equal(wl.logZ, ref_logz) \
                    or not torch.equal(wl.out["grad_em"], ref_gem) \
                    or not torch.equal(wl.vout[1], ref_lab):
                raise RuntimeError("graph replay differs from the eager step")
            launch_mode = "cuda graph (the step captured once, replayed)"
        except Exception as exc:  # keep the eager number
            graph = None
            launch_mode = f"eager (graph capture failed: {str(exc).splitlines()[0][:120]})"
    if world > 1:
        ok = torch.tensor([1 if graph is not None else 0], dtype=torch.int32, device=dev)
        dist.all_reduce(ok, op=dist.ReduceOp.MIN)
        if graph is not None and int(ok.item()) == 0:
            graph, launch_mode = None, "eager (graph capture failed on another rank)"
    if graph is not None:
        def replay():
            graph.replay()
            allreduce_param_grads([wl.out["grad_trans"], wl.out["grad_dur"]])
        if world > 1:
            dist.barrier()
        ms_step = reduce_max(time_steps(replay, steps, stream, flush, dev), dev) / steps
    else:
        ms_step = ms_eager
    clocks = sampler.stop()

    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    hbm = peaks.get("hbm_gbs")
    roofs = {}
    for k, v in kern.items():
        r = kernel_roofline(k, v, K, C, ring_pos.get(k, wl.positions), steps, sm_count, sm_max,
                            hbm, wl.name)
        if r:
            roofs[k] = r
    fb = [k for k in kern if k in FWD_BWD_KERNELS]
    dom_k = max(fb, key=lambda k: kern[k]["ms_total"]) if fb else None
    mufu_peak = sm_count * MUFU_PER_SM_PER_CLK * sm_max * 1e6
    fb_ms = sum(kern[k]["ms_total"] for k in fb) / steps
    res = {
        "workload": wl.name, "B": B, "T": T, "K": K, "C": C, "sum_lengths": wl.positions,
        "edges_per_step": wl.edges, "padded_edges_per_step": B * T * K * C * C,
        "ms_per_step": ms_step, "ms_per_step_eager": ms_eager, "launch": launch_mode,
        "value": wl.edges * world / (ms_step * 1e-3),
        "positions_per_s": wl.positions * world / (ms_step * 1e-3),
        "padded_edge_evals_per_s": B * T * K * C * C * world / (ms_step * 1e-3),
        "fwd_bwd_kernel_ms_per_step": fb_ms,
        "kernels": kern,
        "gpu_launches_per_step": sum(v["launches"] for v in kern.values()) / steps,
        # whole step against the factored count: 2 K C (rings) + K C (posteriors)
        "step_mufu_frac": 3 * K * C * wl.positions / (ms_step * 1e-3) / mufu_peak,
        "roofline": roofs.get(dom_k),
        "roofline_all": {k: {"frac": v["frac"], "achieved": v["achieved"], "peak": v["peak"],
                             "unit": v["unit"]} for k, v in roofs.items()},
        "memory": wl.memory(peak_alloc),
        "clocks": clocks,
    }
    return res, graph


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
    peaks = measured_peaks()
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    name = args.workload
    base = synth.WORKLOADS[name]
    wl = Workload(name, shard_seed(base.seed, rank), dev)
    head, graph = measure(wl, args.steps, args.warmup, flush, world, local, not args.no_graph,
                          peaks, sm_count)
    B, T, C, K = wl.B, wl.T, wl.C, wl.K
    em, lengths, trans, dur, out, logZ = wl.em, wl.lengths, wl.trans, wl.dur, wl.out, wl.logZ
    stream = torch.cuda.current_stream(dev)

    # --- the loss: log Z - score(gold) with its gradient (the gold-path part
    # subtracted from the step's gradients), timed on its own: it is not part
    # of the fwd+bwd metric
    gold = torch.from_numpy(wl.w["gold"]).to(dev)
    gold_start = torch.from_numpy(wl.w["gold_start"]).to(dev)
    nll_grads = {k: torch.zeros_like(out[k]) for k in ("grad_em", "grad_trans", "grad_dur")}
    gscore = torch.empty(B, dtype=torch.float64, device=dev)

    def nll_step():
        semicrf.path_score(em, lengths, trans, dur, gold, gold_start, ws=wl.ws, negate=True,
                           grads=nll_grads, score=gscore)

    for _ in range(max(args.warmup, 3)):
        nll_step()
    semicrf.profile_enable(True)
    nll_ms = reduce_max(time_steps(nll_step, args.steps, stream, flush, dev), dev) / args.steps
    semicrf.profile_enable(False)
    nll_kern = {}
    for k in ("path_terms_kernel", "path_grad_kernel"):
        tot, n = semicrf.profile_read(k)
        if n:
            nll_kern[k] = {"ms_total": tot, "launches": n, "ms_per_launch": tot / n}
    nll_ok = bool(torch.isfinite(gscore).all().item()) and semicrf.get_status(wl.ws) == 0

    # --- end to end: host (pinned) inputs -> device -> results back to host
    h_em = torch.from_numpy(wl.w["em"]).pin_memory()
    h_len = torch.from_numpy(wl.w["lengths"]).pin_memory()
    h_tr = torch.from_numpy(wl.w["trans"]).pin_memory()
    h_du = torch.from_numpy(wl.w["dur"]).pin_memory()
    d_em, d_len, d_tr, d_du = (torch.empty_like(x, device=dev) for x in (h_em, h_len, h_tr, h_du))
    h_out = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in
             [("logZ", logZ)] + list(out.items())}
    h_score = torch.empty(B, dtype=torch.float64).pin_memory()
    h_lab = torch.empty((B, T), dtype=torch.int32).pin_memory()
    h_seg = torch.empty((B, T), dtype=torch.uint8).pin_memory()
    h2d = _nbytes(h_em, h_len, h_tr, h_du)
    d2h = _nbytes(*h_out.values(), h_score, h_lab, h_seg)

    def e2e_step():
        if graph is not None:
            for h, d in ((h_em, em), (h_len, lengths), (h_tr, trans), (h_du, dur)):
                d.copy_(h, non_blocking=True)
            graph.replay()
            allreduce_param_grads([out["grad_trans"], out["grad_dur"]])
            score, lab, seg = wl.vout
        else:
            for h, d in ((h_em, d_em), (h_len, d_len), (h_tr, d_tr), (h_du, d_du)):
                d.copy_(h, non_blocking=True)
            score, lab, seg = wl.lib_step(d_em, d_len, d_tr, d_du)
            allreduce_param_grads([out["grad_trans"], out["grad_dur"]])
        h_out["logZ"].copy_(logZ, non_blocking=True)
        for k, v in out.items():
            h_out[k].copy_(v, non_blocking=True)
        h_score.copy_(score, non_blocking=True)
        h_lab.copy_(lab, non_blocking=True)
        h_seg.copy_(seg, non_blocking=True)

    for _ in range(3):
        e2e_step()
    if world > 1:
        dist.barrier()
    e2e_ms = reduce_max(time_steps(e2e_step, args.steps, stream, flush, dev), dev) / args.steps
    ok = bool(np.allclose(h_out["logZ"].numpy(), logZ.cpu().numpy()))
    del graph

    extras = {}
    if world == 1:
        for ex in [x for x in args.extras.split(",") if x and x != "none" and x != name]:
            wx = Workload(ex, synth.WORKLOADS[ex].seed, dev)
            rx, gx = measure(wx, min(args.steps, args.extra_steps), min(args.warmup, 3), flush, 1,
                             local, not args.no_graph, peaks, sm_count)
            del gx
            if not args.no_cpu_baseline:
                rx["cpu_baseline"] = cpu_baseline(ex, wx.w)
            extras[ex] = rx
            del wx
            torch.cuda.empty_cache()

    line = None
    if rank == 0:
        roof = head["roofline"]
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": head["ms_per_step"],
            "ms_per_step_eager": head["ms_per_step_eager"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": name, "B": B, "T": T, "K": K, "C": C,
                       "sum_lengths": wl.positions, "edges_per_step_per_gpu": wl.edges,
                       "padded_edges_per_step_per_gpu": B * T * K * C * C,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": "flushed between timed steps (256 MB write outside the events)",
                       "step": "prefix sums + forward + backward (log Z, position/start/end "
                               "marginals, grad_em, grad_trans, grad_dur) + Viterbi on a side "
                               "stream",
                       "launch": head["launch"]},
            "positions_per_s": head["positions_per_s"],
            "padded_edge_evals_per_s": head["padded_edge_evals_per_s"],
            "peak_hbm_bytes": head["memory"]["peak_bytes"],
            "memory": head["memory"],
            "kernels": head["kernels"],
            "gpu_launches": int(round(head["gpu_launches_per_step"] * args.steps)),
            "step_mufu_frac": head["step_mufu_frac"],
            "roofline": roof,
            "roofline_all": head["roofline_all"],
            "fwd_bwd_kernel_ms_per_step": head["fwd_bwd_kernel_ms_per_step"],
            "e2e": {"value": wl.edges * world / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "results_checked": bool(ok)},
            "clocks": head["clocks"],
        }
        line["nll"] = {
            "what": "loss log Z - score(gold) and its gradient: semicrf_path_score with "
                    "SEMICRF_FLAG_NEGATE_GRAD on the gradient buffers (gold = the generating "
                    "segmentation), timed alone with L2 flushed between steps",
            "ms_per_step": nll_ms, "kernels": nll_kern,
            "gpu_launches_per_step": sum(v["launches"] for v in nll_kern.values()) / args.steps,
            "scores_finite": nll_ok,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(name, wl.w)
        if extras:
            line["workloads"] = extras
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
    ap.add_argument("--workload", default=HEADLINE,
                    choices=("tiny", "speech", "genomic", "ultra", "large"))
    ap.add_argument("--extras", default=",".join(EXTRAS),
                    help="comma-separated further workloads timed at N=1 ('none' for none)")
    ap.add_argument("--extra-steps", type=int, default=5)
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
