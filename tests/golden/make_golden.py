"""Writes the float64 oracle's expected values for the five full-size workloads.

Usage:  python tests/golden/make_golden.py [tiny speech genomic ultra large]

Calls only the oracle (``oracle/``) on inputs drawn by the seeded generator
(``semi_markov_crf_b200.synth``), and stores, per workload, in
``tests/golden/<name>.npz``:

  logZ [B], grad_trans [C, C], grad_dur [K, C]          exact, in full
  viterbi_score [B]                                     the optimum
  sample_b, sample_u [S]                                seeded sampled positions
  pos_marg, grad_e [S, C]       at (b, u)               sampled outputs
  start_marg, end_marg [S, C]   at boundary (b, u)

The GPU parity tests regenerate the same inputs, run the CUDA path at the
benchmark's launch configuration and compare against these values, so the
oracle (minutes per workload at these sizes) does not run on the GPU machine.
"""

from __future__ import annotations

import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from semi_markov_crf_b200 import synth  # noqa: E402

NAMES = ("tiny", "speech", "genomic", "ultra", "large")


def sample_positions(lengths, C, seed):
    """Seeded (b, u) pairs with 0 <= u < L_b, about 1 MB of samples at most."""
    rng = np.random.default_rng(1000 + seed)
    n = int(min(4000, max(64, 32000 // C)))
    bs = rng.integers(0, len(lengths), size=n)
    us = np.array([rng.integers(0, max(1, int(lengths[b]))) for b in bs], dtype=np.int64)
    return bs.astype(np.int64), us


def make(name: str):
    w = synth.make(name)
    K = w["dur"].shape[0]
    t0 = time.time()
    fb = oracle.forward_backward(w["em"], w["lengths"], w["trans"], w["dur"], K)
    vit = oracle.viterbi(w["em"], w["lengths"], w["trans"], w["dur"], K)
    dt = time.time() - t0
    C = w["em"].shape[2]
    bs, us = sample_positions(w["lengths"], C, synth.CONFIGS[name].seed)
    out = dict(
        logZ=fb["logZ"], logZ_beta=fb["logZ_beta"], grad_trans=fb["grad_trans"],
        grad_dur=fb["grad_dur"], viterbi_score=vit["score"], sample_b=bs, sample_u=us,
        pos_marg=fb["pos_marg"][bs, us], grad_e=fb["grad_e"][bs, us],
        start_marg=fb["start_marg"][bs, us], end_marg=fb["end_marg"][bs, us],
        lengths=w["lengths"], oracle_seconds=np.array(dt))
    path = os.path.join(HERE, f"{name}.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: oracle {dt:.1f} s -> {path} ({os.path.getsize(path)} bytes)", flush=True)


if __name__ == "__main__":
    for n in (sys.argv[1:] or NAMES):
        make(n)
