"""Writes the float64 oracle's expected values for the full-size workloads.

Usage:  python tests/golden/make_golden.py [genomic ultra large ...]

Calls only the oracle (``oracle/``) on inputs drawn by the seeded generator
(``semi_markov_crf_b200.synth``), and stores, per workload, in
``tests/golden/<name>.npz``:

  logZ [B], logZ_beta [B], grad_trans [C, C], grad_dur [K, C]   in full
  viterbi_score [B]                                  the optimum
  viterbi_labels [B, T] int8/int16, viterbi_seg [B, T] packed bits
                                                     the oracle's decoded path, in full
  row_b, row_u [R]              targeted positions (b, u), u < L_b
  q_pos_marg, q_grad_e [R, C]   outputs there
  brow_b, brow_u [S]            targeted boundaries (b, t), t <= L_b
  q_start_marg, q_end_marg [S, C]
                                boundary marginals there

Marginals and emission gradients are stored quantised, round(x * 2^17) as
int32 (error <= 2^-18, far below the 1e-4 tolerance), so that values near
zero compress.  The targeted rows are the positions around the points where
the kernels change state -- both sides of every 8th prefix-sum tile edge
(multiples of 256) and of every cut-normaliser grid point (multiples of
128), two rows either side of every checkpoint at the checkpoint spacing
ceil(sqrt(T K)) and at the library's capped spacing, with the rows K before
and after each checkpoint (segments that straddle it), and the first and
last K + 2 rows of each sequence -- plus seeded random rows.  For wide label
sets (C > 64) only the first and last sequence get the targeted rows.

The tiny and speech workloads are not stored: the GPU tests run the oracle on
them at test time (seconds) and compare every element.  ``long_k`` is the
long-duration case (B=2, T=6,000, K=8000, C=6), stored at every position.

The GPU parity tests regenerate the same inputs, run the CUDA path at the
benchmark's launch configuration and compare against these values, so the
oracle (minutes per workload at these sizes) does not run on the GPU machine.
"""

from __future__ import annotations

import math
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from semi_markov_crf_b200 import synth  # noqa: E402

NAMES = ("genomic", "ultra", "large", "long_k")


def long_k_case():
    """Long durations (the pages' genomic regime of K = 2000-8000): B=2,
    T=6,000 (lengths 6,000 and 4,500), K=8000, C=6, the genomic label
    frequencies with segments of mean length 500.  (The oracle's position
    marginals sum every covering segment explicitly, O(T K^2 C): at this
    size that is minutes, at T = 20,000 hours.)"""
    return synth.make_custom(2, 6_000, 8000, 6, seed=43, lengths=[6_000, 4_500],
                             dur_mean=500.0, amp=2.0,
                             label_p=(0.6, 0.2, 0.1, 0.05, 0.03, 0.02))


def workload(name: str):
    return long_k_case() if name == "long_k" else synth.make(name)
QSCALE = float(1 << 17)
SMS = 148  # B200: the library's checkpoint cap depends on the SM count


def spacings(T: int, K: int, B: int):
    """Checkpoint spacings the rows are aimed at: the pages' ceil(sqrt(T K))
    and the library's spacing on a 148-SM GPU (capped so the posterior pass
    is one wave)."""
    pages = math.isqrt(T * K)
    if pages * pages < T * K:
        pages += 1
    per_seq = max(1, 2 * SMS // max(B, 1))
    lib = min(pages, max(2 * K, -(-T // per_seq)))
    return sorted({pages, max(lib, 1)})


def target_rows(lengths, T: int, K: int, seed: int, n_random: int, targeted):
    """Sorted unique (b, u) position rows and (b, t) boundary rows; the
    sequences in `targeted` get the state-change rows, every sequence the
    random ones."""
    rng = np.random.default_rng(1000 + seed)
    B = len(lengths)
    pos_b, pos_u, bnd_b, bnd_u = [], [], [], []
    for b in range(B):
        L = int(lengths[b])
        pts = set()
        if b in targeted:
            for p in range(256, L, 256):                  # prefix-sum tile edges (every 8th)
                pts.update((p - 1, p))
            for p in range(128, L + 1, 128):              # cut-normaliser grid
                pts.update((p - 1, p))
            for s in spacings(T, K, B):                   # checkpoints, and segments across them
                for p in range(s, L + 1, s):
                    pts.update(range(p - 2, p + 2))
                    pts.update((p - K, p - K + 1, p + K - 1, p + K))
            pts.update(range(0, min(L, K + 2)))
            pts.update(range(max(0, L - K - 2), L + 1))
        pts.update(int(x) for x in rng.integers(0, L + 1, size=n_random))
        rows = sorted(x for x in pts if 0 <= x < L)
        bnds = sorted(x for x in pts if 0 <= x <= L)
        pos_b += [b] * len(rows)
        pos_u += rows
        bnd_b += [b] * len(bnds)
        bnd_u += bnds
    return (np.array(pos_b, np.int32), np.array(pos_u, np.int32),
            np.array(bnd_b, np.int32), np.array(bnd_u, np.int32))


def quantise(x):
    return np.rint(np.asarray(x, np.float64) * QSCALE).astype(np.int32)


def make(name: str):
    w = workload(name)
    K = w["dur"].shape[0]
    B, T, C = w["em"].shape
    t0 = time.time()
    fb = oracle.forward_backward(w["em"], w["lengths"], w["trans"], w["dur"], K)
    vit = oracle.viterbi(w["em"], w["lengths"], w["trans"], w["dur"], K)
    dt = time.time() - t0
    # wide label sets: the state-change rows of the first and last sequence
    targeted = {0, B - 1} if C > 64 else set(range(B))
    n_random = 100 if C > 64 else 300
    seed = 43 if name == "long_k" else synth.WORKLOADS[name].seed
    if name == "long_k":  # every position
        rb, ru = np.nonzero(np.arange(T)[None, :] < w["lengths"][:, None])
        bb, bu = np.nonzero(np.arange(T + 1)[None, :] <= w["lengths"][:, None])
        rb, ru, bb, bu = (x.astype(np.int32) for x in (rb, ru, bb, bu))
    else:
        rb, ru, bb, bu = target_rows(w["lengths"], T, K, seed, n_random, targeted)
    lab_dtype = np.int8 if C <= 127 else np.int16
    out = dict(
        logZ=fb["logZ"], logZ_beta=fb["logZ_beta"], grad_trans=fb["grad_trans"],
        grad_dur=fb["grad_dur"], viterbi_score=vit["score"],
        viterbi_labels=vit["labels"].astype(lab_dtype),
        viterbi_seg=np.packbits(vit["seg_start"].astype(np.uint8), axis=1),
        row_b=rb, row_u=ru, q_pos_marg=quantise(fb["pos_marg"][rb, ru]),
        q_grad_e=quantise(fb["grad_e"][rb, ru]),
        brow_b=bb, brow_u=bu, q_start_marg=quantise(fb["start_marg"][bb, bu]),
        q_end_marg=quantise(fb["end_marg"][bb, bu]),
        qscale=np.array(QSCALE), lengths=w["lengths"], oracle_seconds=np.array(dt))
    path = os.path.join(HERE, f"{name}.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: oracle {dt:.1f} s, {len(rb)} position rows, {len(bb)} boundary rows -> "
          f"{path} ({os.path.getsize(path)} bytes)", flush=True)


if __name__ == "__main__":
    for n in (sys.argv[1:] or NAMES):
        make(n)
