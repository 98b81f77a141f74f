"""Seeded synthetic semi-CRF workloads.

This module only draws random numbers.  It holds none of the semi-CRF
arithmetic (no centering, no prefix sums, no recursions), so both the CUDA
path and the float64 oracle can be fed from it without sharing any of the
method's code.

The workloads mirror the ones the Flash-SemiCRF pages talk about:

* ``tiny``    B=1, T=64, K=8, C=4; emissions N(0,1), trans/dur N(0,0.1), seed 0.
* ``speech``  B=32, lengths uniform in [300, 800] (padded T=800), K=30, C=39.
              Labels uniform, geometric durations (mean 8) capped at K,
              emissions 1.5*onehot + N(0,1).  Stands in for the TIMIT phone
              segmentation task (explainer, section 4 "Results and
              Benchmarks", TIMIT with K=30); TIMIT itself is not used.
* ``genomic`` B=4, T=100000, K=200, C=6.  Label frequencies
              (.6,.2,.1,.05,.03,.02), geometric durations (mean 50) capped at
              K, emissions 2*onehot + N(0,1).  Stands in for the genome-scale
              sequences of the explainer's section 1 (T > 1e5).
* ``ultra``   B=1, T=1000000, same generator as ``genomic``: the
              T=1e6, K=200, C=6 case whose explicit edge tensor is ~29 GB
              (explainer, section 1 "Problem Statement").
* ``large``   B=8, T=10000, K=64, C=128, uniform labels, durations mean 16,
              emissions 1.0*onehot + N(0,1), trans/dur N(0,0.05).

Draw order (fixed, so that a seed reproduces the same arrays everywhere):
lengths for all sequences; then per sequence the (label, duration) pairs
until the sequence is covered (the last segment truncated), then that
sequence's noise; then ``trans``; then ``dur``.  Padding past each length is
zero unless ``pad_value`` says otherwise.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make", "make_custom", "checkpoint_interval"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    K: int
    C: int
    seed: int
    len_lo: int            # lengths drawn uniformly in [len_lo, T]; len_lo == T means fixed
    label_p: tuple | None  # None -> uniform over C; "noise" workloads use mode == "noise"
    dur_mean: float
    amp: float             # onehot amplitude of the true label
    param_std: float       # std of trans and dur
    mode: str = "segments"  # "segments" (onehot + noise) or "noise" (pure N(0,1))


WORKLOADS = {
    "tiny": Workload("tiny", 1, 64, 8, 4, 0, 64, None, 1.0, 0.0, 0.1, mode="noise"),
    "speech": Workload("speech", 32, 800, 30, 39, 1, 300, None, 8.0, 1.5, 0.1),
    "genomic": Workload("genomic", 4, 100_000, 200, 6, 2, 100_000,
                        (0.6, 0.2, 0.1, 0.05, 0.03, 0.02), 50.0, 2.0, 0.1),
    "ultra": Workload("ultra", 1, 1_000_000, 200, 6, 3, 1_000_000,
                      (0.6, 0.2, 0.1, 0.05, 0.03, 0.02), 50.0, 2.0, 0.1),
    "large": Workload("large", 8, 10_000, 64, 128, 4, 10_000, None, 16.0, 1.0, 0.05),
}


def checkpoint_interval(T: int, K: int) -> int:
    """Checkpoint spacing Delta = ceil(sqrt(T*K)) on the padded length."""
    if T <= 0:
        return 1
    d = math.isqrt(T * K)
    if d * d < T * K:
        d += 1
    return max(d, 1)


def _draw(rng, w: Workload, B: int, T: int, K: int, C: int, pad_value):
    if w.len_lo >= T:
        lengths = np.full(B, T, dtype=np.int32)
    else:
        lengths = rng.integers(w.len_lo, T + 1, size=B).astype(np.int32)
    em = np.zeros((B, T, C), dtype=np.float32)
    gold = np.full((B, T), -1, dtype=np.int32)
    gold_start = np.zeros((B, T), dtype=np.uint8)
    for b in range(B):
        L = int(lengths[b])
        if w.mode == "noise":
            em[b, :L] = rng.standard_normal((L, C)).astype(np.float32)
        else:
            labels = np.empty(L, dtype=np.int32)
            pos = 0
            while pos < L:
                if w.label_p is None:
                    c = int(rng.integers(0, C))
                else:
                    c = int(rng.choice(C, p=np.asarray(w.label_p, dtype=np.float64)))
                d = int(rng.geometric(1.0 / w.dur_mean))
                d = min(d, K, L - pos)
                labels[pos:pos + d] = c
                gold_start[b, pos] = 1
                pos += d
            noise = rng.standard_normal((L, C))
            x = noise
            x[np.arange(L), labels] += w.amp
            em[b, :L] = x.astype(np.float32)
            gold[b, :L] = labels
        if pad_value is not None and L < T:
            em[b, L:] = pad_value
    trans = (w.param_std * rng.standard_normal((C, C))).astype(np.float32)
    dur = (w.param_std * rng.standard_normal((K, C))).astype(np.float32)
    return dict(em=em, lengths=lengths, trans=trans, dur=dur, K=K, gold=gold,
                gold_start=gold_start)


def make(name: str, pad_value=None, B: int | None = None, T: int | None = None,
         seed: int | None = None) -> dict:
    """Draw one named workload.

    ``B``/``T`` override the batch size / padded length (keeping every other
    setting; a length range is rescaled proportionally), which the tests use
    to get oracle-sized cases of the same distribution.  Returns a dict with
    ``em`` [B,T,C] float32, ``lengths`` [B] int32, ``trans`` [C,C] float32
    (trans[c_prev, c]), ``dur`` [K,C] float32 (dur[k-1, c] scores duration
    k), ``K`` and the generating segmentation: labels ``gold`` [B,T] (-1 =
    padding) and ``gold_start`` [B,T] uint8 (1 where a drawn segment starts;
    two adjacent drawn segments may share a label).
    """
    w = WORKLOADS[name]
    B_ = w.B if B is None else int(B)
    T_ = w.T if T is None else int(T)
    if T is not None and w.len_lo < w.T:
        lo = max(1, int(round(w.len_lo * T_ / w.T)))
        w = dataclasses.replace(w, len_lo=lo)
    elif T is not None:
        w = dataclasses.replace(w, len_lo=T_)
    rng = np.random.default_rng(w.seed if seed is None else seed)
    out = _draw(rng, w, B_, T_, w.K, w.C, pad_value)
    out["name"] = name
    return out


def make_custom(B: int, T: int, K: int, C: int, seed: int, *, lengths=None,
                amp: float = 1.0, dur_mean: float = 4.0, param_std: float = 0.1,
                label_p=None, mode: str = "segments", pad_value=None) -> dict:
    """Draw a workload of arbitrary shape (edge-case and sweep tests)."""
    if lengths is None:
        len_lo = T
    else:
        len_lo = None
    w = Workload("custom", B, T, K, C, seed, len_lo if len_lo is not None else T,
                 None if label_p is None else tuple(label_p), dur_mean, amp, param_std, mode)
    rng = np.random.default_rng(seed)
    out = _draw(rng, w, B, T, K, C, pad_value)
    if lengths is not None:
        lengths = np.asarray(lengths, dtype=np.int32)
        assert lengths.shape == (B,)
        em = out["em"]
        for b in range(B):
            L = int(lengths[b])
            if L < T:
                em[b, L:] = 0.0 if pad_value is None else pad_value
                out["gold"][b, L:] = -1
                out["gold_start"][b, L:] = 0
        out["lengths"] = lengths
    out["name"] = "custom"
    return out
