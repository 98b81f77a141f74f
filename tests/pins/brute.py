"""Brute-force enumeration of every labelled segmentation (tiny inputs only).

An independent statement of the semi-CRF of the Flash-SemiCRF pages
(explainer section 1, "Problem Statement"): a segmentation splits positions
0..L-1 into consecutive segments of duration 1..K, each with one of C labels;
its score is the sum of segment content (summed centred emissions), the
duration score dur[k-1, c] and the transition trans[c', c] between
consecutive segments.  Here every segmentation is listed and scored one by
one, so log Z, every marginal and the argmax follow from their definitions
with no dynamic programming at all.
"""

from __future__ import annotations

import math

import numpy as np


def segmentations(L: int, K: int, C: int):
    """Yield every segmentation as a tuple of (start, end, label)."""
    def rec(pos):
        if pos == L:
            yield ()
            return
        for k in range(1, min(K, L - pos) + 1):
            for c in range(C):
                for rest in rec(pos + k):
                    yield ((pos, pos + k, c),) + rest
    yield from rec(0)


def score(segs, et, trans, dur, ps=None, pe=None):
    total = 0.0
    prev = None
    for (s, t, c) in segs:
        total += float(sum(et[u, c] for u in range(s, t)))
        total += float(dur[t - s - 1, c])
        if ps is not None:
            total += float(ps[s, c])      # boundary projections: start at s,
        if pe is not None:
            total += float(pe[t - 1, c])  # end at position t-1
        if prev is not None:
            total += float(trans[prev, c])
        prev = c
    return total


def enumerate_all(e, L, trans, dur, center=True, tie_tol=1e-9, ps=None, pe=None):
    """Everything the oracle reports, by enumeration, for one sequence."""
    e = np.asarray(e, dtype=np.float64)[:L]
    trans = np.asarray(trans, dtype=np.float64)
    dur = np.asarray(dur, dtype=np.float64)
    K, C = dur.shape
    nu = e.mean(axis=0) if (center and L > 0) else np.zeros(C)
    et = e - nu
    segs_all = list(segmentations(L, K, C))
    scores = np.array([score(sg, et, trans, dur, ps, pe) for sg in segs_all])
    m = scores.max()
    logZ = m + math.log(np.exp(scores - m).sum())
    probs = np.exp(scores - logZ)
    St = np.zeros((L + 1, C))
    En = np.zeros((L + 1, C))
    mu = np.zeros((L, C))
    gdur = np.zeros((K, C))
    gtrans = np.zeros((C, C))
    segm = np.zeros((max(L, 1), K, C))
    for p, sg in zip(probs, segs_all):
        prev = None
        for (s, t, c) in sg:
            segm[s, t - s - 1, c] += p
            St[s, c] += p
            En[t, c] += p
            mu[s:t, c] += p
            gdur[t - s - 1, c] += p
            if prev is not None:
                gtrans[prev, c] += p
            prev = c
    best = float(scores.max())
    # Every segmentation within tie_tol of the best is optimal.  Swapping the
    # durations of two adjacent same-label segments leaves the score unchanged,
    # so exact ties are structural, not accidental.
    optimal = [sg for sc, sg in zip(scores, segs_all) if sc >= best - tie_tol]
    # The documented tie-break, read from the end of the sequence: smallest
    # final label, then smallest last duration, then smallest previous label,
    # and so on back to the start.
    def key(sg):
        out = [sg[-1][2]]
        for i in range(len(sg) - 1, -1, -1):
            out.append(sg[i][1] - sg[i][0])
            out.append(sg[i - 1][2] if i > 0 else -1)
        return out
    chosen = min(optimal, key=key)
    return dict(logZ=logZ, start_marg=St, end_marg=En, pos_marg=mu, grad_dur=gdur, seg_marg=segm[:L],
                grad_trans=gtrans, best_score=best, optimal=[to_arrays(sg, L) for sg in optimal],
                tie_broken=to_arrays(chosen, L), n_segmentations=len(segs_all))


def to_arrays(segs, L):
    labels = np.full(L, -1, dtype=np.int32)
    seg_start = np.zeros(L, dtype=np.uint8)
    for (s, t, c) in segs:
        labels[s:t] = c
        seg_start[s] = 1
    return labels, seg_start
