"""Textbook linear-chain CRF, written independently of the semi-CRF oracle.

With maximum duration K = 1 every segment is one position long, so the
semi-CRF of the Flash-SemiCRF pages reduces to a linear-chain CRF (the pages
call it the K=1 case: explainer section 1, "Problem Statement").  Its node
score at position u is the centred emission plus the duration-1 score,
x[u, c] = e~[u, c] + dur[0, c], and consecutive labels add trans[c', c];
there is no start or end score.

This module is the classic scaled forward-backward in the probability domain
(Rabiner-style scaling with per-step normalisers) and the classic Viterbi,
so it shares neither structure nor code with the log-domain semi-CRF oracle.
"""

from __future__ import annotations

import numpy as np


def node_scores(e, L, dur0, center=True):
    e = np.asarray(e, dtype=np.float64)[:L]
    nu = e.mean(axis=0) if center else np.zeros(e.shape[1])
    return e - nu + np.asarray(dur0, dtype=np.float64)[None, :]


def forward_backward(x, trans):
    """x [L, C] node log-potentials, trans [C, C].  Returns log Z, node
    marginals [L, C] and expected transition counts [C, C]."""
    x = np.asarray(x, dtype=np.float64)
    L, C = x.shape
    A = np.exp(np.asarray(trans, dtype=np.float64))
    shift = x.max(axis=1, keepdims=True)
    phi = np.exp(x - shift)            # node potentials, rescaled per position
    fwd = np.zeros((L, C))
    scale = np.zeros(L)
    v = phi[0]
    scale[0] = v.sum()
    fwd[0] = v / scale[0]
    for u in range(1, L):
        v = (fwd[u - 1] @ A) * phi[u]
        scale[u] = v.sum()
        fwd[u] = v / scale[u]
    logZ = float(np.log(scale).sum() + shift.sum())
    bwd = np.zeros((L, C))
    bwd[L - 1] = 1.0
    for u in range(L - 2, -1, -1):
        bwd[u] = (A @ (phi[u + 1] * bwd[u + 1])) / scale[u + 1]
    node = fwd * bwd
    pair = np.zeros((C, C))
    for u in range(1, L):
        pair += (fwd[u - 1][:, None] * A * (phi[u] * bwd[u])[None, :]) / scale[u]
    return logZ, node, pair


def viterbi(x, trans):
    """Classic max-product decoding; returns best score and labels [L]."""
    x = np.asarray(x, dtype=np.float64)
    trans = np.asarray(trans, dtype=np.float64)
    L, C = x.shape
    delta = x[0].copy()
    back = np.zeros((L, C), dtype=np.int64)
    for u in range(1, L):
        cand = delta[:, None] + trans          # [c_prev, c]
        back[u] = np.argmax(cand, axis=0)
        delta = cand[back[u], np.arange(C)] + x[u]
    labels = np.zeros(L, dtype=np.int32)
    labels[-1] = int(np.argmax(delta))
    best = float(delta[labels[-1]])
    for u in range(L - 1, 0, -1):
        labels[u - 1] = back[u, labels[u]]
    return best, labels
