"""Float64 CPU oracle for the semi-CRF hot path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports, links or executes anything here, and this package
imports nothing from the product path: the two share only the seeded input
generator, which holds no semi-CRF arithmetic.

The arithmetic lives in ``semicrf_oracle.c`` (plain C, float64, explicit
edges); this module compiles it with gcc on first use and wraps it with
ctypes, running independent sequences of a batch on a thread pool (ctypes
releases the GIL during the call).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "semicrf_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math) into oracle/_build."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_center.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp]
            lib.oracle_center.restype = None
            lib.oracle_prefix.argtypes = [_dp, ctypes.c_int, ctypes.c_int, _dp]
            lib.oracle_prefix.restype = None
            lib.oracle_fb.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp,
                                      ctypes.c_int, ctypes.c_double, _dp, _dp,
                                      _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
            lib.oracle_fb.restype = ctypes.c_int
            lib.oracle_viterbi.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp,
                                           ctypes.c_int, _dp, _ip, _u8p]
            lib.oracle_viterbi.restype = ctypes.c_int
            lib.oracle_path_score.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp,
                                              ctypes.c_int, _ip, _u8p]
            lib.oracle_path_score.restype = ctypes.c_double
            lib.oracle_path_counts.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, _ip, _u8p, _dp, _dp, _dp]
            lib.oracle_path_counts.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a, kind=_dp):
    if a is None:
        return ctypes.cast(None, kind)
    return a.ctypes.data_as(kind)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _threads(n_items: int, threads: int | None) -> int:
    if threads is None:
        threads = os.cpu_count() or 1
    return max(1, min(int(threads), n_items))


def _proj(P, b, L, C):
    """Contiguous float64 [L, C] slice of a [B, T, C] projection array, or None."""
    if P is None:
        return None
    return np.ascontiguousarray(np.asarray(P[b, :max(L, 1)], dtype=np.float64)) if L > 0 else np.zeros((1, C))


def prefix_center(em, lengths, center: bool = True):
    """nu [B, C] and the prefix sums S [B, T+1, C] of the centred emissions.

    Rows t > L_b of S are zero.  Both are float64.
    """
    lib = _load()
    em = _f64(em)
    B, T, C = em.shape
    S = np.zeros((B, T + 1, C))
    nu = np.zeros((B, C))
    for b in range(B):
        L = int(lengths[b])
        e = np.ascontiguousarray(em[b, :L])
        et = np.zeros((max(L, 1), C))
        nub = np.zeros(C)
        lib.oracle_center(_ptr(e), L, C, int(center), _ptr(et), _ptr(nub))
        Sb = np.zeros((L + 1, C))
        lib.oracle_prefix(_ptr(et), L, C, _ptr(Sb))
        S[b, :L + 1] = Sb
        nu[b] = nub
    return S, nu


def forward_backward(em, lengths, trans, dur, K: int | None = None, center: bool = True,
                     grad_logZ=None, threads: int | None = None, want_alpha_beta: bool = False,
                     p_start=None, p_end=None, want_segments: bool = False):
    """Exact log Z, marginals and gradients for a batch.

    ``p_start`` / ``p_end`` [B, T, C] (optional) are boundary projection
    scores: segment [s, t) with label c gains p_start[b, s, c] + p_end[b, t-1, c].

    Returns a dict of float64 arrays:
      logZ [B], logZ_beta [B], start_marg / end_marg [B, T+1, C],
      pos_marg / grad_e [B, T, C], grad_trans [C, C], grad_dur [K, C]
    (and alpha / beta [B, T+1, C] when ``want_alpha_beta``; seg_marg
    [B, T, K, C] when ``want_segments``: P(segment [s, s+k) with label c) at
    [b, s, k-1, c], zero where s + k > L_b).  Entries past a
    sequence's length are zero.  ``grad_logZ`` [B] (default ones) scales the
    three gradients; grad_trans / grad_dur are summed over the batch in batch
    order.
    """
    lib = _load()
    em = _f64(em)
    trans = _f64(trans)
    dur = _f64(dur)
    B, T, C = em.shape
    if K is None:
        K = dur.shape[0]
    assert dur.shape == (K, C) and trans.shape == (C, C)
    g = np.ones(B) if grad_logZ is None else np.asarray(grad_logZ, dtype=np.float64)
    out = dict(logZ=np.zeros(B), logZ_beta=np.zeros(B),
               start_marg=np.zeros((B, T + 1, C)), end_marg=np.zeros((B, T + 1, C)),
               pos_marg=np.zeros((B, T, C)), grad_e=np.zeros((B, T, C)))
    if want_alpha_beta:
        out["alpha"] = np.zeros((B, T + 1, C))
        out["beta"] = np.zeros((B, T + 1, C))
    if want_segments:
        out["seg_marg"] = np.zeros((B, T, K, C))
    gt = np.zeros((B, C, C))
    gd = np.zeros((B, K, C))

    def one(b):
        L = int(lengths[b])
        e = np.ascontiguousarray(em[b, :L]) if L > 0 else np.zeros((1, C))
        lz = np.zeros(1)
        lzb = np.zeros(1)
        St = np.zeros((L + 1, C))
        En = np.zeros((L + 1, C))
        mu = np.zeros((max(L, 1), C))
        ge = np.zeros((max(L, 1), C))
        al = np.zeros((L + 1, C)) if want_alpha_beta else None
        be = np.zeros((L + 1, C)) if want_alpha_beta else None
        sg = np.zeros((max(L, 1), K, C)) if want_segments else None
        rc = lib.oracle_fb(_ptr(e), L, C, K, _ptr(trans), _ptr(dur), _ptr(_proj(p_start, b, L, C)),
                           _ptr(_proj(p_end, b, L, C)), int(center), float(g[b]),
                           _ptr(lz), _ptr(lzb), _ptr(al), _ptr(be), _ptr(St), _ptr(En),
                           _ptr(mu), _ptr(ge), _ptr(gt[b]), _ptr(gd[b]), _ptr(sg))
        if rc != 0:
            raise MemoryError("oracle_fb: allocation failed")
        out["logZ"][b] = lz[0]
        out["logZ_beta"][b] = lzb[0]
        out["start_marg"][b, :L + 1] = St
        out["end_marg"][b, :L + 1] = En
        if L > 0:
            out["pos_marg"][b, :L] = mu[:L]
            out["grad_e"][b, :L] = ge[:L]
        if want_alpha_beta:
            out["alpha"][b, :L + 1] = al
            out["beta"][b, :L + 1] = be
        if want_segments and L > 0:
            out["seg_marg"][b, :L] = sg[:L]

    n = _threads(B, threads)
    if n == 1:
        for b in range(B):
            one(b)
    else:
        with ThreadPoolExecutor(n) as ex:
            list(ex.map(one, range(B)))
    out["grad_trans"] = np.zeros((C, C))
    out["grad_dur"] = np.zeros((K, C))
    for b in range(B):  # fixed order: deterministic sums
        out["grad_trans"] += gt[b]
        out["grad_dur"] += gd[b]
    return out


def log_partition(em, lengths, trans, dur, K: int | None = None, center: bool = True,
                  threads: int | None = None, p_start=None, p_end=None):
    """log Z [B] only (still the full explicit-edge forward-backward)."""
    return forward_backward(em, lengths, trans, dur, K, center, threads=threads,
                            p_start=p_start, p_end=p_end)["logZ"]


def viterbi(em, lengths, trans, dur, K: int | None = None, center: bool = True,
            threads: int | None = None, p_start=None, p_end=None):
    """Best segmentation: score [B] float64, labels [B, T] int32 (-1 past the
    length) and seg_start [B, T] uint8 (1 where a segment starts)."""
    lib = _load()
    em = _f64(em)
    trans = _f64(trans)
    dur = _f64(dur)
    B, T, C = em.shape
    if K is None:
        K = dur.shape[0]
    score = np.zeros(B)
    labels = np.full((B, T), -1, dtype=np.int32)
    seg = np.zeros((B, T), dtype=np.uint8)

    def one(b):
        L = int(lengths[b])
        e = np.ascontiguousarray(em[b, :L]) if L > 0 else np.zeros((1, C))
        sc = np.zeros(1)
        lab = np.full(max(L, 1), -1, dtype=np.int32)
        ss = np.zeros(max(L, 1), dtype=np.uint8)
        rc = lib.oracle_viterbi(_ptr(e), L, C, K, _ptr(trans), _ptr(dur),
                                _ptr(_proj(p_start, b, L, C)), _ptr(_proj(p_end, b, L, C)),
                                int(center), _ptr(sc),
                                _ptr(lab, _ip), _ptr(ss, _u8p))
        if rc != 0:
            raise MemoryError("oracle_viterbi: allocation failed")
        score[b] = sc[0]
        if L > 0:
            labels[b, :L] = lab[:L]
            seg[b, :L] = ss[:L]

    n = _threads(B, threads)
    if n == 1:
        for b in range(B):
            one(b)
    else:
        with ThreadPoolExecutor(n) as ex:
            list(ex.map(one, range(B)))
    return dict(score=score, labels=labels, seg_start=seg)


def path_score(em, lengths, trans, dur, labels, seg_start, K: int | None = None,
               center: bool = True, p_start=None, p_end=None):
    """float64 score [B] of the given segmentations (NaN where malformed)."""
    lib = _load()
    em = _f64(em)
    trans = _f64(trans)
    dur = _f64(dur)
    B, T, C = em.shape
    if K is None:
        K = dur.shape[0]
    out = np.zeros(B)
    for b in range(B):
        L = int(lengths[b])
        e = np.ascontiguousarray(em[b, :L]) if L > 0 else np.zeros((1, C))
        lab = np.ascontiguousarray(np.asarray(labels[b, :max(L, 1)], dtype=np.int32))
        ss = np.ascontiguousarray(np.asarray(seg_start[b, :max(L, 1)], dtype=np.uint8))
        out[b] = lib.oracle_path_score(_ptr(e), L, C, K, _ptr(trans), _ptr(dur),
                                       _ptr(_proj(p_start, b, L, C)), _ptr(_proj(p_end, b, L, C)),
                                       int(center),
                                       _ptr(lab, _ip), _ptr(ss, _u8p))
    return out


def path_counts(lengths, labels, seg_start, C: int, K: int, center: bool = True):
    """Derivatives of the path score of given segmentations (float64).

    Returns ``grad_em`` [B, T, C] (d score_b / d em[b, u, c], zero past L_b),
    ``trans_count`` [B, C, C], ``dur_count`` [B, K, C], ``p_start_count`` /
    ``p_end_count`` [B, T, C] (derivatives with respect to boundary
    projections; per sequence, not weighted) and ``valid`` [B] (False where the path is malformed; its
    counts are zero).  Their weighted sums are the gold-score part of the
    gradient of the loss log Z - score.
    """
    lib = _load()
    labels = np.asarray(labels)
    seg_start = np.asarray(seg_start)
    B, T = labels.shape
    grad_em = np.zeros((B, T, C))
    tc = np.zeros((B, C, C))
    dc = np.zeros((B, K, C))
    valid = np.ones(B, dtype=bool)
    for b in range(B):
        L = int(lengths[b])
        lab = np.ascontiguousarray(np.asarray(labels[b, :max(L, 1)], dtype=np.int32))
        ss = np.ascontiguousarray(np.asarray(seg_start[b, :max(L, 1)], dtype=np.uint8))
        de = np.zeros((max(L, 1), C))
        dt = np.zeros((C, C))
        dd = np.zeros((K, C))
        rc = lib.oracle_path_counts(L, C, K, int(center), _ptr(lab, _ip), _ptr(ss, _u8p),
                                    _ptr(de), _ptr(dt), _ptr(dd))
        valid[b] = rc == 0
        if L > 0:
            grad_em[b, :L] = de[:L]
        tc[b] = dt
        dc[b] = dd
    # boundary projections: the path score gains p_start at each segment's
    # first position and p_end at its last, so those are its derivatives
    ps_c = np.zeros((B, T, C))
    pe_c = np.zeros((B, T, C))
    for b in range(B):
        L = int(lengths[b])
        if not valid[b]:
            continue
        for u in range(L):
            if seg_start[b, u]:
                ps_c[b, u, labels[b, u]] = 1.0
            if u == L - 1 or seg_start[b, u + 1]:
                pe_c[b, u, labels[b, u]] = 1.0
    return dict(grad_em=grad_em, trans_count=tc, dur_count=dc, valid=valid,
                p_start_count=ps_c, p_end_count=pe_c)
