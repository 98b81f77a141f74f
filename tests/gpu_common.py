"""Helpers shared by the GPU parity tests: run the CUDA path through the
binding and compare it with the oracle at the stated tolerances.

Tolerances:
  log Z                        1e-5 relative (absolute below |log Z| = 1)
  marginals, emission grads    1e-4 absolute
  grad_trans, grad_dur         1e-4 * max(1, |expected count|): these are
                               expected counts, up to ~10^4 on the long
                               workloads, so the 1e-4 bound is taken
                               relative to the count once it exceeds one
"""

from __future__ import annotations

import numpy as np
import torch

LOGZ_RTOL = 1e-5
MARG_ATOL = 1e-4
COUNT_RTOL = 1e-4
# Viterbi: a stretch where the GPU's path differs from the oracle's is a tie
# when the two float64 scores over it agree to 2^-20 of the stretch's own
# magnitude (sum of |terms|): a few float32 ulps per term
TIE_RTOL = 2.0 ** -20


def to_dev(case, dev="cuda"):
    return (torch.from_numpy(np.ascontiguousarray(case["em"])).to(dev),
            torch.from_numpy(np.ascontiguousarray(case["lengths"])).to(dev),
            torch.from_numpy(np.ascontiguousarray(case["trans"])).to(dev),
            torch.from_numpy(np.ascontiguousarray(case["dur"])).to(dev))


def gpu_fb(case, center=True, grad_logZ=None, forward_only=False, log_domain=False):
    from semi_markov_crf_b200 import semicrf
    em, lengths, trans, dur = to_dev(case)
    g = None if grad_logZ is None else torch.as_tensor(grad_logZ, dtype=torch.float64, device="cuda")
    logZ, ws = semicrf.forward(em, lengths, trans, dur, center=center, forward_only=forward_only,
                               log_domain=log_domain)
    out = semicrf.backward(ws, lengths, trans, dur, grad_logZ=g, marginals=True)
    status = semicrf.get_status(ws)
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["logZ"] = logZ.cpu().numpy()
    res["status"] = status
    return res


def gpu_viterbi(case, center=True):
    from semi_markov_crf_b200 import semicrf
    em, lengths, trans, dur = to_dev(case)
    score, labels, seg = semicrf.viterbi(em, lengths, trans, dur, center=center)
    return dict(score=score.cpu().numpy(), labels=labels.cpu().numpy(), seg_start=seg.cpu().numpy())


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0


def assert_fb_close(got, ref, lengths, label=""):
    lz_g, lz_r = got["logZ"], ref["logZ"]
    err = np.abs(lz_g - lz_r) / np.maximum(1.0, np.abs(lz_r))
    assert np.all(err <= LOGZ_RTOL), f"{label} logZ rel err {err.max():.3e}"
    B = len(lengths)
    for key in ("pos_marg", "grad_e"):
        gk = "grad_em" if key == "grad_e" else key
        e = max_abs(got[gk], ref[key])
        assert e <= MARG_ATOL, f"{label} {key} max abs err {e:.3e}"
    for key in ("start_marg", "end_marg"):
        e = max_abs(got[key], ref[key])
        assert e <= MARG_ATOL, f"{label} {key} max abs err {e:.3e}"
    for key in ("grad_trans", "grad_dur"):
        d = np.abs(got[key].astype(np.float64) - ref[key])
        lim = COUNT_RTOL * np.maximum(1.0, np.abs(ref[key]))
        assert np.all(d <= lim), f"{label} {key} worst ratio {(d / lim).max():.3f}"
    # padding is exactly zero
    for b in range(B):
        L = int(lengths[b])
        assert np.all(got["grad_em"][b, L:] == 0) and np.all(got["pos_marg"][b, L:] == 0)
        assert np.all(got["start_marg"][b, L + 1:] == 0) and np.all(got["end_marg"][b, L + 1:] == 0)


def errors(got, ref):
    """Worst errors, for reporting."""
    out = dict(logZ_rel=float(np.max(np.abs(got["logZ"] - ref["logZ"]) / np.maximum(1, np.abs(ref["logZ"])))))
    out["pos_marg"] = max_abs(got["pos_marg"], ref["pos_marg"])
    out["grad_e"] = max_abs(got["grad_em"], ref["grad_e"])
    out["start_marg"] = max_abs(got["start_marg"], ref["start_marg"])
    out["end_marg"] = max_abs(got["end_marg"], ref["end_marg"])
    for key in ("grad_trans", "grad_dur"):
        out[key] = float(np.max(np.abs(got[key] - ref[key]) / np.maximum(1, np.abs(ref[key]))))
    return out


def assert_viterbi_ok(got, ref, case, center=True, label="", p_start=None, p_end=None):
    """Scores agree; paths are bit-exact or, where they differ, the GPU path is
    a valid segmentation whose float64 re-score is optimal within the
    tolerance (a tie in the model, resolved differently by float32 rounding)."""
    import oracle
    lengths = case["lengths"]
    sc_r = ref["score"]
    err = np.abs(got["score"] - sc_r) / np.maximum(1.0, np.abs(sc_r))
    assert np.all(err <= LOGZ_RTOL), f"{label} viterbi score rel err {err.max():.3e}"
    rescored = oracle.path_score(case["em"], lengths, case["trans"], case["dur"], got["labels"],
                                 got["seg_start"], K=case["dur"].shape[0], center=center,
                                 p_start=p_start, p_end=p_end)
    n_diff = 0
    for b in range(len(lengths)):
        L = int(lengths[b])
        assert np.all(got["labels"][b, L:] == -1) and np.all(got["seg_start"][b, L:] == 0)
        same = (np.array_equal(got["labels"][b, :L], ref["labels"][b, :L]) and
                np.array_equal(got["seg_start"][b, :L], ref["seg_start"][b, :L]))
        if not same:
            n_diff += 1
            assert np.isfinite(rescored[b]), f"{label} seq {b}: GPU path is not a valid segmentation"
    if n_diff:
        # every stretch where the paths differ is a tie of the model, resolved
        # differently by float32 rounding: equal float64 scores over the
        # stretch to within rounding of its own terms (reading O7)
        for r in local_tie_report(case, got["labels"], got["seg_start"], ref["labels"],
                                  ref["seg_start"], center=center, p_start=p_start, p_end=p_end):
            assert abs(r["diff"]) <= TIE_RTOL * max(1.0, r["mag"]), (label, r)
    return n_diff


# ----------------------------------------------------------------------------- Viterbi ties
def differing_stretches(lab_a, seg_a, lab_b, seg_b, L):
    """Maximal stretches [a, b) of positions where two segmentations of
    0..L-1 differ.  Both have a segment boundary at a and at b, and the
    segment just before a and the one starting at b (when they exist) are
    the same in both.  Returns a list of (w0, a, b, w1): [w0, a) is the
    shared segment before the stretch (w0 = a = 0 when none), [b, w1) the
    shared one after it (w1 = b = L when none)."""
    if L == 0:
        return []
    ba = np.flatnonzero(seg_a[:L]).tolist() + [L]
    bb = np.flatnonzero(seg_b[:L]).tolist() + [L]
    common = sorted(set(ba) & set(bb))
    sa, sb = set(ba), set(bb)
    ia = np.asarray(ba)
    ib = np.asarray(bb)
    same = []
    for p, q in zip(common[:-1], common[1:]):
        # one segment each (no boundary strictly inside) with the same label
        inside_a = np.searchsorted(ia, q) - np.searchsorted(ia, p, side="right")
        inside_b = np.searchsorted(ib, q) - np.searchsorted(ib, p, side="right")
        same.append(inside_a == 0 and inside_b == 0 and lab_a[p] == lab_b[p])
    out = []
    i = 0
    n = len(same)
    while i < n:
        if same[i]:
            i += 1
            continue
        j = i
        while j < n and not same[j]:
            j += 1
        a, b = common[i], common[j]
        w0 = common[i - 1] if i > 0 else a
        w1 = common[j + 1] if j < n else b
        out.append((w0, a, b, w1))
        i = j
    del sa, sb
    return out


def local_tie_report(case, got_lab, got_seg, ref_lab, ref_seg, center=True, p_start=None,
                     p_end=None):
    """For every sequence and every stretch where the GPU's decoded path
    differs from the oracle's: the float64 score difference of the two paths
    over the stretch (GPU minus oracle; the rest of both paths is the same,
    so the differences add up to the difference of the total scores), and
    the size of the stretch's score (sum of |terms| along the oracle path),
    both from the oracle's path_score on the window of the stretch plus its
    shared neighbouring segments, on emissions centred with the whole
    sequence's mean."""
    import oracle
    em = np.asarray(case["em"], np.float64)
    lengths = case["lengths"]
    K = case["dur"].shape[0]
    C = em.shape[2]
    reports = []
    for b in range(len(lengths)):
        L = int(lengths[b])
        st = differing_stretches(got_lab[b], got_seg[b], ref_lab[b], ref_seg[b], L)
        if not st:
            continue
        nu = em[b, :L].mean(axis=0) if center else np.zeros(C)
        for (w0, a, b1, w1) in st:
            n = w1 - w0
            e = (em[b, w0:w1] - nu)[None]
            ps = None if p_start is None else np.asarray(p_start, np.float64)[b, w0:w1][None]
            pe = None if p_end is None else np.asarray(p_end, np.float64)[b, w0:w1][None]
            sc = []
            for lab, seg in ((got_lab, got_seg), (ref_lab, ref_seg)):
                ll = np.ascontiguousarray(lab[b, w0:w1][None].astype(np.int32))
                ss = np.ascontiguousarray(seg[b, w0:w1][None].astype(np.uint8))
                ss[0, 0] = 1
                sc.append(float(oracle.path_score(e, np.array([n], np.int32), case["trans"],
                                                  case["dur"], ll, ss, K=K, center=False,
                                                  p_start=ps, p_end=pe)[0]))
            rl = ref_lab[b, w0:w1]
            mag = float(np.abs(e[0, np.arange(n), rl]).sum()
                        + np.abs(case["dur"]).max() * n + np.abs(case["trans"]).max() * n)
            for P in (ps, pe):
                if P is not None:
                    mag += float(np.abs(P[0, np.arange(n), rl]).sum())
            reports.append(dict(b=b, start=a, end=b1, window=(w0, w1), diff=sc[0] - sc[1],
                                mag=mag))
    return reports
