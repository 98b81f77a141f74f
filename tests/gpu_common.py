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
            tol = LOGZ_RTOL * max(1.0, abs(sc_r[b]))
            assert rescored[b] >= sc_r[b] - tol, (
                f"{label} seq {b}: GPU path scores {rescored[b]} < optimum {sc_r[b]} - {tol}")
    return n_diff
