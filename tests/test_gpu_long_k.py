"""Long durations, 2048 < K <= 8192 (the pages' genomic regime of K =
2000-8000: explainer section 4 and the Chinese explainer's section 4).
These sizes run on the exponential-domain rings and the pipelined decoder,
one label per CTA of a thread-block cluster, with the posterior pass staging
the segment ends in chunks and the cut normaliser label by label.

- K = 8000, C = 6, T = 6,000 (lengths 6,000 and 4,500: segments up to the
  whole sequence) against the float64 oracle at every position
  (tests/golden/long_k.npz; the oracle's explicit covering sums make larger
  T a matter of hours): log Z,
  marginals, emission gradients, transition and duration gradients, and the
  decoded path (bit-exact except at ties of the model).
- K = 3000 at C = 1 and C = 3 (one CTA, and a cluster of three) against the
  oracle computed now.
- T = 10^6, K = 8000, C = 6: the any-size invariants.
- A sequence outside the exponent range is reported as unsupported (status
  2, log Z NaN, zero posteriors) next to a normal one, which still matches
  the oracle; forcing the log domain is refused on the host.
"""

import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import (COUNT_RTOL, LOGZ_RTOL, MARG_ATOL, TIE_RTOL, assert_fb_close,
                        assert_viterbi_ok, errors, gpu_fb, gpu_viterbi, local_tie_report, to_dev)
from semi_markov_crf_b200 import semicrf, synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "long_k.npz")


def _long_k_case():
    return synth.make_custom(2, 6_000, 8000, 6, seed=43, lengths=[6_000, 4_500],
                             dur_mean=500.0, amp=2.0, label_p=(0.6, 0.2, 0.1, 0.05, 0.03, 0.02))


def test_k8000_matches_the_oracle_everywhere():
    if not os.path.exists(GOLDEN):
        pytest.skip("tests/golden/long_k.npz not generated")
    g = dict(np.load(GOLDEN))
    case = _long_k_case()
    assert np.array_equal(case["lengths"], g["lengths"])
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    shape = semicrf.launch_shape(B, T, C, K)
    assert shape["ring_ctas"] == 6 and shape["log_threads"] == 0, shape
    got = gpu_fb(case)
    assert got["status"] == 0
    q = float(g["qscale"])
    err = np.abs(got["logZ"] - g["logZ"]) / np.maximum(1.0, np.abs(g["logZ"]))
    assert np.all(err <= LOGZ_RTOL), err
    rb, ru, bb, bu = g["row_b"], g["row_u"], g["brow_b"], g["brow_u"]
    rep = {}
    for key, gk, (b, u) in (("q_pos_marg", "pos_marg", (rb, ru)), ("q_grad_e", "grad_em", (rb, ru)),
                            ("q_start_marg", "start_marg", (bb, bu)),
                            ("q_end_marg", "end_marg", (bb, bu))):
        rep[gk] = float(np.max(np.abs(got[gk][b, u].astype(np.float64) - g[key] / q)))
        assert rep[gk] <= MARG_ATOL + 0.5 / q, (gk, rep[gk])
    for key in ("grad_trans", "grad_dur"):
        d = np.abs(got[key].astype(np.float64) - g[key])
        rep[key] = float(np.max(d / np.maximum(1.0, np.abs(g[key]))))
        assert rep[key] <= COUNT_RTOL, (key, rep[key])
    print("K=8000", rep, "positions", len(rb))
    vit = gpu_viterbi(case)
    ref = dict(score=g["viterbi_score"], labels=g["viterbi_labels"].astype(np.int32),
               seg_start=np.unpackbits(g["viterbi_seg"], axis=1, count=T))
    assert_viterbi_ok(vit, ref, case, label="K=8000")
    n_same = sum(np.array_equal(vit["labels"][b], ref["labels"][b]) for b in range(B))
    print("K=8000 viterbi bit-exact sequences", n_same, "of", B)


@pytest.mark.parametrize("C,n", [(1, 1), (3, 3)])
def test_k3000_small_label_sets_match_oracle(C, n):
    case = synth.make_custom(2, 3200, 3000, C, seed=44 + C, lengths=[3200, 2100],
                             dur_mean=400.0, amp=2.0)
    B, T, _ = case["em"].shape
    K = case["dur"].shape[0]
    assert semicrf.launch_shape(B, T, C, K)["ring_ctas"] == n
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"], K)
    got = gpu_fb(case)
    assert got["status"] == 0
    print(C, errors(got, ref))
    assert_fb_close(got, ref, case["lengths"], f"K=3000 C={C}")
    vref = oracle.viterbi(case["em"], case["lengths"], case["trans"], case["dur"], K)
    assert_viterbi_ok(gpu_viterbi(case), vref, case, label=f"K=3000 C={C}")


def test_k8000_million_positions_invariants():
    case = synth.make_custom(1, 1_000_000, 8000, 6, seed=45, dur_mean=500.0, amp=2.0,
                             label_p=(0.6, 0.2, 0.1, 0.05, 0.03, 0.02))
    L = 1_000_000
    got = gpu_fb(case)
    assert got["status"] == 0 and np.isfinite(got["logZ"]).all()
    mu = got["pos_marg"][0].astype(np.float64)
    assert np.max(np.abs(mu.sum(axis=1) - 1.0)) <= MARG_ATOL
    K = 8000
    gd = got["grad_dur"].astype(np.float64)
    gt = got["grad_trans"].astype(np.float64)
    covered = float((np.arange(1, K + 1)[:, None] * gd).sum())
    assert abs(covered - L) <= COUNT_RTOL * L, covered
    assert abs(gd.sum() - gt.sum() - 1.0) <= COUNT_RTOL * max(1.0, gd.sum())
    assert np.max(np.abs(got["grad_em"][0].astype(np.float64).sum(axis=0))) <= MARG_ATOL * np.sqrt(L)
    vit = gpu_viterbi(case)
    resc = oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"], vit["labels"],
                             vit["seg_start"], K)
    assert np.isfinite(resc[0])
    assert abs(resc[0] - vit["score"][0]) <= 1e-8 * abs(resc[0]), (resc[0], vit["score"][0])


def test_k4000_outside_the_exponent_range_is_reported():
    """Sequence 1's emissions are scaled far outside the exponential-domain
    rings' head-room: it is reported (status 2, log Z NaN, zero posteriors)
    while sequence 0 is computed as usual."""
    case = synth.make_custom(2, 3000, 4000, 4, seed=46, dur_mean=300.0, amp=2.0)
    case["em"][1] *= 60.0
    K = case["dur"].shape[0]
    em, lengths, trans, dur = to_dev(case)
    logZ, ws = semicrf.forward(em, lengths, trans, dur)
    out = semicrf.backward(ws, lengths, trans, dur, marginals=True)
    assert semicrf.get_status(ws) == 2
    assert semicrf.ring_domains(ws) == [1, 2, 1, 2]
    lz = logZ.cpu().numpy()
    assert np.isnan(lz[1]) and np.isfinite(lz[0])
    for k in ("grad_em", "pos_marg", "start_marg", "end_marg"):
        assert torch.count_nonzero(out[k][1]) == 0, k
    one = dict(case, em=case["em"][:1], lengths=case["lengths"][:1])
    ref = oracle.forward_backward(one["em"], one["lengths"], case["trans"], case["dur"], K)
    got = {k: v[:1].cpu().numpy() if v.dim() == 3 else v.cpu().numpy() for k, v in out.items()}
    got["logZ"] = lz[:1]
    assert_fb_close(got, ref, one["lengths"], "K=4000 with a declined sequence")
    with pytest.raises(semicrf.SemiCRFError) as info:
        semicrf.forward(em, lengths, trans, dur, log_domain=True)
    assert info.value.code == 2
