"""GPU parity of the segment marginals P(segment [s, s+k) with label c)
(semicrf_backward_segments) against the float64 oracle, element by element,
in both ring domains, with the bookkeeping that ties them to the other
outputs: summed over durations they are the start marginals, over starts the
duration gradient (g = 1), and nothing runs past a sequence's end."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import MARG_ATOL, to_dev
from semi_markov_crf_b200 import semicrf, synth

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": lambda: synth.make("tiny"),
    "speech_small": lambda: synth.make("speech", B=3, T=150),
    "genomic_small": lambda: synth.make("genomic", B=2, T=1200),
    "large_small": lambda: synth.make("large", B=2, T=120),
    "ragged_with_empty": lambda: synth.make_custom(4, 60, 9, 5, seed=19, lengths=[60, 0, 1, 37]),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    c = CASES[request.param]()
    ref = oracle.forward_backward(c["em"], c["lengths"], c["trans"], c["dur"], c["dur"].shape[0],
                                  want_segments=True)
    return request.param, c, ref


@pytest.mark.parametrize("log_domain", [False, True])
def test_segment_marginals_match_oracle(case, log_domain):
    name, c, ref = case
    em, lengths, trans, dur = to_dev(c)
    logZ, ws = semicrf.forward(em, lengths, trans, dur, log_domain=log_domain)
    out = semicrf.backward(ws, lengths, trans, dur, marginals=True, segments=True)
    assert semicrf.get_status(ws) == 0
    sm = out["seg_marg"].cpu().numpy().astype(np.float64)
    err = float(np.max(np.abs(sm - ref["seg_marg"])))
    print(name, "log" if log_domain else "exp", "seg_marg max abs err", err)
    assert err <= MARG_ATOL
    # bookkeeping against the call's own other outputs
    st = out["start_marg"].cpu().numpy().astype(np.float64)
    gd = out["grad_dur"].cpu().numpy().astype(np.float64)
    T = c["em"].shape[1]
    assert np.max(np.abs(sm.sum(axis=2) - st[:, :T])) <= MARG_ATOL
    assert np.max(np.abs(sm.sum(axis=(0, 1)) - gd) / np.maximum(1.0, np.abs(gd))) <= 1e-4
    for b, L in enumerate(c["lengths"]):
        L = int(L)
        assert np.all(sm[b, L:] == 0)
        for s in range(max(0, L - c["dur"].shape[0]), L):
            assert np.all(sm[b, s, L - s:] == 0)


def test_segment_marginals_leave_the_other_outputs_unchanged(case):
    name, c, _ = case
    em, lengths, trans, dur = to_dev(c)
    logZ, ws = semicrf.forward(em, lengths, trans, dur)
    a = semicrf.backward(ws, lengths, trans, dur, marginals=True)
    a = {k: v.clone() for k, v in a.items()}
    logZ, ws = semicrf.forward(em, lengths, trans, dur)
    b = semicrf.backward(ws, lengths, trans, dur, marginals=True, segments=True)
    for k in a:
        assert torch.equal(a[k], b[k]), k
