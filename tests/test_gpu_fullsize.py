"""GPU parity at the five full workload sizes (tiny, speech, genomic, ultra,
large), in the launch configuration bench.py times.

The expected values come from tests/golden/<name>.npz, written by
tests/golden/make_golden.py, which runs only the float64 oracle on the same
seeded inputs: log Z, the full transition and duration gradients, the
Viterbi optimum, and marginals / emission gradients at seeded sampled
positions.  Properties that hold at any size are checked on every output:
position marginals sum to one over labels, every position is covered by
exactly one segment (sum_k k * grad_dur = sum_b L_b), segments minus
transitions is one per sequence, and the centering Jacobian sums the
emission gradient to zero over positions.
"""

import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import COUNT_RTOL, LOGZ_RTOL, MARG_ATOL, gpu_fb, gpu_viterbi
from semi_markov_crf_b200 import synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
NAMES = ["tiny", "speech", "genomic", "ultra", "large"]


def _golden(name):
    path = os.path.join(GOLDEN, f"{name}.npz")
    if not os.path.exists(path):
        pytest.skip(f"{path} not generated")
    return dict(np.load(path))


@pytest.fixture(scope="module", params=NAMES)
def full(request):
    name = request.param
    gold = _golden(name)
    case = synth.make(name)
    assert np.array_equal(case["lengths"], gold["lengths"]), "generator drifted from the golden file"
    got = gpu_fb(case)
    return name, case, gold, got


def test_fullsize_forward_backward_matches_oracle(full):
    name, case, gold, got = full
    assert got["status"] == 0
    err = np.abs(got["logZ"] - gold["logZ"]) / np.maximum(1.0, np.abs(gold["logZ"]))
    print(name, "logZ rel err", err.max())
    assert np.all(err <= LOGZ_RTOL)
    b, u = gold["sample_b"], gold["sample_u"]
    report = {}
    for key, gk in (("pos_marg", "pos_marg"), ("grad_e", "grad_em"), ("start_marg", "start_marg"),
                    ("end_marg", "end_marg")):
        e = float(np.max(np.abs(got[gk][b, u].astype(np.float64) - gold[key])))
        report[key] = e
    for key in ("grad_trans", "grad_dur"):
        d = np.abs(got[key].astype(np.float64) - gold[key])
        report[key] = float(np.max(d / np.maximum(1.0, np.abs(gold[key]))))
    print(name, report)
    for key in ("pos_marg", "grad_e", "start_marg", "end_marg"):
        assert report[key] <= MARG_ATOL, (key, report[key])
    for key in ("grad_trans", "grad_dur"):
        assert report[key] <= COUNT_RTOL, (key, report[key])


def test_fullsize_invariants(full):
    name, case, gold, got = full
    lengths = case["lengths"]
    K = case["dur"].shape[0]
    for bb in range(len(lengths)):
        L = int(lengths[bb])
        s = got["pos_marg"][bb, :L].astype(np.float64).sum(axis=1)
        assert np.max(np.abs(s - 1.0)) <= MARG_ATOL, (name, bb, np.max(np.abs(s - 1.0)))
        colsum = got["grad_em"][bb, :L].astype(np.float64).sum(axis=0)
        assert np.max(np.abs(colsum)) <= MARG_ATOL * max(1.0, np.sqrt(L)), (name, colsum)
    gd = got["grad_dur"].astype(np.float64)
    gt = got["grad_trans"].astype(np.float64)
    covered = float((np.arange(1, K + 1)[:, None] * gd).sum())
    total = float(lengths.sum())
    assert abs(covered - total) <= COUNT_RTOL * total, (covered, total)
    assert abs(gd.sum() - gt.sum() - len(lengths)) <= COUNT_RTOL * max(1.0, gd.sum())


def test_fullsize_viterbi_is_optimal(full):
    name, case, gold, _ = full
    got = gpu_viterbi(case)
    best = gold["viterbi_score"]
    err = np.abs(got["score"] - best) / np.maximum(1.0, np.abs(best))
    assert np.all(err <= LOGZ_RTOL), err.max()
    # the decoded path is a valid segmentation whose float64 score is optimal
    rescored = oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"],
                                 got["labels"], got["seg_start"], K=case["dur"].shape[0])
    assert np.all(np.isfinite(rescored))
    assert np.all(rescored >= best - LOGZ_RTOL * np.maximum(1.0, np.abs(best))), (rescored - best)
