"""GPU parity of the cluster-split rings: the exponential-domain forward and
backward rings and the pipelined decoder with each ring spread over a
thread-block cluster of N CTAs (labels split across the CTAs, the label
vector exchanged through distributed shared memory every step), for every
cluster size the library instantiates, against the float64 oracle and
against the one-CTA kernels.  SEMICRF_XCLUSTER selects the cluster size
(a tuning switch read at every call)."""

import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import assert_fb_close, assert_viterbi_ok, errors, gpu_fb, gpu_viterbi
from semi_markov_crf_b200 import semicrf, synth

pytestmark = pytest.mark.gpu


def _cases():
    return {
        # wide label sets: ragged tails, several checkpoint segments and tiles
        "large_small": (lambda: synth.make("large", B=3, T=400), (1, 2, 4, 8)),
        "wide_ragged": (lambda: synth.make_custom(3, 333, 40, 100, seed=31, lengths=[333, 1, 250],
                                                  dur_mean=6.0), (1, 2, 4, 8)),
        # narrower sets on small clusters
        "speech_small": (lambda: synth.make("speech", B=4, T=200), (1, 2)),
    }


CASES = _cases()


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    make, sizes = CASES[request.param]
    c = make()
    K = c["dur"].shape[0]
    ref = oracle.forward_backward(c["em"], c["lengths"], c["trans"], c["dur"], K)
    vref = oracle.viterbi(c["em"], c["lengths"], c["trans"], c["dur"], K)
    return request.param, c, sizes, ref, vref


def _with_cluster(n, fn):
    old = os.environ.get("SEMICRF_XCLUSTER")
    os.environ["SEMICRF_XCLUSTER"] = str(n)
    try:
        return fn()
    finally:
        if old is None:
            del os.environ["SEMICRF_XCLUSTER"]
        else:
            os.environ["SEMICRF_XCLUSTER"] = old


def test_cluster_rings_match_oracle(case):
    name, c, sizes, ref, vref = case
    B, T, C = c["em"].shape
    K = c["dur"].shape[0]
    outs = {}
    for n in sizes:
        shape = _with_cluster(n, lambda: semicrf.launch_shape(B, T, C, K))
        assert shape["ring_ctas"] == n, (name, n, shape)
        got = _with_cluster(n, lambda: gpu_fb(c))
        assert got["status"] == 0
        print(name, n, errors(got, ref))
        assert_fb_close(got, ref, c["lengths"], f"{name} N={n}")
        vit = _with_cluster(n, lambda: gpu_viterbi(c))
        assert_viterbi_ok(vit, vref, c, label=f"{name} N={n}")
        outs[n] = (got, vit)
    # the decoded path does not depend on the cluster size: the same float
    # sums are compared in the same order
    for n in sizes[1:]:
        assert np.array_equal(outs[n][1]["labels"], outs[sizes[0]][1]["labels"])
        assert np.array_equal(outs[n][1]["score"], outs[sizes[0]][1]["score"])


def test_cluster_rings_are_deterministic(case):
    name, c, sizes, _, _ = case
    n = sizes[-1]
    a = _with_cluster(n, lambda: gpu_fb(c))
    b = _with_cluster(n, lambda: gpu_fb(c))
    for k in ("logZ", "grad_em", "grad_trans", "grad_dur", "pos_marg"):
        assert np.array_equal(a[k], b[k]), k
