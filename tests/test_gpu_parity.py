"""GPU parity: the CUDA path against the float64 oracle on the same seeded
inputs (oracle-sized cases spanning several tiles, several checkpoint
segments and ragged tails), plus edge cases, determinism and status
reporting.  Every call goes through the C ABI via the binding."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import (assert_fb_close, assert_viterbi_ok, errors, gpu_fb, gpu_viterbi, to_dev)
from semi_markov_crf_b200 import synth

pytestmark = pytest.mark.gpu


def _cases():
    return {
        "tiny": lambda: synth.make("tiny"),
        "speech_small": lambda: synth.make("speech", B=6, T=160),
        "genomic_small": lambda: synth.make("genomic", B=2, T=3000),
        "large_small": lambda: synth.make("large", B=2, T=160),
        "single_position": lambda: synth.make_custom(2, 5, 4, 3, seed=5, lengths=[1, 5]),
        "shorter_than_K": lambda: synth.make_custom(3, 12, 20, 5, seed=6, lengths=[7, 12, 3]),
        "k_equals_1": lambda: synth.make_custom(2, 90, 1, 7, seed=7, lengths=[90, 41]),
        "one_label": lambda: synth.make_custom(2, 70, 6, 1, seed=8, lengths=[70, 33]),
        "mixed_with_empty": lambda: synth.make_custom(4, 80, 9, 5, seed=9, lengths=[80, 0, 1, 57]),
        "delta_not_multiple_of_K": lambda: synth.make_custom(1, 501, 7, 3, seed=10),
        "many_segments_small_K": lambda: synth.make_custom(2, 1200, 3, 4, seed=11, lengths=[1200, 999]),
        # C = 64: the traceback stages a few hundred rows at a time, so these
        # lengths take several stages
        "traceback_in_stages": lambda: synth.make_custom(2, 900, 16, 64, seed=13, lengths=[900, 777]),
        # long durations: K above 512 takes the 64-durations-per-lane shape
        "k_700": lambda: synth.make_custom(2, 2600, 700, 4, seed=42, lengths=[2600, 1900],
                                           dur_mean=100.0, amp=2.0),
        "k_2000_genomic_like": lambda: synth.make_custom(
            2, 5000, 2000, 6, seed=41, lengths=[5000, 3333], dur_mean=50.0, amp=2.0,
            label_p=(0.6, 0.2, 0.1, 0.05, 0.03, 0.02)),
    }


CASES = _cases()


@pytest.fixture(scope="module", params=sorted(CASES))
def fb_case(request):
    case = CASES[request.param]()
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"],
                                  case["dur"].shape[0])
    return request.param, case, ref


def test_forward_backward_matches_oracle(fb_case):
    name, case, ref = fb_case
    got = gpu_fb(case)
    assert got["status"] == 0
    print(name, errors(got, ref))
    assert_fb_close(got, ref, case["lengths"], name)


def test_log_domain_rings_match_oracle(fb_case):
    """The same cases with every ring forced into the log-domain kernel."""
    name, case, ref = fb_case
    got = gpu_fb(case, log_domain=True)
    assert got["status"] == 0
    print(name, errors(got, ref))
    assert_fb_close(got, ref, case["lengths"], name)


def _wide_range_cases():
    """Inputs outside the exponential-domain kernel's exponent head-room:
    forbidden (-inf) transitions and durations, and emissions of about a
    hundred nats per position; the library runs them in the log domain.
    (Float32 log-domain values carry ulp(|one step's score|): at scores of
    several hundred log2 units per position -- emissions x25 here -- that
    alone reaches 1e-4 on marginals.)"""
    forbidden = synth.make("speech", B=3, T=120, seed=21)
    forbidden["trans"][0, 1] = -np.inf
    forbidden["trans"][2, :5] = -np.inf
    forbidden["dur"][3, 7] = -np.inf
    loud = synth.make("speech", B=3, T=120, seed=22)
    loud["em"] *= np.float32(10.0)
    long_loud = synth.make("genomic", B=1, T=2500, seed=23)
    long_loud["em"] *= np.float32(10.0)
    return {"forbidden": forbidden, "loud": loud, "long_loud": long_loud}


def test_ring_domain_choice():
    """Workload-like inputs run in the exponential domain, the wide-range ones
    and log_domain=True in the log domain; both give the oracle's results."""
    from semi_markov_crf_b200 import semicrf
    case = synth.make("speech", B=4, T=200, seed=24)
    em, lengths, trans, dur = to_dev(case)
    _, ws = semicrf.forward(em, lengths, trans, dur)
    assert semicrf.ring_domains(ws) == [1] * 8
    _, ws = semicrf.forward(em, lengths, trans, dur, log_domain=True)
    assert semicrf.ring_domains(ws) == [2] * 8
    for name, c in _wide_range_cases().items():
        em, lengths, trans, dur = to_dev(c)
        _, ws = semicrf.forward(em, lengths, trans, dur)
        B = len(c["lengths"])
        assert semicrf.ring_domains(ws) == [2] * (2 * B), name


def test_log_domain_ignores_a_stale_workspace():
    """A workspace whose bytes say that every ring ran in the exponential
    domain and kept its values (int32 ones everywhere) must not mislead a
    log-domain forward-backward on it."""
    from semi_markov_crf_b200 import semicrf
    case = synth.make("genomic", B=2, T=3000, seed=26)
    em, lengths, trans, dur = to_dev(case)
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    ws = semicrf.Workspace(B, T, C, K, semicrf.FLAG_LOG_DOMAIN, em.device)
    ws.buf.view(torch.int32).fill_(1)
    logZ, ws = semicrf.forward(em, lengths, trans, dur, ws=ws, log_domain=True)
    out = semicrf.backward(ws, lengths, trans, dur, marginals=True)
    assert semicrf.get_status(ws) == 0
    got = {k: v.cpu().numpy() for k, v in out.items()}
    got["logZ"] = logZ.cpu().numpy()
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"], K)
    print(errors(got, ref))
    assert_fb_close(got, ref, case["lengths"], "stale workspace")


def test_moderately_loud_inputs_stay_exact_in_the_exponential_domain():
    """Emissions x3 (per-step exponent span about 60 of fp32's 126): still the
    exponential domain, still within tolerance."""
    from semi_markov_crf_b200 import semicrf
    case = synth.make("genomic", B=2, T=2000, seed=25)
    case["em"] *= np.float32(3.0)
    em, lengths, trans, dur = to_dev(case)
    _, ws = semicrf.forward(em, lengths, trans, dur)
    assert semicrf.ring_domains(ws) == [1] * 4
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"],
                                  case["dur"].shape[0])
    got = gpu_fb(case)
    print(errors(got, ref))
    assert_fb_close(got, ref, case["lengths"], "loud x3")


@pytest.mark.parametrize("name", ["forbidden", "loud", "long_loud"])
def test_wide_range_inputs_match_oracle(name):
    case = _wide_range_cases()[name]
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"],
                                  case["dur"].shape[0])
    got = gpu_fb(case)
    assert got["status"] == 0
    print(name, errors(got, ref))
    assert_fb_close(got, ref, case["lengths"], name)


def test_viterbi_matches_oracle(fb_case):
    name, case, _ = fb_case
    ref = oracle.viterbi(case["em"], case["lengths"], case["trans"], case["dur"], case["dur"].shape[0])
    got = gpu_viterbi(case)
    n = assert_viterbi_ok(got, ref, case, label=name)
    print(name, "paths differing at ties:", n)


def test_prefix_center_matches_oracle():
    from semi_markov_crf_b200 import semicrf
    case = synth.make("speech", B=5, T=300, pad_value=1e30)
    em, lengths, _, _ = to_dev(case)
    for center in (True, False):
        S, nu = semicrf.prefix_center(em, lengths, center=center)
        S_ref, nu_ref = oracle.prefix_center(case["em"], case["lengths"], center=center)
        S = S.cpu().numpy()
        assert np.max(np.abs(S - S_ref)) <= 1e-9 * max(1.0, np.max(np.abs(S_ref)))
        assert np.max(np.abs(nu.cpu().numpy() - nu_ref)) <= 1e-6 * max(1.0, np.max(np.abs(nu_ref)))


def test_garbage_padding_changes_nothing():
    clean = synth.make("speech", B=4, T=100)
    dirty = synth.make("speech", B=4, T=100, pad_value=np.nan)
    assert np.any(np.isnan(dirty["em"]))
    a, b = gpu_fb(clean), gpu_fb(dirty)
    for k in ("logZ", "grad_em", "grad_trans", "grad_dur", "pos_marg", "start_marg", "end_marg"):
        assert np.array_equal(a[k], b[k]), k
    huge = synth.make("speech", B=4, T=100, pad_value=1e30)
    c = gpu_fb(huge)
    assert np.array_equal(a["logZ"], c["logZ"]) and np.array_equal(a["grad_em"], c["grad_em"])
    va, vb = gpu_viterbi(clean), gpu_viterbi(dirty)
    for k in va:
        assert np.array_equal(va[k], vb[k])


def test_results_are_deterministic():
    case = synth.make("genomic", B=2, T=2500)
    a, b = gpu_fb(case), gpu_fb(case)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_forward_only_flag_gives_the_same_backward():
    case = synth.make("speech", B=3, T=120)
    a = gpu_fb(case)
    b = gpu_fb(case, forward_only=True)
    for k in ("logZ", "grad_em", "grad_trans", "grad_dur", "pos_marg"):
        assert np.array_equal(a[k], b[k]), k


def test_no_center_and_upstream_gradient():
    case = synth.make("speech", B=3, T=120)
    g = np.array([1.0, -2.5, 0.25])
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"], 30,
                                  center=False, grad_logZ=g)
    got = gpu_fb(case, center=False, grad_logZ=g)
    assert_fb_close(got, ref, case["lengths"], "no_center")


def test_bad_length_is_reported_and_zeroed():
    from semi_markov_crf_b200 import semicrf
    case = synth.make_custom(3, 40, 5, 3, seed=3, lengths=[40, 20, 10])
    case["lengths"] = np.array([40, 41, -1], dtype=np.int32)
    got = gpu_fb(case)
    assert got["status"] == 6
    assert np.isnan(got["logZ"][1]) and np.isnan(got["logZ"][2]) and np.isfinite(got["logZ"][0])
    assert np.all(got["grad_em"][1:] == 0) and np.all(got["pos_marg"][1:] == 0)
    v = gpu_viterbi(case)
    assert np.all(v["labels"][1:] == -1)
    ok = synth.make_custom(1, 40, 5, 3, seed=3)
    assert gpu_fb(ok)["status"] == 0


def test_bounded_wait_gives_up_with_a_status():
    from semi_markov_crf_b200 import semicrf
    ws = semicrf.Workspace(1, 8, 2, 2)
    assert semicrf.selftest_bounded_wait(ws, 1000) == 5
    # the context is still usable afterwards
    case = synth.make("tiny")
    assert gpu_fb(case)["status"] == 0
