"""GPU parity of the path score and the loss gradient (semicrf_path_score)
against the float64 oracle, through the C ABI via the binding: the score of
gold, decoded and random segmentations, the per-sequence weighted counts it
adds to the gradients, the NLL gradient log Z - score assembled from
semicrf_backward and semicrf_path_score, malformed paths, bad lengths, and
that the call leaves a pending forward / backward pair untouched.

Tolerances: the score is a float64 sum of float32 inputs on both sides, in a
different order, so it agrees to ~1e-13 relative; 1e-9 is used.  Gradients
are float32 outputs: emission entries 1e-4 absolute, counts
1e-4 * max(1, |count|), as for the backward pass.
"""

import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import COUNT_RTOL, MARG_ATOL, gpu_fb, max_abs, to_dev
from semi_markov_crf_b200 import synth

pytestmark = pytest.mark.gpu

SCORE_RTOL = 1e-9


def _random_paths(rng, lengths, T, K, C):
    labels = np.full((len(lengths), T), -1, dtype=np.int32)
    seg = np.zeros((len(lengths), T), dtype=np.uint8)
    for b, L in enumerate(lengths):
        pos = 0
        while pos < L:
            d = int(rng.integers(1, min(K, L - pos) + 1))
            labels[b, pos:pos + d] = rng.integers(0, C)
            seg[b, pos] = 1
            pos += d
    return labels, seg


def _gpu_path(case, labels, seg, g=None, negate=False, grads=None, center=True, ws=None):
    from semi_markov_crf_b200 import semicrf
    em, lengths, trans, dur = to_dev(case)
    lab = torch.from_numpy(np.ascontiguousarray(labels, dtype=np.int32)).cuda()
    ss = torch.from_numpy(np.ascontiguousarray(seg, dtype=np.uint8)).cuda()
    gs = None if g is None else torch.as_tensor(g, dtype=torch.float64, device="cuda")
    score = semicrf.path_score(em, lengths, trans, dur, lab, ss, center=center, ws=ws,
                               grad_score=gs, negate=negate, grads=grads)
    return score.cpu().numpy()


def _zero_grads(case):
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    return dict(grad_em=torch.zeros((B, T, C), dtype=torch.float32, device="cuda"),
                grad_trans=torch.zeros((C, C), dtype=torch.float32, device="cuda"),
                grad_dur=torch.zeros((K, C), dtype=torch.float32, device="cuda"))


def _expected(case, labels, seg, g, center=True):
    C = case["em"].shape[2]
    K = case["dur"].shape[0]
    cnt = oracle.path_counts(case["lengths"], labels, seg, C, K, center=center)
    w = np.asarray(g, dtype=np.float64) * cnt["valid"]
    return dict(grad_em=cnt["grad_em"] * w[:, None, None],
                grad_trans=np.einsum("b,bij->ij", w, cnt["trans_count"]),
                grad_dur=np.einsum("b,bij->ij", w, cnt["dur_count"]))


def _assert_grads(got, ref, label):
    e = max_abs(got["grad_em"].cpu().numpy(), ref["grad_em"])
    assert e <= MARG_ATOL, f"{label} grad_em {e:.3e}"
    for key in ("grad_trans", "grad_dur"):
        d = np.abs(got[key].cpu().numpy().astype(np.float64) - ref[key])
        r = float(np.max(d / np.maximum(1.0, np.abs(ref[key])))) if d.size else 0.0
        assert r <= COUNT_RTOL, f"{label} {key} {r:.3e}"


def _assert_scores(got, ref, label):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), (label, got, ref)
    err = np.abs(got[fin] - ref[fin]) / np.maximum(1.0, np.abs(ref[fin]))
    assert err.size == 0 or err.max() <= SCORE_RTOL, (label, err.max())


CASES = {
    "tiny": lambda: synth.make("tiny"),
    "speech_small": lambda: synth.make("speech", B=6, T=160),
    "genomic_small": lambda: synth.make("genomic", B=2, T=3000),
    "large_small": lambda: synth.make("large", B=2, T=160),
    "mixed_with_empty": lambda: synth.make_custom(4, 80, 9, 5, seed=9, lengths=[80, 0, 1, 57]),
    "k_equals_1": lambda: synth.make_custom(2, 90, 1, 7, seed=7, lengths=[90, 41]),
    "several_chunks": lambda: synth.make_custom(3, 2600, 12, 3, seed=21, lengths=[2600, 1025, 1024]),
    "k_2000": lambda: synth.make_custom(2, 5000, 2000, 6, seed=41, lengths=[5000, 3333],
                                        dur_mean=400.0, amp=2.0),
}


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("center", [True, False])
def test_path_score_and_counts_match_oracle(name, center):
    case = CASES[name]()
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    rng = np.random.default_rng(17)
    paths = {"random": _random_paths(rng, case["lengths"], T, K, C)}
    if np.any(case["gold"] >= 0):
        paths["gold"] = (case["gold"], case["gold_start"])
    vit = oracle.viterbi(case["em"], case["lengths"], case["trans"], case["dur"], K, center=center)
    paths["viterbi"] = (vit["labels"], vit["seg_start"])
    g = rng.uniform(-2.0, 2.0, size=B)
    for pname, (labels, seg) in paths.items():
        ref = oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"], labels, seg,
                                K, center=center)
        grads = _zero_grads(case)
        got = _gpu_path(case, labels, seg, g=g, grads=grads, center=center)
        _assert_scores(got, ref, f"{name}/{pname}")
        _assert_grads(grads, _expected(case, labels, seg, g, center), f"{name}/{pname}")
    # decoding optimum: the decoded path scores the Viterbi score
    assert np.allclose(_gpu_path(case, vit["labels"], vit["seg_start"], center=center),
                       vit["score"], rtol=SCORE_RTOL, atol=SCORE_RTOL)


@pytest.mark.parametrize("name", ["speech_small", "genomic_small", "large_small"])
def test_nll_gradient_matches_oracle(name):
    """backward(g) then path_score(g, negate) on the same buffers gives the
    gradient of g * (log Z - score(gold))."""
    from semi_markov_crf_b200 import semicrf
    case = CASES[name]()
    B = case["em"].shape[0]
    K = case["dur"].shape[0]
    g = np.linspace(0.5, 1.5, B)
    em, lengths, trans, dur = to_dev(case)
    gt = torch.as_tensor(g, dtype=torch.float64, device="cuda")
    logZ, ws = semicrf.forward(em, lengths, trans, dur)
    lab = torch.from_numpy(case["gold"]).cuda()
    ss = torch.from_numpy(case["gold_start"]).cuda()
    out = semicrf.backward(ws, lengths, trans, dur, grad_logZ=gt)
    score = semicrf.path_score(em, lengths, trans, dur, lab, ss, ws=ws, grad_score=gt, negate=True,
                               grads=out)
    assert semicrf.get_status(ws) == 0
    fb = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"], K,
                                 grad_logZ=g)
    ps = oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"], case["gold"],
                           case["gold_start"], K)
    gold = _expected(case, case["gold"], case["gold_start"], g)
    ref = dict(grad_em=fb["grad_e"] - gold["grad_em"], grad_trans=fb["grad_trans"] - gold["grad_trans"],
               grad_dur=fb["grad_dur"] - gold["grad_dur"])
    _assert_grads(out, ref, name)
    nll = logZ.cpu().numpy() - score.cpu().numpy()
    nll_ref = fb["logZ"] - ps
    assert np.all(nll_ref > 0)
    assert np.max(np.abs(nll - nll_ref) / np.maximum(1.0, np.abs(fb["logZ"]))) <= 1e-5


def test_malformed_paths_score_nan_and_add_no_gradient():
    case = synth.make_custom(5, 30, 4, 3, seed=31)
    B, T, C = case["em"].shape
    K = 4
    rng = np.random.default_rng(32)
    labels, seg = _random_paths(rng, case["lengths"], T, K, C)
    seg[1, 0] = 0                                # no start at position 0
    labels[2, 7] = C                             # label out of range
    labels[3, :] = 1; seg[3, :] = 0; seg[3, 0] = 1  # one segment longer than K
    j = int(np.flatnonzero(seg[4, 1:] == 0)[0]) + 1  # a label change inside a segment
    labels[4, j] = (labels[4, j - 1] + 1) % C
    ref = oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"], labels, seg, K)
    assert np.isfinite(ref[0]) and np.all(np.isnan(ref[1:]))
    grads = _zero_grads(case)
    got = _gpu_path(case, labels, seg, grads=grads)
    _assert_scores(got, ref, "malformed")
    _assert_grads(grads, _expected(case, labels, seg, np.ones(B)), "malformed")
    assert np.all(grads["grad_em"][1:].cpu().numpy() == 0)


def test_bad_length_sets_the_status():
    from semi_markov_crf_b200 import semicrf
    case = synth.make_custom(2, 40, 5, 3, seed=3)
    labels, seg = case["gold"], case["gold_start"]
    case["lengths"] = np.array([40, 41], dtype=np.int32)
    em, lengths, trans, dur = to_dev(case)
    ws = semicrf.Workspace(2, 40, 3, 5)
    s = semicrf.path_score(em, lengths, trans, dur, torch.from_numpy(labels).cuda(),
                           torch.from_numpy(seg).cuda(), ws=ws).cpu().numpy()
    assert semicrf.get_status(ws) == 6
    assert np.isfinite(s[0]) and np.isnan(s[1])


def test_path_score_between_forward_and_backward_changes_nothing():
    from semi_markov_crf_b200 import semicrf
    case = synth.make("speech", B=4, T=200)
    em, lengths, trans, dur = to_dev(case)
    logZ, ws = semicrf.forward(em, lengths, trans, dur)
    ref = {k: v.clone() for k, v in semicrf.backward(ws, lengths, trans, dur, marginals=True).items()}
    logZ2, ws = semicrf.forward(em, lengths, trans, dur, ws=ws)
    semicrf.path_score(em, lengths, trans, dur, torch.from_numpy(case["gold"]).cuda(),
                       torch.from_numpy(case["gold_start"]).cuda(), ws=ws)
    got = semicrf.backward(ws, lengths, trans, dur, marginals=True)
    assert torch.equal(logZ, logZ2)
    for k in ref:
        assert torch.equal(ref[k], got[k]), k


def test_path_score_is_deterministic():
    case = synth.make("genomic", B=2, T=5000)
    a_g, b_g = _zero_grads(case), _zero_grads(case)
    a = _gpu_path(case, case["gold"], case["gold_start"], g=[0.3, -1.7], grads=a_g)
    b = _gpu_path(case, case["gold"], case["gold_start"], g=[0.3, -1.7], grads=b_g)
    assert np.array_equal(a, b)
    for k in a_g:
        assert torch.equal(a_g[k], b_g[k]), k
