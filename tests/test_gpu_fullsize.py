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


@pytest.mark.parametrize("name", NAMES)
def test_fullsize_gold_path_score_and_counts(name):
    """The path score of the generating segmentation (a random one for the
    noise-only tiny workload) and the counts it adds to the gradients, at the
    full size, against the oracle (cheap: one pass over the path)."""
    from gpu_common import to_dev
    from semi_markov_crf_b200 import semicrf
    case = synth.make(name)
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    labels, seg = case["gold"], case["gold_start"]
    if not np.any(labels >= 0):
        rng = np.random.default_rng(5)
        labels = np.full((B, T), -1, dtype=np.int32)
        seg = np.zeros((B, T), dtype=np.uint8)
        for b, L in enumerate(case["lengths"]):
            pos = 0
            while pos < L:
                d = int(rng.integers(1, min(K, L - pos) + 1))
                labels[b, pos:pos + d] = rng.integers(0, C)
                seg[b, pos] = 1
                pos += d
    em, lengths, trans, dur = to_dev(case)
    grads = dict(grad_em=torch.zeros((B, T, C), dtype=torch.float32, device="cuda"),
                 grad_trans=torch.zeros((C, C), dtype=torch.float32, device="cuda"),
                 grad_dur=torch.zeros((K, C), dtype=torch.float32, device="cuda"))
    g = np.linspace(-1.0, 2.0, B) if B > 1 else np.array([0.75])
    score = semicrf.path_score(em, lengths, trans, dur, torch.from_numpy(labels).cuda(),
                               torch.from_numpy(seg).cuda(),
                               grad_score=torch.as_tensor(g, device="cuda"), grads=grads)
    score = score.cpu().numpy()
    ref = oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"], labels, seg, K)
    assert np.all(np.isfinite(ref))
    err = np.abs(score - ref) / np.maximum(1.0, np.abs(ref))
    print(name, "path score rel err", err.max())
    assert err.max() <= 1e-9
    cnt = oracle.path_counts(case["lengths"], labels, seg, C, K)
    e = float(np.max(np.abs(grads["grad_em"].cpu().numpy() - cnt["grad_em"] * g[:, None, None])))
    assert e <= MARG_ATOL, e
    for key, ck in (("grad_trans", "trans_count"), ("grad_dur", "dur_count")):
        ref_c = np.einsum("b,bij->ij", g, cnt[ck])
        d = np.abs(grads[key].cpu().numpy().astype(np.float64) - ref_c)
        assert np.max(d / np.maximum(1.0, np.abs(ref_c))) <= COUNT_RTOL, key
