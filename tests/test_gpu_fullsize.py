"""GPU parity at the five full workload sizes (tiny, speech, genomic, ultra,
large), in the launch configuration bench.py times.

Tiny and speech: the float64 oracle runs here, on the same seeded inputs
(seconds), and every output is compared element by element: log Z, every
position / start / end marginal and emission gradient, the full transition
and duration gradients, and the decoded path.

Genomic, ultra and large: the oracle takes minutes, so its values come from
tests/golden/<name>.npz (written by tests/golden/make_golden.py, which runs
only the oracle): log Z, the full transition and duration gradients, the
oracle's full decoded path, and the marginals and emission gradients at
every position near the points where the kernels change state (prefix-sum
tile edges, the cut-normaliser grid, checkpoints, segments straddling them,
both ends of each sequence) plus random rows.

Viterbi paths are compared bit for bit.  Where the GPU's path differs from
the oracle's, each differing stretch must be a tie: the float64 scores of
the two paths over that stretch agree to within float32 rounding of the
stretch's own terms (reading O7).  The number of differing stretches is
printed per workload.

Properties that hold at any size are checked on every output: position
marginals sum to one over labels, every position is covered by exactly one
segment (sum_k k * grad_dur = sum_b L_b), segments minus transitions is one
per sequence, and the centering Jacobian sums the emission gradient to zero
over positions.
"""

import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import (COUNT_RTOL, LOGZ_RTOL, MARG_ATOL, TIE_RTOL, gpu_fb, gpu_viterbi,
                        local_tie_report)
from semi_markov_crf_b200 import synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
NAMES = ["tiny", "speech", "genomic", "ultra", "large"]
LIVE = ("tiny", "speech")   # the oracle runs at test time


def _reference(name, case):
    """Oracle values: computed now (LIVE) or read from the golden file."""
    K = case["dur"].shape[0]
    if name in LIVE:
        fb = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"], K)
        vit = oracle.viterbi(case["em"], case["lengths"], case["trans"], case["dur"], K)
        B, T = case["em"].shape[:2]
        rb, ru = np.nonzero(np.arange(T)[None, :] < case["lengths"][:, None])
        bb, bu = np.nonzero(np.arange(T + 1)[None, :] <= case["lengths"][:, None])
        return dict(logZ=fb["logZ"], grad_trans=fb["grad_trans"], grad_dur=fb["grad_dur"],
                    viterbi_score=vit["score"], labels=vit["labels"], seg_start=vit["seg_start"],
                    row_b=rb, row_u=ru, pos_marg=fb["pos_marg"][rb, ru],
                    grad_e=fb["grad_e"][rb, ru], brow_b=bb, brow_u=bu,
                    start_marg=fb["start_marg"][bb, bu], end_marg=fb["end_marg"][bb, bu],
                    quant=0.0)
    path = os.path.join(GOLDEN, f"{name}.npz")
    if not os.path.exists(path):
        pytest.skip(f"{path} not generated")
    g = dict(np.load(path))
    assert np.array_equal(case["lengths"], g["lengths"]), "generator drifted from the golden file"
    q = float(g["qscale"])
    T = case["em"].shape[1]
    return dict(logZ=g["logZ"], grad_trans=g["grad_trans"], grad_dur=g["grad_dur"],
                viterbi_score=g["viterbi_score"], labels=g["viterbi_labels"].astype(np.int32),
                seg_start=np.unpackbits(g["viterbi_seg"], axis=1, count=T),
                row_b=g["row_b"], row_u=g["row_u"], pos_marg=g["q_pos_marg"] / q,
                grad_e=g["q_grad_e"] / q, brow_b=g["brow_b"], brow_u=g["brow_u"],
                start_marg=g["q_start_marg"] / q, end_marg=g["q_end_marg"] / q,
                quant=0.5 / q)


@pytest.fixture(scope="module", params=NAMES)
def full(request):
    name = request.param
    case = synth.make(name)
    ref = _reference(name, case)
    got = gpu_fb(case)
    return name, case, ref, got


def test_fullsize_forward_backward_matches_oracle(full):
    name, case, ref, got = full
    assert got["status"] == 0
    err = np.abs(got["logZ"] - ref["logZ"]) / np.maximum(1.0, np.abs(ref["logZ"]))
    assert np.all(err <= LOGZ_RTOL), err.max()
    rb, ru, bb, bu = ref["row_b"], ref["row_u"], ref["brow_b"], ref["brow_u"]
    report = {"logZ_rel": float(err.max()), "position_rows": int(len(rb)),
              "boundary_rows": int(len(bb))}
    for key, gk, (b, u) in (("pos_marg", "pos_marg", (rb, ru)), ("grad_e", "grad_em", (rb, ru)),
                            ("start_marg", "start_marg", (bb, bu)),
                            ("end_marg", "end_marg", (bb, bu))):
        report[key] = float(np.max(np.abs(got[gk][b, u].astype(np.float64) - ref[key])))
    for key in ("grad_trans", "grad_dur"):
        d = np.abs(got[key].astype(np.float64) - ref[key])
        report[key] = float(np.max(d / np.maximum(1.0, np.abs(ref[key]))))
    print(name, report)
    for key in ("pos_marg", "grad_e", "start_marg", "end_marg"):
        assert report[key] <= MARG_ATOL + ref["quant"], (key, report[key])
    for key in ("grad_trans", "grad_dur"):
        assert report[key] <= COUNT_RTOL, (key, report[key])


def test_fullsize_invariants(full):
    name, case, ref, got = full
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


def test_fullsize_viterbi_matches_oracle(full):
    name, case, ref, _ = full
    got = gpu_viterbi(case)
    best = ref["viterbi_score"]
    err = np.abs(got["score"] - best) / np.maximum(1.0, np.abs(best))
    assert np.all(err <= LOGZ_RTOL), err.max()
    lengths = case["lengths"]
    for b in range(len(lengths)):
        L = int(lengths[b])
        assert np.all(got["labels"][b, L:] == -1) and np.all(got["seg_start"][b, L:] == 0)
    same = [np.array_equal(got["labels"][b], ref["labels"][b]) and
            np.array_equal(got["seg_start"][b], ref["seg_start"][b]) for b in range(len(lengths))]
    rep = local_tie_report(case, got["labels"], got["seg_start"], ref["labels"],
                           ref["seg_start"])
    worst = max((abs(r["diff"]) / max(1.0, r["mag"]) for r in rep), default=0.0)
    print(name, f"viterbi: {sum(same)}/{len(same)} sequences bit-exact, {len(rep)} differing "
                f"stretches, worst |diff|/mag {worst:.2e}",
          [(r["b"], r["start"], r["end"], round(r["diff"], 9)) for r in rep[:8]])
    assert all(same) == (not rep)
    for r in rep:
        assert abs(r["diff"]) <= TIE_RTOL * max(1.0, r["mag"]), r
    # the decoded path's float64 score is the optimum
    rescored = oracle.path_score(case["em"], lengths, case["trans"], case["dur"], got["labels"],
                                 got["seg_start"], K=case["dur"].shape[0])
    assert np.all(np.isfinite(rescored))


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
