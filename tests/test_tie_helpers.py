"""Host checks of the Viterbi comparison helpers the GPU tests use: the
differing stretches between two segmentations, and that a stretch's score
difference from the oracle's windowed path score equals the difference of
the total scores (the rest of both paths is shared)."""

import numpy as np

import oracle
from gpu_common import differing_stretches, local_tie_report
from semi_markov_crf_b200 import synth


def _path(L, segs):
    lab = np.full(L + 3, -1, np.int32)
    seg = np.zeros(L + 3, np.uint8)
    for s, t, c in segs:
        lab[s:t] = c
        seg[s] = 1
    return lab, seg


def test_identical_paths_have_no_stretch():
    la, sa = _path(10, [(0, 3, 1), (3, 10, 2)])
    assert differing_stretches(la, sa, la, sa, 10) == []


def test_one_stretch_with_shared_neighbours():
    # shared [0,2) label 0, then 2..6 differ, shared [6,9) label 1
    la, sa = _path(9, [(0, 2, 0), (2, 4, 2), (4, 6, 2), (6, 9, 1)])
    lb, sb = _path(9, [(0, 2, 0), (2, 5, 2), (5, 6, 2), (6, 9, 1)])
    assert differing_stretches(la, sa, lb, sb, 9) == [(0, 2, 6, 9)]


def test_label_change_only_and_stretch_at_both_ends():
    la, sa = _path(6, [(0, 3, 0), (3, 6, 1)])
    lb, sb = _path(6, [(0, 3, 2), (3, 6, 1)])
    assert differing_stretches(la, sa, lb, sb, 6) == [(0, 0, 3, 6)]
    lc, sc = _path(6, [(0, 3, 0), (3, 6, 2)])
    assert differing_stretches(la, sa, lc, sc, 6) == [(0, 3, 6, 6)]
    # two stretches separated by a shared segment
    la, sa = _path(12, [(0, 2, 0), (2, 6, 1), (6, 8, 0), (8, 12, 1)])
    lb, sb = _path(12, [(0, 2, 1), (2, 6, 1), (6, 8, 0), (8, 12, 0)])
    assert differing_stretches(la, sa, lb, sb, 12) == [(0, 0, 2, 6), (6, 8, 12, 12)]


def test_stretch_differences_add_up_to_the_total_difference():
    case = synth.make_custom(1, 40, 5, 3, seed=11)
    K = 5
    la, sa = _path(40, [(0, 4, 0), (4, 9, 1), (9, 12, 1), (12, 17, 2), (17, 20, 0),
                        (20, 25, 1), (25, 30, 2), (30, 35, 0), (35, 40, 2)])
    lb, sb = _path(40, [(0, 4, 0), (4, 7, 1), (7, 12, 1), (12, 17, 2), (17, 20, 0),
                        (20, 25, 0), (25, 30, 2), (30, 33, 0), (33, 35, 0), (35, 40, 2)])
    la, sa, lb, sb = (x[None, :40] for x in (la, sa, lb, sb))
    rep = local_tie_report(case, la, sa, lb, sb)
    assert [(r["start"], r["end"]) for r in rep] == [(4, 12), (20, 25), (30, 35)]
    tot = oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"], la, sa, K) - \
        oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"], lb, sb, K)
    assert np.isfinite(tot[0]) and tot[0] != 0
    assert abs(sum(r["diff"] for r in rep) - float(tot[0])) < 1e-9
