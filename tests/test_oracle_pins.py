"""Pins for the float64 oracle (CPU only).

Each test checks the oracle against something other than itself: brute-force
enumeration, a separately written textbook linear-chain CRF, closed forms,
finite differences, and identities the model must satisfy (explainer
section 4, "Correctness": marginals summing to one, valid boundary
probabilities, mass conservation, finite-difference gradient checks).
Chosen so that a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.
"""

import math

import numpy as np
import pytest

import oracle
from pins import brute, linear_chain
from semi_markov_crf_b200 import synth


def _rand_case(rng, B, T, K, C, lengths=None, scale=1.0, pstd=0.5):
    em = (scale * rng.standard_normal((B, T, C))).astype(np.float64)
    if lengths is None:
        lengths = np.full(B, T, dtype=np.int32)
    lengths = np.asarray(lengths, dtype=np.int32)
    trans = pstd * rng.standard_normal((C, C))
    dur = pstd * rng.standard_normal((K, C))
    return em, lengths, trans, dur


# ---------------------------------------------------------------- (v) prefix sums
def test_prefix_sum_equals_explicit_segment_sum():
    rng = np.random.default_rng(11)
    em, lengths, _, _ = _rand_case(rng, 3, 40, 6, 5, lengths=[40, 17, 1], scale=3.0)
    S, nu = oracle.prefix_center(em, lengths, center=True)
    for b in range(3):
        L = int(lengths[b])
        assert np.allclose(nu[b], em[b, :L].mean(axis=0), rtol=0, atol=1e-13)
        et = em[b, :L] - em[b, :L].mean(axis=0)
        for t in range(1, L + 1):
            for k in range(1, min(6, t) + 1):
                explicit = et[t - k:t].sum(axis=0)
                assert np.max(np.abs(S[b, t] - S[b, t - k] - explicit)) < 1e-12
        # centering identity: the centred sum over the whole sequence is zero
        assert np.max(np.abs(S[b, L])) < 1e-12
        assert np.all(S[b, L + 1:] == 0)
    S0, nu0 = oracle.prefix_center(em, lengths, center=False)
    assert np.all(nu0 == 0)
    assert np.allclose(S0[0, 40], em[0].sum(axis=0), atol=1e-12)


# ---------------------------------------------------------------- (i) brute force
BRUTE_CASES = [
    # (L, K, C, center, seed)
    (1, 3, 3, True, 1),
    (2, 1, 2, True, 2),
    (3, 4, 3, False, 3),
    (5, 2, 3, True, 4),
    (6, 3, 2, True, 5),
    (7, 4, 2, False, 6),
    (8, 4, 2, True, 7),
    (7, 3, 3, True, 8),
    (10, 4, 2, True, 9),
]


@pytest.mark.parametrize("L,K,C,center,seed", BRUTE_CASES)
def test_bruteforce_logZ_and_marginals(L, K, C, center, seed):
    rng = np.random.default_rng(seed)
    em, lengths, trans, dur = _rand_case(rng, 1, L, K, C, pstd=0.7)
    ref = brute.enumerate_all(em[0], L, trans, dur, center=center)
    out = oracle.forward_backward(em, lengths, trans, dur, K, center=center, threads=1)
    assert abs(out["logZ"][0] - ref["logZ"]) <= 1e-12 * max(1.0, abs(ref["logZ"]))
    assert abs(out["logZ_beta"][0] - ref["logZ"]) <= 1e-12 * max(1.0, abs(ref["logZ"]))
    for key in ("start_marg", "end_marg", "pos_marg"):
        got = out[key][0][: ref[key].shape[0]]
        assert np.max(np.abs(got - ref[key])) < 1e-12, key
    assert np.max(np.abs(out["grad_dur"] - ref["grad_dur"])) < 1e-12
    assert np.max(np.abs(out["grad_trans"] - ref["grad_trans"])) < 1e-12


@pytest.mark.parametrize("L,K,C,center,seed", BRUTE_CASES)
def test_bruteforce_segment_marginals(L, K, C, center, seed):
    """P(segment [s, s+k) with label c), the quantity behind the pages'
    "boundary probabilities are valid" check (explainer section 4,
    Correctness), against enumeration; and its bookkeeping: summed over
    durations it is the start marginal, over starts the duration count,
    over the segments covering u the position marginal."""
    rng = np.random.default_rng(seed)
    em, lengths, trans, dur = _rand_case(rng, 1, L, K, C, pstd=0.7)
    ref = brute.enumerate_all(em[0], L, trans, dur, center=center)
    out = oracle.forward_backward(em, lengths, trans, dur, K, center=center, threads=1,
                                  want_segments=True)
    sm = out["seg_marg"][0]
    assert sm.shape == (L, K, C)
    assert np.max(np.abs(sm - ref["seg_marg"])) < 1e-12
    assert np.max(np.abs(sm.sum(axis=1) - out["start_marg"][0, :L])) < 1e-12
    assert np.max(np.abs(sm.sum(axis=0) - out["grad_dur"])) < 1e-12
    cover = np.zeros((L, C))
    for s_ in range(L):
        for k in range(1, K + 1):
            cover[s_:s_ + k] += sm[s_, k - 1]
    assert np.max(np.abs(cover - out["pos_marg"][0, :L])) < 1e-12
    for s_ in range(L):   # no segment runs past the end
        assert np.all(sm[s_, L - s_:] == 0)


@pytest.mark.parametrize("L,K,C,center,seed", BRUTE_CASES)
def test_bruteforce_viterbi(L, K, C, center, seed):
    rng = np.random.default_rng(100 + seed)
    em, lengths, trans, dur = _rand_case(rng, 1, L, K, C, pstd=0.7)
    ref = brute.enumerate_all(em[0], L, trans, dur, center=center)
    vit = oracle.viterbi(em, lengths, trans, dur, K, center=center, threads=1)
    assert abs(vit["score"][0] - ref["best_score"]) < 1e-12
    # the decoded path is one of the optimal segmentations
    assert any(np.array_equal(vit["labels"][0, :L], lab) and np.array_equal(vit["seg_start"][0, :L], ss)
               for lab, ss in ref["optimal"])
    rescored = oracle.path_score(em, lengths, trans, dur, vit["labels"], vit["seg_start"], K,
                                 center=center)
    assert abs(rescored[0] - ref["best_score"]) < 1e-12


def test_viterbi_tie_break_prefers_short_duration_then_small_label():
    # All-zero model: every segmentation scores 0, so the documented tie-break
    # (smallest k, then smallest previous label, then smallest final label)
    # decides: unit-length segments, all labelled 0.
    L, K, C = 6, 3, 3
    em = np.zeros((1, L, C))
    vit = oracle.viterbi(em, [L], np.zeros((C, C)), np.zeros((K, C)), K)
    assert vit["score"][0] == 0.0
    assert np.array_equal(vit["labels"][0], np.zeros(L, dtype=np.int32))
    assert np.array_equal(vit["seg_start"][0], np.ones(L, dtype=np.uint8))


@pytest.mark.parametrize("seed", [1, 2, 3, 4, 5])
def test_viterbi_exact_ties_follow_the_tie_break(seed):
    # Small integer inputs make every score exact in float64, so structural
    # ties (same-label neighbours with swapped durations) are exact and the
    # tie-break alone picks the path; enumeration applies the same rule.
    rng = np.random.default_rng(300 + seed)
    L, K, C = 8, 4, 2
    em = rng.integers(-2, 3, size=(1, L, C)).astype(np.float64)
    trans = rng.integers(-1, 2, size=(C, C)).astype(np.float64)
    dur = rng.integers(-1, 2, size=(K, C)).astype(np.float64)
    ref = brute.enumerate_all(em[0], L, trans, dur, center=False, tie_tol=0.0)
    vit = oracle.viterbi(em, [L], trans, dur, K, center=False)
    assert vit["score"][0] == ref["best_score"]
    assert len(ref["optimal"]) >= 1
    lab, ss = ref["tie_broken"]
    assert np.array_equal(vit["labels"][0], lab)
    assert np.array_equal(vit["seg_start"][0], ss)


# ---------------------------------------------------------------- (ii) K = 1 is a linear-chain CRF
@pytest.mark.parametrize("center", [True, False])
def test_k1_equals_linear_chain_crf(center):
    rng = np.random.default_rng(21)
    L, C = 25, 4
    em, lengths, trans, dur = _rand_case(rng, 1, L, 1, C, scale=2.0, pstd=0.8)
    out = oracle.forward_backward(em, lengths, trans, dur, 1, center=center, threads=1)
    x = linear_chain.node_scores(em[0], L, dur[0], center=center)
    logZ, node, pair = linear_chain.forward_backward(x, trans)
    assert abs(out["logZ"][0] - logZ) < 1e-10 * max(1, abs(logZ))
    assert np.max(np.abs(out["pos_marg"][0] - node)) < 1e-12
    assert np.max(np.abs(out["grad_trans"] - pair)) < 1e-11
    assert np.max(np.abs(out["grad_dur"][0] - node.sum(axis=0))) < 1e-11
    # a K = 1 segment ending at boundary t is the label of position t-1
    assert np.max(np.abs(out["end_marg"][0, 1:] - node)) < 1e-12
    assert np.max(np.abs(out["start_marg"][0, :L] - node)) < 1e-12
    # every boundary is a segment boundary when K = 1
    assert np.allclose(out["end_marg"][0, 1:].sum(axis=1), 1.0, atol=1e-12)


def test_k1_viterbi_equals_textbook_viterbi():
    rng = np.random.default_rng(22)
    L, C = 30, 5
    em, lengths, trans, dur = _rand_case(rng, 1, L, 1, C, scale=2.0, pstd=0.8)
    vit = oracle.viterbi(em, lengths, trans, dur, 1)
    x = linear_chain.node_scores(em[0], L, dur[0])
    best, labels = linear_chain.viterbi(x, trans)
    assert abs(vit["score"][0] - best) < 1e-10
    assert np.array_equal(vit["labels"][0], labels)
    assert np.all(vit["seg_start"][0] == 1)


# ---------------------------------------------------------------- (iii) normalisation
def test_marginals_normalise():
    rng = np.random.default_rng(31)
    B, T, K, C = 3, 120, 12, 5
    em, _, trans, dur = _rand_case(rng, B, T, K, C, pstd=0.5)
    lengths = np.array([120, 77, 5], dtype=np.int32)
    out = oracle.forward_backward(em, lengths, trans, dur, K, threads=3)
    for b in range(B):
        L = int(lengths[b])
        assert np.allclose(out["pos_marg"][b, :L].sum(axis=1), 1.0, atol=1e-12)
        assert abs(out["end_marg"][b, L].sum() - 1.0) < 1e-12
        assert abs(out["start_marg"][b, 0].sum() - 1.0) < 1e-12
        # a boundary strictly inside the sequence both ends and starts a segment
        assert np.allclose(out["start_marg"][b, 1:L].sum(axis=1),
                           out["end_marg"][b, 1:L].sum(axis=1), atol=1e-12)
        assert np.all(out["end_marg"][b, :L + 1] <= 1 + 1e-12)
        assert np.all(out["start_marg"][b, :L + 1] >= 0)
        assert np.all(out["pos_marg"][b, L:] == 0)
        assert abs(out["logZ"][b] - out["logZ_beta"][b]) < 1e-10 * abs(out["logZ"][b])


# ---------------------------------------------------------------- (iv) finite differences
def _fd(f, x, idx, h=1e-5):
    xp = x.copy(); xp[idx] += h
    xm = x.copy(); xm[idx] -= h
    return (f(xp) - f(xm)) / (2 * h)


@pytest.mark.parametrize("center", [True, False])
def test_gradients_match_central_finite_differences(center):
    rng = np.random.default_rng(41)
    B, T, K, C = 2, 9, 4, 3
    em, _, trans, dur = _rand_case(rng, B, T, K, C, pstd=0.6)
    lengths = np.array([9, 6], dtype=np.int32)
    g = np.array([1.5, -0.75])
    out = oracle.forward_backward(em, lengths, trans, dur, K, center=center, grad_logZ=g, threads=1)

    def loss_e(x):
        return float(g @ oracle.log_partition(x, lengths, trans, dur, K, center=center, threads=1))

    def loss_t(x):
        return float(g @ oracle.log_partition(em, lengths, x, dur, K, center=center, threads=1))

    def loss_d(x):
        return float(g @ oracle.log_partition(em, lengths, trans, x, K, center=center, threads=1))

    for b in range(B):
        for u in range(T):
            for c in range(C):
                fd = _fd(loss_e, em, (b, u, c))
                if u >= lengths[b]:
                    assert abs(fd) < 1e-9 and out["grad_e"][b, u, c] == 0
                else:
                    assert abs(fd - out["grad_e"][b, u, c]) < 1e-6, (b, u, c)
    for i in range(C):
        for j in range(C):
            assert abs(_fd(loss_t, trans, (i, j)) - out["grad_trans"][i, j]) < 1e-6
    for k in range(K):
        for c in range(C):
            assert abs(_fd(loss_d, dur, (k, c)) - out["grad_dur"][k, c]) < 1e-6


# ---------------------------------------------------------------- closed forms
def _z_count(L, K, C):
    z = [1] + [0] * L
    for t in range(1, L + 1):
        z[t] = C * sum(z[t - k] for k in range(1, min(K, t) + 1))
    return z[L]


@pytest.mark.parametrize("L,K,C", [(10, 2, 1), (13, 5, 3), (6, 8, 4), (30, 7, 2), (9, 9, 3)])
def test_closed_form_partition_counts(L, K, C):
    # trans = 0, dur = 0 and constant emissions (centred to zero): every
    # segmentation scores 0 and Z counts them.
    em = np.full((1, L, C), 0.37)
    out = oracle.forward_backward(em, [L], np.zeros((C, C)), np.zeros((K, C)), K, threads=1)
    assert abs(out["logZ"][0] - math.log(_z_count(L, K, C))) < 1e-12 * max(1, L)
    if C == 1 and K == 2:  # Fibonacci: z[L] = F(L+1)
        fib = [0, 1]
        while len(fib) < L + 2:
            fib.append(fib[-1] + fib[-2])
        assert abs(out["logZ"][0] - math.log(fib[L + 1])) < 1e-12
    if K >= L:  # C (C + 1)^(L - 1)
        assert abs(out["logZ"][0] - (math.log(C) + (L - 1) * math.log(C + 1))) < 1e-12
    # label symmetry: every position marginal is exactly 1/C
    assert np.max(np.abs(out["pos_marg"][0] - 1.0 / C)) < 1e-12


def test_adaptive_duration_prior_identity():
    # Centering subtracts nu_c per position, i.e. k * nu_c per segment of
    # duration k: log Z with centering equals log Z without it once dur is
    # replaced by dur[k-1, c] - k * nu_c (explainer section 2, "Emission
    # Baseline Centering", the induced duration prior -nu * k).
    rng = np.random.default_rng(51)
    T, K, C = 40, 6, 4
    em, lengths, trans, dur = _rand_case(rng, 1, T, K, C, scale=1.0)
    em[0] += np.array([2.0, -1.0, 0.5, 3.0])  # label-dependent means
    lz_c = oracle.log_partition(em, lengths, trans, dur, K, center=True)[0]
    nu = em[0].mean(axis=0)
    dur2 = dur - np.arange(1, K + 1)[:, None] * nu[None, :]
    lz_u = oracle.log_partition(em, lengths, trans, dur2, K, center=False)[0]
    assert abs(lz_c - lz_u) < 1e-10 * max(1, abs(lz_c))


# ---------------------------------------------------------------- conservation laws
def test_mass_conservation_segment_count_and_centering_jacobian():
    rng = np.random.default_rng(61)
    B, T, K, C = 3, 60, 7, 4
    em, _, trans, dur = _rand_case(rng, B, T, K, C)
    lengths = np.array([60, 33, 1], dtype=np.int32)
    g = np.array([1.0, 2.0, -0.5])
    out = oracle.forward_backward(em, lengths, trans, dur, K, grad_logZ=g, threads=3)
    ks = np.arange(1, K + 1)[:, None]
    # every position is covered by exactly one segment
    assert abs((ks * out["grad_dur"]).sum() - float(g @ lengths)) < 1e-10
    # #segments - #transitions = 1 per (non-empty) sequence
    assert abs(out["grad_dur"].sum() - out["grad_trans"].sum() - g.sum()) < 1e-10
    # the centering Jacobian removes the per-label mean of the gradient
    for b in range(B):
        assert np.max(np.abs(out["grad_e"][b].sum(axis=0))) < 1e-10


def test_empty_sequence_has_logZ_zero():
    C, K = 3, 4
    em = np.zeros((2, 5, C))
    out = oracle.forward_backward(em, [0, 5], np.zeros((C, C)), np.zeros((K, C)), K, threads=1)
    assert out["logZ"][0] == 0.0
    assert np.all(out["pos_marg"][0] == 0)


def test_path_score_rejects_malformed_paths():
    rng = np.random.default_rng(71)
    T, K, C = 12, 3, 3
    em, lengths, trans, dur = _rand_case(rng, 1, T, K, C)
    vit = oracle.viterbi(em, lengths, trans, dur, K)
    ok = oracle.path_score(em, lengths, trans, dur, vit["labels"], vit["seg_start"], K)
    assert abs(ok[0] - vit["score"][0]) < 1e-12
    bad = vit["seg_start"].copy(); bad[0, 0] = 0
    assert math.isnan(oracle.path_score(em, lengths, trans, dur, vit["labels"], bad, K)[0])
    long = np.zeros_like(vit["seg_start"]); long[0, 0] = 1   # one 12-long segment > K
    lab = np.zeros_like(vit["labels"])
    assert math.isnan(oracle.path_score(em, lengths, trans, dur, lab, long, K)[0])


# ---------------------------------------------------------------- generator
def test_synthetic_generator_is_reproducible_and_shaped():
    a = synth.make("speech", B=4, T=100)
    b = synth.make("speech", B=4, T=100)
    for key in ("em", "lengths", "trans", "dur", "gold"):
        assert np.array_equal(a[key], b[key])
    assert a["em"].shape == (4, 100, 39) and a["em"].dtype == np.float32
    assert a["trans"].shape == (39, 39) and a["dur"].shape == (30, 39)
    assert np.all((a["lengths"] >= 1) & (a["lengths"] <= 100))
    t = synth.make("tiny")
    assert t["em"].shape == (1, 64, 4) and int(t["lengths"][0]) == 64 and t["K"] == 8
    g = synth.make("genomic", B=2, T=3000)
    assert np.all((g["gold"] >= 0) & (g["gold"] < 6))
    # the imbalanced label frequencies show up in the generating segmentation
    freq = np.bincount(g["gold"].ravel(), minlength=6) / g["gold"].size
    assert freq[0] > 0.4 and freq[5] < 0.1
    assert synth.checkpoint_interval(1_000_000, 200) == 14143
    assert synth.checkpoint_interval(800, 30) == 155


# ------------------------------------------------------- path score and loss
def _as_arrays(segs, L):
    lab = np.full(L, -1, dtype=np.int32)
    ss = np.zeros(L, dtype=np.uint8)
    for (s, t, c) in segs:
        lab[s:t] = c
        ss[s] = 1
    return lab, ss


@pytest.mark.parametrize("L,K,C,center,seed", BRUTE_CASES[:4])
def test_path_scores_of_all_segmentations_give_logZ_and_expected_counts(L, K, C, center, seed):
    # log Z is the log-sum-exp of the scores of every segmentation, and the
    # gradient of log Z is the posterior expectation of the path counts.
    rng = np.random.default_rng(300 + seed)
    em, lengths, trans, dur = _rand_case(rng, 1, L, K, C, pstd=0.7)
    segs = list(brute.segmentations(L, K, C))
    labs = np.stack([_as_arrays(sg, L)[0] for sg in segs])
    sss = np.stack([_as_arrays(sg, L)[1] for sg in segs])
    n = len(segs)
    emb = np.repeat(em, n, axis=0)
    scores = oracle.path_score(emb, np.full(n, L), trans, dur, labs, sss, K, center=center)
    m = scores.max()
    logZ = m + math.log(np.exp(scores - m).sum())
    fb = oracle.forward_backward(em, lengths, trans, dur, K, center=center, threads=1)
    assert abs(logZ - fb["logZ"][0]) < 1e-12 * max(1.0, abs(logZ))
    cnt = oracle.path_counts(np.full(n, L), labs, sss, C, K, center=center)
    assert cnt["valid"].all()
    p = np.exp(scores - logZ)
    assert np.max(np.abs(np.einsum("n,nij->ij", p, cnt["trans_count"]) - fb["grad_trans"])) < 1e-12
    assert np.max(np.abs(np.einsum("n,nij->ij", p, cnt["dur_count"]) - fb["grad_dur"])) < 1e-12
    assert np.max(np.abs(np.einsum("n,nuc->uc", p, cnt["grad_em"][:, :L])
                         - fb["grad_e"][0, :L])) < 1e-12


def _random_path(rng, L, K, C):
    lab = np.empty(L, dtype=np.int32)
    ss = np.zeros(L, dtype=np.uint8)
    pos = 0
    while pos < L:
        d = int(rng.integers(1, min(K, L - pos) + 1))
        lab[pos:pos + d] = rng.integers(0, C)
        ss[pos] = 1
        pos += d
    return lab, ss


@pytest.mark.parametrize("center", [True, False])
def test_path_counts_are_the_finite_differences_of_the_path_score(center):
    # The path score is linear in em, trans and dur, so a central difference
    # with a large step is exact up to rounding.
    rng = np.random.default_rng(311)
    T, K, C = 17, 5, 4
    em, lengths, trans, dur = _rand_case(rng, 1, T, K, C, lengths=[14])
    lab, ss = _random_path(rng, 14, K, C)
    labels = np.full((1, T), -1, dtype=np.int32); labels[0, :14] = lab
    seg = np.zeros((1, T), dtype=np.uint8); seg[0, :14] = ss
    cnt = oracle.path_counts(lengths, labels, seg, C, K, center=center)
    h = 0.25

    def sc(e=em, t=trans, d=dur):
        return oracle.path_score(e, lengths, t, d, labels, seg, K, center=center)[0]

    for (u, c) in [(0, 0), (3, 1), (7, 2), (13, 3), (10, 0)]:
        ep, emn = em.copy(), em.copy()
        ep[0, u, c] += h; emn[0, u, c] -= h
        assert abs((sc(e=ep) - sc(e=emn)) / (2 * h) - cnt["grad_em"][0, u, c]) < 1e-9
    for (a, c) in [(0, 1), (2, 3), (1, 1), (3, 0)]:
        tp, tm = trans.copy(), trans.copy()
        tp[a, c] += h; tm[a, c] -= h
        assert abs((sc(t=tp) - sc(t=tm)) / (2 * h) - cnt["trans_count"][0, a, c]) < 1e-9
    for (k, c) in [(0, 0), (1, 2), (4, 3), (2, 1)]:
        dp, dm = dur.copy(), dur.copy()
        dp[k, c] += h; dm[k, c] -= h
        assert abs((sc(d=dp) - sc(d=dm)) / (2 * h) - cnt["dur_count"][0, k, c]) < 1e-9
    # the rows past L_b carry no gradient
    assert np.all(cnt["grad_em"][0, 14:] == 0)
    # boundary projections enter the score linearly too
    ps = rng.normal(0, 1, size=(1, T, C))
    pe = rng.normal(0, 1, size=(1, T, C))

    def scp(a, z):
        return oracle.path_score(em, lengths, trans, dur, labels, seg, K, center=center,
                                 p_start=a, p_end=z)[0]

    for (u, c) in [(0, lab[0]), (5, 1), (13, 2), (9, 0)]:
        a, z = ps.copy(), ps.copy()
        a[0, u, c] += h; z[0, u, c] -= h
        assert abs((scp(a, pe) - scp(z, pe)) / (2 * h) - cnt["p_start_count"][0, u, c]) < 1e-9
        a, z = pe.copy(), pe.copy()
        a[0, u, c] += h; z[0, u, c] -= h
        assert abs((scp(ps, a) - scp(ps, z)) / (2 * h) - cnt["p_end_count"][0, u, c]) < 1e-9


def test_path_counts_reject_what_the_path_score_rejects():
    rng = np.random.default_rng(312)
    T, K, C = 12, 3, 3
    em, lengths, trans, dur = _rand_case(rng, 1, T, K, C)
    lab, ss = _random_path(rng, T, K, C)
    cases = []
    s0 = ss.copy(); s0[0] = 0; cases.append((lab, s0))            # no start at 0
    l1 = lab.copy(); l1[5] = C; cases.append((l1, ss))             # label out of range
    one = np.zeros(T, dtype=np.uint8); one[0] = 1                  # one segment longer than K
    cases.append((np.zeros(T, dtype=np.int32), one))
    for (a, s) in cases:
        out = oracle.path_counts(lengths, a[None], s[None], C, K)
        assert not out["valid"][0] and np.all(out["trans_count"] == 0)
        assert math.isnan(oracle.path_score(em, lengths, trans, dur, a[None], s[None], K)[0])
    ok = oracle.path_counts(lengths, lab[None], ss[None], C, K)
    assert ok["valid"][0]
    # segments - transitions = 1; durations sum to L; centred emission rows sum to 0
    assert ok["dur_count"].sum() - ok["trans_count"].sum() == 1
    assert (ok["dur_count"][0] * np.arange(1, K + 1)[:, None]).sum() == T
    assert np.max(np.abs(ok["grad_em"][0].sum(axis=1))) < 1e-12


def test_gold_segmentation_of_the_generator_is_a_valid_path():
    w = synth.make("genomic", B=2, T=3000)
    cnt = oracle.path_counts(w["lengths"], w["gold"], w["gold_start"], 6, w["K"])
    assert cnt["valid"].all()
    nll = (oracle.log_partition(w["em"], w["lengths"], w["trans"], w["dur"], w["K"])
           - oracle.path_score(w["em"], w["lengths"], w["trans"], w["dur"], w["gold"],
                               w["gold_start"], w["K"]))
    assert np.all(nll > 0)


# ------------------------------------------------------- boundary projections
@pytest.mark.parametrize("L,K,C,center,seed", BRUTE_CASES[:5])
def test_projections_bruteforce(L, K, C, center, seed):
    rng = np.random.default_rng(400 + seed)
    em, lengths, trans, dur = _rand_case(rng, 1, L, K, C, pstd=0.7)
    ps = rng.normal(0, 0.8, size=(1, L, C))
    pe = rng.normal(0, 0.8, size=(1, L, C))
    ref = brute.enumerate_all(em[0], L, trans, dur, center=center, ps=ps[0], pe=pe[0])
    out = oracle.forward_backward(em, lengths, trans, dur, K, center=center, threads=1,
                                  p_start=ps, p_end=pe)
    assert abs(out["logZ"][0] - ref["logZ"]) <= 1e-12 * max(1.0, abs(ref["logZ"]))
    assert abs(out["logZ_beta"][0] - ref["logZ"]) <= 1e-12 * max(1.0, abs(ref["logZ"]))
    for key in ("start_marg", "end_marg", "pos_marg"):
        assert np.max(np.abs(out[key][0][: ref[key].shape[0]] - ref[key])) < 1e-12, key
    assert np.max(np.abs(out["grad_dur"] - ref["grad_dur"])) < 1e-12
    assert np.max(np.abs(out["grad_trans"] - ref["grad_trans"])) < 1e-12
    vit = oracle.viterbi(em, lengths, trans, dur, K, center=center, threads=1, p_start=ps, p_end=pe)
    assert abs(vit["score"][0] - ref["best_score"]) < 1e-12
    assert any(np.array_equal(vit["labels"][0, :L], lab) and np.array_equal(vit["seg_start"][0, :L], ss)
               for lab, ss in ref["optimal"])
    rs = oracle.path_score(em, lengths, trans, dur, vit["labels"], vit["seg_start"], K,
                           center=center, p_start=ps, p_end=pe)
    assert abs(rs[0] - ref["best_score"]) < 1e-12


def test_projection_gradients_are_the_boundary_marginals():
    # d log Z / d p_start[s, c] = P(a label-c segment starts at s) and
    # d log Z / d p_end[u, c] = P(a label-c segment ends after position u).
    rng = np.random.default_rng(411)
    T, K, C = 15, 4, 3
    em, lengths, trans, dur = _rand_case(rng, 1, T, K, C, lengths=[13])
    ps = rng.normal(0, 0.5, size=(1, T, C))
    pe = rng.normal(0, 0.5, size=(1, T, C))
    out = oracle.forward_backward(em, lengths, trans, dur, K, threads=1, p_start=ps, p_end=pe)

    def lz(a, b_):
        return oracle.log_partition(em, lengths, trans, dur, K, threads=1, p_start=a, p_end=b_)[0]

    for (u, c) in [(0, 0), (4, 2), (12, 1), (7, 0)]:
        a, b_ = ps.copy(), ps.copy()
        a[0, u, c] += 1e-5; b_[0, u, c] -= 1e-5
        assert abs((lz(a, pe) - lz(b_, pe)) / 2e-5 - out["start_marg"][0, u, c]) < 1e-6
        a, b_ = pe.copy(), pe.copy()
        a[0, u, c] += 1e-5; b_[0, u, c] -= 1e-5
        assert abs((lz(ps, a) - lz(ps, b_)) / 2e-5 - out["end_marg"][0, u + 1, c]) < 1e-6
    # entries past the length change nothing
    a = ps.copy(); a[0, 13:] += 5.0
    assert lz(a, pe) == lz(ps, pe)


def test_label_constant_projections_are_a_duration_shift():
    # p_start[s, c] = a[c] and p_end[u, c] = z[c] for every position add
    # a[c] + z[c] to every label-c segment, which is dur[k-1, c] + a[c] + z[c].
    rng = np.random.default_rng(412)
    B, T, K, C = 2, 40, 6, 4
    em, lengths, trans, dur = _rand_case(rng, B, T, K, C, lengths=[40, 23])
    a = rng.normal(0, 1, size=C)
    z = rng.normal(0, 1, size=C)
    ps = np.broadcast_to(a, (B, T, C)).copy()
    pe = np.broadcast_to(z, (B, T, C)).copy()
    got = oracle.forward_backward(em, lengths, trans, dur, K, threads=1, p_start=ps, p_end=pe)
    ref = oracle.forward_backward(em, lengths, trans, dur + a + z, K, threads=1)
    assert np.max(np.abs(got["logZ"] - ref["logZ"])) < 1e-10
    assert np.max(np.abs(got["pos_marg"] - ref["pos_marg"])) < 1e-10
    assert np.max(np.abs(got["grad_dur"] - ref["grad_dur"])) < 1e-10
