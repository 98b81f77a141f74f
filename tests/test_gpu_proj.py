"""GPU parity with boundary projections (the semicrf_*_proj entry points)
against the float64 oracle: log Z, marginals and every gradient (the
projection gradients included), decoding, the path score and its counts,
and that a plain call after a projection call on the same workspace is a
plain call again.  Every forward-backward case runs twice: on the default
path (exponential-domain rings, the kept-row posterior pass and the
pipelined decoder, which carry the projection terms) and with the rings
forced into the log domain.  Tolerances as in gpu_common."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import (COUNT_RTOL, MARG_ATOL, assert_fb_close, assert_viterbi_ok, max_abs,
                        to_dev)
from semi_markov_crf_b200 import synth

pytestmark = pytest.mark.gpu

CASES = {
    "speech_small": lambda: synth.make("speech", B=6, T=160),
    "genomic_small": lambda: synth.make("genomic", B=2, T=3000),
    "large_small": lambda: synth.make("large", B=2, T=160),
    "mixed_with_empty": lambda: synth.make_custom(4, 80, 9, 5, seed=9, lengths=[80, 0, 1, 57]),
    "k_equals_1": lambda: synth.make_custom(2, 90, 1, 7, seed=7, lengths=[90, 41]),
    "k_700": lambda: synth.make_custom(2, 1500, 700, 4, seed=42, lengths=[1500, 1100],
                                       dur_mean=100.0, amp=2.0),
}


def _proj(case, seed, scale=0.5):
    rng = np.random.default_rng(seed)
    B, T, C = case["em"].shape
    ps = (scale * rng.standard_normal((B, T, C))).astype(np.float32)
    pe = (scale * rng.standard_normal((B, T, C))).astype(np.float32)
    return ps, pe


def _masked(x, lengths):
    x = np.array(x, dtype=np.float64)
    for b, L in enumerate(lengths):
        x[b, int(L):] = 0.0
    return x


@pytest.mark.parametrize("log_domain", [False, True])
@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_backward_with_projections_match_oracle(name, log_domain):
    from semi_markov_crf_b200 import semicrf
    case = CASES[name]()
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    ps, pe = _proj(case, 51)
    g = np.linspace(0.5, 1.5, B)
    em, lengths, trans, dur = to_dev(case)
    tp, te = torch.from_numpy(ps).cuda(), torch.from_numpy(pe).cuda()
    logZ, ws = semicrf.forward(em, lengths, trans, dur, p_start=tp, p_end=te,
                               log_domain=log_domain)
    out = semicrf.backward(ws, lengths, trans, dur, marginals=True,
                           grad_logZ=torch.as_tensor(g, device="cuda"))
    assert semicrf.get_status(ws) == 0
    dom = semicrf.ring_domains(ws)
    nonempty = [b for b in range(B) if case["lengths"][b] > 0]
    want = 2 if log_domain else 1
    assert all(dom[b] == want and dom[B + b] == want for b in nonempty), dom
    got = {k: v.cpu().numpy() for k, v in out.items()}
    got["logZ"] = logZ.cpu().numpy()
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"], K,
                                  grad_logZ=g, p_start=ps, p_end=pe)
    assert_fb_close(got, ref, case["lengths"], name)
    # projection gradients: g times the start marginal at u and the end
    # marginal after u
    eps = _masked(g[:, None, None] * ref["start_marg"][:, :T], case["lengths"])
    epe = _masked(g[:, None, None] * ref["end_marg"][:, 1:], case["lengths"])
    assert max_abs(got["grad_p_start"], eps) <= MARG_ATOL
    assert max_abs(got["grad_p_end"], epe) <= MARG_ATOL
    # the same without the caller's marginal buffers
    logZ2, ws2 = semicrf.forward(em, lengths, trans, dur, p_start=tp, p_end=te,
                                 log_domain=log_domain)
    out2 = semicrf.backward(ws2, lengths, trans, dur, grad_logZ=torch.as_tensor(g, device="cuda"))
    assert torch.equal(out2["grad_p_start"], out["grad_p_start"])
    assert torch.equal(out2["grad_p_end"], out["grad_p_end"])


@pytest.mark.parametrize("name", ["speech_small", "genomic_small", "k_700", "mixed_with_empty"])
def test_viterbi_and_path_score_with_projections_match_oracle(name):
    from semi_markov_crf_b200 import semicrf
    case = CASES[name]()
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    ps, pe = _proj(case, 52)
    em, lengths, trans, dur = to_dev(case)
    tp, te = torch.from_numpy(ps).cuda(), torch.from_numpy(pe).cuda()
    score, labels, seg = semicrf.viterbi(em, lengths, trans, dur, p_start=tp, p_end=te)
    got = dict(score=score.cpu().numpy(), labels=labels.cpu().numpy(), seg_start=seg.cpu().numpy())
    ref = oracle.viterbi(case["em"], case["lengths"], case["trans"], case["dur"], K,
                         p_start=ps, p_end=pe)
    assert_viterbi_ok(got, ref, case, label=name, p_start=ps, p_end=pe)
    # path score of the gold (or decoded) path, with counts for every parameter
    if np.any(case["gold"] >= 0):
        lab, ss = case["gold"], case["gold_start"]
    else:
        lab, ss = ref["labels"], ref["seg_start"]
    g = np.linspace(-1.0, 1.0, B)
    grads = {k: torch.zeros(s, dtype=torch.float32, device="cuda") for k, s in (
        ("grad_em", (B, T, C)), ("grad_trans", (C, C)), ("grad_dur", (K, C)),
        ("grad_p_start", (B, T, C)), ("grad_p_end", (B, T, C)))}
    sc = semicrf.path_score(em, lengths, trans, dur, torch.from_numpy(lab).cuda(),
                            torch.from_numpy(ss).cuda(), grad_score=torch.as_tensor(g, device="cuda"),
                            grads=grads, p_start=tp, p_end=te).cpu().numpy()
    rs = oracle.path_score(case["em"], case["lengths"], case["trans"], case["dur"], lab, ss, K,
                           p_start=ps, p_end=pe)
    fin = np.isfinite(rs)
    assert np.array_equal(np.isfinite(sc), fin)
    assert np.all(np.abs(sc[fin] - rs[fin]) <= 1e-9 * np.maximum(1.0, np.abs(rs[fin])))
    cnt = oracle.path_counts(case["lengths"], lab, ss, C, K)
    w = g * cnt["valid"]
    assert max_abs(grads["grad_em"].cpu().numpy(), cnt["grad_em"] * w[:, None, None]) <= MARG_ATOL
    assert max_abs(grads["grad_p_start"].cpu().numpy(), cnt["p_start_count"] * w[:, None, None]) <= MARG_ATOL
    assert max_abs(grads["grad_p_end"].cpu().numpy(), cnt["p_end_count"] * w[:, None, None]) <= MARG_ATOL
    for key, ck in (("grad_trans", "trans_count"), ("grad_dur", "dur_count")):
        r = np.einsum("b,bij->ij", w, cnt[ck])
        d = np.abs(grads[key].cpu().numpy().astype(np.float64) - r)
        assert np.max(d / np.maximum(1.0, np.abs(r))) <= COUNT_RTOL, key


@pytest.mark.parametrize("log_domain", [False, True])
def test_zero_projections_equal_the_plain_run(log_domain):
    from semi_markov_crf_b200 import semicrf
    case = CASES["speech_small"]()
    B, T, C = case["em"].shape
    em, lengths, trans, dur = to_dev(case)
    z = torch.zeros((B, T, C), dtype=torch.float32, device="cuda")
    lz_p, ws_p = semicrf.forward(em, lengths, trans, dur, p_start=z, p_end=z, log_domain=log_domain)
    out_p = semicrf.backward(ws_p, lengths, trans, dur, marginals=True)
    lz, ws = semicrf.forward(em, lengths, trans, dur, log_domain=log_domain)
    out = semicrf.backward(ws, lengths, trans, dur, marginals=True)
    assert torch.equal(lz_p, lz)
    for k in ("grad_em", "grad_trans", "grad_dur", "pos_marg", "start_marg", "end_marg"):
        assert torch.equal(out_p[k], out[k]), k
    # decoding: zero projections change nothing either
    a = semicrf.viterbi(em, lengths, trans, dur, p_start=z, p_end=z)
    b = semicrf.viterbi(em, lengths, trans, dur)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_loud_projections_leave_the_exponential_domain():
    """Projections of several hundred nats per position exceed the
    exponential-domain kernels' exponent head-room: those sequences run in
    the log domain and still match the oracle."""
    from semi_markov_crf_b200 import semicrf
    case = synth.make("speech", B=3, T=60, seed=23)
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    ps, pe = _proj(case, 56, scale=30.0)
    em, lengths, trans, dur = to_dev(case)
    tp, te = torch.from_numpy(ps).cuda(), torch.from_numpy(pe).cuda()
    logZ, ws = semicrf.forward(em, lengths, trans, dur, p_start=tp, p_end=te)
    out = semicrf.backward(ws, lengths, trans, dur, marginals=True)
    assert semicrf.get_status(ws) == 0
    assert all(v == 2 for v in semicrf.ring_domains(ws))
    got = {k: v.cpu().numpy() for k, v in out.items()}
    got["logZ"] = logZ.cpu().numpy()
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"], K,
                                  p_start=ps, p_end=pe)
    err = np.abs(got["logZ"] - ref["logZ"]) / np.maximum(1.0, np.abs(ref["logZ"]))
    assert np.all(err <= 1e-5), err


def test_plain_call_after_a_projection_call_clears_the_switch():
    from semi_markov_crf_b200 import semicrf
    case = CASES["speech_small"]()
    em, lengths, trans, dur = to_dev(case)
    ps, pe = _proj(case, 53, scale=2.0)
    lz0, ws = semicrf.forward(em, lengths, trans, dur)
    ref = {k: v.clone() for k, v in semicrf.backward(ws, lengths, trans, dur, marginals=True).items()}
    semicrf.forward(em, lengths, trans, dur, ws=ws, p_start=torch.from_numpy(ps).cuda(),
                    p_end=torch.from_numpy(pe).cuda())
    semicrf.backward(ws, lengths, trans, dur)
    lz1, ws = semicrf.forward(em, lengths, trans, dur, ws=ws)
    got = semicrf.backward(ws, lengths, trans, dur, marginals=True)
    assert torch.equal(lz0, lz1)
    for k in ref:
        assert torch.equal(ref[k], got[k]), k


def test_projections_without_centering_and_forward_only():
    from semi_markov_crf_b200 import semicrf
    case = CASES["speech_small"]()
    B, T, C = case["em"].shape
    K = case["dur"].shape[0]
    ps, pe = _proj(case, 54)
    g = np.linspace(-1.0, 2.0, B)
    em, lengths, trans, dur = to_dev(case)
    tp, te = torch.from_numpy(ps).cuda(), torch.from_numpy(pe).cuda()
    gt = torch.as_tensor(g, device="cuda")
    ref = oracle.forward_backward(case["em"], case["lengths"], case["trans"], case["dur"], K,
                                  center=False, grad_logZ=g, p_start=ps, p_end=pe)
    for fo in (False, True):
        logZ, ws = semicrf.forward(em, lengths, trans, dur, center=False, forward_only=fo,
                                   p_start=tp, p_end=te)
        out = semicrf.backward(ws, lengths, trans, dur, marginals=True, grad_logZ=gt)
        assert semicrf.get_status(ws) == 0
        got = {k: v.cpu().numpy() for k, v in out.items()}
        got["logZ"] = logZ.cpu().numpy()
        assert_fb_close(got, ref, case["lengths"], f"no_center forward_only={fo}")
        eps = _masked(g[:, None, None] * ref["start_marg"][:, :T], case["lengths"])
        assert max_abs(got["grad_p_start"], eps) <= MARG_ATOL


def test_projections_with_a_bad_length():
    from semi_markov_crf_b200 import semicrf
    case = synth.make_custom(3, 40, 5, 3, seed=3, lengths=[40, 20, 10])
    ps, pe = _proj(case, 55)
    case["lengths"] = np.array([40, 41, 10], dtype=np.int32)
    em, lengths, trans, dur = to_dev(case)
    logZ, ws = semicrf.forward(em, lengths, trans, dur, p_start=torch.from_numpy(ps).cuda(),
                               p_end=torch.from_numpy(pe).cuda())
    out = semicrf.backward(ws, lengths, trans, dur)
    assert semicrf.get_status(ws) == 6
    lz = logZ.cpu().numpy()
    assert np.isnan(lz[1]) and np.isfinite(lz[0]) and np.isfinite(lz[2])
    assert np.all(out["grad_p_start"][1].cpu().numpy() == 0)
    assert np.all(out["grad_p_end"][1].cpu().numpy() == 0)
