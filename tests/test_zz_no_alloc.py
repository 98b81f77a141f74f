"""GPU test of semicrf_forward_noalloc, the log Z entry point for callers that
cannot allocate device memory when they run (it keeps its scratch in a fixed
array inside the library instead of a caller workspace).

It is called through the C ABI and compared with the float64 oracle and
with semicrf_forward (the workspace path) on the same inputs, on two calls in
a row, at the log Z tolerance the other parity tests use, in both ring
domains; a length outside [0, T] gives NaN for that sequence only.  This file
is named so that pytest collects it last; it must pass alone in a fresh
process and after the rest.
"""

import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from gpu_common import LOGZ_RTOL, to_dev
from semi_markov_crf_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc_logz(lib, em, lengths, trans, dur, out, flags=0):
    B, T, C = em.shape
    K = dur.shape[0]
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.semicrf_forward_noalloc(
        ctypes.c_void_p(em.data_ptr()), ctypes.c_void_p(lengths.data_ptr()),
        ctypes.c_void_p(trans.data_ptr()), ctypes.c_void_p(dur.data_ptr()), B, T, C, K,
        ctypes.c_uint(flags), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(stream))
    assert rc == 0, rc
    torch.cuda.synchronize()
    return out.cpu().numpy().copy()


@pytest.mark.parametrize("log_domain", [False, True])
def test_noalloc_forward_matches_oracle_and_workspace_forward_twice(log_domain):
    from semi_markov_crf_b200 import semicrf
    lib = semicrf.lib
    flags = semicrf.FLAG_LOG_DOMAIN if log_domain else 0
    cases = (synth.make("tiny"), synth.make("speech", B=6, T=240),
             synth.make("genomic", B=2, T=2500), synth.make("large", B=2, T=150))
    for case in cases:
        K = case["dur"].shape[0]
        lz_oracle = oracle.log_partition(case["em"], case["lengths"], case["trans"], case["dur"], K)
        em, lengths, trans, dur = to_dev(case)
        ref, _ = semicrf.forward(em, lengths, trans, dur, log_domain=log_domain)
        ref = ref.cpu().numpy()
        out = torch.full((em.shape[0],), float("nan"), dtype=torch.float64, device="cuda")
        a = _noalloc_logz(lib, em, lengths, trans, dur, out, flags)
        out.fill_(float("nan"))
        b = _noalloc_logz(lib, em, lengths, trans, dur, out, flags)
        for got in (a, b):
            for want in (lz_oracle, ref):
                err = np.abs(got - want) / np.maximum(1.0, np.abs(want))
                assert np.all(err <= LOGZ_RTOL), err.max()


def test_noalloc_bad_length_gives_nan_for_that_sequence_only():
    from semi_markov_crf_b200 import semicrf
    case = synth.make("speech", B=3, T=64)
    em, lengths, trans, dur = to_dev(case)
    lengths[1] = 65        # > T
    lengths[2] = -1
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    got = _noalloc_logz(semicrf.lib, em, lengths, trans, dur, out)
    assert np.isnan(got[1]) and np.isnan(got[2]) and np.isfinite(got[0])
    one = dict(case, em=case["em"][:1], lengths=case["lengths"][:1])
    want = oracle.log_partition(one["em"], one["lengths"], case["trans"], case["dur"],
                                case["dur"].shape[0])
    assert abs(got[0] - want[0]) <= LOGZ_RTOL * max(1.0, abs(want[0]))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from semi_markov_crf_b200 import semicrf
    # about 8 * B * (T+1) * C bytes of prefix sums alone: far above 32 MiB
    B, T, C, K = 8, 200_000, 8, 16
    em = torch.zeros((B, T, C), dtype=torch.float32, device="cuda")
    lengths = torch.full((B,), T, dtype=torch.int32, device="cuda")
    trans = torch.zeros((C, C), dtype=torch.float32, device="cuda")
    dur = torch.zeros((K, C), dtype=torch.float32, device="cuda")
    with pytest.raises(semicrf.SemiCRFError) as info:
        semicrf.forward_noalloc(em, lengths, trans, dur)
    assert info.value.code == 2
