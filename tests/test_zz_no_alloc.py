"""GPU test of semicrf_forward_noalloc, the log Z entry point for callers that
cannot allocate device memory when they run (it keeps its scratch in a fixed
array inside the library instead of a caller workspace).

It is called through the C ABI and compared with semicrf_forward (the
workspace path) on the same inputs, on two calls in a row, at the log Z
tolerance the other parity tests use.  This file is named so that pytest
collects it last; it must pass alone in a fresh process and after the rest.
"""

import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from gpu_common import LOGZ_RTOL, to_dev
from semi_markov_crf_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc_logz(lib, em, lengths, trans, dur, out):
    B, T, C = em.shape
    K = dur.shape[0]
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.semicrf_forward_noalloc(
        ctypes.c_void_p(em.data_ptr()), ctypes.c_void_p(lengths.data_ptr()),
        ctypes.c_void_p(trans.data_ptr()), ctypes.c_void_p(dur.data_ptr()), B, T, C, K,
        ctypes.c_uint(0), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(stream))
    assert rc == 0, rc
    torch.cuda.synchronize()
    return out.cpu().numpy().copy()


def test_noalloc_forward_matches_workspace_forward_twice():
    from semi_markov_crf_b200 import semicrf
    lib = semicrf.lib
    first = synth.make("speech", B=6, T=240)
    second = synth.make("genomic", B=2, T=2500)
    for case in (first, second):
        em, lengths, trans, dur = to_dev(case)
        ref, _ = semicrf.forward(em, lengths, trans, dur)
        ref = ref.cpu().numpy()
        out = torch.full((em.shape[0],), float("nan"), dtype=torch.float64, device="cuda")
        a = _noalloc_logz(lib, em, lengths, trans, dur, out)
        out.fill_(float("nan"))
        b = _noalloc_logz(lib, em, lengths, trans, dur, out)
        for got in (a, b):
            err = np.abs(got - ref) / np.maximum(1.0, np.abs(ref))
            assert np.all(err <= LOGZ_RTOL), err.max()


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
