"""Runs the hot path through the bounds-checking debug build
(libsemicrf_b200_check.so, loaded with SEMICRF_LIBRARY=check) on cases that
reach every kernel and lane shape family, and prints one JSON line with the
status word after each call and the worst log Z error against the oracle.
Started by tests/test_gpu_bounds.py in a process of its own."""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import numpy as np
import torch

import oracle
from gpu_common import to_dev
from semi_markov_crf_b200 import semicrf, synth


def cases():
    return {
        "tiny": synth.make("tiny"),
        "speech_small": synth.make("speech", B=4, T=200),
        "traceback_in_stages": synth.make_custom(2, 900, 16, 64, seed=13, lengths=[900, 777]),
        "k_2000_genomic_like": synth.make_custom(
            2, 5000, 2000, 6, seed=41, lengths=[5000, 3333], dur_mean=50.0, amp=2.0,
            label_p=(0.6, 0.2, 0.1, 0.05, 0.03, 0.02)),
        "large_cluster": synth.make("large", B=2, T=300),
        "ragged_with_empty": synth.make_custom(4, 80, 9, 5, seed=9, lengths=[80, 0, 1, 57]),
    }


def main():
    assert semicrf.library_path.endswith("libsemicrf_b200_check.so"), semicrf.library_path
    out = {"library": os.path.basename(semicrf.library_path), "digest": semicrf.source_digest(),
           "cases": {}}
    ws0 = semicrf.Workspace(1, 8, 2, 2, 0, "cuda")
    out["selftest_status"] = semicrf.selftest_bounds(ws0)
    for name, c in cases().items():
        em, lengths, trans, dur = to_dev(c)
        K = c["dur"].shape[0]
        rec = {}
        for log_domain in (False, True):
            logZ, ws = semicrf.forward(em, lengths, trans, dur, log_domain=log_domain)
            semicrf.backward(ws, lengths, trans, dur, marginals=True,
                             segments=c["em"].shape[1] * K * c["em"].shape[2] <= 4_000_000)
            rec["fb_log" if log_domain else "fb_exp"] = semicrf.get_status(ws)
            ref = oracle.log_partition(c["em"], c["lengths"], c["trans"], c["dur"], K)
            err = np.abs(logZ.cpu().numpy() - ref) / np.maximum(1.0, np.abs(ref))
            rec["logZ_err_" + ("log" if log_domain else "exp")] = float(err.max())
        vws = semicrf.Workspace(*c["em"].shape[:2], c["em"].shape[2], K, 0, "cuda")
        sc, lab, seg = semicrf.viterbi(em, lengths, trans, dur, ws=vws)
        rec["viterbi"] = semicrf.get_status(vws)
        semicrf.path_score(em, lengths, trans, dur, lab, seg, ws=vws)
        rec["path_score"] = semicrf.get_status(vws)
        out["cases"][name] = rec
    torch.cuda.synchronize()
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
