"""The bounds-checking debug build (libsemicrf_b200_check.so, built with
-DSEMICRF_BOUNDS_CHECK) stands in for a race and bounds checker: every
guarded access of the kernels -- TMA tile sources and row pointers into the
staged tiles, ring windows and slots, label-vector stores (cluster peers
included), kept rows, the traceback's staging and marks, the posterior
pass's tiles -- records the first failing site in the status word instead of
making the access.  A child process loads that build and runs forward,
backward (with segment marginals where they fit), Viterbi and the path
score on cases that reach every kernel and lane-shape family; every status
must be 0 and log Z must still match the oracle.  The self-test makes one
deliberately out-of-range guarded store and must see its site recorded."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CHECK_LIB = os.path.join(os.path.dirname(HERE), "semi_markov_crf_b200", "libsemicrf_b200_check.so")


def test_bounds_checked_build_runs_clean():
    if not os.path.exists(CHECK_LIB):
        pytest.fail("libsemicrf_b200_check.so is not built (python -m semi_markov_crf_b200.build "
                    "--bounds-check)")
    env = dict(os.environ, SEMICRF_LIBRARY="check")
    res = subprocess.run([sys.executable, os.path.join(HERE, "bounds_child.py")], env=env,
                         capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    out = json.loads(res.stdout.strip().splitlines()[-1])
    print(json.dumps(out))
    assert out["library"] == "libsemicrf_b200_check.so"
    # the debug build is of the current sources (a stale one would test old code)
    from semi_markov_crf_b200.build import source_digest
    assert out["digest"] == source_digest(), "libsemicrf_b200_check.so is stale: rebuild it"
    st = out["selftest_status"]
    assert st & 0xff == 7 and st >> 8 == 13, st   # SEMICRF_ERR_BOUNDS at the self-test's site
    for name, rec in out["cases"].items():
        for key, v in rec.items():
            if key.startswith("logZ_err"):
                assert v <= 1e-5, (name, key, v)
            else:
                assert v == 0, (name, key, v)
