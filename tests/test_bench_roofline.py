"""bench.py's roofline arithmetic on the host: the algorithmic work counts
of the factored recursion (never the nominal per-edge count), the achieved /
peak figures of a kernel entry, the HBM entries of the streaming kernels,
and that a stored ncu traffic figure is reported only for the kernel sources
and workload it was measured on."""

import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("K,C", [(30, 39), (200, 6), (64, 128)])
def test_counts_are_the_factored_fan_in(bench, K, C):
    ring = bench.algorithmic_ops_per_position("chain_exp_kernel", K, C)
    post = bench.algorithmic_ops_per_position("posterior_kernel", K, C)
    assert ring == (2 * K * C, "mufu") and post == (K * C, "mufu")
    assert bench.algorithmic_ops_per_position("chain_kernel", K, C) == ring
    assert bench.algorithmic_ops_per_position("segment_kernel", K, C) == (2 * K * C, "mufu")
    assert bench.algorithmic_ops_per_position("viterbi_pipe_kernel", K, C) == \
        (2 * (K * C + C * C), "fp32")
    # nothing is credited per edge: K C^2 appears only in the metric's unit
    for k in ("chain_exp_kernel", "posterior_kernel", "viterbi_pipe_kernel"):
        assert bench.algorithmic_ops_per_position(k, K, C)[0] < K * C * C or C <= 2
    assert bench.algorithmic_ops_per_position("prefix_scan_kernel", K, C) is None
    assert bench.edges_of([300, 500], K, C) == 800 * K * C * C


def test_kernel_roofline_entry(bench):
    K, C, P, steps = 64, 128, 80000, 10
    info = {"launches": 10, "ms_per_launch": 20.0, "ms_total": 200.0}
    r = bench.kernel_roofline("chain_exp_kernel", info, K, C, P, steps, 148, 1965.0)
    ops = 2 * K * C * P
    achieved = ops / 20e-3
    peak = 148 * bench.MUFU_PER_SM_PER_CLK * 1965.0e6
    assert r["bound"] == "alu" and r["unit"] == "Gop/s"
    assert r["ops_per_launch"] == ops
    assert abs(r["achieved"] - achieved / 1e9) < 1e-6 * achieved / 1e9
    assert abs(r["peak"] - peak / 1e9) < 1e-6 * peak / 1e9
    assert abs(r["frac"] - achieved / peak) < 1e-12
    assert r["frac"] < 1.0
    # two launches per step halve the work of one launch
    r2 = bench.kernel_roofline("chain_exp_kernel", dict(info, launches=20), K, C, P, steps, 148,
                               1965.0)
    assert r2["ops_per_launch"] == ops // 2
    # the fp32 unit for the decoder
    rv = bench.kernel_roofline("viterbi_pipe_kernel", info, K, C, P, steps, 148, 1965.0)
    assert abs(rv["peak"] - 148 * bench.FP32_PER_SM_PER_CLK * 1965.0e6 / 1e9) < 1e-6
    assert rv["ops_per_launch"] == 2 * (K * C + C * C) * P
    # streaming kernels: HBM entries against the measured copy bandwidth
    rp = bench.kernel_roofline("prefix_scan_kernel", dict(info, ms_per_launch=0.01), K, C, P,
                               steps, 148, 1965.0, hbm_gbs=6538.0)
    assert rp["bound"] == "hbm" and rp["bytes_per_launch"] == 12 * C * P
    assert abs(rp["achieved"] - 12 * C * P / 1e-5 / 1e9) < 1e-6 * rp["achieved"]
    assert bench.kernel_roofline("prefix_scan_kernel", info, K, C, P, steps, 148, 1965.0) is None
    assert bench.kernel_roofline("finalize_positions_kernel", info, K, C, P, steps, 148, 1965.0,
                                 hbm_gbs=6538.0) is None


def test_stored_traffic_only_for_the_sources_it_was_measured_on(bench, monkeypatch):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    with open(path) as f:
        stored = json.load(f)
    monkeypatch.setattr(bench, "csrc_digest", lambda: stored["csrc_sha256"])
    wl, kernels = next(iter(stored["workloads"].items()))
    k, v = next(iter(kernels.items()))
    assert bench.stored_traffic(k, wl) == v
    assert bench.stored_traffic(k, "no-such-workload") is None
    monkeypatch.setattr(bench, "csrc_digest", lambda: "0" * 64)
    assert bench.stored_traffic(k, wl) is None


def test_cpu_sample_is_a_prefix_of_the_workload(bench):
    from semi_markov_crf_b200 import synth
    w = synth.make("speech", B=4, T=100)
    em, lengths = bench.sample_of(w, 3, 40)
    assert em.shape == (3, 40, w["em"].shape[2])
    assert (em == w["em"][:3, :40]).all()
    assert list(lengths) == [min(int(x), 40) for x in w["lengths"][:3]]
