"""bench.py's roofline arithmetic on the host: the per-edge work counts of
the hot-path table, the achieved / peak figures of a kernel entry, the
issued-operation counts, and that a stored ncu traffic figure is reported
only for the kernel sources it was measured on."""

import importlib.util
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
def test_per_edge_counts_add_up_to_three_exponentials_per_edge(bench, K, C):
    ring = bench.edge_ops_per_position("chain_exp_kernel", K, C)
    post = bench.edge_ops_per_position("posterior_kernel", K, C)
    assert ring == (2 * K * C * C, "mufu") and post == (K * C * C, "mufu")
    assert ring[0] + post[0] == 3 * K * C * C          # forward + backward, per edge
    assert bench.edge_ops_per_position("viterbi_pipe_kernel", K, C) == (2 * K * C * C, "fp32")
    assert bench.edge_ops_per_position("prefix_scan_kernel", K, C) is None
    assert bench.edges_of([300, 500], K, C) == 800 * K * C * C


def test_kernel_roofline_entry(bench):
    K, C, P, steps = 30, 39, 17580, 10
    info = {"launches": 10, "ms_per_launch": 0.5, "ms_total": 5.0}
    r = bench.kernel_roofline("chain_exp_kernel", info, K, C, P, steps, 148, 1965.0)
    ops = 2 * K * C * C * P
    achieved = ops / 0.5e-3
    peak = 148 * bench.MUFU_PER_SM_PER_CLK * 1965.0e6
    assert r["bound"] == "alu" and r["unit"] == "Gop/s"
    assert r["ops_per_launch"] == ops
    assert abs(r["achieved"] - achieved / 1e9) < 1e-6 * achieved / 1e9
    assert abs(r["peak"] - peak / 1e9) < 1e-6 * peak / 1e9
    assert abs(r["frac"] - achieved / peak) < 1e-12
    # two launches per step halve the work of one launch
    r2 = bench.kernel_roofline("chain_exp_kernel", dict(info, launches=20), K, C, P, steps, 148, 1965.0)
    assert r2["ops_per_launch"] == ops // 2
    # issued operations: the grouped fan-ins
    ri = bench.kernel_roofline("chain_exp_kernel", info, K, C, P, steps, 148, 1965.0, issued=True)
    assert ri["ops_per_launch"] == 2 * (K * C + 3 * C) * P
    # the fp32 unit for the decoder
    rv = bench.kernel_roofline("viterbi_pipe_kernel", info, K, C, P, steps, 148, 1965.0)
    assert abs(rv["peak"] - 148 * bench.FP32_PER_SM_PER_CLK * 1965.0e6 / 1e9) < 1e-6
    # HBM-bound kernels have no entry of this kind
    assert bench.kernel_roofline("prefix_scan_kernel", info, K, C, P, steps, 148, 1965.0) is None


def test_stored_traffic_only_for_the_sources_it_was_measured_on(bench, monkeypatch):
    import json
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        stored = json.load(f)
    monkeypatch.setattr(bench, "csrc_digest", lambda: stored["csrc_sha256"])
    k, v = next(iter(stored["kernels"].items()))
    assert bench.stored_traffic(k) == v
    monkeypatch.setattr(bench, "csrc_digest", lambda: "0" * 64)
    assert bench.stored_traffic(k) is None
