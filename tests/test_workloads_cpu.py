"""The seeded input generator and the CPU legs of bench.py (CPU only)."""
import io
import json
import sys
from contextlib import redirect_stdout

import numpy as np

import workloads


def test_topk_rule_against_sorted_with_ties():
    rng = np.random.default_rng(3)
    for E, K in [(8, 3), (16, 16), (32, 5), (7, 1)]:
        lg = rng.integers(-3, 3, size=(200, E)).astype(np.float32)   # many exact ties
        got = workloads._topk_rows(lg, K)
        for i in range(lg.shape[0]):
            want = sorted(range(E), key=lambda e: (-lg[i, e], e))[:K]
            assert list(got[i]) == want


def test_routing_is_seeded_and_normalised():
    wl = workloads.reduced(workloads.WORKLOADS["kimi_r64_e896_k16"], S=9)
    a_idx, a_w = workloads.routing(wl, seed=0)
    b_idx, b_w = workloads.routing(wl, seed=0)
    c_idx, _ = workloads.routing(wl, seed=1)
    assert np.array_equal(a_idx, b_idx) and np.array_equal(a_w, b_w)
    assert not np.array_equal(a_idx, c_idx)
    assert a_idx.shape == (wl.N, wl.K) and a_idx.dtype == np.int32
    assert np.all((a_idx >= 0) & (a_idx < wl.E))
    assert np.all(np.sort(a_idx, axis=1)[:, 1:] != np.sort(a_idx, axis=1)[:, :-1])  # distinct
    assert np.allclose(a_w.sum(axis=1), 1.0, atol=1e-6) and np.all(a_w > 0)


def test_adversarial_and_hot_recipes():
    wl = workloads.reduced(workloads.WORKLOADS["skew_r32_adversarial"], S=5)
    idx, w = workloads.routing(wl)
    assert np.array_equal(np.sort(idx, axis=1), np.tile(np.arange(wl.K), (wl.N, 1)))
    wl3 = workloads.reduced(workloads.WORKLOADS["r16_e256_h7168"], S=200)
    idx3, w3 = workloads.routing(wl3)
    hot = np.random.default_rng(0).choice(wl3.E, 8, replace=False)
    share = np.isin(idx3, hot).mean()
    assert share > 8 / wl3.E * 2          # the +2.0 logit bias makes the 8 chosen experts hot
    assert np.allclose(w3.sum(axis=1), 1.0, atol=1e-6)


def test_roundrobin_is_balanced():
    idx, w = workloads.roundrobin_routing(4, 6, 8, 4)
    assert np.array_equal(np.bincount(idx.reshape(-1), minlength=8), np.full(8, 12))
    assert np.allclose(w, 0.25)


def test_reference_arm_prints_one_line(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "0")
    args = type("A", (), dict(workload="tiny_r4_e16", steps=1, warmup=0, gpus=1))()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["metric"] == bench.METRIC
    # the same config keys and values as the GPU arm's line
    assert line["config"] == bench.bench_config(workloads.WORKLOADS["tiny_r4_e16"], 1)
    # the oracle runs through the plan's own slots, not sequential ones
    assert "via the plan's src_pair" in line["cpu_baseline"]["sample"]
    assert "via the plan's slots" in line["cpu_baseline"]["sample"]


def test_roofline_traffic_follows_the_kernel_source(monkeypatch):
    """bench reports the committed DRAM traffic of a kernel only while its
    source is the one the counters were taken on, and reads the measured
    copy peak from MEASURED_PEAKS.json when present."""
    import os

    import bench
    rows = [ln.split() for ln in open(os.path.join(bench.ROOT, "profiles", "dram_traffic.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert {r[0] for r in rows} >= {"plan", "dispatch", "combine", "reduce"}
    for name, workload, nbytes, sha, *_ in rows:
        monkeypatch.setattr(bench, "kernel_sha", lambda n, sha=sha: sha)
        assert bench.dram_traffic(name, workload) == float(nbytes)        # same source
        assert bench.dram_traffic(name, "kimi_r64_e896_k16") is None       # no capture there
        monkeypatch.setattr(bench, "kernel_sha", lambda n: "000000000000")
        assert bench.dram_traffic(name, workload) is None                  # kernel changed
    peak, kind = bench.measured_peak()
    assert peak > 1000 and kind in ("measured", "fallback")


def test_end_to_end_host_sources_fit_the_budget():
    """The end-to-end leg pins its large inputs whole when they fit the host
    budget, else their first rows (in proportion), and the row copy fills
    every device row from that source."""
    import torch

    import bench
    y = torch.arange(40, dtype=torch.float32).reshape(10, 4)
    G = torch.arange(12, dtype=torch.float32).reshape(6, 2)
    hy, hG, d = bench.pinned_sources({"y": y, "G": G}, 10 ** 9, pin=False)
    assert d == {"y": "pinned whole", "G": "pinned whole"} and torch.equal(hy, y) and torch.equal(hG, G)
    hy, hG, d = bench.pinned_sources({"y": y, "G": None}, 60, pin=False)   # 160 B > 60 B
    assert hG is None and hy.shape == (3, 4) and torch.equal(hy, y[:3])
    assert d == {"y": "first 3 of 10 rows pinned, copied 4 times per step"}
    dst = torch.empty(10, 4)
    bench.copy_rows(dst, hy)
    assert torch.equal(dst, y[torch.tensor([0, 1, 2, 0, 1, 2, 0, 1, 2, 0])])
    assert bench.host_pin_budget(8) > 0
