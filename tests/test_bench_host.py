"""Host-side logic of bench.py (no GPU): the traffic records' scaling and gating, the
phase tables printed by --trace, and the config dict both arms print."""
import argparse

import numpy as np

import bench
import workload as wl


def test_union_traffic_scales_with_table_lengths_and_is_gated():
    cfg = wl.CONFIGS[4]
    t = bench.UNION_TRAFFIC
    rows = [[3000] * 64, [3400] * 64]
    want = sum(t["fixed_per_layer"] * 64 + t["per_neuron"] * sum(r) for r in rows) / 2
    got = bench.union_traffic(cfg, 32, None, False, rows)
    if bench.decode_sources_sha256(bench.UNION_SOURCES) == t["sha256"]:
        assert abs(got - want) <= 1e-6 * want
        # 1.5% above the algorithmic bytes at the capture's table length, as captured
        alg = 2 * (cfg.H * cfg.d + cfg.n * cfg.H) + 5639.17 * (4 * cfg.d + 6)
        assert 1.0 < (t["fixed_per_layer"] + 5639.17 * t["per_neuron"]) / alg < 1.05
    else:
        assert got is None                       # sources changed since the capture: no claim
    # another workload, batch, rate or look-ahead: no claim either
    assert bench.union_traffic(wl.CONFIGS[2], 32, None, False, rows) is None
    assert bench.union_traffic(cfg, 16, None, False, rows) is None
    assert bench.union_traffic(cfg, 32, 0.05, False, rows) is None
    assert bench.union_traffic(cfg, 32, None, True, rows) is None


def test_decode_traffic_scales_with_layers_and_is_gated():
    cfg = wl.CONFIGS[1]
    t = bench.DECODE_TRAFFIC
    got = bench.decode_traffic(cfg, 8, 1, None, False)
    if bench.decode_sources_sha256() == t["sha256"]:
        assert abs(got - 8 * t["bytes_per_layer"]) < 1.0
    else:
        assert got is None
    assert bench.decode_traffic(cfg, 8, 2, None, False) is None
    assert bench.decode_traffic(cfg, 8, 1, None, True) is None


def test_union_phase_table_reads_the_stamp_layout():
    G, L = 4, 2
    nl = 4 * L
    t = np.zeros((nl, G, 8), dtype=np.int64)
    for i in range(nl):
        base = 1_000_000 * (i + 1)
        t[i, :, 0] = base + np.arange(G) * 10
        t[i, :, 1] = base + 5_000              # 5 us wait
        t[i, :, 2] = base + 6_000
        t[i, :, 3] = base + 26_000             # 20 us streaming
        t[i, :, 4] = base + 27_000
        t[i, :, 5] = base + 30_000 + np.arange(G) * 1_000   # tail to the slowest CTA: 6 us
    table = bench.union_phase_table(t.ravel(), nl, G)
    lines = table.splitlines()
    assert len(lines) == 5
    for line in lines[1:]:
        wait, stream, tail = (float(v) for v in line.split()[-3:])
        assert (wait, stream, tail) == (5.0, 20.0, 6.0)


def test_fused_phase_table_skips_layer_zero_and_reports_the_period():
    G, L, M = 3, 4, 16
    t = np.zeros((G, L, M), dtype=np.int64)
    for l in range(L):
        for m in range(12):
            t[:, l, m] = 10_000_000 + l * 25_000 + m * 2_000 + np.arange(G) * 100
    lines = bench.fused_phase_table(t.ravel(), G, L, M).splitlines()
    assert lines[-1].split()[-1] == "25.0"
    first = dict((ln.rsplit(None, 2)[0].strip(), float(ln.split()[-2])) for ln in lines[1:-1])
    assert first["input formed"] == 0.1 and first["hidden layer done"] == 4.1


def test_both_arms_print_the_same_config():
    ap = argparse.Namespace(rate=None, lookahead=False, l2_hot_rows=0, union_stack=2, flush_l2=False)
    cfg = wl.CONFIGS[4]
    a = bench.config_dict(cfg, ap, 1)
    b = bench.config_dict(cfg, ap, 1)
    assert a == b
    assert a["workload"] == cfg.name and a["batch"] == 32 and a["global_batch"] == 32
