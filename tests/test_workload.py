"""The seeded input generator: known-answer vectors, exact rounding, and the
rate calibration the workload recipe promises."""
import math

import numpy as np
import pytest

import oracle as O
import workload as wl


def test_philox_known_answers():
    # Known-answer vectors published with Random123 for Philox4x32-10.
    assert wl.philox4x32_10([0, 0, 0, 0], [0, 0]) == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    assert wl.philox4x32_10([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2) == [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]
    assert wl.philox4x32_10([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0]) == \
        [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]


def test_normals_moments_and_counter_addressing():
    z = wl.normals(wl.stream_id(wl.T_X, 3, 7), 400_000)
    assert abs(z.mean()) < 4 / math.sqrt(4e5) and abs(z.std() - 1) < 0.01
    # element e is addressable on its own
    part = wl.normals(wl.stream_id(wl.T_X, 3, 7), 1000, e0=12345)
    assert np.array_equal(part, z[12345:13345])
    rows = np.array([5, 0, 9])
    full = wl.fill(wl.stream_id(wl.T_W1, 2), 10 * 16, 0.25, 0).reshape(10, 16)
    assert np.array_equal(wl.fill_rows(wl.stream_id(wl.T_W1, 2), 16, rows, 0.25, 0), full[rows])


def test_f16_rounding_matches_numpy():
    r = np.random.default_rng(0)
    v = np.concatenate([r.standard_normal(200_000) * 10.0 ** r.integers(-9, 5, 200_000),
                        np.array([65504.0, 65519.99, 65520.0, 1e-8, 2.0 ** -25, 2.0 ** -24 * 1.5, 0.0, -0.0])])
    # ties: halfway between adjacent binary16 values
    h = r.integers(1, 0x7BFF, 5000).astype(np.uint16).view(np.float16).astype(np.float64)
    h2 = (h.astype(np.float16).view(np.uint16) + 1).view(np.float16).astype(np.float64)
    v = np.concatenate([v, (h + h2) / 2])
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(wl.round_to(v, 0), want)


def test_bf16_rounding_is_nearest_even():
    r = np.random.default_rng(1)
    v = r.standard_normal(100_000) * 10.0 ** r.integers(-30, 30, 100_000)
    bits = wl.round_to(v, 1)
    got = wl.widen(bits, 1)
    # neighbours of the result on the bf16 grid
    up = wl.widen((bits.astype(np.int32) + 1).astype(np.uint16), 1)
    dn = wl.widen((bits.astype(np.int32) - 1).astype(np.uint16), 1)
    err = np.abs(got - v)
    assert np.all(err <= np.abs(up - v)) and np.all(err <= np.abs(dn - v))
    # exact ties go to the even pattern
    base = r.integers(0x3C00, 0x4400, 2000).astype(np.uint16)
    lo, hi = wl.widen(base, 1), wl.widen(base + 1, 1)
    tb = wl.round_to((lo + hi) / 2, 1)
    assert np.all(tb % 2 == 0)


def test_widen_is_exact_inverse():
    b = np.arange(0, 0x7C00, dtype=np.uint16)
    assert np.array_equal(wl.round_to(wl.widen(b, 0), 0), b)
    b = np.arange(0, 0x7F80, dtype=np.uint16)
    assert np.array_equal(wl.round_to(wl.widen(b, 1), 1), b)


@pytest.mark.parametrize("cfg_id", [0, 1, 2, 3, 4])
def test_power_law_rates_mean_and_shape(cfg_id):
    cfg = wl.CONFIGS[cfg_id]
    for rate in (cfg.rates or (cfg.rate,)):
        p = wl.power_law_rates(cfg.n, cfg.alpha, rate, layer=1)
        assert abs(p.mean() - rate) < 1e-9
        rank = wl.neuron_ranks(cfg.n, 1)
        order = np.argsort(rank)
        assert np.all(np.diff(p[order]) <= 0)         # hotter rank -> higher rate
        assert p.max() <= wl.PMAX
    # hot neurons start scattered over the physical slots
    rank = wl.neuron_ranks(cfg.n, 1)
    assert sorted(rank.tolist()) == list(range(1, cfg.n + 1))
    assert np.nonzero(rank <= 32)[0].max() > cfg.n // 2


def test_fc1_bias_realises_rates():
    """Empirical P(z_i > 0) over 4096 tokens within a binomial 5-sigma band of p_i."""
    cfg = wl.CONFIGS[0]
    L = wl.host_layer(cfg, layer=0)
    X = wl.widen(wl.tokens(cfg, 4096, aux=1, tensor=wl.T_XPROF), 0)
    z = O.fc1_preactivation(L.f64("W1"), L.f64("b1"), X)
    f = (z > 0).mean(axis=0)
    sd = np.sqrt(L.p * (1 - L.p) / 4096)
    # ||W1[i]|| is ~1 with spread ~1/sqrt(2d); allow that on top of sampling noise
    assert np.mean(np.abs(f - L.p) <= 5 * sd + 0.03 * L.p + 1e-3) > 0.99
    assert abs(f.mean() - cfg.rate) < 0.05 * cfg.rate


def test_predictor_bias_realises_rates():
    cfg = wl.CONFIGS[0]
    L = wl.host_layer(cfg, layer=0)
    X = wl.widen(wl.tokens(cfg, 512, aux=2), 0)
    h = O.predictor_hidden(L.f64("Wp1"), X)
    l = O.predictor_logits(L.f64("Wp2"), h, L.f64("bp2"))
    f = (l > 0).mean(axis=0)
    assert abs(f.mean() - cfg.rate) < 0.1 * cfg.rate
    # union over B tokens ~ mean(1 - (1-p)^B)
    for B in (4, 16):
        u = np.mean([np.any(l[t:t + B] > 0, axis=0).mean() for t in range(0, 512, B)])
        want = np.mean(1 - (1 - L.p) ** B)
        assert abs(u - want) < 0.15 * want
