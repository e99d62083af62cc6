"""Pins for the oracle's calibration (Eq. (2), Eq. (4)) and smoothing/fold
(Eq. (1)) of "W4A4 Quantization for Inference on Wan2.2-I2V-A14B"."""
import numpy as np
import pytest

import oracle
from conftest import golden_path
from outlier_split_mixed_b200 import synth


def _f32(h):
    return synth.bf16_bits_to_f32(h).astype(np.float64)


@pytest.fixture(scope="module")
def small_layer():
    X = synth.acts_heavy_tailed(300, 256, seed=11, frac=0.05)
    W = synth.weights_gaussian(256, 96, seed=12, sigma=0.05)
    return X, W


def test_statistics_are_column_and_row_maxima(small_layer):
    X, W = small_layer
    assert np.array_equal(oracle.act_amax(X), np.abs(_f32(X)).max(axis=0).astype(np.float32))
    assert np.array_equal(oracle.weight_amax(W), np.abs(_f32(W)).max(axis=1).astype(np.float32))


def test_topk_equals_full_sort_with_low_index_tiebreak():
    rng = np.random.default_rng(3)
    K = 500
    amax = rng.integers(0, 40, K).astype(np.float32) * np.float32(0.25)  # many exact ties
    wmax = np.full(K, 0.1, np.float32)
    for k in (0, 1, 7, 64, 499, 500):
        _, _, O = oracle.calibrate(amax, wmax, 0.5, k)
        order = np.lexsort((np.arange(K), -amax.astype(np.float64)))  # score desc, index asc
        assert np.array_equal(O, np.sort(order[:k]).astype(np.int32)), k
        assert np.all(np.diff(O) > 0)


def test_alpha_half_balances_act_and_weight_ranges(small_layer):
    # For alpha = 1/2, Eq. (2) gives max_t|x_tj|/s_j = max_n|w_jn| s_j = sqrt(a_j w_j).
    X, W = small_layer
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, _ = oracle.calibrate(amax, wmax, 0.5, 0)
    lhs = amax.astype(np.float64) * inv_s.astype(np.float64)
    rhs = wmax.astype(np.float64) * s.astype(np.float64)
    assert np.allclose(lhs, rhs, rtol=3e-7, atol=0)
    assert np.allclose(lhs, np.sqrt(amax.astype(np.float64) * wmax.astype(np.float64)), rtol=3e-7)


def test_larger_alpha_moves_range_into_weights(small_layer):
    # The spread of the smoothed activation maxima across channels is the
    # spread of a_j*w_j raised to (1-alpha): larger alpha flattens the
    # activations and roughens the weights.
    X, W = small_layer
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    spreads_x, spreads_w = [], []
    for alpha in (0.2, 0.4, 0.5, 0.6, 0.8):
        s, inv_s, _ = oracle.calibrate(amax, wmax, alpha, 0)
        xa = amax * inv_s
        wa = wmax * s
        spreads_x.append(xa.max() / xa.min())
        spreads_w.append(wa.max() / wa.min())
    assert all(a > b for a, b in zip(spreads_x, spreads_x[1:]))
    assert all(a < b for a, b in zip(spreads_w, spreads_w[1:]))


def test_statistics_are_floored_and_nonfinite_rejected():
    amax = np.array([0.0, 1.0, 4.0], np.float32)
    wmax = np.array([0.5, 0.0, 0.25], np.float32)
    s, inv_s, _ = oracle.calibrate(amax, wmax, 0.5, 1)
    assert np.isclose(s[0], np.sqrt(1e-5) / np.sqrt(0.5), rtol=1e-6)
    assert np.isclose(s[1], 1.0 / np.sqrt(1e-5), rtol=1e-6)
    with pytest.raises(ValueError):
        oracle.calibrate(np.array([np.inf, 1.0], np.float32), np.ones(2, np.float32), 0.5, 1)
    with pytest.raises(ValueError):
        oracle.calibrate(np.ones(2, np.float32), np.array([1.0, np.nan], np.float32), 0.5, 1)


def test_eq1_smoothing_is_equivalent_up_to_bf16_rounding(small_layer):
    # Eq. (1): (X / s)(s W) = X W. With both smoothed operands rounded to BF16
    # (relative error <= 2^-9 each, plus one FP32 rounding), every product
    # moves by at most (2^-8 + 2^-17) of its magnitude.
    X, W = small_layer
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, _ = oracle.calibrate(amax, wmax, 0.6, 0)
    Xs, Ws = oracle.smooth_act(X, inv_s), oracle.fold_weights(W, s)
    x, w = _f32(X), _f32(W)
    y_ref = x @ w
    y_s = _f32(Xs) @ _f32(Ws)
    bound = (2.0 ** -8 + 2.0 ** -17) * (np.abs(x) @ np.abs(w))
    assert np.all(np.abs(y_s - y_ref) <= bound)
    # and the smoothing really moved range: the smoothed activation maxima are flatter
    assert (np.abs(_f32(Xs)).max(0).max() / np.abs(_f32(Xs)).max(0).min()) < (amax.max() / amax.min())


def test_eq1_wrong_channel_would_be_caught(small_layer):
    # The Eq. (1) bound is tight enough that pairing s_j with the wrong
    # channel (a plausible indexing mistake) violates it.
    X, W = small_layer
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, _ = oracle.calibrate(amax, wmax, 0.6, 0)
    Xs = oracle.smooth_act(X, np.roll(inv_s, 1))
    Ws = oracle.fold_weights(W, s)
    x, w = _f32(X), _f32(W)
    bound = (2.0 ** -8 + 2.0 ** -17) * (np.abs(x) @ np.abs(w))
    assert np.any(np.abs(_f32(Xs) @ _f32(Ws) - x @ w) > bound)


# ---- tail-aware (percentile) channel score -------------------------------

def _golden_percentiles():
    rows = []
    with open(golden_path("percentile_rank.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                q, r, v = line.split()
                rows.append((float(q), int(r), float(v)))
    return rows


def test_percentile_golden_column():
    col = np.array([3, -1, 4, 1, -5, 9, 2, 6], np.float32)
    X = synth.to_bf16_bits(col[:, None] * np.ones((1, 32), np.float32))
    for q, r, v in _golden_percentiles():
        assert oracle.percentile_rank(q, 8) == r, q
        score = oracle.act_percentile(X, r)
        assert np.all(score == np.float32(v)), (q, score[0], v)


def test_percentile_at_q1_is_the_maximum_and_monotone_in_q():
    X = synth.acts_heavy_tailed(200, 96, seed=31, frac=0.05)
    T = X.shape[0]
    amax = oracle.act_amax(X)
    assert np.array_equal(oracle.act_percentile(X, oracle.percentile_rank(1.0, T)), amax)
    prev = None
    for q in (0.5, 0.9, 0.99, 0.999, 1.0):
        sc = oracle.act_percentile(X, oracle.percentile_rank(q, T))
        assert np.all(sc <= amax)
        if prev is not None:
            assert np.all(sc >= prev)
        prev = sc


def test_scored_calibration_reduces_to_eq4_with_the_maximum():
    rng = np.random.default_rng(41)
    K, k = 300, 17
    amax = np.exp(rng.normal(0, 1, K)).astype(np.float32)
    wmax = rng.uniform(0.01, 0.5, K).astype(np.float32)
    a = oracle.calibrate(amax, wmax, 0.55, k)
    b = oracle.calibrate_scored(amax, amax, wmax, 0.55, k)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    # s does not depend on the score; O does
    score = rng.permutation(amax)
    c = oracle.calibrate_scored(amax, score, wmax, 0.55, k)
    assert np.array_equal(c[0], a[0]) and np.array_equal(c[1], a[1])
    assert np.array_equal(c[2], np.sort(np.argsort(-score, kind="stable")[:k]))


def test_percentile_score_ignores_a_single_token_spike():
    # The purpose of the tail-aware score: a channel whose maximum comes from
    # one rare token is an outlier for Eq. (4)'s max score but not for a
    # percentile score, while a channel with a consistently heavy tail is
    # an outlier for both.
    T, K = 512, 64
    rng = np.random.default_rng(5)
    x = rng.normal(0, 0.3, (T, K)).astype(np.float32)
    x[7, 10] = 40.0                                   # one spike
    x[:, 20] = rng.standard_t(2, T).astype(np.float32) * 3.0   # heavy tail throughout
    X = synth.to_bf16_bits(x)
    amax = oracle.act_amax(X)
    score = oracle.act_percentile(X, oracle.percentile_rank(0.99, T))
    wmax = np.full(K, 0.3, np.float32)
    O_max = oracle.calibrate(amax, wmax, 0.5, 2)[2]
    O_pct = oracle.calibrate_scored(amax, score, wmax, 0.5, 2)[2]
    assert 10 in O_max and 20 in O_max
    assert 10 not in O_pct and 20 in O_pct


def test_library_host_finalize_equals_the_oracle():
    # osm_calibrate_finalize(_scored) is host code in libosm: no GPU needed.
    import outlier_split_mixed_b200 as osm
    rng = np.random.default_rng(3)
    K, k = 777, 31
    a = np.exp(rng.normal(0, 1, K)).astype(np.float32)
    a[::50] = a[1]                                    # ties
    sc = rng.permutation(a)
    w = rng.uniform(0.01, 0.5, K).astype(np.float32)
    for got, want in ((osm.calibrate_finalize(a, w, 0.6, k), oracle.calibrate(a, w, 0.6, k)),
                      (osm.calibrate_finalize_scored(a, sc, w, 0.6, k), oracle.calibrate_scored(a, sc, w, 0.6, k))):
        for x, y in zip(got, want):
            assert np.array_equal(x, y)
