"""The seeded synthetic inputs follow their stated recipes (the stand-ins for
the paper's calibration data: activation column maxima above 6 on a few
heavy-tailed channels with a tail beyond |x| > 1.5, weight column maxima
below 0.6), are valid BF16 and are reproducible from their seeds."""
import numpy as np

from outlier_split_mixed_b200 import synth


def _f(h):
    return synth.bf16_bits_to_f32(h)


def test_heavy_tailed_activations():
    M, K = 2048, 1024
    x = _f(synth.acts_heavy_tailed(M, K, seed=7, frac=0.01))
    colmax = np.abs(x).max(axis=0)
    heavy = np.flatnonzero(colmax > 3.0)
    assert len(heavy) == round(0.01 * K)                      # 1 % of the channels
    assert np.allclose(colmax[heavy], 6.0, rtol=2 ** -8)      # rescaled to column max 6 (one BF16 rounding)
    bulk = np.setdiff1d(np.arange(K), heavy)
    assert abs(float(x[:, bulk].std()) - 0.3) < 0.01          # N(0, 0.3) bulk
    assert (np.abs(x[:, heavy]) > 1.5).sum() > 0              # a tail beyond 1.5


def test_spiked_and_gelu_activations():
    x = _f(synth.acts_gaussian_spiked(256, 512, seed=0))
    colmax = np.abs(x).max(axis=0)
    assert (np.abs(colmax - 6.0) <= 6.0 * 2 ** -8).sum() == 8  # eight spiked channels at max 6
    g = _f(synth.acts_gelu_boosted(512, 1024, seed=3, frac=0.005))
    gm = np.abs(g).max(axis=0)
    boosted = np.abs(gm - 8.0) <= 8.0 * 2 ** -8
    assert boosted.sum() == round(0.005 * 1024)
    assert g[:, ~boosted].min() > -0.2                         # GELU is bounded below (about -0.17)


def test_weights_stay_below_0_6():
    w = _f(synth.weights_gaussian(512, 384, seed=5, sigma=0.2))
    assert np.abs(w).max() < 0.6
    assert abs(float(w.std()) - 0.2) < 0.02


def test_generators_are_reproducible_and_bf16():
    a = synth.acts_heavy_tailed(64, 256, seed=11)
    b = synth.acts_heavy_tailed(64, 256, seed=11)
    c = synth.acts_heavy_tailed(64, 256, seed=12)
    assert a.dtype == np.uint16 and np.array_equal(a, b) and not np.array_equal(a, c)
    # a BF16 bit pattern round-trips through FP32
    assert np.array_equal(synth.to_bf16_bits(_f(a)), a)
    cfg = synth.UP
    assert np.array_equal(cfg.make_x(32), synth.acts_heavy_tailed(32, cfg.K, cfg.x_seed))
