"""Pins for the oracle's scalar arithmetic: BF16 rounding, the E2M1 element
codec and the MX shared-exponent rule (OCP MX v1.0, the 4-bit format the
paper's HiF4/MXFP4 kernels use)."""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import golden_path


def _read_pairs(name):
    rows = []
    with open(golden_path(name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                a, b = line.split()
                rows.append((a, b))
    return rows


def test_e2m1_decode_matches_format_table():
    for code_s, val_s in _read_pairs("e2m1_codes.txt"):
        code, val = int(code_s, 16), float(val_s)
        got = oracle.e2m1_decode(code)
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), (code, got, val)


def test_e2m1_every_code_round_trips():
    for code_s, val_s in _read_pairs("e2m1_codes.txt"):
        code, val = int(code_s, 16), float(val_s)
        assert oracle.e2m1_encode(val, negative=math.copysign(1.0, val) < 0) == code


def test_e2m1_rounding_table():
    for v_s, code_s in _read_pairs("e2m1_rounding.txt"):
        v = float(v_s)
        assert oracle.e2m1_encode(v, negative=math.copysign(1.0, v) < 0) == int(code_s, 16), v_s


def _brute_e2m1(v):
    """Argmin over the 15 distinct E2M1 values; ties -> even mantissa bit;
    the sign bit is always the sign of v (so a rounded-to-zero negative is 0x8)."""
    mags = [(c, abs(oracle.e2m1_decode(c))) for c in range(8)]
    best = None
    for c, m in mags:
        d = abs(abs(v) - m)
        key = (d, c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1] | (8 if math.copysign(1.0, v) < 0 else 0)


def test_e2m1_encode_equals_bruteforce_argmin():
    rng = np.random.default_rng(123)
    vals = np.concatenate([rng.uniform(-8, 8, 4000),
                           np.arange(-8, 8.0001, 0.125)])  # every quarter-step, incl. all ties
    for v in vals:
        assert oracle.e2m1_encode(float(v)) == _brute_e2m1(float(v)), v


def test_mx_scale_exponent_table():
    for a_s, x_s in _read_pairs("mx_scale_exponent.txt"):
        assert oracle.mx_scale_exponent(float(a_s)) == int(x_s), a_s


def test_mx_scale_exponent_puts_amax_in_top_binade():
    # Unless clamped, the rule leaves amax / 2^X in [4, 8): the top binade of E2M1.
    rng = np.random.default_rng(5)
    for a in np.exp(rng.uniform(-80, 80, 3000)):
        X = oracle.mx_scale_exponent(float(a))
        if -127 < X < 127:
            r = a / 2.0 ** X
            assert 4.0 <= r < 8.0, (a, X)


def _f32(u):
    return float(np.array([u], dtype=np.uint32).view(np.float32)[0])


def test_bf16_rounding_matches_torch_cast():
    rng = np.random.default_rng(9)
    bits = rng.integers(0, 2**32, 20000, dtype=np.uint64).astype(np.uint32)
    edge = np.array([0x3F808000, 0x3F818000, 0x3F80C000, 0x7F7FFFFF, 0x7F7F8000, 0x7F7F7FFF,
                     0x00000001, 0x00008000, 0x00018000, 0x80008000, 0xBF808000, 0x3F7FFFFF,
                     0x00000000, 0x80000000], dtype=np.uint32)
    bits = np.concatenate([bits, edge])
    f = bits.view(np.float32)
    finite = np.isfinite(f)
    f = f[finite]
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round_array(f)
    assert np.array_equal(got, want)


def test_bf16_ties_go_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: even significand is 1.0.
    assert oracle.f32_to_bf16(_f32(0x3F808000)) == 0x3F80
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    assert oracle.f32_to_bf16(_f32(0x3F818000)) == 0x3F82
    # just above the largest finite BF16 by half an ulp rounds to infinity
    assert oracle.f32_to_bf16(_f32(0x7F7F8000)) == 0x7F80
    assert oracle.f32_to_bf16(_f32(0x7F7F7FFF)) == 0x7F7F


# ---- GELU (tanh form) of the FFN, FP64 ------------------------------------

def test_gelu_tanh_equals_torch_tanh_gelu_in_fp64():
    # PyTorch's GELU with approximate="tanh" is the same definition,
    # 0.5 x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3))); in float64 the two
    # agree to FP64 rounding (relative, plus the absolute |x| 2^-52 that the
    # cancellation in 1 + tanh(u) leaves in the far negative tail).
    xs = np.concatenate([np.linspace(-12, 12, 4801), np.linspace(-1e-3, 1e-3, 201), [-40.0, 40.0, 1e-300]])
    want = torch.nn.functional.gelu(torch.from_numpy(xs), approximate="tanh").numpy()
    got = oracle.gelu(xs)
    assert np.all(np.abs(got - want) <= 4e-16 * np.abs(want) + 2.0 ** -52 * np.abs(xs) + 1e-300)


def test_gelu_tanh_is_within_the_known_distance_of_the_erf_gelu():
    # The tanh form approximates x * Phi(x) to within 4.8e-4 everywhere
    # (max |difference| 4.73e-4 near |x| = 2); a dropped cubic term (0.034),
    # a sigmoid form x sigma(1.702 x) (0.020) or sqrt(2/pi) misread as 0.8
    # (6.4e-4) all exceed that bound.
    from scipy.special import erf
    xs = np.linspace(-10, 10, 20001)
    exact = 0.5 * xs * (1.0 + erf(xs / math.sqrt(2.0)))
    err = np.abs(oracle.gelu(xs) - exact)
    assert err.max() <= 4.8e-4 and err.max() > 4.0e-4


def test_gelu_tanh_special_values_and_odd_part():
    # GELU(x) - GELU(-x) = x (tanh is odd), GELU(0) = 0, GELU(x) -> x for large
    # x and -> -0 for large negative x (tanh saturates to -1 in FP64).
    for x in [1e-8, 0.1, 0.5, 1.0, 2.3, 5.0, 9.0]:
        assert abs(oracle.gelu_tanh(x) - oracle.gelu_tanh(-x) - x) <= 2e-16 * abs(x)
    assert oracle.gelu_tanh(0.0) == 0.0
    assert oracle.gelu_tanh(40.0) == 40.0
    r = oracle.gelu_tanh(-40.0)
    assert r == 0.0 and math.copysign(1.0, r) == -1.0
    # slope 1/2 at the origin
    assert abs(oracle.gelu_tanh(1e-9) / 1e-9 - 0.5) <= 1e-9


def _bf16_nearest_exact(v: float) -> int:
    # brute force with exact rationals: the nearest BF16 value among the
    # finite candidates around v (ties: even significand), as bit patterns
    from fractions import Fraction
    f32 = np.float32(v) if abs(v) < 3.4e38 else np.float32(np.copysign(3.3e38, v))
    base = int(np.array([f32], np.float32).view(np.uint32)[0]) >> 16
    cands = []
    for d in range(-2, 3):
        b = (base + d) & 0xFFFF
        fv = float(np.array([b << 16], np.uint32).view(np.float32)[0])
        if math.isfinite(fv):
            cands.append((b, fv))
    fv_ = Fraction(v)
    best = min(cands, key=lambda c: (abs(Fraction(c[1]) - fv_), c[0] & 1))
    return best[0]


def test_f64_to_bf16_is_one_correct_rounding():
    rng = np.random.default_rng(23)
    vals = list(np.ldexp(1.0 + rng.random(3000), rng.integers(-130, 60, 3000)) * rng.choice([-1, 1], 3000))
    # exact midpoints between BF16 neighbours (ties), and values one FP64 ulp
    # off them, where rounding through binary32 first would go wrong
    for _ in range(500):
        b = int(rng.integers(0x0080, 0x7F00))
        lo = float(np.array([b << 16], np.uint32).view(np.float32)[0])
        hi = float(np.array([(b + 1) << 16], np.uint32).view(np.float32)[0])
        mid = (lo + hi) / 2
        vals += [mid, np.nextafter(mid, 0.0), np.nextafter(mid, np.inf)]
    for v in vals:
        v = float(v)
        assert oracle.f64_to_bf16(v) == _bf16_nearest_exact(v), v
    # a value one FP64 ulp above a BF16 tie whose binary32 rounding lands on
    # the tie: one-step rounding goes up, rounding through binary32 goes to even
    mid = 1.0 + 2.0 ** -8
    v = np.nextafter(mid, 2.0)
    assert oracle.f64_to_bf16(v) == 0x3F81
    assert oracle.f32_to_bf16(float(np.float32(v))) == 0x3F80
    # binary32 values convert as oracle_f32_to_bf16 does
    f = np.float32(rng.standard_normal(2000) * 100).astype(np.float64)
    assert all(oracle.f64_to_bf16(float(x)) == oracle.f32_to_bf16(float(x)) for x in f)
    assert oracle.f64_to_bf16(0.0) == 0 and oracle.f64_to_bf16(-0.0) == 0x8000
    assert oracle.f64_to_bf16(3.5e38) == 0x7F80 and oracle.f64_to_bf16(2.0 ** -133) == 0x0001
    assert oracle.f64_to_bf16(2.0 ** -134) == 0x0000 and oracle.f64_to_bf16(1.5 * 2.0 ** -134) == 0x0001


# ---- binary16 (FP16 outlier branch) --------------------------------------

def test_f16_rounding_matches_numpy_cast():
    rng = np.random.default_rng(19)
    # magnitudes across the whole half range, subnormals and overflow included
    mag = np.ldexp(1.0 + rng.random(20000), rng.integers(-27, 17, 20000))
    scaled = (mag * rng.choice([-1.0, 1.0], 20000)).astype(np.float32)
    edge = np.array([65504.0, 65519.0, 65520.0, 65536.0, 2.0**-14, 2.0**-24, 2.0**-25, 1.5 * 2.0**-25,
                     3 * 2.0**-26, 1.0 + 2.0**-11, 1.0 + 3 * 2.0**-11, -0.0, 0.0, -2.0**-25], np.float32)
    with np.errstate(over="ignore"):  # the overflow cases are intended (they round to infinity)
        wants = np.concatenate([scaled, edge]).astype(np.float16).view(np.uint16)
    for v, want in zip(np.concatenate([scaled, edge]), wants):
        assert oracle.f32_to_f16(float(v)) == int(want), float(v)


def test_f16_decode_of_every_code():
    codes = np.arange(65536, dtype=np.uint16)
    want = codes.view(np.float16).astype(np.float64)
    for c in range(0, 65536, 7):
        got = oracle.f16_to_f64(c)
        w = want[c]
        assert (np.isnan(got) and np.isnan(w)) or got == w, c
