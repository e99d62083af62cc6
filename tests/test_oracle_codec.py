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


@pytest.mark.parametrize("x", [-8.0, -3.0, -1.0, -0.5, -1e-3, 0.0, 1e-3, 0.3, 1.0, 2.5, 6.0, 10.0])
def test_gelu_tanh_close_to_libm(x):
    # Exact bits of the FP32 routine are a specification (parity unpinned);
    # here it is held to the FP64 libm formula within a small error bound.
    want = 0.5 * x * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))
    got = oracle.gelu_tanh_f32(x)
    assert abs(got - want) <= 4e-7 * abs(x) + 1e-7 * abs(want) + 1e-30


def test_gelu_recip_within_one_ulp_on_one_to_two():
    # Newton's iteration from the linear seed: 1/d to within one FP32 ulp of
    # the exact reciprocal over [1, 2] (dense sample plus both ends).
    rng = np.random.default_rng(17)
    ds = np.concatenate([np.linspace(1.0, 2.0, 20001), rng.uniform(1.0, 2.0, 20000), [1.0, 2.0]]).astype(np.float32)
    for d in ds:
        got = np.float32(oracle.gelu_recip(float(d)))
        exact = 1.0 / float(d)
        ulp = float(np.spacing(np.float32(exact)))
        assert abs(float(got) - exact) <= ulp, (float(d), float(got), exact)
    assert oracle.gelu_recip(1.0) == 1.0 and oracle.gelu_recip(2.0) == 0.5


def test_gelu_tanh_dense_against_fp64_formula():
    # Over the range the FFN accumulators span, the FP32 routine stays within
    # a few FP32 ulps of the FP64 formula (and is exactly 0 at 0).
    xs = np.concatenate([np.linspace(-12, 12, 24001), np.linspace(-1e-3, 1e-3, 2001)]).astype(np.float32)
    for x in xs:
        x = float(x)
        want = 0.5 * x * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))
        got = oracle.gelu_tanh_f32(x)
        assert abs(got - want) <= 5e-7 * abs(want) + 2e-8 * abs(x) + 1e-37, (x, got, want)
    assert oracle.gelu_tanh_f32(0.0) == 0.0


def test_gelu_exp_close_to_libm():
    for x in np.linspace(-86, 0, 2001):
        want = math.exp(float(np.float32(x)))
        got = oracle.gelu_exp_neg(float(x))
        assert abs(got - want) <= 3e-7 * want + 1e-38, x


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
