"""Pins for the oracle's NVFP4 path (E2M1 elements, a UE4M3 scale per 16
elements, a power-of-two factor per tensor): the E4M3 codec against
PyTorch's float8_e4m3fn, the element multiplier against exact rational
arithmetic, the per-tensor exponent by its defining inequalities, block
encodes by round trips and by an independent dequantised error bound, and
the dual product by an FP64 triple loop over values decoded with PyTorch's
float8 type."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from outlier_split_mixed_b200 import synth

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _torch_e4m3_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decode_equals_torch_float8():
    want = _torch_e4m3_decode(np.arange(256))
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if math.isnan(want[c]):
            assert math.isnan(got), c
        else:
            assert got == want[c] and math.copysign(1, got) == math.copysign(1, want[c]), (c, got, want[c])
    # format anchors: largest finite, smallest normal, smallest subnormal, one
    assert (oracle.e4m3_decode(0x7E), oracle.e4m3_decode(0x08), oracle.e4m3_decode(0x01),
            oracle.e4m3_decode(0x38)) == (448.0, 2.0 ** -6, 2.0 ** -9, 1.0)


def test_e4m3_encode_equals_torch_rne_below_overflow():
    rng = np.random.default_rng(5)
    vals = np.concatenate([
        rng.uniform(0, 464, 3000), np.exp(rng.uniform(-12, 6, 3000)),
        _torch_e4m3_decode(np.arange(127)),                               # every finite value
        (_torch_e4m3_decode(np.arange(126)) + _torch_e4m3_decode(np.arange(1, 127))) / 2,   # every tie
    ]).astype(np.float32)
    vals = vals[vals < 464]
    want = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in vals], np.uint8)
    assert np.array_equal(got, want)
    assert np.array_equal(np.array([oracle.e4m3_encode(-float(v)) for v in vals[:200]], np.uint8), want[:200] | 0x80)


def test_e4m3_encode_saturates():
    for v in (448.0, 463.9, 464.0, 480.0, 1e6, float("inf")):
        assert oracle.e4m3_encode(v) == 0x7E
    assert oracle.e4m3_encode(float("-inf")) == 0xFE
    assert oracle.e4m3_encode(float("nan")) == 0x7F


def _f32_round_exact(q: Fraction) -> float:
    """Nearest binary32 to the rational q > 0 (ties to even), by exact
    comparison with the neighbours of a candidate."""
    c = np.float32(float(q))
    cands = [np.nextafter(c, np.float32(0)), c, np.nextafter(c, np.float32(np.inf))]
    best = None
    for x in cands:
        d = abs(Fraction(float(x)) - q)
        even = (int(np.array(x, np.float32).view(np.uint32)) & 1) == 0
        key = (d, not even)
        if best is None or key < best[0]:
            best = (key, float(x))
    return best[1]


@pytest.mark.parametrize("g", [-100, -9, 0, 3, 100])
def test_nvfp4_recip_is_the_correctly_rounded_reciprocal(g):
    for S in range(1, 127):
        D = Fraction(oracle.e4m3_decode(S)) * Fraction(2) ** g
        assert oracle.nvfp4_recip(S, g) == _f32_round_exact(1 / D), (S, g)
    assert oracle.nvfp4_recip(0, g) == 0.0


def test_nvfp4_tensor_exponent_by_definition():
    rng = np.random.default_rng(9)
    for a in np.concatenate([np.exp(rng.uniform(-60, 60, 400)), [2688.0, 2688.0 * 2, 2688.0 * 2 ** -30, 1.0]]):
        g = oracle.nvfp4_tensor_exponent(float(a))
        assert a <= 2688.0 * 2.0 ** g
        assert a > 2688.0 * 2.0 ** (g - 1)
    assert oracle.nvfp4_tensor_exponent(2688.0) == 0
    assert oracle.nvfp4_tensor_exponent(np.nextafter(2688.0, 3000.0)) == 1
    assert oracle.nvfp4_tensor_exponent(0.0) == 0
    assert oracle.nvfp4_tensor_exponent(1e-300) == -100 and oracle.nvfp4_tensor_exponent(1e300) == 100


def test_nvfp4_scale_of_six_times_a_scale_is_that_scale():
    # amax = 6 * S_dec * 2^g is a BF16 value; fp32(1/6) is within 3e-8 of 1/6,
    # so the E4M3 rounding gives back S
    for g in (-20, 0, 7):
        for S in range(1, 127):
            amax = 6.0 * oracle.e4m3_decode(S) * 2.0 ** g
            assert oracle.nvfp4_scale(amax, g) == S, (S, g)
    assert oracle.nvfp4_scale(0.0, 0) == 0


def test_nvfp4_scale_equals_exact_then_torch_rounding():
    rng = np.random.default_rng(21)
    k6 = Fraction(float(np.float32(1.0 / 6.0)))
    for g in (-5, 0, 4):
        am = synth.bf16_bits_to_f32(synth.to_bf16_bits(np.exp(rng.uniform(-14, 9, 300)).astype(np.float32)))
        for a in am:
            sc = np.float32(_f32_round_exact(Fraction(float(a)) * k6 * Fraction(2) ** (-g)))
            want = int(torch.tensor([sc]).clamp(max=448.0).to(torch.float8_e4m3fn).view(torch.uint8)[0])
            assert oracle.nvfp4_scale(float(a), g) == want, (a, g)


def _bf16(vals):
    return synth.to_bf16_bits(np.asarray(vals, np.float32))


def test_quantize_act_nv_exact_grid_round_trips():
    # s = 1, k = 0; each 16-block is e2m1 values times 2^g S with one value at
    # 6: the block scale is S and every code decodes back to its input.
    rng = np.random.default_rng(3)
    K, M = 128, 6
    g = -3
    vals = np.zeros((M, K), np.float32)
    want_codes = np.zeros((M, K), np.uint8)
    want_scales = np.zeros((M, K // 16), np.uint8)
    for t in range(M):
        for b in range(K // 16):
            S = int(rng.integers(16, 110))           # normal E4M3 scales
            c = rng.integers(0, 16, 16).astype(np.uint8)
            c[int(rng.integers(0, 16))] = 7 | (8 if rng.integers(0, 2) else 0)   # a +-6
            vals[t, 16 * b:16 * b + 16] = [(-1 if x & 8 else 1) * E2M1[x & 7] * oracle.e4m3_decode(S) * 2.0 ** g
                                           for x in c]
            want_codes[t, 16 * b:16 * b + 16] = c
            want_scales[t, b] = S
    X = _bf16(vals)
    assert np.array_equal(synth.bf16_bits_to_f32(X), vals)     # exactly representable
    inv_s = np.ones(K, np.float32)
    codes, scales, a_hp = oracle.quantize_act_nv(X, inv_s, np.zeros(0, np.int32), g)
    assert np.array_equal(scales, want_scales)
    unpacked = np.stack([codes & 15, codes >> 4], axis=-1).reshape(M, K)
    # +0 encodes as code 0 and -0 as 8: compare values, then signs of non-zeros
    assert np.array_equal(unpacked & 7, want_codes & 7)
    nz = (want_codes & 7) != 0
    assert np.array_equal((unpacked & 8)[nz], (want_codes & 8)[nz])
    assert a_hp.shape == (M, 0)


def test_quantize_act_nv_error_bound_and_outlier_slots():
    rng = np.random.default_rng(8)
    M, K, k = 40, 512, 24
    X = synth.acts_heavy_tailed(M, K, 77, frac=0.02)
    inv_s = np.exp(rng.uniform(-0.7, 0.7, K)).astype(np.float32)
    O = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    Xs = oracle.smooth_act(X, inv_s)
    J = np.setdiff1d(np.arange(K), O)
    g = oracle.nvfp4_tensor_exponent(float(np.abs(synth.bf16_bits_to_f32(Xs[:, J])).max()))
    codes, scales, a_hp = oracle.quantize_act_nv(X, inv_s, O, g)
    Kbp = oracle.kbp(K, k)
    assert codes.shape == (M, Kbp // 2) and scales.shape == (M, Kbp // 16)
    # outlier slots: x' * 2^-g, exact (no subnormals here)
    assert np.array_equal(synth.bf16_bits_to_f32(a_hp[:, :k]),
                          synth.bf16_bits_to_f32(Xs[:, O]) * np.float32(2.0 ** -g))
    assert np.all(a_hp[:, k:] == 0)
    # bulk: decoded value within half an E2M1 step (of the block scale) of x',
    # plus the saturation overshoot when the E4M3 scale rounded down
    xb = synth.bf16_bits_to_f32(Xs[:, J]).astype(np.float64)
    dec_s = _torch_e4m3_decode(scales) * 2.0 ** g
    c = np.stack([codes & 15, codes >> 4], axis=-1).reshape(M, Kbp)[:, :K - k]
    e = np.array([E2M1[x & 7] * (-1 if x & 8 else 1) for x in c.ravel()]).reshape(c.shape)
    dq = e * np.repeat(dec_s, 16, axis=1)[:, :K - k]
    xpad = np.zeros((M, Kbp))
    xpad[:, :K - k] = np.abs(xb)                            # the tail block is ragged (488 = 30.5 x 16)
    blk_amax = xpad.reshape(M, -1, 16).max(axis=2)
    step = np.repeat(dec_s, 16, axis=1)[:, :K - k]          # half the largest E2M1 gap (2), times S
    over = np.maximum(np.repeat(blk_amax, 16, axis=1)[:, :K - k] - 6 * step, 0)
    assert np.all(np.abs(dq - xb) <= step + over + 1e-30)
    assert np.all(np.sign(dq[dq != 0]) == np.sign(xb[dq != 0]))
    # padding scale bytes are zero
    assert np.all(scales[:, (K - k + 15) // 16:] == 0)


def test_plan_exponents_match_smoothed_calibration_data():
    rng = np.random.default_rng(12)
    M, K, N, k = 64, 256, 64, 16
    X = synth.acts_heavy_tailed(M, K, 5, frac=0.03)
    W = synth.weights_gaussian(K, N, 6, 0.05)
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, O = oracle.calibrate(amax, wmax, 0.5, k)
    ga, gw = oracle.nvfp4_plan_exponents(amax, wmax, s, inv_s, O)
    J = np.setdiff1d(np.arange(K), O)
    xs = np.abs(synth.bf16_bits_to_f32(oracle.smooth_act(X, inv_s))[:, J]).max()
    ws = np.abs(synth.bf16_bits_to_f32(oracle.fold_weights(W, s))[J, :]).max()
    assert (ga, gw) == (oracle.nvfp4_tensor_exponent(float(xs)), oracle.nvfp4_tensor_exponent(float(ws)))
    assert rng is not None


def _decode_nv(codes, scales, g):
    rows = codes.shape[0]
    Kbp = codes.shape[1] * 2
    c = np.stack([codes & 15, codes >> 4], axis=-1).reshape(rows, Kbp)
    e = np.array([E2M1[x & 7] * (-1 if x & 8 else 1) for x in c.ravel()]).reshape(c.shape)
    return e * np.repeat(_torch_e4m3_decode(scales), 16, axis=1) * 2.0 ** g


@pytest.mark.parametrize("k", [0, 20, 64])
def test_dual_gemm_nv_equals_triple_loop(k):
    M, K, N = 6, 192, 40
    rng = np.random.default_rng(40 + k)
    X = synth.acts_heavy_tailed(M, K, 31 + k, frac=0.05)
    W = synth.weights_gaussian(K, N, 32 + k, 0.05)
    s = np.exp(rng.uniform(-0.5, 0.5, K)).astype(np.float32)
    inv_s = (np.float32(1.0) / s).astype(np.float32)
    O = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    ga, gw = -4, -7
    ac, asc, ah = oracle.quantize_act_nv(X, inv_s, O, ga)
    wc, wsc, wh = oracle.pack_weights_nv(W, s, O, gw)
    bias = rng.standard_normal(N).astype(np.float32)
    y, T = oracle.dual_gemm_rows_nv(ac, asc, ah, np.arange(M), wc, wsc, wh, ga, gw, bias)
    A = _decode_nv(ac, asc, ga)
    B = _decode_nv(wc, wsc, gw)
    Ah = synth.bf16_bits_to_f32(ah).astype(np.float64) * 2.0 ** ga
    Bh = synth.bf16_bits_to_f32(wh).astype(np.float64) * 2.0 ** gw
    for t in range(M):
        for n in range(N):
            terms = [A[t, p] * B[n, p] for p in range(A.shape[1])] + [Ah[t, i] * Bh[n, i] for i in range(Ah.shape[1])]
            ref = math.fsum(terms) + float(bias[n])
            assert abs(y[t, n] - ref) <= 1e-12 * (sum(abs(x) for x in terms) + 1), (t, n)
            assert abs(T[t, n] - sum(abs(x) for x in terms)) <= 1e-12 * (T[t, n] + 1)


def test_dual_gemm_nv_all_outliers_is_the_bf16_product():
    # k = K: no bulk; the 2^-g scalings of the BF16 operands are exact, so y
    # is the FP64 product of the smoothed and folded BF16 values
    M, K, N = 5, 64, 24
    X = synth.acts_heavy_tailed(M, K, 3, frac=0.05)
    W = synth.weights_gaussian(K, N, 4, 0.05)
    s = np.exp(np.random.default_rng(1).uniform(-0.5, 0.5, K)).astype(np.float32)
    inv_s = (np.float32(1.0) / s).astype(np.float32)
    O = np.arange(K, dtype=np.int32)
    ga, gw = 5, -9
    ac, asc, ah = oracle.quantize_act_nv(X, inv_s, O, ga)
    wc, wsc, wh = oracle.pack_weights_nv(W, s, O, gw)
    y, _ = oracle.dual_gemm_rows_nv(ac, asc, ah, np.arange(M), wc, wsc, wh, ga, gw)
    xs = synth.bf16_bits_to_f32(oracle.smooth_act(X, inv_s)).astype(np.float64)
    ws = synth.bf16_bits_to_f32(oracle.fold_weights(W, s)).astype(np.float64)
    np.testing.assert_allclose(y, xs @ ws, rtol=1e-12, atol=1e-12)


def test_library_host_exponents_equal_the_oracle():
    # osm_nvfp4_tensor_exponent / osm_nvfp4_plan_exponents are host code in
    # libosm: no GPU needed.
    import outlier_split_mixed_b200 as osm
    rng = np.random.default_rng(17)
    for a in np.concatenate([np.exp(rng.uniform(-50, 50, 200)), [0.0, 2688.0, 2689.0]]).astype(np.float32):
        assert osm.nvfp4_tensor_exponent(float(a)) == oracle.nvfp4_tensor_exponent(float(a))
    for seed, k in ((1, 0), (2, 17), (3, 200)):
        M, K, N = 96, 512, 64
        X = synth.acts_heavy_tailed(M, K, seed, frac=0.03)
        W = synth.weights_gaussian(K, N, seed + 50, 0.05)
        amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
        s, inv_s, O = oracle.calibrate(amax, wmax, 0.6, k)
        assert osm.nvfp4_plan_exponents(amax, wmax, s, inv_s, O) == oracle.nvfp4_plan_exponents(amax, wmax, s, inv_s, O)


def _golden_lines(name):
    from conftest import golden_path
    with open(golden_path(name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                yield line


def test_e4m3_encode_hand_table():
    for line in _golden_lines("e4m3_rounding.txt"):
        v, code = line.split()
        assert oracle.e4m3_encode(float(v)) == int(code, 16), line


def test_nvfp4_blocks_hand_derived():
    for line in _golden_lines("nvfp4_blocks.txt"):
        g, vals, sc, codes = (x.strip() for x in line.split("|"))
        v = np.array([float(x) for x in vals.split()], np.float32)
        X = np.zeros((1, 32), np.uint16)
        X[0, :16] = synth.to_bf16_bits(v)
        # every value but 0.1 is a BF16 number; bf16(0.1) = 0.10009766 still codes to 0
        c, s, _ = oracle.quantize_act_nv(X, np.ones(32, np.float32), np.zeros(0, np.int32), int(g))
        assert s[0, 0] == int(sc, 16), line
        assert c[0, :8].tolist() == [int(x, 16) for x in codes.split()], line
        assert s[0, 1] == 0 and not c[0, 8:].any()                         # the all-zero second block
