"""Pins for the oracle's runtime activation path, weight packing and the
dual-branch product (Eq. (3)/(5) of "W4A4 Quantization for Inference on
Wan2.2-I2V-A14B"; block packing of its Fig. 8 paragraph)."""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import golden_path
from outlier_split_mixed_b200 import synth


def _f64(h):
    return synth.bf16_bits_to_f32(h).astype(np.float64)


def _read_blocks():
    blocks, cur = [], None
    with open(golden_path("mxfp4_blocks.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, _, rest = line.partition(" ")
            if key == "block":
                cur = {"name": rest}
                blocks.append(cur)
            elif key == "values":
                cur["values"] = [float(v) for v in rest.split()]
            elif key == "scale_code":
                cur["scale"] = int(rest)
            elif key == "codes":
                cur["codes"] = [int(c, 16) for c in rest.split()]
    return blocks


def _unpack(codes_row):
    out = np.empty(codes_row.shape[0] * 2, np.uint8)
    out[0::2] = codes_row & 15
    out[1::2] = codes_row >> 4
    return out


@pytest.mark.parametrize("blk", _read_blocks(), ids=lambda b: b["name"])
def test_quantize_act_golden_blocks(blk):
    # One row, K = 32, no outliers, s = 1: the bulk row is the input itself.
    x = synth.to_bf16_bits(np.array([blk["values"]], np.float32))
    assert np.array_equal(_f64(x)[0], np.array(blk["values"]))  # values are exact in BF16
    codes, scales, a_hp = oracle.quantize_act(x, np.ones(32, np.float32), np.zeros(0, np.int32))
    assert codes.shape == (1, 64) and scales.shape == (1, 4) and a_hp.shape == (1, 0)
    assert scales[0, 0] == blk["scale"]
    assert list(_unpack(codes[0])[:32]) == blk["codes"]
    # the three padded blocks of the 128-wide bulk row hold code 0 and scale 0
    assert np.all(_unpack(codes[0])[32:] == 0) and np.all(scales[0, 1:] == 0)


# ---------------------------------------------------------------------------
# Brute force on a 4 x 32 x 4 layer: independent loops, every quantiser
# decision re-derived by search from the OCP MX definition.
# ---------------------------------------------------------------------------

E2M1 = {c: (-1 if c & 8 else 1) * [0, 0.5, 1, 1.5, 2, 3, 4, 6][c & 7] for c in range(16)}


def _brute_code(v):
    best = None
    for c in range(8):
        d = abs(abs(v) - E2M1[c])
        key = (d, c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1] | (8 if math.copysign(1.0, v) < 0 else 0)


def _brute_X(amax):
    # the unique integer X with 4 <= amax / 2^X < 8, clamped to [-127, 127]
    if amax == 0:
        return -127
    for X in range(-200, 200):
        if 4 <= amax / 2.0 ** X < 8:
            return max(-127, min(127, X))
    raise AssertionError


def _brute_quant(vals):
    """vals: list of floats of one block (real elements). -> (X, [codes])"""
    X = _brute_X(max(abs(v) for v in vals))
    return X, [_brute_code(v / 2.0 ** X) for v in vals]


def _brute_layer(X16, W16, alpha, k, wmode):
    M, K = X16.shape
    N = W16.shape[1]
    x, w = _f64(X16), _f64(W16)
    amax = [max(abs(x[t, j]) for t in range(M)) for j in range(K)]
    wmax = [max(abs(w[j, n]) for n in range(N)) for j in range(K)]
    s, inv_s, O_or = oracle.calibrate(np.array(amax, np.float32), np.array(wmax, np.float32), alpha, k)
    # outlier set by a full sort written here (score desc, index asc)
    O = sorted(sorted(range(K), key=lambda j: (-amax[j], j))[:k])
    assert list(O_or) == O
    J = [j for j in range(K) if j not in O]
    # smoothing: one FP32 multiply, RNE to BF16 (via torch's cast)
    xs = _f64(synth.to_bf16_bits((x.astype(np.float32) * inv_s[None, :]).astype(np.float32)))
    ws = _f64(synth.to_bf16_bits((w.astype(np.float32) * s[:, None]).astype(np.float32)))
    Kb = len(J)
    blocks = [list(range(p, min(p + 32, Kb))) for p in range(0, Kb, 32)]
    # activations: 1x32 blocks over the compacted bulk index
    aq = {}
    for t in range(M):
        for bi, blk in enumerate(blocks):
            Xa, cs = _brute_quant([xs[t, J[p]] for p in blk])
            aq[t, bi] = (Xa, cs)
    # weights: block exponent from the block / tile / strip amax
    def wamax(n, bi):
        return max(abs(ws[J[p], n]) for p in blocks[bi])
    wq = {}
    for n in range(N):
        for bi, blk in enumerate(blocks):
            if wmode == 0:
                am = wamax(n, bi)
            elif wmode == 1:
                am = max(wamax(nn, bi) for nn in range(n // 32 * 32, min(N, n // 32 * 32 + 32)))
            else:
                am = max(wamax(n, bb) for bb in range(bi // 4 * 4, min(len(blocks), bi // 4 * 4 + 4)))
            Xw = _brute_X(am)
            wq[n, bi] = (Xw, [_brute_code(ws[J[p], n] / 2.0 ** Xw) for p in blk])
    y = np.zeros((M, N))
    for t in range(M):
        for n in range(N):
            terms = []
            for bi, blk in enumerate(blocks):
                Xa, ca = aq[t, bi]
                Xw, cw = wq[n, bi]
                for i in range(len(blk)):
                    terms.append(Fraction(E2M1[ca[i]]) * Fraction(E2M1[cw[i]]) * Fraction(2) ** (Xa + Xw))
            for j in O:
                terms.append(Fraction(xs[t, j]) * Fraction(ws[j, n]))
            y[t, n] = float(sum(terms))
    return y, s, inv_s, np.array(O, np.int32), aq, wq, blocks


@pytest.mark.parametrize("wmode", [0, 1, 2])
@pytest.mark.parametrize("k", [0, 3, 32])
def test_bruteforce_4x32x4_layer(k, wmode):
    X = synth.acts_heavy_tailed(4, 32, seed=21 + k, frac=0.1)
    W = synth.weights_gaussian(32, 4, seed=22 + k, sigma=0.2)
    y_bf, s, inv_s, O, aq, wq, blocks = _brute_layer(X, W, 0.6, k, wmode)
    ac, asc, ahp = oracle.quantize_act(X, inv_s, O)
    wc, wsc, whp = oracle.pack_weights(W, s, O, wmode)
    for (t, bi), (Xa, cs) in aq.items():
        assert asc[t, bi] == Xa + 127
        assert list(_unpack(ac[t])[32 * bi:32 * bi + len(cs)]) == cs
    for (n, bi), (Xw, cs) in wq.items():
        assert wsc[n, bi] == Xw + 127
        assert list(_unpack(wc[n])[32 * bi:32 * bi + len(cs)]) == cs
    y, T = oracle.dual_gemm_rows(ac, asc, ahp, np.arange(4), wc, wsc, whp)
    assert np.allclose(y, y_bf, rtol=1e-13, atol=1e-300)
    assert np.all(T >= np.abs(y) * (1 - 1e-12))


def test_k_equals_K_is_a_plain_bf16_gemm():
    # Eq. (5) with O = all channels: the bulk branch is empty and the result
    # is the exact product of the smoothed BF16 operands.
    X = synth.acts_heavy_tailed(40, 96, seed=31)
    W = synth.weights_gaussian(96, 48, seed=32, sigma=0.05)
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, O = oracle.calibrate(amax, wmax, 0.5, 96)
    assert oracle.kbp(96, 96) == 0
    ac, asc, ahp = oracle.quantize_act(X, inv_s, O)
    wc, wsc, whp = oracle.pack_weights(W, s, O, 0)
    assert ac.shape == (40, 0) and asc.shape == (40, 0) and ahp.shape == (40, 128)
    y, _ = oracle.dual_gemm_rows(ac, asc, ahp, np.arange(40), wc, wsc, whp)
    ref = _f64(oracle.smooth_act(X, inv_s)) @ _f64(oracle.fold_weights(W, s))
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_k_zero_is_pure_w4a4_and_s_one_is_native():
    X = synth.acts_heavy_tailed(8, 64, seed=41)
    W = synth.weights_gaussian(64, 16, seed=42, sigma=0.05)
    ones = np.ones(64, np.float32)
    ac, asc, ahp = oracle.quantize_act(X, ones, np.zeros(0, np.int32))
    wc, wsc, whp = oracle.pack_weights(W, ones, np.zeros(0, np.int32), 0)
    assert ahp.shape == (8, 0) and whp.shape == (16, 0)
    # native W4A4 (s = 1, k = 0): bulk codes are the plain MXFP4 encodings of X
    for t in range(8):
        for b in range(2):
            Xa, cs = _brute_quant(list(_f64(X)[t, 32 * b:32 * b + 32]))
            assert asc[t, b] == Xa + 127 and list(_unpack(ac[t])[32 * b:32 * b + 32]) == cs
    y, _ = oracle.dual_gemm_rows(ac, asc, ahp, np.arange(8), wc, wsc, whp)
    deq_a = np.array([[E2M1[c] for c in _unpack(ac[t])] for t in range(8)]) * \
        np.repeat(2.0 ** (asc.astype(np.float64) - 127), 32, axis=1)
    deq_w = np.array([[E2M1[c] for c in _unpack(wc[n])] for n in range(16)]) * \
        np.repeat(2.0 ** (wsc.astype(np.float64) - 127), 32, axis=1)
    assert np.allclose(y, deq_a @ deq_w.T, rtol=1e-13, atol=1e-300)


def test_weight_modes_agree_with_1x32_exponents():
    # A tile or strip exponent is floor(log2(max amax)) - 2, i.e. the max of
    # the 1x32 exponents inside it (floor(log2) is monotone).
    K, N, k = 300, 96, 20
    W = synth.weights_gaussian(K, N, seed=51, sigma=0.05)
    rng = np.random.default_rng(52)
    s = np.exp(rng.uniform(-1, 1, K)).astype(np.float32)
    O = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    _, s1, _ = oracle.pack_weights(W, s, O, 0)
    _, st, _ = oracle.pack_weights(W, s, O, 1)
    _, ss, _ = oracle.pack_weights(W, s, O, 2)
    Kb = K - k
    nb_real = (Kb + 31) // 32
    for n in range(N):
        for b in range(s1.shape[1]):
            if b >= nb_real:
                assert s1[n, b] == st[n, b] == ss[n, b] == 0
                continue
            assert st[n, b] == s1[n // 32 * 32:n // 32 * 32 + 32, b].max()
            assert ss[n, b] == s1[n, b // 4 * 4:min(nb_real, b // 4 * 4 + 4)].max()


def test_split_routes_every_channel_once():
    # a_hp holds exactly the smoothed outlier columns; the bulk codes
    # dequantise to within one E2M1 half-step of the smoothed bulk columns.
    K, k = 200, 13
    X = synth.acts_heavy_tailed(16, K, seed=61, frac=0.05)
    rng = np.random.default_rng(62)
    inv_s = np.exp(rng.uniform(-0.5, 0.5, K)).astype(np.float32)
    O = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    J = np.setdiff1d(np.arange(K), O)
    ac, asc, ahp = oracle.quantize_act(X, inv_s, O)
    xs = _f64(oracle.smooth_act(X, inv_s))
    assert np.array_equal(_f64(ahp[:, :k]), xs[:, O]) and np.all(ahp[:, k:] == 0)
    deq = np.array([[E2M1[c] for c in _unpack(ac[t])] for t in range(16)]) * \
        np.repeat(2.0 ** (asc.astype(np.float64) - 127), 32, axis=1)
    step = np.repeat(2.0 ** (asc.astype(np.float64) - 127), 32, axis=1)  # 2^X
    err = np.abs(deq[:, :K - k] - xs[:, J])
    assert np.all(err <= 2.0 * step[:, :K - k] + 1e-300)   # saturation region [6, 8)
    assert np.all(deq[:, K - k:] == 0)


def test_error_falls_as_k_grows():
    # The paper's rationale (smoothing + a few high-precision columns) as a
    # sanity invariant on heavy-tailed data: relative error vs the unquantised
    # product falls as k grows.
    M, K, N = 64, 512, 64
    X = synth.acts_heavy_tailed(M, K, seed=71, frac=0.02)
    W = synth.weights_gaussian(K, N, seed=72, sigma=0.05)
    ref = _f64(X) @ _f64(W)
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    errs = []
    for k in (0, 4, 16, 64, 256):
        s, inv_s, O = oracle.calibrate(amax, wmax, 0.6, k)
        ac, asc, ahp = oracle.quantize_act(X, inv_s, O)
        wc, wsc, whp = oracle.pack_weights(W, s, O, 0)
        y, _ = oracle.dual_gemm_rows(ac, asc, ahp, np.arange(M), wc, wsc, whp)
        errs.append(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    assert errs[-1] < errs[0]
    assert errs[2] < errs[0]


def test_channel_reordering_is_invisible_to_quantize_act():
    # Permuting the channels to [J | O] (bulk ascending, then outliers
    # ascending), permuting inv_s alike and declaring the last k channels the
    # outliers gives the same codes, scales and slots as the natural layout:
    # the reading under which an FFN up-projection may emit its output columns
    # pre-ordered for the down-projection.
    M, K, k = 24, 320, 37
    X = synth.acts_heavy_tailed(M, K, seed=81, frac=0.03)
    rng = np.random.default_rng(82)
    inv_s = np.exp(rng.uniform(-0.6, 0.6, K)).astype(np.float32)
    O = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    order = np.concatenate([np.setdiff1d(np.arange(K), O), O])
    nat = oracle.quantize_act(X, inv_s, O)
    perm = oracle.quantize_act(X[:, order], inv_s[order], np.arange(K - k, K, dtype=np.int32))
    for a, b in zip(nat, perm):
        assert np.array_equal(a, b)
    # ...while reversing the bulk channels (a different compaction) changes them
    other = np.concatenate([np.setdiff1d(np.arange(K), O)[::-1], O])
    moved = oracle.quantize_act(X[:, other], inv_s[other], np.arange(K - k, K, dtype=np.int32))
    assert not np.array_equal(moved[0], nat[0])
    assert np.array_equal(moved[2], nat[2])


def test_gelu_bf16_special_values():
    # GELU(0) = 0, GELU(x) = x for large x and -0 for large -x; every value is
    # the FP64 GELU rounded once to BF16.
    y = np.array([0.0, 12.0, 300.0, -12.0, -300.0, 1.0, -1.0, 0.5, 3.0, -2.5])
    h = oracle.gelu_bf16(y)
    f = synth.bf16_bits_to_f32(h).astype(np.float64)
    assert f[0] == 0.0 and f[1] == 12.0 and f[2] == 300.0
    assert f[3] == 0.0 and f[4] == 0.0
    for yi, hi, fi in zip(y, h, f):
        assert hi == oracle.f64_to_bf16(oracle.gelu_tanh(yi))
        want = 0.5 * yi * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (yi + 0.044715 * yi ** 3)))
        assert abs(fi - want) <= 2.0 ** -8 * abs(want) + 1e-30, yi  # half a BF16 ulp


def test_fp16_outlier_branch_k_equals_K_is_a_plain_fp16_gemm():
    # With every channel on the outlier branch in FP16, y is the FP64 sum of
    # the FP16-rounded smoothed operands' products (a textbook GEMM).
    M, K, N = 8, 64, 16
    X = synth.acts_heavy_tailed(M, K, seed=91, frac=0.1)
    W = synth.weights_gaussian(K, N, seed=92, sigma=0.1)
    rng = np.random.default_rng(93)
    s = np.exp(rng.uniform(-0.5, 0.5, K)).astype(np.float32)
    inv_s = (np.float32(1.0) / s).astype(np.float32)
    O = np.arange(K, dtype=np.int32)
    ac, asc, ah = oracle.quantize_act(X, inv_s, O, hp_fp16=True)
    wc, wsc, wh = oracle.pack_weights(W, s, O, 0, hp_fp16=True)
    y, _ = oracle.dual_gemm_rows(ac, asc, ah, np.arange(M), wc, wsc, wh, hp_fp16=True)
    xs = (synth.bf16_bits_to_f32(X) * inv_s[None, :]).astype(np.float32).astype(np.float16).astype(np.float64)
    ws = (synth.bf16_bits_to_f32(W) * s[:, None]).astype(np.float32).astype(np.float16).astype(np.float64)
    assert np.allclose(y, xs @ ws, rtol=1e-13, atol=0.0)
    # bulk untouched by the outlier type
    ac2, asc2, _ = oracle.quantize_act(X, inv_s, np.arange(4, dtype=np.int32), hp_fp16=True)
    ac3, asc3, _ = oracle.quantize_act(X, inv_s, np.arange(4, dtype=np.int32), hp_fp16=False)
    assert np.array_equal(ac2, ac3) and np.array_equal(asc2, asc3)


def test_fp16_outlier_branch_is_closer_than_bf16():
    # Same outlier set: the outlier contribution (y minus the same layer with
    # the outlier slots zeroed) carries 3 more significand bits in FP16, so
    # it is closer to the exact product of the smoothed, unrounded operands.
    M, K, N, k = 64, 256, 32, 32
    X = synth.acts_heavy_tailed(M, K, seed=95, frac=0.05)
    W = synth.weights_gaussian(K, N, seed=96, sigma=0.05)
    s, inv_s, O = oracle.calibrate(oracle.act_amax(X), oracle.weight_amax(W), 0.5, k)
    xs = _f64(X)[:, O] * inv_s[O].astype(np.float64)
    ws = _f64(W)[O, :] * s[O, None].astype(np.float64)
    exact = xs @ ws
    err = {}
    for fp16 in (False, True):
        ac, asc, ah = oracle.quantize_act(X, inv_s, O, hp_fp16=fp16)
        wc, wsc, wh = oracle.pack_weights(W, s, O, 0, hp_fp16=fp16)
        y, _ = oracle.dual_gemm_rows(ac, asc, ah, np.arange(M), wc, wsc, wh, hp_fp16=fp16)
        y0, _ = oracle.dual_gemm_rows(ac, asc, np.zeros_like(ah), np.arange(M), wc, wsc, wh, hp_fp16=fp16)
        err[fp16] = np.linalg.norm((y - y0) - exact)
    assert err[True] < err[False] / 4
