"""Accumulation accuracy of the dual-branch GEMM and the error-vs-k series.

1. Stress of the block-scaled MMA's accumulation (Eq. (3) of "W4A4
   Quantization for Inference on Wan2.2-I2V-A14B" fixes the exact value:
   the per-group-scaled sum of exact products). One large product at the
   start of K = 13824 and thousands of small products after it. The MMAs
   add partial sums into the FP32 accumulator -- at most one per scale
   group (32 FP4 values of K) and one per 16 BF16 values -- so the result
   can be off by at most one FP32 ulp of the running sum per addition:
       |y - y_ref| <= (n_add + 1) 2^-23 sum|a w| + 1e-6
   with n_add = Kbp/32 + kp/16 (the directed-rounding bound of the FP32
   accumulation as the tensor cores perform it). This construction is the
   adversarial case for that bound -- every small partial sum is a few
   hundred ulps of the large accumulator, all of one sign -- and the
   tensor cores' accumulation rounds toward zero there (measured: the error
   is one-signed, about half an ulp per instruction, 1.25e-5 sum|a w| at
   K = 13824, above the 1e-5 sum|a w| that realistic data stays far below).
   A sum that lost whole small products (too few alignment bits inside an
   instruction) would exceed the bound by orders of magnitude. Cases: small
   products of one sign after the large one; a large product cancelled by
   an equal and opposite one near the end, with small products of both
   signs between; and small products on the BF16 outlier branch, whose
   MMAs run after every bulk MMA into the already large accumulator.

2. The Eq. (5) argument of the paper: keeping a handful of outlier columns
   in high precision stops the largest activation tails from collapsing
   the 4-bit blocks, so the layer's relative error against the unquantised
   product falls as k grows. Measured on the Wan-like up-projection data
   (4096 tokens x 5120 -> 13824, alpha 0.6, 128x1 stripes) through the CUDA
   path for k in {0, 16, 64, 128, 256}, against the unquantised product of
   the same BF16 operands (PyTorch FP32 matmul); reported, and checked to
   fall from k = 0 to k = 256.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import outlier_split_mixed_b200 as osm  # noqa: E402
from outlier_split_mixed_b200 import synth  # noqa: E402
from gpu_helpers import assert_bitexact, to_dev_bf16, unswizzle  # noqa: E402

pytestmark = pytest.mark.gpu

E2M1 = np.array([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    osm.lib()


def _stress_inputs(case, M=256, K=13824, N=256, seed=0):
    """X [M][K], W [K][N] as float64 values on E2M1 grids times powers of two
    (exact in BF16), and the outlier set."""
    rng = np.random.default_rng(seed)
    X = np.zeros((M, K))
    W = np.zeros((K, N))
    # one large product at k = 0: +-6 x 6
    X[:, 0] = 6.0 * rng.choice([-1.0, 1.0], M)
    W[0, :] = 6.0
    small = slice(32, K)                 # every later 32-block
    xs = rng.choice(E2M1, (M, K - 32)) * 2.0 ** -10
    ws = rng.choice(E2M1, (K - 32, N)) * 2.0 ** -10
    O = np.zeros(0, np.int32)
    if case == "same_sign":
        # small products all of the large product's sign
        X[:, small] = xs * np.sign(X[:, :1])
        W[small, :] = ws
    elif case == "cancel":
        # the large product cancelled near the end of K; small products of both signs between
        X[:, small] = xs * rng.choice([-1.0, 1.0], (M, K - 32))
        W[small, :] = ws
        X[:, K - 32] = -X[:, 0]              # alone in the last 32-block of each row
        X[:, K - 31:] = 0.0
        W[K - 32, :] = 6.0
    elif case == "outlier_tail":
        # bulk: the large product and nothing else; 256 small products of one
        # sign on the BF16 branch (outlier channels), after every bulk MMA
        O = np.sort(rng.choice(np.arange(64, K), 256, replace=False)).astype(np.int32)
        X[:, O] = xs[:, :256] * 16.0 * np.sign(X[:, :1])
        W[O, :] = ws[:256] * 16.0
    else:
        raise ValueError(case)
    to = lambda a: synth.to_bf16_bits(a.astype(np.float32))  # noqa: E731  (exact: grid values)
    Xb, Wb = to(X), to(W)
    assert np.array_equal(synth.bf16_bits_to_f32(Xb), X.astype(np.float32))
    assert np.array_equal(synth.bf16_bits_to_f32(Wb), W.astype(np.float32))
    return Xb, Wb, O


@pytest.mark.parametrize("case", ["same_sign", "cancel", "outlier_tail"])
def test_block_scaled_accumulation_stress(case):
    X, W, O = _stress_inputs(case)
    M, K = X.shape
    N = W.shape[1]
    k = O.size
    s = np.ones(K, np.float32)
    plan = osm.Plan(K, N, k, s, O, osm.WSCALE_1x32)
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    ac, asc, ah = plan.alloc_packed(M)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    wc, wsc, wh = plan.alloc_packed(N)
    osm.pack_weights(plan, Wd, wc, wsc, wh)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y)
    torch.cuda.synchronize()
    assert plan.status() == 0

    ones = np.ones(K, np.float32)
    a_o = oracle.quantize_act(X, ones, O)
    w_o = oracle.pack_weights(W, ones, O, osm.WSCALE_1x32)
    assert_bitexact("a codes", ac.cpu().numpy().reshape(M, plan.Kbp // 2), a_o[0])
    assert_bitexact("a scales", unswizzle(asc.cpu().numpy(), M, plan.Kbp // 32)[:M], a_o[1])
    y, T = oracle.dual_gemm_rows(*a_o, np.arange(M), *w_o)
    # the grid values encode exactly, so the oracle's sum is X W (FP64 sums of
    # exact products; only the summation order differs)
    exact = synth.bf16_bits_to_f32(X).astype(np.float64) @ synth.bf16_bits_to_f32(W).astype(np.float64)
    assert np.all(np.abs(y - exact) <= 1e-13 * T)
    small = T - 36.0 * (2 if case == "cancel" else 1)
    assert np.all(small > 1e-3 * T) or case == "cancel", "the small products must matter at the tolerance"
    n_add = plan.Kbp // 32 + plan.kp // 16
    Yg = Y.cpu().numpy().astype(np.float64)
    err = Yg - y
    bound = (n_add + 1) * 2.0 ** -23 * T + 1e-6
    bad = np.abs(err) > bound
    assert not bad.any(), (case, int(bad.sum()), float(np.max(np.abs(err) / T)))
    print(f"{case}: n_add {n_add}, max |err| / sum|a w| = {np.max(np.abs(err) / T):.3e} "
          f"(bound {(n_add + 1) * 2.0 ** -23:.3e}), mean signed err / sum|a w| = {np.mean(err / T):.3e}")


def test_relative_error_falls_as_k_grows():
    cfg = synth.UP
    X, W = cfg.make_x(), cfg.make_w()
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    ref = Xd.float() @ Wd.float()                       # unquantised product of the same BF16 operands
    series = []
    for k in (0, 16, 64, 128, 256):
        s, _, O, _, _ = osm.calibrate([Xd], Wd, cfg.alpha, k)
        plan = osm.Plan(cfg.K, cfg.N, k, s, O, cfg.wmode)
        wc, wsc, wh = plan.alloc_packed(cfg.N)
        osm.pack_weights(plan, Wd, wc, wsc, wh)
        ac, asc, ah = plan.alloc_packed(cfg.M)
        osm.quantize_act(plan, Xd, ac, asc, ah)
        Y = torch.empty((cfg.M, cfg.N), dtype=torch.float32, device="cuda")
        osm.dual_gemm(plan, ac, asc, ah, cfg.M, wc, wsc, wh, Y)
        e, n = osm.error_norms(Y, ref)
        assert plan.status() == 0
        plan.close()
        series.append((k, float(np.sqrt(e / n))))
    print("relative Frobenius error vs k:", ", ".join(f"k={k}: {r:.4f}" for k, r in series))
    rel = [r for _, r in series]
    assert rel[-1] < rel[0]
    assert all(b <= a * 1.01 for a, b in zip(rel, rel[1:])), series
