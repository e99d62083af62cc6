"""The FFN epilogues of dual_gemm: OSM_EPI_GELU_BF16 and the fused
OSM_EPI_GELU_REQUANT, which hands the hidden activations of an FFN
up-projection to the down-projection already smoothed, split and
MXFP4-encoded (implementation paragraph of "W4A4 Quantization for
Inference on Wan2.2-I2V-A14B": activations divided by s, quantised,
routed).

The oracle's GELU is the plain FP64 definition; the kernel evaluates its
own FP32 routine, so its BF16 output is held to the FP64 value by a bound
(the accumulation bound carried through GELU, |GELU'| <= 1.13, plus one BF16
rounding and the routine's own error), while the fused requantisation is
checked bit for bit against the oracle's quantize_act applied to the
GPU's hidden activations from the same accumulators (the GELU_BF16
epilogue's output)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import outlier_split_mixed_b200 as osm  # noqa: E402
from outlier_split_mixed_b200 import synth  # noqa: E402
from gpu_helpers import assert_bitexact, gelu_tolerance, to_dev_bf16, to_np_u16, unswizzle  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    osm.lib()


def _grid_values(rng, shape, scale_exp):
    # magnitudes 4 or 6 (E2M1 values, so every 32-block has exponent 0 before
    # the power-of-two scale) with random signs: every product and every
    # partial sum of the layer is then exact in FP32
    mags = rng.choice(np.array([4.0, 6.0], np.float32), size=shape)
    signs = rng.choice(np.array([-1.0, 1.0], np.float32), size=shape)
    return synth.to_bf16_bits(mags * signs * np.float32(2.0 ** scale_exp))


def _order(K, O):
    return np.concatenate([np.setdiff1d(np.arange(K), O), O]).astype(np.int32)


def _assert_gelu_close(H_gpu, y, T, name):
    """H_gpu (BF16 as float64) against GELU(y) of the oracle's FP64
    accumulators y, within gelu_tolerance."""
    g = oracle.gelu(y)
    tol = gelu_tolerance(y, T, g)
    err = np.abs(H_gpu - g)
    bad = err > tol
    assert not bad.any(), (name, int(bad.sum()), np.argwhere(bad)[:3].tolist())
    return float(np.max(err / np.maximum(np.abs(g), 1e-30)))


def test_fused_requant_is_bitexact_with_exact_accumulators():
    rng = np.random.default_rng(2024)
    M, K, N, k = 300, 512, 768, 32            # up-projection: K -> N = next K
    Nn, kn = 256, 64                          # next (down) layer: N -> Nn with kn outliers
    X = _grid_values(rng, (M, K), 0)
    W = _grid_values(rng, (K, N), -10)
    O_up = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    s_up = np.ones(K, np.float32)
    s_next = np.exp(rng.uniform(-0.7, 0.7, N)).astype(np.float32)
    O_next = np.sort(rng.choice(N, kn, replace=False)).astype(np.int32)
    inv_next = (np.float32(1.0) / s_next).astype(np.float32)
    order = _order(N, O_next)

    # ---- CUDA path
    up = osm.Plan(K, N, k, s_up, O_up, osm.WSCALE_STRIP128x1)
    nxt = osm.Plan(N, Nn, kn, s_next, O_next, osm.WSCALE_1x32)
    assert np.array_equal(nxt.channel_order(), order)
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    ac, asc, ah = up.alloc_packed(M)
    osm.quantize_act(up, Xd, ac, asc, ah)
    wc, wsc, wh = up.alloc_packed(N)
    osm.pack_weights_for_next(up, nxt, Wd, wc, wsc, wh)
    nc, ns, nh = nxt.alloc_packed(M)
    osm.dual_gemm(up, ac, asc, ah, M, wc, wsc, wh, None, epi=osm.EPI_GELU_REQUANT, next_plan=nxt,
                  next_buffers=(nc, ns, nh))
    # GELU_BF16 on the natural packing
    wc2, wsc2, wh2 = up.alloc_packed(N)
    osm.pack_weights(up, Wd, wc2, wsc2, wh2)
    H = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    osm.dual_gemm(up, ac, asc, ah, M, wc2, wsc2, wh2, H, epi=osm.EPI_GELU_BF16)
    torch.cuda.synchronize()
    assert up.status() == 0

    # ---- oracle: natural order
    ac_o, asc_o, ah_o = oracle.quantize_act(X, s_up, O_up)
    wc_o, wsc_o, wh_o = oracle.pack_weights(W, s_up, O_up, osm.WSCALE_STRIP128x1)
    y, T = oracle.dual_gemm_rows(ac_o, asc_o, ah_o, np.arange(M), wc_o, wsc_o, wh_o)
    assert np.array_equal(y, y.astype(np.float32).astype(np.float64)), "construction: accumulators exact in FP32"
    # GELU of exact accumulators: only the routine's error and one rounding remain
    H_gpu = to_np_u16(H)
    _assert_gelu_close(synth.bf16_bits_to_f32(H_gpu).astype(np.float64), y, np.zeros_like(T), "GELU_BF16")
    # fused requantisation = the oracle's quantize_act of the GPU's H, bit for bit
    nc_o, ns_o, nh_o = oracle.quantize_act(H_gpu, inv_next, O_next)
    assert_bitexact("next codes", nc.cpu().numpy().reshape(M, nxt.Kbp // 2), nc_o)
    sc = unswizzle(ns.cpu().numpy(), M, nxt.Kbp // 32)
    assert_bitexact("next scales", sc[:M], ns_o)
    assert np.all(sc[M:] == 0)
    assert_bitexact("next outlier slots", to_np_u16(nh).reshape(M, nxt.kp), nh_o)


@pytest.mark.parametrize("shape", [(512, 1024, 1536, 32, 48, False), (130, 512, 1024, 0, 64, False),
                                   (256, 512, 768, 64, 0, False), (512, 1024, 1536, 32, 48, True)],
                         ids=["partial_bulk_block", "up_k0", "next_k0", "next_fp16_outliers"])
def test_fused_requant_equals_gelu_bf16_then_quantize(shape):
    # Realistic data: the fused epilogue must equal the unfused pipeline
    # (GELU_BF16 epilogue, then quantize_act of the next layer) bit for bit,
    # since both see the same FP32 accumulators.
    M, K, N, k, kn, next_fp16 = shape
    X = synth.acts_heavy_tailed(M, K, seed=600 + K, frac=0.02)
    W = synth.weights_gaussian(K, N, seed=601 + K, sigma=0.04)
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    s, _, O, _, _ = osm.calibrate([Xd], Wd, 0.6, k)
    up = osm.Plan(K, N, k, s, O, osm.WSCALE_STRIP128x1)
    ac, asc, ah = up.alloc_packed(M)
    osm.quantize_act(up, Xd, ac, asc, ah)
    wc, wsc, wh = up.alloc_packed(N)
    osm.pack_weights(up, Wd, wc, wsc, wh)
    H = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    osm.dual_gemm(up, ac, asc, ah, M, wc, wsc, wh, H, epi=osm.EPI_GELU_BF16)
    Wn = synth.weights_gaussian(N, 256, seed=602 + K, sigma=0.02)
    sn, _, On, _, _ = osm.calibrate([H], to_dev_bf16(Wn), 0.5, kn)
    nxt = osm.Plan(N, 256, kn, sn, On, osm.WSCALE_TILE32x32, hp_fp16=next_fp16)
    c1, s1, h1 = nxt.alloc_packed(M)
    osm.quantize_act(nxt, H, c1, s1, h1)
    wc2, wsc2, wh2 = up.alloc_packed(N)
    osm.pack_weights_for_next(up, nxt, Wd, wc2, wsc2, wh2)
    c2, s2, h2 = nxt.alloc_packed(M)
    for t in (c2, s2):
        t.fill_(0xAB)          # stale bytes must all be overwritten
    h2.fill_(3.0)
    osm.dual_gemm(up, ac, asc, ah, M, wc2, wsc2, wh2, None, epi=osm.EPI_GELU_REQUANT, next_plan=nxt,
                  next_buffers=(c2, s2, h2))
    torch.cuda.synchronize()
    assert up.status() == 0
    # against the oracle: its quantize_act of the GPU's H with the next plan
    H_gpu = to_np_u16(H)
    s_o, inv_o, O_o = oracle.calibrate(oracle.act_amax(H_gpu), oracle.weight_amax(Wn), 0.5, kn)
    s_p, inv_p, O_p = nxt.tables()
    assert_bitexact("next s", s_p, s_o)
    assert_bitexact("next O", O_p, O_o)
    nc_o, ns_o, nh_o = oracle.quantize_act(H_gpu, inv_o, O_o, hp_fp16=next_fp16)
    assert_bitexact("next codes", c2.cpu().numpy().reshape(M, nxt.Kbp // 2), nc_o)
    sc = unswizzle(s2.cpu().numpy(), M, nxt.Kbp // 32)
    assert_bitexact("next scales", sc[:M], ns_o)
    assert np.all(sc[M:] == 0)
    assert_bitexact("next outlier slots", to_np_u16(h2).reshape(M, nxt.kp), nh_o)
    # and the unfused GPU pipeline gives the same bytes
    assert torch.equal(c1, c2)
    assert torch.equal(s1, s2)
    assert torch.equal(h1.view(torch.int16), h2.view(torch.int16))


def test_gelu_bf16_epilogue_tracks_the_oracle_on_real_data():
    # Accumulators differ from the FP64 sums by FP32 rounding, so compare the
    # GELU outputs with the FP64 GELU of the oracle's sums within the
    # accumulation bound pushed through GELU (|GELU'| <= 1.13), one BF16
    # rounding and the routine's error.
    M, K, N, k = 200, 768, 512, 48
    X = synth.acts_heavy_tailed(M, K, seed=611, frac=0.02)
    W = synth.weights_gaussian(K, N, seed=612, sigma=0.04)
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    s, inv_s, O, _, _ = osm.calibrate([Xd], Wd, 0.6, k)
    plan = osm.Plan(K, N, k, s, O, osm.WSCALE_1x32)
    ac, asc, ah = plan.alloc_packed(M)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    wc, wsc, wh = plan.alloc_packed(N)
    osm.pack_weights(plan, Wd, wc, wsc, wh)
    H = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, H, epi=osm.EPI_GELU_BF16)
    torch.cuda.synchronize()
    so, inv_so, Oo = oracle.calibrate(oracle.act_amax(X), oracle.weight_amax(W), 0.6, k)
    ac_o, asc_o, ah_o = oracle.quantize_act(X, inv_so, Oo)
    wc_o, wsc_o, wh_o = oracle.pack_weights(W, so, Oo, 0)
    y, T = oracle.dual_gemm_rows(ac_o, asc_o, ah_o, np.arange(M), wc_o, wsc_o, wh_o)
    h = H.float().cpu().numpy().astype(np.float64)
    _assert_gelu_close(h, y, T, "GELU_BF16 on real data")


def test_gelu_epilogue_on_every_bf16_value_against_the_fp64_definition():
    # Exact accumulators acc = w: X is the identity (64 x 64), every channel
    # on the BF16 branch with s = 1, so row t of Y is GELU of row t of W. W
    # holds every BF16 value with 2^-20 <= |w| < 16 (both signs) plus 0, so
    # the epilogue's FP32 routine is checked on every input it can meet in
    # that range: |h - GELU(w)| <= 5e-7 |GELU(w)| + 2e-8 |w| + half a BF16 ulp.
    mags = np.arange(0x3580, 0x4180, dtype=np.uint32)          # 2^-20 .. 16 (exclusive)
    vals = np.concatenate([mags, mags | 0x8000, [0]]).astype(np.uint16)
    K = 64
    N = -(-vals.size // K // 32) * 32
    Wb = np.zeros(K * N, np.uint16)
    Wb[:vals.size] = vals
    W = Wb.reshape(K, N)
    X = np.zeros((K, K), np.uint16)
    X[np.arange(K), np.arange(K)] = 0x3F80                      # 1.0
    plan = osm.Plan(K, N, K, np.ones(K, np.float32), np.arange(K, dtype=np.int32), osm.WSCALE_1x32)
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    ac, asc, ah = plan.alloc_packed(K)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    wc, wsc, wh = plan.alloc_packed(N)
    osm.pack_weights(plan, Wd, wc, wsc, wh)
    H = torch.empty((K, N), dtype=torch.bfloat16, device="cuda")
    osm.dual_gemm(plan, ac, asc, ah, K, wc, wsc, wh, H, epi=osm.EPI_GELU_BF16)
    torch.cuda.synchronize()
    assert plan.status() == 0
    y = synth.bf16_bits_to_f32(W).astype(np.float64)
    h = H.float().cpu().numpy().astype(np.float64)
    g = oracle.gelu(y)
    tol = 5e-7 * np.abs(g) + 2e-8 * np.abs(y) + 2.0 ** -8 * (1.0 + 1e-6) * np.abs(g) + 1e-38
    bad = np.abs(h - g) > tol
    assert not bad.any(), [(y[i], h[i], g[i]) for i in map(tuple, np.argwhere(bad)[:3])]
    # away from the far left tail (where GELU is tiny and the routine's
    # relative error grows with |u|) the result is the correctly rounded BF16
    # of GELU(w) but for inputs whose GELU lies within the routine's error of
    # a BF16 rounding boundary
    exact = np.array([oracle.f64_to_bf16(v) for v in g.ravel()], np.uint16).reshape(g.shape)
    core = y >= -3.0
    assert np.mean((to_np_u16(H) == exact)[core]) > 0.995


def test_gelu_routine_against_the_fp64_definition():
    # the epilogues' FP32 routine itself (osm_gelu_f32), no BF16 rounding:
    # within 5e-7 |GELU(x)| + 2e-8 |x| of the FP64 GELU, on a dense grid over
    # the range FFN accumulators take and on random magnitudes up to 1e4
    rng = np.random.default_rng(31)
    x = np.concatenate([np.linspace(-12.0, 12.0, 2_000_001), np.linspace(-1e-3, 1e-3, 20001),
                        rng.standard_normal(1_000_000) * 3.0,
                        np.ldexp(rng.uniform(1, 2, 100000), rng.integers(-40, 14, 100000))
                        * rng.choice([-1.0, 1.0], 100000), [0.0, -0.0, 1e-30, -1e-30, 80.0, -80.0]]
                       ).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    g = osm.gelu_f32(xd).cpu().numpy().astype(np.float64)
    xs = x.astype(np.float64)
    G = oracle.gelu(xs)
    err = np.abs(g - G)
    tol = 5e-7 * np.abs(G) + 2e-8 * np.abs(xs) + 1e-38
    bad = err > tol
    assert not bad.any(), [(float(xs[i]), float(g[i]), float(G[i])) for i in np.argwhere(bad)[:3, 0]]
    print(f"GELU routine: max |err| / (5e-7 |G| + 2e-8 |x|) = {np.max(err / tol):.3f}")
