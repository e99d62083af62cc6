"""NVFP4 bulk format on the CUDA path vs the oracle, through the C ABI.
Bit-exact: the per-tensor exponents, E2M1 codes, UE4M3 scales (after
un-swizzle), the 2^-g-scaled BF16 outlier buffers. Tolerance on Y:
|y_gpu - y_ref| <= 1e-5 sum|a w| + 1e-6 (+ 2^-8 |y| for BF16 outputs)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import outlier_split_mixed_b200 as osm  # noqa: E402
from outlier_split_mixed_b200 import synth  # noqa: E402
from gpu_helpers import assert_y_close, compare_layer, gpu_layer, oracle_layer, to_dev_bf16  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    osm.lib()


# (name, M, K, N, alpha, k, epi, bias, x_kind)
CASES = [
    ("tiny", 256, 512, 1024, 0.5, 16, osm.EPI_F32, False, "spiked"),
    ("ragged", 300, 1024, 768, 0.6, 100, osm.EPI_F32, False, "heavy"),      # Kb = 924: a ragged 16-block
    ("odd_atoms", 200, 640, 352, 0.6, 64, osm.EPI_F32, True, "heavy"),      # Kbp = 640: a partial ring slot
    ("k0", 130, 512, 256, 0.5, 0, osm.EPI_F32, False, "heavy"),
    ("kK", 64, 256, 512, 0.5, 256, osm.EPI_F32, False, "heavy"),
    ("m1", 1, 512, 256, 0.5, 32, osm.EPI_F32, False, "heavy"),
    ("bf16_bias", 257, 768, 512, 0.7, 48, osm.EPI_BF16, True, "gelu"),
    ("long_k", 257, 5120, 512, 0.6, 128, osm.EPI_F32, False, "heavy"),       # wraps the 5-slot ring
    ("wide_k_staged", 40, 32768, 64, 0.5, 64, osm.EPI_F32, False, "heavy"),
]


def _inputs(M, K, N, x_kind, seed):
    if x_kind == "spiked":
        X = synth.acts_gaussian_spiked(M, K, seed)
    elif x_kind == "heavy":
        X = synth.acts_heavy_tailed(M, K, seed, frac=0.02)
    else:
        X = synth.acts_gelu_boosted(M, K, seed, frac=0.02)
    W = synth.weights_gaussian(K, N, seed + 1, sigma=0.04)
    return X, W


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_nvfp4_layer_parity(case):
    name, M, K, N, alpha, k, epi, use_bias, x_kind = case
    seed = 2000 + sum(map(ord, name))
    X, W = _inputs(M, K, N, x_kind, seed)
    bias = (np.random.default_rng(seed).standard_normal(N).astype(np.float32) * 0.1) if use_bias else None
    g = gpu_layer(X, W, alpha, k, osm.WSCALE_1x32, epi=epi, bias=bias, batches=2 if M > 2 else 1, nv=True)
    o = oracle_layer(X, W, alpha, k, osm.WSCALE_1x32, bias=bias, nv=True)
    compare_layer(g, o)
    assert_y_close(g["Y"], o["y"], o["T"], bf16=(epi == osm.EPI_BF16))


def test_nvfp4_gelu_bf16_epilogue():
    # GELU_BF16 applies GELU to 2^(g_a+g_w) acc: checked by tolerance against
    # the FP64 GELU of the oracle's accumulators
    M, K, N, k = 128, 512, 256, 32
    X, W = _inputs(M, K, N, "heavy", 5)
    g = gpu_layer(X, W, 0.5, k, osm.WSCALE_1x32, epi=osm.EPI_GELU_BF16, nv=True)
    o = oracle_layer(X, W, 0.5, k, osm.WSCALE_1x32, nv=True)
    compare_layer(g, o)
    import oracle
    want = oracle.gelu(o["y"])
    # |GELU'| <= 1.13: the accumulation bound carried through GELU, plus one
    # BF16 rounding and the FP32 routine's error against the FP64 definition
    tol = (1.13 * (1e-5 * o["T"] + 1e-6) + 5e-7 * np.abs(want) + 2e-8 * np.abs(o["y"])
           + 2.0 ** -8 * (1.0 + 1e-6) * np.abs(want) + 1e-30)
    assert np.all(np.abs(g["Y"] - want) <= tol)


def test_full_size_ffn_up_nvfp4():
    cfg = synth.UP
    X, W = cfg.make_x(), cfg.make_w()
    rows = synth.sample_rows(cfg.M, 64)
    g = gpu_layer(X, W, cfg.alpha, cfg.k, osm.WSCALE_1x32, rows=rows, nv=True)
    o = oracle_layer(X, W, cfg.alpha, cfg.k, osm.WSCALE_1x32, rows=rows, nv=True)
    rng = np.random.default_rng(3)
    groups = np.sort(rng.choice(cfg.N // 32, 12, replace=False))
    wr = (groups[:, None] * 32 + np.arange(32)[None, :]).ravel()
    compare_layer(g, o, check_weights_rows=wr)
    assert_y_close(g["Y"], o["y"], o["T"], bf16=False)


def test_nvfp4_requires_mx_for_fused_requant_and_1x32_mode():
    rng = np.random.default_rng(0)
    K, N = 256, 256
    s = np.ones(K, np.float32)
    O = np.arange(16, dtype=np.int32)
    with pytest.raises(osm.OsmError):
        osm.Plan(K, N, 16, s, O, osm.WSCALE_TILE32x32, fmt=osm.FMT_NVFP4)
    with pytest.raises(osm.OsmError):
        osm.Plan(K, N, 16, s, O, osm.WSCALE_1x32, hp_fp16=True, fmt=osm.FMT_NVFP4)
    with pytest.raises(osm.OsmError):
        osm.Plan(K, N, 16, s, O, osm.WSCALE_1x32, fmt=osm.FMT_NVFP4, g_act=101)
    up = osm.Plan(K, N, 16, s, O, osm.WSCALE_1x32, fmt=osm.FMT_NVFP4, g_act=-3, g_w=-5)
    nxt = osm.Plan(N, 128, 16, np.ones(N, np.float32), O, osm.WSCALE_1x32)
    W = to_dev_bf16(synth.weights_gaussian(K, N, 1, 0.05))
    X = to_dev_bf16(synth.acts_heavy_tailed(64, K, 2))
    wc, wsc, wh = up.alloc_packed(N)
    osm.pack_weights_for_next(up, nxt, W, wc, wsc, wh)
    ac, asc, ah = up.alloc_packed(64)
    osm.quantize_act(up, X, ac, asc, ah)
    nc, ns, nh = nxt.alloc_packed(64)
    with pytest.raises(osm.OsmError):
        osm.dual_gemm(up, ac, asc, ah, 64, wc, wsc, wh, None, epi=osm.EPI_GELU_REQUANT, next_plan=nxt,
                      next_buffers=(nc, ns, nh))
    torch.cuda.synchronize()
    assert up.status() == 0
    assert rng is not None


def test_nvfp4_scales_buffer_size():
    K, N, k = 1024, 256, 100
    plan = osm.Plan(K, N, k, np.ones(K, np.float32), np.arange(k, dtype=np.int32), osm.WSCALE_1x32)
    _, mx_bytes, _ = plan.sizes(300)
    plan.set_format(osm.FMT_NVFP4, 0, 0)
    _, nv_bytes, _ = plan.sizes(300)
    assert nv_bytes == 2 * mx_bytes == 384 * (plan.Kbp // 16)
