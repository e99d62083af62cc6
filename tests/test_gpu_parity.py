"""CUDA path vs the oracle, through the C ABI, on seeded synthetic inputs.
Bit-exact: statistics, s / inv_s, O, E2M1 codes, E8M0 scales, the BF16
outlier buffers. Tolerance on Y: |y_gpu - y_ref| <= 1e-5 sum|a w| + 1e-6."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import outlier_split_mixed_b200 as osm  # noqa: E402
from outlier_split_mixed_b200 import synth  # noqa: E402
from gpu_helpers import (assert_bitexact, assert_y_close, compare_layer, gpu_layer, oracle_layer,  # noqa: E402
                         to_np_u16, unswizzle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    osm.lib()


# (name, M, K, N, alpha, k, mode, epi, bias, x_kind)
SMALL = [
    ("tiny_cfg", 256, 512, 1024, 0.5, 16, osm.WSCALE_1x32, osm.EPI_F32, False, "spiked"),
    ("ragged_tile32", 300, 1024, 768, 0.6, 100, osm.WSCALE_TILE32x32, osm.EPI_F32, False, "heavy"),
    ("odd_atoms_strip", 200, 640, 352, 0.6, 64, osm.WSCALE_STRIP128x1, osm.EPI_F32, True, "heavy"),
    ("k0_native", 130, 512, 256, 0.5, 0, osm.WSCALE_1x32, osm.EPI_F32, False, "heavy"),
    ("kK_pure_bf16", 64, 256, 512, 0.5, 256, osm.WSCALE_1x32, osm.EPI_F32, False, "heavy"),
    ("m1", 1, 512, 256, 0.5, 32, osm.WSCALE_1x32, osm.EPI_F32, False, "heavy"),
    ("bf16_out_bias", 257, 768, 512, 0.7, 48, osm.WSCALE_1x32, osm.EPI_BF16, True, "gelu"),
    ("long_k_wraps_ring", 257, 5120, 512, 0.6, 128, osm.WSCALE_STRIP128x1, osm.EPI_F32, False, "heavy"),
    ("k_all_but_32", 96, 512, 256, 0.5, 480, osm.WSCALE_TILE32x32, osm.EPI_F32, False, "heavy"),
    # rows too wide for the streaming quantize_act ring: the staged form
    ("wide_k_staged", 40, 32768, 64, 0.5, 64, osm.WSCALE_1x32, osm.EPI_F32, False, "heavy"),
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


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_layer_parity_small(case):
    name, M, K, N, alpha, k, mode, epi, use_bias, x_kind = case
    seed = 1000 + sum(map(ord, name))
    X, W = _inputs(M, K, N, x_kind, seed)
    bias = (np.random.default_rng(seed).standard_normal(N).astype(np.float32) * 0.1) if use_bias else None
    g = gpu_layer(X, W, alpha, k, mode, epi=epi, bias=bias, batches=3 if M > 3 else 1)
    o = oracle_layer(X, W, alpha, k, mode, bias=bias)
    compare_layer(g, o)
    assert_y_close(g["Y"], o["y"], o["T"], bf16=(epi == osm.EPI_BF16))


FP16_CASES = [c for c in SMALL if c[0] in ("tiny_cfg", "ragged_tile32", "odd_atoms_strip", "kK_pure_bf16",
                                             "bf16_out_bias", "long_k_wraps_ring", "wide_k_staged")]


@pytest.mark.parametrize("case", FP16_CASES, ids=[c[0] + "_fp16" for c in FP16_CASES])
def test_layer_parity_fp16_outlier_branch(case):
    # The FP16 outlier branch: outlier slots rounded to binary16, FP16 MMAs.
    name, M, K, N, alpha, k, mode, epi, use_bias, x_kind = case
    seed = 1000 + sum(map(ord, name))
    X, W = _inputs(M, K, N, x_kind, seed)
    bias = (np.random.default_rng(seed).standard_normal(N).astype(np.float32) * 0.1) if use_bias else None
    g = gpu_layer(X, W, alpha, k, mode, epi=epi, bias=bias, hp_fp16=True)
    o = oracle_layer(X, W, alpha, k, mode, bias=bias, hp_fp16=True)
    compare_layer(g, o)
    assert_y_close(g["Y"], o["y"], o["T"], bf16=(epi == osm.EPI_BF16))


def test_tiny_config_exact_shapes():
    cfg = synth.TINY
    X, W = cfg.make_x(), cfg.make_w()
    g = gpu_layer(X, W, cfg.alpha, cfg.k, cfg.wmode)
    o = oracle_layer(X, W, cfg.alpha, cfg.k, cfg.wmode)
    compare_layer(g, o)
    assert_y_close(g["Y"], o["y"], o["T"], bf16=False)


def _full_size(cfg, n_rows, n_wgroups=12):
    X, W = cfg.make_x(), cfg.make_w()
    epi = osm.EPI_BF16 if cfg.out_bf16 else osm.EPI_F32
    rows = synth.sample_rows(cfg.M, n_rows)
    g = gpu_layer(X, W, cfg.alpha, cfg.k, cfg.wmode, epi=epi, rows=rows)
    o = oracle_layer(X, W, cfg.alpha, cfg.k, cfg.wmode, rows=rows)
    rng = np.random.default_rng(3)
    groups = np.sort(rng.choice(cfg.N // 32, n_wgroups, replace=False))
    wr = (groups[:, None] * 32 + np.arange(32)[None, :]).ravel()
    compare_layer(g, o, check_weights_rows=wr)
    return assert_y_close(g["Y"], o["y"], o["T"], bf16=cfg.out_bf16)


def test_full_size_ffn_up():
    _full_size(synth.UP, 96)


def test_full_size_ffn_down():
    _full_size(synth.DOWN, 48)


def test_full_size_long_sequence_bf16():
    _full_size(synth.LONG, 48)


def test_short_wait_limit_reports_timeout_and_context_survives():
    # Failure detection without a fault: a wait limit far below the time
    # the pipeline needs makes the kernel's bounded waits run out; the kernel
    # must report OSM_STATUS_TIMEOUT and return, and the context must stay
    # usable for a correct run right after.
    cfg = synth.UP
    M = 1024
    X, W = cfg.make_x(M), cfg.make_w()
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    s, inv_s, O, _, _ = osm.calibrate([Xd], Wd, cfg.alpha, cfg.k)
    plan = osm.Plan(cfg.K, cfg.N, cfg.k, s, O, cfg.wmode)
    wc, wsc, wh = plan.alloc_packed(cfg.N)
    osm.pack_weights(plan, Wd, wc, wsc, wh)
    ac, asc, ah = plan.alloc_packed(M)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    Y = torch.empty((M, cfg.N), dtype=torch.float32, device="cuda")
    plan.set_wait_limit(1000)  # 1 us
    osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y)
    st = plan.status(clear=True)
    assert st & osm.STATUS_TIMEOUT
    plan.set_wait_limit(2_000_000_000)
    Y2 = torch.empty_like(Y)
    osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y2)
    assert plan.status(clear=True) == 0
    Y3 = torch.empty_like(Y)
    osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y3)
    torch.cuda.synchronize()
    assert torch.equal(Y2, Y3)  # deterministic and complete


def test_quantize_act_wait_limit_reports_timeout_and_recovers():
    # Failure detection without a fault: with the starve flag every row
    # group's wait expects bytes that never come, so each bounded wait runs
    # out (1 ms limit); the kernel reports OSM_STATUS_TIMEOUT, lets its copies
    # land and returns; the context stays usable and a normal run right after
    # equals a run on a fresh plan.
    cfg = synth.UP
    M = 1024
    X = cfg.make_x(M)
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    rng = np.random.default_rng(11)
    s = np.exp(rng.uniform(-0.5, 0.5, cfg.K)).astype(np.float32)
    O = np.sort(rng.choice(cfg.K, cfg.k, replace=False)).astype(np.int32)
    plan = osm.Plan(cfg.K, cfg.N, cfg.k, s, O, cfg.wmode)
    ac, asc, ah = plan.alloc_packed(M)
    plan.set_wait_limit(1_000_000)
    plan.set_debug(osm.DEBUG_STARVE_QUANTIZE)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    assert plan.status(clear=True) & osm.STATUS_TIMEOUT
    plan.set_debug(0)
    plan.set_wait_limit(2_000_000_000)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    assert plan.status(clear=True) == 0
    fresh = osm.Plan(cfg.K, cfg.N, cfg.k, s, O, cfg.wmode)
    bc, bsc, bh = fresh.alloc_packed(M)
    osm.quantize_act(fresh, Xd, bc, bsc, bh)
    torch.cuda.synchronize()
    assert torch.equal(ac, bc) and torch.equal(asc, bsc) and torch.equal(ah.view(torch.int16), bh.view(torch.int16))


def test_quant_linear_and_host_entry_point_agree():
    cfg = synth.TINY
    X, W = cfg.make_x(), cfg.make_w()
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    s, inv_s, O, _, _ = osm.calibrate([Xd], Wd, cfg.alpha, cfg.k)
    plan = osm.Plan(cfg.K, cfg.N, cfg.k, s, O, cfg.wmode)
    lin = osm.QuantLinear(plan, Wd)
    Y = lin.forward(Xd)
    Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((cfg.M, cfg.N), dtype=torch.float32).pin_memory()
    ws = torch.empty(osm.linear_workspace_size(plan, cfg.M), dtype=torch.uint8, device="cuda")
    osm.linear_host(plan, Xh, cfg.M, lin.w_codes, lin.w_scales, lin.w_hp, Yh, ws)
    torch.cuda.synchronize()
    assert torch.equal(Y.cpu(), Yh)


@pytest.mark.parametrize("M", [8191, 8193, 8194])
def test_quantize_act_large_batches_ragged_last_group(M):
    # Batches of 8192 rows and more at K = 5120 run the three-CTA form whose
    # register-held pairs cover K/2 exactly; an odd M leaves its last row
    # group with one row. Codes, scales (padding rows 0) and outlier slots
    # are bit-exact against the oracle on every row.
    K, k = 5120, 128
    X = synth.acts_heavy_tailed(M, K, 4242 + M, frac=0.02)
    W = synth.weights_gaussian(K, 256, 4243, sigma=0.04)
    s, inv_s, O = oracle.calibrate(oracle.act_amax(X), oracle.weight_amax(W), 0.6, k)
    plan = osm.Plan(K, 256, k, s, O, osm.WSCALE_STRIP128x1)
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda().view(torch.bfloat16)
    ac, asc, ah = plan.alloc_packed(M)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    torch.cuda.synchronize()
    assert plan.status() == 0
    codes, scales, hp = oracle.quantize_act(X, inv_s, O)
    nb = plan.Kbp // 32
    assert_bitexact("a_codes", ac.cpu().numpy().reshape(M, plan.Kbp // 2), codes)
    sc = unswizzle(asc.cpu().numpy(), M, nb)
    assert_bitexact("a_scales", sc[:M], scales)
    assert np.all(sc[M:] == 0), "padding rows of a_scales must be 0"
    assert_bitexact("a_hp", to_np_u16(ah).reshape(M, plan.kp), hp)



@pytest.mark.parametrize("fmt", ["fp16_outliers", "nvfp4"])
def test_quantize_act_large_batch_other_encodings(fmt):
    # The three-CTA paired form at K = 5120 with the FP16 outlier slots and
    # with the NVFP4 bulk encoding (E4M3 scales per 16, the per-tensor
    # exponent), odd M: bit-exact against the oracle on every row.
    M, K, k = 8193, 5120, 128
    X = synth.acts_heavy_tailed(M, K, 777, frac=0.02)
    W = synth.weights_gaussian(K, 256, 778, sigma=0.04)
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, O = oracle.calibrate(amax, wmax, 0.6, k)
    if fmt == "nvfp4":
        g_act, g_w = oracle.nvfp4_plan_exponents(amax, wmax, s, inv_s, O)
        plan = osm.Plan(K, 256, k, s, O, osm.WSCALE_1x32, fmt=osm.FMT_NVFP4, g_act=g_act, g_w=g_w)
        codes, scales, hp = oracle.quantize_act_nv(X, inv_s, O, g_act)
    else:
        plan = osm.Plan(K, 256, k, s, O, osm.WSCALE_1x32, hp_fp16=True)
        codes, scales, hp = oracle.quantize_act(X, inv_s, O, hp_fp16=True)
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda().view(torch.bfloat16)
    ac, asc, ah = plan.alloc_packed(M)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    torch.cuda.synchronize()
    assert plan.status() == 0
    nb = plan.nblocks
    assert_bitexact("a_codes", ac.cpu().numpy().reshape(M, plan.Kbp // 2), codes)
    sc = unswizzle(asc.cpu().numpy(), M, nb)
    assert_bitexact("a_scales", sc[:M], scales)
    assert np.all(sc[M:] == 0), "padding rows of a_scales must be 0"
    assert_bitexact("a_hp", to_np_u16(ah).reshape(M, plan.kp), hp)
