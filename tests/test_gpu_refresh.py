"""On-device re-calibration (osm_plan_refresh): Eq. (2) and Eq. (4) of
"W4A4 Quantization for Inference on Wan2.2-I2V-A14B" recomputed from device
statistics, compared with the oracle's calibration, and a refreshed plan
compared with a plan built on the host from the same s and O."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import outlier_split_mixed_b200 as osm  # noqa: E402
from outlier_split_mixed_b200 import synth  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    osm.lib()


def _stats(K, seed, kind):
    rng = np.random.default_rng(seed)
    if kind == "ties":
        amax = rng.choice(np.array([0.5, 1.0, 2.0, 6.0], np.float32), K)   # many equal maxima
    elif kind == "all_equal":
        amax = np.full(K, 3.0, np.float32)
    else:
        amax = np.exp(rng.normal(0.0, 1.0, K)).astype(np.float32)
        amax[rng.choice(K, max(1, K // 100), replace=False)] *= 20.0
        amax[rng.choice(K, max(1, K // 200), replace=False)] = 0.0          # floored at 1e-5
        amax[rng.choice(K, max(1, K // 200), replace=False)] = 3e-6
    wmax = (rng.uniform(0.01, 0.6, K)).astype(np.float32)
    wmax[rng.choice(K, max(1, K // 300), replace=False)] = 0.0
    return amax, wmax


def _ulps(a, b):
    ai = a.view(np.int32).astype(np.int64)
    bi = b.view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


CASES = [(512, 16, "random"), (5120, 128, "random"), (13824, 256, "random"), (1024, 0, "random"),
         (256, 256, "random"), (65536, 1000, "random"), (4096, 100, "ties"), (2048, 37, "all_equal")]


@pytest.mark.parametrize("K,k,kind", CASES, ids=[f"K{c[0]}_k{c[1]}_{c[2]}" for c in CASES])
def test_refresh_matches_oracle_calibration(K, k, kind):
    amax, wmax = _stats(K, 100 + K + k, kind)
    alpha = 0.6
    O0 = np.arange(K - k, K, dtype=np.int32)       # a different initial set
    plan = osm.Plan(K, 64, k, np.full(K, 2.0, np.float32), O0, osm.WSCALE_1x32)
    plan.refresh(torch.from_numpy(amax).cuda(), torch.from_numpy(wmax).cuda(), alpha)
    torch.cuda.synchronize()
    assert plan.status(clear=True) == 0
    s_g, inv_g, O_g = plan.tables()
    s_o, inv_o, O_o = oracle.calibrate(amax, wmax, alpha, k)
    assert np.array_equal(O_g, O_o)
    d = _ulps(s_g, s_o)
    assert d.max() <= 1 and np.count_nonzero(d) <= max(1, K // 1000)
    assert np.array_equal(inv_g, (np.float32(1.0) / s_g).astype(np.float32))
    J = np.setdiff1d(np.arange(K), O_o).astype(np.int32)
    assert np.array_equal(plan.channel_order(), np.concatenate([J, O_o]))
    if kind == "all_equal":
        assert np.array_equal(O_g, np.arange(k))


def test_refreshed_plan_equals_host_built_plan():
    # Statistics taken on the device from a batch, the plan refreshed in
    # place, weights packed again: every packed byte and Y equal those of a
    # plan created on the host from the refreshed s and O.
    M, K, N, k, alpha = 300, 1024, 512, 48, 0.6
    X = synth.acts_heavy_tailed(M, K, 71, frac=0.02)
    W = synth.weights_gaussian(K, N, 72, 0.04)
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    wmax = torch.empty(K, dtype=torch.float32, device="cuda")
    osm.act_amax_accumulate(Xd, amax)
    osm.weight_amax(Wd, wmax)
    plan = osm.Plan(K, N, k, np.ones(K, np.float32), np.arange(k, dtype=np.int32), osm.WSCALE_TILE32x32)
    plan.refresh(amax, wmax, alpha)

    def run(pl):
        wc, wsc, wh = pl.alloc_packed(N)
        osm.pack_weights(pl, Wd, wc, wsc, wh)
        ac, asc, ah = pl.alloc_packed(M)
        osm.quantize_act(pl, Xd, ac, asc, ah)
        Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        osm.dual_gemm(pl, ac, asc, ah, M, wc, wsc, wh, Y)
        torch.cuda.synchronize()
        return [wc, wsc, wh.view(torch.int16), ac, asc, ah.view(torch.int16), Y]

    got = run(plan)
    s_g, _, O_g = plan.tables()
    ref_plan = osm.Plan(K, N, k, s_g, O_g, osm.WSCALE_TILE32x32)
    want = run(ref_plan)
    for a, b in zip(got, want):
        assert torch.equal(a, b)
    # and the statistics themselves are the oracle's
    s_o, _, O_o = oracle.calibrate(oracle.act_amax(X), oracle.weight_amax(W), alpha, k)
    assert np.array_equal(O_g, O_o)
    assert _ulps(s_g, s_o).max() <= 1


def test_refresh_follows_the_batch():
    # Two batches with different outlier channels: after each refresh the
    # plan's O is that batch's top-k, as a dynamic (per-step) outlier set
    # requires.
    K, N, k = 2048, 256, 32
    wmax = torch.full((K,), 0.3, dtype=torch.float32, device="cuda")
    plan = osm.Plan(K, N, k, np.ones(K, np.float32), np.arange(k, dtype=np.int32), osm.WSCALE_1x32)
    for seed in (1, 2):
        X = synth.acts_heavy_tailed(128, K, seed, frac=0.02)
        Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
        amax = torch.zeros(K, dtype=torch.float32, device="cuda")
        osm.act_amax_accumulate(Xd, amax)
        plan.refresh(amax, wmax, 0.5)
        _, _, O_g = plan.tables()
        _, _, O_o = oracle.calibrate(oracle.act_amax(X), np.full(K, 0.3, np.float32), 0.5, k)
        assert np.array_equal(O_g, O_o)


def test_refresh_with_non_finite_statistics_keeps_the_plan():
    K, k = 1024, 20
    amax, wmax = _stats(K, 5, "random")
    plan = osm.Plan(K, 64, k, np.full(K, 1.5, np.float32), np.arange(k, dtype=np.int32), osm.WSCALE_1x32)
    before = plan.tables(), plan.channel_order()
    bad = amax.copy()
    bad[17] = np.nan
    plan.refresh(torch.from_numpy(bad).cuda(), torch.from_numpy(wmax).cuda(), 0.5)
    torch.cuda.synchronize()
    assert plan.status(clear=True) & osm.STATUS_NONFINITE
    after = plan.tables(), plan.channel_order()
    for a, b in zip(before[0], after[0]):
        assert np.array_equal(a, b)
    assert np.array_equal(before[1], after[1])
    wbad = wmax.copy()
    wbad[3] = np.inf
    plan.refresh(torch.from_numpy(amax).cuda(), torch.from_numpy(wbad).cuda(), 0.5)
    torch.cuda.synchronize()
    assert plan.status(clear=True) & osm.STATUS_NONFINITE


@pytest.mark.parametrize("T,K,q", [(2048, 512, 0.999), (2048, 512, 0.99), (1000, 256, 0.5), (7, 64, 0.9),
                                   (1, 32, 0.3), (513, 1024, 1.0)])
def test_act_percentile_matches_oracle(T, K, q):
    X = synth.acts_heavy_tailed(T, K, seed=T + K, frac=0.03)
    X[: T // 3, ::5] = X[0, ::5]                       # many equal values in some columns
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    score = torch.empty(K, dtype=torch.float32, device="cuda")
    osm.act_percentile(Xd, q, score)
    want = oracle.act_percentile(X, oracle.percentile_rank(q, T))
    assert np.array_equal(score.cpu().numpy(), want)
    if q == 1.0:
        assert np.array_equal(want, oracle.act_amax(X))


def test_scored_refresh_matches_oracle():
    T, K, k, alpha = 1024, 2048, 40, 0.55
    X = synth.acts_heavy_tailed(T, K, seed=91, frac=0.02)
    quiet = int(np.argmin(oracle.act_amax(X)))
    X[3, quiet] = synth.to_bf16_bits(np.array([60.0], np.float32))[0]   # a one-token spike
    W = synth.weights_gaussian(K, 128, 92, 0.04)
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    score = torch.empty(K, dtype=torch.float32, device="cuda")
    wmax = torch.empty(K, dtype=torch.float32, device="cuda")
    osm.act_amax_accumulate(Xd, amax)
    osm.act_percentile(Xd, 0.99, score)
    osm.weight_amax(Wd, wmax)
    plan = osm.Plan(K, 128, k, np.ones(K, np.float32), np.arange(k, dtype=np.int32), osm.WSCALE_1x32)
    plan.refresh_scored(amax, score, wmax, alpha)
    s_g, _, O_g = plan.tables()
    am_o, wm_o = oracle.act_amax(X), oracle.weight_amax(W)
    sc_o = oracle.act_percentile(X, oracle.percentile_rank(0.99, T))
    s_o, _, O_o = oracle.calibrate_scored(am_o, sc_o, wm_o, alpha, k)
    assert np.array_equal(O_g, O_o)
    assert _ulps(s_g, s_o).max() <= 1
    assert quiet not in O_g                           # the spike does not decide the mask
    assert quiet in oracle.calibrate(am_o, wm_o, alpha, k)[2]           # ... while the maximum would
    # the host path on the same device statistics agrees
    h = osm.calibrate_finalize_scored(amax.cpu().numpy(), score.cpu().numpy(), wmax.cpu().numpy(), alpha, k)
    assert np.array_equal(h[2], O_g)
