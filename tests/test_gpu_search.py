"""Per-layer alpha / k search on the CUDA path against the same search on the
oracle: every candidate's relative output error, and the choice."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import outlier_split_mixed_b200 as osm  # noqa: E402
from outlier_split_mixed_b200 import synth  # noqa: E402
from outlier_split_mixed_b200.search import search_alpha_k  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    osm.lib()


def test_error_norms_match_fp64():
    rng = np.random.default_rng(1)
    y = rng.normal(0, 1, (777, 333)).astype(np.float32)
    r = (y + rng.normal(0, 0.01, y.shape)).astype(np.float32)
    e, n = osm.error_norms(torch.from_numpy(y).cuda(), torch.from_numpy(r).cuda())
    d = y.astype(np.float64) - r.astype(np.float64)
    assert abs(e - np.sum(d * d)) <= 1e-12 * np.sum(d * d)
    assert abs(n - np.sum(r.astype(np.float64) ** 2)) <= 1e-12 * np.sum(r.astype(np.float64) ** 2)


def _oracle_rel_err(X, W, alpha, k, mode):
    s, inv_s, O = oracle.calibrate(oracle.act_amax(X), oracle.weight_amax(W), alpha, k)
    ac, asc, ah = oracle.quantize_act(X, inv_s, O)
    wc, wsc, wh = oracle.pack_weights(W, s, O, mode)
    y, _ = oracle.dual_gemm_rows(ac, asc, ah, np.arange(X.shape[0]), wc, wsc, wh)
    ref = synth.bf16_bits_to_f32(X).astype(np.float64) @ synth.bf16_bits_to_f32(W).astype(np.float64)
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def test_search_matches_the_oracle():
    M, K, N = 256, 512, 256
    X = synth.acts_heavy_tailed(M, K, seed=51, frac=0.03)
    W = synth.weights_gaussian(K, N, 52, 0.04)
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    alphas, ks = [0.3, 0.5, 0.7], [0, 16, 64]
    r = search_alpha_k(Xd, Wd, alphas, ks, wmode=osm.WSCALE_1x32)
    want = {(a, k): _oracle_rel_err(X, W, a, k, osm.WSCALE_1x32) for k in ks for a in alphas}
    for a, k, e in r.table:
        assert abs(e - want[(a, k)]) <= 1e-5, (a, k, e, want[(a, k)])
    best = min(want.items(), key=lambda kv: kv[1])
    second = sorted(want.values())[1]
    if second - best[1] > 1e-4:
        assert (r.alpha, r.k) == best[0]
    # more outlier channels help on heavy-tailed data
    assert min(e for a, k, e in r.table if k == 64) < min(e for a, k, e in r.table if k == 0)
