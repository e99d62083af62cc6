"""The allocation-free forward (osm_linear_noalloc) against the regular
entry points (osm_quantize_act + osm_dual_gemm on caller-owned buffers).

osm_linear_noalloc exists for callers that cannot allocate device memory
while the layer runs (a serving runtime whose pool owns the GPU's memory,
a plug-in that its host framework hands only tensors and a stream); its
packed activations live in a static device array inside the library. Both
paths run the same kernels on the same operands, so their outputs must be
bit-identical: any difference would be a fault in the shared scratch's
layout. This module is self-contained so it passes alone in a fresh
process and after the rest of the suite."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import outlier_split_mixed_b200 as osm  # noqa: E402
from outlier_split_mixed_b200 import synth  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from outlier_split_mixed_b200 import build
    build.build()
    cfg = synth.UP
    W = cfg.make_w()
    X = cfg.make_x(1024)
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    s, inv_s, O, _, _ = osm.calibrate([Xd], Wd, cfg.alpha, cfg.k)
    plan = osm.Plan(cfg.K, cfg.N, cfg.k, s, O, cfg.wmode)
    wc, wsc, wh = plan.alloc_packed(cfg.N)
    osm.pack_weights(plan, Wd, wc, wsc, wh)
    bias = torch.from_numpy(np.random.default_rng(5).standard_normal(cfg.N).astype(np.float32) * 0.1).cuda()
    return cfg, plan, (wc, wsc, wh), bias


def _reference(plan, X, wpack, bias, epi):
    M = X.shape[0]
    ac, asc, ah = plan.alloc_packed(M)
    osm.quantize_act(plan, X, ac, asc, ah)
    Y = torch.empty((M, plan.N), dtype=torch.float32 if epi == osm.EPI_F32 else torch.bfloat16, device="cuda")
    osm.dual_gemm(plan, ac, asc, ah, M, *wpack, Y, bias=bias, epi=epi)
    return Y


def _same(a, b):
    # bit for bit: the same kernels on the same packed operands
    assert a.dtype == b.dtype and a.shape == b.shape
    assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a.view(torch.int16),
                       b.view(torch.int32) if b.dtype == torch.float32 else b.view(torch.int16))


@pytest.mark.parametrize("epi", [osm.EPI_F32, osm.EPI_BF16])
def test_two_calls_in_a_row_match_the_regular_path(layer, epi):
    cfg, plan, wpack, bias = layer
    # two different batches back to back: the second call must not see the
    # first call's leftovers in the shared scratch
    X1 = torch.from_numpy(synth.acts_heavy_tailed(1000, cfg.K, seed=77).view(np.int16)).cuda().view(torch.bfloat16)
    X2 = torch.from_numpy(synth.acts_heavy_tailed(333, cfg.K, seed=78).view(np.int16)).cuda().view(torch.bfloat16)
    ydt = torch.float32 if epi == osm.EPI_F32 else torch.bfloat16
    Y1 = torch.empty((1000, cfg.N), dtype=ydt, device="cuda")
    Y2 = torch.empty((333, cfg.N), dtype=ydt, device="cuda")
    osm.linear_noalloc(plan, X1, *wpack, Y1, bias=bias, epi=epi)
    osm.linear_noalloc(plan, X2, *wpack, Y2, bias=bias, epi=epi)
    torch.cuda.synchronize()
    assert plan.status() == 0
    _same(Y1, _reference(plan, X1, wpack, bias, epi))
    _same(Y2, _reference(plan, X2, wpack, bias, epi))


def test_allocates_nothing_and_rejects_oversized_batches(layer):
    cfg, plan, wpack, bias = layer
    X = torch.from_numpy(synth.acts_heavy_tailed(512, cfg.K, seed=79).view(np.int16)).cuda().view(torch.bfloat16)
    Y = torch.empty((512, cfg.N), dtype=torch.float32, device="cuda")
    osm.linear_noalloc(plan, X, *wpack, Y)  # first call on the device sets up the scratch address
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        osm.linear_noalloc(plan, X, *wpack, Y)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    # a batch whose packed activations exceed the static scratch is refused up front
    cb, sb, hb = plan.sizes(1)
    too_many = osm.NOALLOC_SCRATCH_BYTES // (cb + hb) + 256
    Xbig = torch.empty((too_many, cfg.K), dtype=torch.bfloat16, device="cuda")
    Ybig = torch.empty((1, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(osm.OsmError) as e:
        osm._check(osm.lib().osm_linear_noalloc(plan.handle, osm._ptr(Xbig, "X"), too_many,
                                                osm._ptr(wpack[0], "w"), osm._ptr(wpack[1], "s"),
                                                osm._ptr(wpack[2], "h"), None, osm.EPI_F32, osm._ptr(Ybig, "Y"),
                                                osm._stream(None)))
    assert e.value.code == osm.ERR_UNSUPPORTED and "static scratch" in str(e.value)
    # absurd batch sizes are refused before the size arithmetic (whose 64-bit
    # products would wrap to a small number at M = 2^59 for this plan)
    for huge in (1 << 59, (1 << 63) - 1, osm.NOALLOC_SCRATCH_BYTES + 1):
        with pytest.raises(osm.OsmError) as e:
            osm._check(osm.lib().osm_linear_noalloc(plan.handle, osm._ptr(Xbig, "X"), huge,
                                                    osm._ptr(wpack[0], "w"), osm._ptr(wpack[1], "s"),
                                                    osm._ptr(wpack[2], "h"), None, osm.EPI_F32,
                                                    osm._ptr(Ybig, "Y"), osm._stream(None)))
        assert e.value.code == osm.ERR_UNSUPPORTED and "static scratch" in str(e.value)
    torch.cuda.synchronize()
    assert plan.status() == 0
