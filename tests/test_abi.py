"""The C ABI boundary on the host: libosm loads, exports every entry point
that include/osm.h declares, and its host-only entry points agree with the
oracle. No device work is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import outlier_split_mixed_b200 as osm
from conftest import ROOT
from outlier_split_mixed_b200 import synth


@pytest.fixture(scope="module", autouse=True)
def built():
    from outlier_split_mixed_b200 import build
    build.build()


def _declared():
    txt = open(os.path.join(ROOT, "include", "osm.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(osm_[a-z_0-9]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 15
    L = ctypes.CDLL(osm.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(osm._SIGNATURES), "binding and header disagree"


def test_library_is_built_for_sm100a_only():
    # the fatbinary in the library carries sm_100a code (checked via the
    # build flags, which are the single source of the architecture)
    from outlier_split_mixed_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.FLAGS)


def test_calibrate_finalize_matches_oracle_bitexact():
    for seed, (T, K, N, alpha, k) in enumerate([(200, 512, 64, 0.5, 16), (97, 1024, 96, 0.6, 128),
                                               (64, 256, 32, 0.7, 256), (50, 320, 64, 0.3, 0)]):
        X = synth.acts_heavy_tailed(T, K, seed=100 + seed, frac=0.03)
        W = synth.weights_gaussian(K, N, seed=200 + seed, sigma=0.03)
        amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
        amax[::37] = 0.0  # exercise the 1e-5 floor
        s, inv_s, O = osm.calibrate_finalize(amax, wmax, alpha, k)
        so, inv_so, Oo = oracle.calibrate(amax, wmax, alpha, k)
        assert np.array_equal(s.view(np.uint32), so.view(np.uint32))
        assert np.array_equal(inv_s.view(np.uint32), inv_so.view(np.uint32))
        assert np.array_equal(O, Oo)


def test_calibrate_finalize_ties_and_errors():
    amax = np.array([1, 3, 3, 2, 3, 0], np.float32)
    wmax = np.ones(6, np.float32)
    _, _, O = osm.calibrate_finalize(amax, wmax, 0.5, 2)
    assert list(O) == [1, 2]
    with pytest.raises(osm.OsmError) as e:
        osm.calibrate_finalize(np.array([1, np.nan], np.float32), np.ones(2, np.float32), 0.5, 1)
    assert e.value.code == osm.ERR_NONFINITE
    for bad_alpha in (0.0, 1.0, -0.1):
        with pytest.raises(osm.OsmError) as e:
            osm.calibrate_finalize(np.ones(4, np.float32), np.ones(4, np.float32), bad_alpha, 1)
        assert e.value.code == osm.ERR_INVALID_ARG
    with pytest.raises(osm.OsmError):
        osm.calibrate_finalize(np.ones(4, np.float32), np.ones(4, np.float32), 0.5, 5)


def _unswizzle(sw, rows, nb):
    # the atom layout written out independently: 128-row x 4-block atoms of
    # 512 bytes, K-atoms contiguous; inside, (r % 32) * 16 + (r // 32 % 4) * 4 + b % 4
    out = np.zeros((rows, nb), np.uint8)
    katoms = nb // 4
    for r in range(rows):
        for b in range(nb):
            out[r, b] = sw[((r // 128) * katoms + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4]
    return out


def test_scales_to_logical_matches_layout_definition():
    rows, nb = 300, 12
    rng = np.random.default_rng(0)
    sw = rng.integers(0, 255, ((rows + 127) // 128) * 128 * nb, dtype=np.uint8)
    assert np.array_equal(osm.scales_to_logical(sw, rows, nb), _unswizzle(sw, rows, nb))


def test_argument_errors_need_no_gpu():
    L = osm.lib()
    h = ctypes.c_void_p()
    s = np.ones(64, np.float32)
    O = np.array([5, 3], np.int32)   # not ascending
    rc = L.osm_plan_create(64, 64, 2, ctypes.c_void_p(s.ctypes.data), ctypes.c_void_p(O.ctypes.data), 0,
                           ctypes.byref(h))
    assert rc == osm.ERR_INVALID_ARG and "ascending" in osm.last_error()
    rc = L.osm_plan_create(48, 64, 0, ctypes.c_void_p(s.ctypes.data), None, 0, ctypes.byref(h))
    assert rc == osm.ERR_INVALID_ARG   # K % 32 != 0
    rc = L.osm_plan_create(64, 64, 0, ctypes.c_void_p(s.ctypes.data), None, 7, ctypes.byref(h))
    assert rc == osm.ERR_INVALID_ARG   # unknown mode
    s2 = s.copy()
    s2[3] = 0.0
    rc = L.osm_plan_create(64, 64, 0, ctypes.c_void_p(s2.ctypes.data), None, 0, ctypes.byref(h))
    assert rc == osm.ERR_INVALID_ARG   # s must be positive
    assert L.osm_dual_gemm(None, *([None] * 3), 1, *([None] * 4), 0, None, None, None, None, None, None) \
        == osm.ERR_INVALID_ARG
    # the FFN block entry points refuse missing plans before touching a device
    assert L.osm_ffn_workspace_size(None, None, 128) == 0
    assert L.osm_ffn_host_workspace_size(None, None, 128) == 0
    assert L.osm_ffn_block(None, None, None, 128, *([None] * 7), None, None, 0, None) == osm.ERR_INVALID_ARG
    assert L.osm_ffn_block_host(None, None, None, 128, *([None] * 7), None, None, 0, None) == osm.ERR_INVALID_ARG


def test_nvfp4_host_helpers_reject_bad_statistics():
    for bad in (-1.0, float("nan"), float("inf")):
        with pytest.raises(osm.OsmError) as e:
            osm.nvfp4_tensor_exponent(bad)
        assert e.value.code == osm.ERR_INVALID_ARG
    ones = np.ones(64, np.float32)
    with pytest.raises(osm.OsmError):
        osm.nvfp4_plan_exponents(ones, ones, ones, ones, np.array([64], np.int32))      # O out of range
    nan_stats = ones.copy()
    nan_stats[5] = np.nan
    with pytest.raises(osm.OsmError):
        osm.nvfp4_plan_exponents(nan_stats, ones, ones, ones, np.zeros(0, np.int32))
    # a NaN on an outlier channel does not enter the bulk maxima
    assert osm.nvfp4_plan_exponents(nan_stats, ones, ones, ones, np.array([5], np.int32)) == (
        osm.nvfp4_tensor_exponent(1.0), osm.nvfp4_tensor_exponent(1.0))
