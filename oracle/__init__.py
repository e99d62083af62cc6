"""Reference oracle for the smoothed, outlier-split W4A4 linear layer.

TEST INFRASTRUCTURE ONLY: a plain, slow CPU implementation (C in
``osm_oracle.c``, FP64 accumulation) of what the layer computes, following
"W4A4 Quantization for Inference on Wan2.2-I2V-A14B" (Eq. (1)-(5) and the
implementation paragraph) and the OCP MX v1.0 definition of MXFP4.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA
library ``outlier_split_mixed_b200``; only the seeded input generators
(``outlier_split_mixed_b200.synth``, which hold none of the method's
arithmetic) feed both.

Pinned functions (see tests/test_oracle_*.py): BF16 rounding, E2M1 codec,
MX scale exponent, calibration (Eq. (2), Eq. (4), the tail-aware percentile
score), smoothing/folding
(Eq. (1)), quantize_act, pack_weights (all three block-scale modes),
dual_gemm_rows (Eq. (5)), and the NVFP4 forms (E4M3 codec, block scale,
element multiplier, per-tensor exponent, quantize_act_nv, pack_weights_nv,
dual_gemm_rows_nv), and the FFN's tanh-form GELU (its FP64 definition) with
the one-step FP64 -> BF16 rounding.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "osm_oracle.c")
_LIB = os.path.join(_HERE, "libosm_oracle.so")
_lock = threading.Lock()
_lib = None

WSCALE_1x32, WSCALE_TILE32x32, WSCALE_STRIP128x1 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FP contraction, OpenMP over rows)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.oracle_bf16_to_f64.restype = ctypes.c_double
            lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
            lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.oracle_e2m1_decode.restype = ctypes.c_double
            lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e2m1_encode.restype = ctypes.c_uint8
            lib.oracle_e2m1_encode.argtypes = [ctypes.c_double, ctypes.c_int]
            lib.oracle_mx_scale_exponent.restype = ctypes.c_int
            lib.oracle_mx_scale_exponent.argtypes = [ctypes.c_double]
            lib.oracle_kbp.restype = I64
            lib.oracle_kbp.argtypes = [I64, I64]
            lib.oracle_kp.restype = I64
            lib.oracle_kp.argtypes = [I64]
            lib.oracle_act_amax.argtypes = [P, I64, I64, P]
            lib.oracle_weight_amax.argtypes = [P, I64, I64, P]
            lib.oracle_calibrate.restype = ctypes.c_int
            lib.oracle_calibrate.argtypes = [P, P, I64, ctypes.c_float, I64, P, P, P]
            lib.oracle_calibrate_scored.restype = ctypes.c_int
            lib.oracle_calibrate_scored.argtypes = [P, P, P, I64, ctypes.c_float, I64, P, P, P]
            lib.oracle_percentile_rank.restype = I64
            lib.oracle_percentile_rank.argtypes = [ctypes.c_double, I64]
            lib.oracle_act_percentile.argtypes = [P, I64, I64, I64, P]
            lib.oracle_smooth_act.argtypes = [P, I64, I64, P, P]
            lib.oracle_fold_weights.argtypes = [P, I64, I64, P, P]
            lib.oracle_quantize_act_ex.argtypes = [P, I64, I64, I64, P, P, P, P, P, ctypes.c_int]
            lib.oracle_pack_weights_ex.argtypes = [P, I64, I64, I64, P, P, ctypes.c_int, P, P, P, ctypes.c_int]
            lib.oracle_dual_gemm_rows_ex.argtypes = [P, P, P, P, I64, P, P, P, I64, I64, I64, P, P, P, ctypes.c_int]
            lib.oracle_f32_to_f16.restype = ctypes.c_uint16
            lib.oracle_f32_to_f16.argtypes = [ctypes.c_float]
            lib.oracle_f16_to_f64.restype = ctypes.c_double
            lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
            lib.oracle_gelu_tanh.restype = ctypes.c_double
            lib.oracle_gelu_tanh.argtypes = [ctypes.c_double]
            lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
            lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
            lib.oracle_gelu_rows.argtypes = [P, I64, P]
            lib.oracle_gelu_bf16_rows.argtypes = [P, I64, P]
            lib.oracle_e4m3_decode.restype = ctypes.c_double
            lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_encode_satfinite.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode_satfinite.argtypes = [ctypes.c_float]
            lib.oracle_nvfp4_tensor_exponent.restype = ctypes.c_int
            lib.oracle_nvfp4_tensor_exponent.argtypes = [ctypes.c_double]
            lib.oracle_nvfp4_scale.restype = ctypes.c_uint8
            lib.oracle_nvfp4_scale.argtypes = [ctypes.c_double, ctypes.c_int]
            lib.oracle_nvfp4_recip.restype = ctypes.c_float
            lib.oracle_nvfp4_recip.argtypes = [ctypes.c_uint8, ctypes.c_int]
            lib.oracle_nvfp4_plan_exponents.argtypes = [P, P, P, P, P, I64, I64, P, P]
            lib.oracle_quantize_act_nv.argtypes = [P, I64, I64, I64, P, P, ctypes.c_int, P, P, P]
            lib.oracle_pack_weights_nv.argtypes = [P, I64, I64, I64, P, P, ctypes.c_int, P, P, P]
            lib.oracle_dual_gemm_rows_nv.argtypes = [P, P, P, P, I64, P, P, P, I64, I64, I64, ctypes.c_int,
                                                     ctypes.c_int, P, P, P]
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- sizes --------------------------------------------------------------

def kbp(K: int, k: int) -> int:
    """Bulk width K-k rounded up to 128 (one scale atom = 4 blocks of 32)."""
    return int(_load().oracle_kbp(K, k))


def kp(k: int) -> int:
    """Outlier width k rounded up to 64 (one 128-byte BF16 chunk)."""
    return int(_load().oracle_kp(k))


# ---- scalars -------------------------------------------------------------

def bf16_to_f64(h: int) -> float:
    return float(_load().oracle_bf16_to_f64(int(h)))


def f32_to_bf16(f: float) -> int:
    return int(_load().oracle_f32_to_bf16(float(np.float32(f))))


def e2m1_decode(code: int) -> float:
    return float(_load().oracle_e2m1_decode(int(code)))


def e2m1_encode(v: float, negative: bool | None = None) -> int:
    if negative is None:
        negative = np.signbit(v)
    return int(_load().oracle_e2m1_encode(float(v), int(bool(negative))))


def mx_scale_exponent(amax: float) -> int:
    return int(_load().oracle_mx_scale_exponent(float(amax)))


def gelu_tanh(x: float) -> float:
    """GELU(x) = 0.5 x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3))) in FP64."""
    return float(_load().oracle_gelu_tanh(float(x)))


def f64_to_bf16(v: float) -> int:
    """RNE of an FP64 value to BF16 in one step (bit pattern)."""
    return int(_load().oracle_f64_to_bf16(float(v)))


# ---- arrays --------------------------------------------------------------

def bf16_round_array(x32: np.ndarray) -> np.ndarray:
    """Element-wise oracle_f32_to_bf16 over a float32 array (slow, scalar)."""
    lib = _load()
    flat = np.ascontiguousarray(x32, dtype=np.float32).ravel()
    out = np.empty(flat.shape, dtype=np.uint16)
    for i, v in enumerate(flat):
        out[i] = lib.oracle_f32_to_bf16(float(v))
    return out.reshape(np.shape(x32))


def act_amax(X: np.ndarray) -> np.ndarray:
    X = _c(X, np.uint16)
    T, K = X.shape
    out = np.empty(K, np.float32)
    _load().oracle_act_amax(_p(X), T, K, _p(out))
    return out


def weight_amax(W: np.ndarray) -> np.ndarray:
    W = _c(W, np.uint16)
    K, N = W.shape
    out = np.empty(K, np.float32)
    _load().oracle_weight_amax(_p(W), K, N, _p(out))
    return out


def calibrate(amax: np.ndarray, wmax: np.ndarray, alpha: float, k: int):
    """Eq. (2) smoothing vector and Eq. (4) top-k outlier set.
    Returns (s, inv_s, O) or raises ValueError on non-finite statistics."""
    amax = _c(amax, np.float32)
    wmax = _c(wmax, np.float32)
    K = amax.shape[0]
    s = np.empty(K, np.float32)
    inv_s = np.empty(K, np.float32)
    O = np.empty(max(k, 1), np.int32)
    rc = _load().oracle_calibrate(_p(amax), _p(wmax), K, float(alpha), k, _p(s), _p(inv_s), _p(O))
    if rc != 0:
        raise ValueError("non-finite calibration statistics")
    return s, inv_s, O[:k].copy()


def calibrate_scored(amax: np.ndarray, score: np.ndarray, wmax: np.ndarray, alpha: float, k: int):
    """Eq. (2) from the maxima, Eq. (4)'s top-k by a separate score."""
    amax = _c(amax, np.float32)
    score = _c(score, np.float32)
    wmax = _c(wmax, np.float32)
    K = amax.shape[0]
    s = np.empty(K, np.float32)
    inv_s = np.empty(K, np.float32)
    O = np.empty(max(k, 1), np.int32)
    rc = _load().oracle_calibrate_scored(_p(amax), _p(score), _p(wmax), K, float(alpha), k, _p(s), _p(inv_s), _p(O))
    if rc != 0:
        raise ValueError("non-finite calibration statistics")
    return s, inv_s, O[:k].copy()


def percentile_rank(q: float, T: int) -> int:
    """Nearest rank ceil(q T), clamped to [1, T]."""
    return int(_load().oracle_percentile_rank(float(q), int(T)))


def act_percentile(X: np.ndarray, rank: int) -> np.ndarray:
    """score[j] = the rank-th smallest |x_tj| (rank 1-based)."""
    X = _c(X, np.uint16)
    T, K = X.shape
    out = np.empty(K, np.float32)
    _load().oracle_act_percentile(_p(X), T, K, int(rank), _p(out))
    return out


def smooth_act(X: np.ndarray, inv_s: np.ndarray) -> np.ndarray:
    X = _c(X, np.uint16)
    inv_s = _c(inv_s, np.float32)
    M, K = X.shape
    out = np.empty_like(X)
    _load().oracle_smooth_act(_p(X), M, K, _p(inv_s), _p(out))
    return out


def fold_weights(W: np.ndarray, s: np.ndarray) -> np.ndarray:
    W = _c(W, np.uint16)
    s = _c(s, np.float32)
    K, N = W.shape
    out = np.empty_like(W)
    _load().oracle_fold_weights(_p(W), K, N, _p(s), _p(out))
    return out


def f32_to_f16(f: float) -> int:
    return int(_load().oracle_f32_to_f16(float(np.float32(f))))


def f16_to_f64(h: int) -> float:
    return float(_load().oracle_f16_to_f64(int(h)))


def quantize_act(X: np.ndarray, inv_s: np.ndarray, O: np.ndarray, hp_fp16: bool = False):
    """Returns (codes [M][Kbp/2] u8, scales [M][Kbp/32] u8 logical, a_hp [M][kp] u16);
    hp_fp16: outlier slots in binary16 instead of BF16."""
    X = _c(X, np.uint16)
    inv_s = _c(inv_s, np.float32)
    O = _c(O, np.int32)
    M, K = X.shape
    k = O.shape[0]
    Kbp, kpp = kbp(K, k), kp(k)
    codes = np.zeros((M, Kbp // 2), np.uint8)
    scales = np.zeros((M, Kbp // 32), np.uint8)
    a_hp = np.zeros((M, kpp), np.uint16)
    Op = O if k else np.zeros(1, np.int32)
    _load().oracle_quantize_act_ex(_p(X), M, K, k, _p(inv_s), _p(Op), _p(codes), _p(scales), _p(a_hp),
                                   int(bool(hp_fp16)))
    return codes, scales, a_hp


def pack_weights(W: np.ndarray, s: np.ndarray, O: np.ndarray, mode: int, hp_fp16: bool = False):
    """Returns (codes [N][Kbp/2] u8, scales [N][Kbp/32] u8 logical, w_hp [N][kp] u16)."""
    W = _c(W, np.uint16)
    s = _c(s, np.float32)
    O = _c(O, np.int32)
    K, N = W.shape
    k = O.shape[0]
    Kbp, kpp = kbp(K, k), kp(k)
    codes = np.zeros((N, Kbp // 2), np.uint8)
    scales = np.zeros((N, Kbp // 32), np.uint8)
    w_hp = np.zeros((N, kpp), np.uint16)
    Op = O if k else np.zeros(1, np.int32)
    _load().oracle_pack_weights_ex(_p(W), K, N, k, _p(s), _p(Op), int(mode), _p(codes), _p(scales), _p(w_hp),
                                   int(bool(hp_fp16)))
    return codes, scales, w_hp


def gelu(y: np.ndarray) -> np.ndarray:
    """GELU_tanh(y) element-wise in FP64."""
    y = _c(y, np.float64)
    out = np.empty(y.shape, np.float64)
    _load().oracle_gelu_rows(_p(y), y.size, _p(out))
    return out


def gelu_bf16(y: np.ndarray) -> np.ndarray:
    """h = bf16(GELU_tanh(y)) element-wise for FP64 accumulators y (GELU in
    FP64, rounded once to BF16)."""
    y = _c(y, np.float64)
    out = np.empty(y.shape, np.uint16)
    _load().oracle_gelu_bf16_rows(_p(y), y.size, _p(out))
    return out


def dual_gemm_rows(a_codes, a_scales, a_hp, rows, w_codes, w_scales, w_hp, bias=None, hp_fp16=False):
    """Eq. (5) for the given activation rows. Returns (y [r][N] f64, T [r][N] f64)."""
    a_codes = _c(a_codes, np.uint8)
    a_scales = _c(a_scales, np.uint8)
    a_hp = _c(a_hp, np.uint16)
    w_codes = _c(w_codes, np.uint8)
    w_scales = _c(w_scales, np.uint8)
    w_hp = _c(w_hp, np.uint16)
    rows = _c(rows, np.int64)
    N = w_codes.shape[0]
    Kbp = w_codes.shape[1] * 2
    kpp = w_hp.shape[1]
    assert a_codes.shape[1] * 2 == Kbp and a_hp.shape[1] == kpp
    y = np.empty((rows.shape[0], N), np.float64)
    T = np.empty((rows.shape[0], N), np.float64)
    bptr = None
    if bias is not None:
        bias = _c(bias, np.float32)
        bptr = _p(bias)
    _load().oracle_dual_gemm_rows_ex(_p(a_codes), _p(a_scales), _p(a_hp), _p(rows), rows.shape[0],
                                     _p(w_codes), _p(w_scales), _p(w_hp), N, Kbp, kpp, bptr,
                                     _p(y), _p(T), int(bool(hp_fp16)))
    return y, T


# ---- NVFP4 ---------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    return float(_load().oracle_e4m3_decode(int(code)))


def e4m3_encode(f: float) -> int:
    """Nearest E4M3 code (ties to even), saturating at 448."""
    return int(_load().oracle_e4m3_encode_satfinite(float(np.float32(f))))


def nvfp4_tensor_exponent(amax: float) -> int:
    return int(_load().oracle_nvfp4_tensor_exponent(float(amax)))


def nvfp4_scale(amax: float, g: int) -> int:
    return int(_load().oracle_nvfp4_scale(float(amax), int(g)))


def nvfp4_recip(S: int, g: int) -> float:
    return float(_load().oracle_nvfp4_recip(int(S), int(g)))


def nvfp4_plan_exponents(amax, wmax, s, inv_s, O):
    """(g_act, g_w) of a plan from its calibration statistics."""
    amax, wmax = _c(amax, np.float32), _c(wmax, np.float32)
    s, inv_s = _c(s, np.float32), _c(inv_s, np.float32)
    O = _c(O, np.int32)
    K, k = amax.shape[0], O.shape[0]
    ga, gw = ctypes.c_int(0), ctypes.c_int(0)
    Op = O if k else np.zeros(1, np.int32)
    _load().oracle_nvfp4_plan_exponents(_p(amax), _p(wmax), _p(s), _p(inv_s), _p(Op), K, k,
                                        ctypes.byref(ga), ctypes.byref(gw))
    return ga.value, gw.value


def quantize_act_nv(X: np.ndarray, inv_s: np.ndarray, O: np.ndarray, g_act: int):
    """NVFP4 activations: (codes [M][Kbp/2], scales [M][Kbp/16] logical UE4M3, a_hp [M][kp])."""
    X = _c(X, np.uint16)
    inv_s = _c(inv_s, np.float32)
    O = _c(O, np.int32)
    M, K = X.shape
    k = O.shape[0]
    Kbp, kpp = kbp(K, k), kp(k)
    codes = np.zeros((M, Kbp // 2), np.uint8)
    scales = np.zeros((M, Kbp // 16), np.uint8)
    a_hp = np.zeros((M, kpp), np.uint16)
    Op = O if k else np.zeros(1, np.int32)
    _load().oracle_quantize_act_nv(_p(X), M, K, k, _p(inv_s), _p(Op), int(g_act), _p(codes), _p(scales), _p(a_hp))
    return codes, scales, a_hp


def pack_weights_nv(W: np.ndarray, s: np.ndarray, O: np.ndarray, g_w: int):
    """NVFP4 weights: (codes [N][Kbp/2], scales [N][Kbp/16] logical UE4M3, w_hp [N][kp])."""
    W = _c(W, np.uint16)
    s = _c(s, np.float32)
    O = _c(O, np.int32)
    K, N = W.shape
    k = O.shape[0]
    Kbp, kpp = kbp(K, k), kp(k)
    codes = np.zeros((N, Kbp // 2), np.uint8)
    scales = np.zeros((N, Kbp // 16), np.uint8)
    w_hp = np.zeros((N, kpp), np.uint16)
    Op = O if k else np.zeros(1, np.int32)
    _load().oracle_pack_weights_nv(_p(W), K, N, k, _p(s), _p(Op), int(g_w), _p(codes), _p(scales), _p(w_hp))
    return codes, scales, w_hp


def dual_gemm_rows_nv(a_codes, a_scales, a_hp, rows, w_codes, w_scales, w_hp, g_act, g_w, bias=None):
    """Eq. (5) with NVFP4 operands. Returns (y [r][N] f64, T [r][N] f64)."""
    a_codes, a_scales, a_hp = _c(a_codes, np.uint8), _c(a_scales, np.uint8), _c(a_hp, np.uint16)
    w_codes, w_scales, w_hp = _c(w_codes, np.uint8), _c(w_scales, np.uint8), _c(w_hp, np.uint16)
    rows = _c(rows, np.int64)
    N = w_codes.shape[0]
    Kbp = w_codes.shape[1] * 2
    kpp = w_hp.shape[1]
    assert a_codes.shape[1] * 2 == Kbp and a_hp.shape[1] == kpp
    assert a_scales.shape[1] == Kbp // 16 and w_scales.shape[1] == Kbp // 16
    y = np.empty((rows.shape[0], N), np.float64)
    T = np.empty((rows.shape[0], N), np.float64)
    bptr = None
    if bias is not None:
        bias = _c(bias, np.float32)
        bptr = _p(bias)
    _load().oracle_dual_gemm_rows_nv(_p(a_codes), _p(a_scales), _p(a_hp), _p(rows), rows.shape[0],
                                     _p(w_codes), _p(w_scales), _p(w_hp), N, Kbp, kpp, int(g_act), int(g_w),
                                     bptr, _p(y), _p(T))
    return y, T
