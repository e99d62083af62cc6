"""B200 (sm_100a) smoothed, outlier-split W4A4 linear layer.

Python binding of libosm (``include/osm.h``): each function below marshals
torch tensors / numpy arrays into the C entry point of the same name
(``osm_<name>``) and raises :class:`OsmError` on a non-zero return code.
There is no fallback: every computation runs in the CUDA library, and a
missing library raises at first use.

Method: "W4A4 Quantization for Inference on Wan2.2-I2V-A14B" -- SmoothQuant
smoothing (Eq. (1), (2)), a static top-k outlier split (Eq. (4), (5)) and a
dual-branch GEMM whose bulk branch is MXFP4 (E2M1 + E8M0 per 32) and whose
outlier branch is BF16 (Eq. (3)).
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libosm.so")

OK = 0
ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_NONFINITE, ERR_NOMEM = 1, 2, 3, 4, 5, 6
STATUS_TIMEOUT = 1
HP_BF16, HP_FP16 = 0, 1
FMT_MXFP4, FMT_NVFP4 = 0, 1
STATUS_NONFINITE = 2
DEBUG_STARVE_QUANTIZE = 1
WSCALE_1x32, WSCALE_TILE32x32, WSCALE_STRIP128x1 = 0, 1, 2
EPI_F32, EPI_BF16, EPI_GELU_REQUANT, EPI_GELU_BF16 = 0, 1, 2, 3

# Every entry point declared in include/osm.h, with its ctypes signature.
_P, _I64, _I, _U64, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
_SIGNATURES = {
    "osm_act_amax_accumulate": (_I, [_P, _I64, _I64, _P, _P]),
    "osm_weight_amax": (_I, [_P, _I64, _I64, _P, _P]),
    "osm_calibrate_finalize": (_I, [_P, _P, _I64, ctypes.c_float, _I64, _P, _P, _P]),
    "osm_plan_create": (_I, [_I64, _I64, _I64, _P, _P, _I, ctypes.POINTER(_P)]),
    "osm_plan_destroy": (_I, [_P]),
    "osm_plan_sizes": (_I, [_P, _I64, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]),
    "osm_plan_dims": (_I, [_P] + [ctypes.POINTER(_I64)] * 6),
    "osm_plan_status": (_I, [_P, _P, ctypes.POINTER(ctypes.c_uint32), _I]),
    "osm_plan_set_wait_limit": (_I, [_P, _U64]),
    "osm_plan_set_debug": (_I, [_P, ctypes.c_uint32]),
    "osm_plan_set_outlier_dtype": (_I, [_P, _I]),
    "osm_plan_set_format": (_I, [_P, _I, _I, _I]),
    "osm_nvfp4_tensor_exponent": (_I, [ctypes.c_float, ctypes.POINTER(_I)]),
    "osm_nvfp4_plan_exponents": (_I, [_P, _P, _P, _P, _P, _I64, _I64, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "osm_plan_refresh": (_I, [_P, _P, _P, ctypes.c_float, _P]),
    "osm_plan_refresh_scored": (_I, [_P, _P, _P, _P, ctypes.c_float, _P]),
    "osm_act_percentile": (_I, [_P, _I64, _I64, ctypes.c_float, _P, _P]),
    "osm_error_norms": (_I, [_P, _P, _I64, _P, _P]),
    "osm_calibrate_finalize_scored": (_I, [_P, _P, _P, _I64, ctypes.c_float, _I64, _P, _P, _P]),
    "osm_plan_tables": (_I, [_P, _P, _P, _P]),
    "osm_pack_weights": (_I, [_P, _P, _P, _P, _P, _P]),
    "osm_pack_weights_for_next": (_I, [_P, _P, _P, _P, _P, _P, _P]),
    "osm_plan_channel_order": (_I, [_P, _P]),
    "osm_quantize_act": (_I, [_P, _P, _I64, _P, _P, _P, _P]),
    "osm_dual_gemm": (_I, [_P, _P, _P, _P, _I64, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P]),
    "osm_linear_workspace_size": (_SZ, [_P, _I64, _I]),
    "osm_linear_host": (_I, [_P, _P, _I64, _P, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "osm_scales_to_logical": (_I, [_P, _I64, _I64, _P]),
    "osm_linear_noalloc": (_I, [_P, _P, _I64, _P, _P, _P, _P, _I, _P, _P]),
    "osm_gelu_f32": (_I, [_P, _P, _I64, _P]),
    "osm_ffn_workspace_size": (_SZ, [_P, _P, _I64]),
    "osm_ffn_host_workspace_size": (_SZ, [_P, _P, _I64]),
    "osm_ffn_block": (_I, [_P, _P, _P, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "osm_ffn_block_host": (_I, [_P, _P, _P, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "osm_last_error": (ctypes.c_char_p, []),
}

_lock = threading.Lock()
_lib = None


class OsmError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libosm error {code}: {msg}")
        self.code = code


def lib():
    """The loaded libosm (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m outlier_split_mixed_b200.build` (nvcc, sm_100a)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def last_error() -> str:
    v = lib().osm_last_error()
    return v.decode() if v else ""


def _check(rc: int):
    if rc != OK:
        raise OsmError(rc, last_error())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, name, dtypes=None, numel=None, allow_none=False):
    """Device pointer of a contiguous CUDA tensor (or None)."""
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if numel is not None and t.numel() * t.element_size() < numel:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, needs {numel}")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _bf16_types():
    import torch
    return (torch.bfloat16, torch.int16, torch.uint16)


def _u8_types():
    import torch
    return (torch.uint8,)


# ----------------------------------------------------------------- plans

class Plan:
    """An osm_plan: K, N, k, the smoothing vector s, the outlier set O and
    the weight block-scale mode, with its device tables; optionally the FP16
    outlier branch (hp_fp16) or the NVFP4 bulk format (fmt = FMT_NVFP4 with
    the per-tensor exponents g_act, g_w)."""

    def __init__(self, K: int, N: int, k: int, s: np.ndarray, O: np.ndarray, wscale_mode: int = WSCALE_1x32,
                 hp_fp16: bool = False, fmt: int = FMT_MXFP4, g_act: int = 0, g_w: int = 0):
        s = np.ascontiguousarray(s, dtype=np.float32)
        O = np.ascontiguousarray(O, dtype=np.int32)
        if s.shape != (K,) or O.shape != (k,):
            raise ValueError("s must have shape (K,) and O shape (k,)")
        h = ctypes.c_void_p()
        _check(lib().osm_plan_create(K, N, k, _host_ptr(s), _host_ptr(O) if k else None, int(wscale_mode),
                                     ctypes.byref(h)))
        self._h = h
        self.s, self.O, self.wscale_mode = s, O, int(wscale_mode)
        d = [ctypes.c_int64() for _ in range(6)]
        _check(lib().osm_plan_dims(self._h, *[ctypes.byref(x) for x in d]))
        self.K, self.N, self.k, self.Kb, self.Kbp, self.kp = (int(x.value) for x in d)
        self.hp_fp16 = bool(hp_fp16)
        if hp_fp16:
            _check(lib().osm_plan_set_outlier_dtype(self._h, HP_FP16))
        self.fmt, self.g_act, self.g_w = FMT_MXFP4, 0, 0
        if fmt != FMT_MXFP4:
            self.set_format(fmt, g_act, g_w)

    def set_format(self, fmt: int, g_act: int = 0, g_w: int = 0):
        """osm_plan_set_format: the 4-bit block format of the bulk branch."""
        _check(lib().osm_plan_set_format(self._h, int(fmt), int(g_act), int(g_w)))
        self.fmt = int(fmt)
        self.g_act, self.g_w = (int(g_act), int(g_w)) if fmt == FMT_NVFP4 else (0, 0)

    @property
    def nblocks(self) -> int:
        """Scale blocks per row: Kbp/32 (MXFP4) or Kbp/16 (NVFP4)."""
        return self.Kbp // (16 if self.fmt == FMT_NVFP4 else 32)

    @property
    def handle(self):
        return self._h

    def sizes(self, rows: int):
        """(codes_bytes, scales_bytes, hp_bytes) for `rows` rows."""
        c, s, h = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().osm_plan_sizes(self._h, rows, ctypes.byref(c), ctypes.byref(s), ctypes.byref(h)))
        return int(c.value), int(s.value), int(h.value)

    def status(self, clear: bool = True, stream=None) -> int:
        v = ctypes.c_uint32()
        _check(lib().osm_plan_status(self._h, _stream(stream), ctypes.byref(v), int(clear)))
        return int(v.value)

    def channel_order(self) -> np.ndarray:
        """[J ascending | O ascending] (osm_plan_channel_order)."""
        out = np.empty(self.K, np.int32)
        _check(lib().osm_plan_channel_order(self._h, _host_ptr(out)))
        return out

    def set_wait_limit(self, ns: int):
        _check(lib().osm_plan_set_wait_limit(self._h, int(ns)))

    def set_debug(self, flags: int):
        _check(lib().osm_plan_set_debug(self._h, int(flags)))

    def refresh(self, amax, wmax, alpha: float, stream=None):
        """Re-calibrate on the device from device statistics (osm_plan_refresh):
        s, inv_s, O and the routing tables are rebuilt; pack the weights again."""
        import torch
        _check(lib().osm_plan_refresh(self._h, _ptr(amax, "amax", (torch.float32,), self.K * 4),
                                      _ptr(wmax, "wmax", (torch.float32,), self.K * 4), float(alpha),
                                      _stream(stream)))

    def refresh_scored(self, amax, score, wmax, alpha: float, stream=None):
        """As refresh, with the top-k by `score` (osm_plan_refresh_scored)."""
        import torch
        f32 = (torch.float32,)
        _check(lib().osm_plan_refresh_scored(self._h, _ptr(amax, "amax", f32, self.K * 4),
                                             _ptr(score, "score", f32, self.K * 4),
                                             _ptr(wmax, "wmax", f32, self.K * 4), float(alpha), _stream(stream)))

    def tables(self):
        """(s, inv_s, O) copied to host numpy arrays (osm_plan_tables)."""
        s = np.empty(self.K, np.float32)
        inv_s = np.empty(self.K, np.float32)
        O = np.empty(max(self.k, 1), np.int32)
        _check(lib().osm_plan_tables(self._h, _host_ptr(s), _host_ptr(inv_s), _host_ptr(O)))
        return s, inv_s, O[:self.k].copy()

    def alloc_packed(self, rows: int, device="cuda"):
        """Allocate (codes, scales, hp) torch buffers for `rows` rows."""
        import torch
        cb, sb, hb = self.sizes(rows)
        codes = torch.empty(max(cb, 16), dtype=torch.uint8, device=device)[:cb]
        scales = torch.empty(max(sb, 16), dtype=torch.uint8, device=device)[:sb]
        hp = torch.empty(max(hb // 2, 8), dtype=torch.bfloat16, device=device)[:hb // 2]
        return codes, scales, hp

    def close(self):
        if getattr(self, "_h", None):
            lib().osm_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ----------------------------------------------------------------- calibration

def act_amax_accumulate(X, amax, stream=None):
    """amax = max(amax, max_t |X[t]|) on the device (osm_act_amax_accumulate)."""
    T, K = X.shape
    import torch
    _check(lib().osm_act_amax_accumulate(_ptr(X, "X", _bf16_types()), T, K,
                                         _ptr(amax, "amax", (torch.float32,), K * 4), _stream(stream)))


def act_percentile(X, q: float, score, stream=None):
    """score[j] = nearest-rank q-percentile of |X[:, j]| on the device (osm_act_percentile)."""
    T, K = X.shape
    import torch
    _check(lib().osm_act_percentile(_ptr(X, "X", _bf16_types()), T, K, float(q),
                                    _ptr(score, "score", (torch.float32,), K * 4), _stream(stream)))


def error_norms(Y, Yref, stream=None):
    """(sum (Y - Yref)^2, sum Yref^2) in FP64 on the device (osm_error_norms)."""
    import torch
    if Y.shape != Yref.shape:
        raise ValueError("Y and Yref differ in shape")
    out = torch.zeros(2, dtype=torch.float64, device=Y.device)
    _check(lib().osm_error_norms(_ptr(Y, "Y", (torch.float32,)), _ptr(Yref, "Yref", (torch.float32,)), Y.numel(),
                                 _ptr(out, "out", (torch.float64,)), _stream(stream)))
    e, n = out.cpu().tolist()
    return e, n


def gelu_f32(x, y=None, stream=None):
    """The FFN epilogues' FP32 GELU routine element-wise (osm_gelu_f32)."""
    import torch
    if y is None:
        y = torch.empty_like(x)
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel():
        raise ValueError("x and y must be float32 tensors of one size")
    _check(lib().osm_gelu_f32(_ptr(x, "x"), _ptr(y, "y"), x.numel(), _stream(stream)))
    return y


def weight_amax(W, wmax, stream=None):
    """wmax[j] = max_n |W[j][n]| (osm_weight_amax)."""
    K, N = W.shape
    import torch
    _check(lib().osm_weight_amax(_ptr(W, "W", _bf16_types()), K, N, _ptr(wmax, "wmax", (torch.float32,), K * 4),
                                 _stream(stream)))


def calibrate_finalize(amax_host: np.ndarray, wmax_host: np.ndarray, alpha: float, k: int):
    """Eq. (2) and Eq. (4) on host statistics -> (s, inv_s, O) (osm_calibrate_finalize)."""
    amax_host = np.ascontiguousarray(amax_host, dtype=np.float32)
    wmax_host = np.ascontiguousarray(wmax_host, dtype=np.float32)
    K = amax_host.shape[0]
    s = np.empty(K, np.float32)
    inv_s = np.empty(K, np.float32)
    O = np.empty(max(k, 1), np.int32)
    _check(lib().osm_calibrate_finalize(_host_ptr(amax_host), _host_ptr(wmax_host), K, float(alpha), int(k),
                                        _host_ptr(s), _host_ptr(inv_s), _host_ptr(O)))
    return s, inv_s, O[:k].copy()


def nvfp4_tensor_exponent(amax: float) -> int:
    """osm_nvfp4_tensor_exponent: smallest g in [-100, 100] with amax <= 6 * 448 * 2^g."""
    g = ctypes.c_int()
    _check(lib().osm_nvfp4_tensor_exponent(float(amax), ctypes.byref(g)))
    return int(g.value)


def nvfp4_plan_exponents(amax_host, wmax_host, s, inv_s, O):
    """osm_nvfp4_plan_exponents: (g_act, g_w) from the calibration statistics."""
    a = np.ascontiguousarray(amax_host, dtype=np.float32)
    w = np.ascontiguousarray(wmax_host, dtype=np.float32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    inv_s = np.ascontiguousarray(inv_s, dtype=np.float32)
    O = np.ascontiguousarray(O, dtype=np.int32)
    ga, gw = ctypes.c_int(), ctypes.c_int()
    _check(lib().osm_nvfp4_plan_exponents(_host_ptr(a), _host_ptr(w), _host_ptr(s), _host_ptr(inv_s),
                                          _host_ptr(O) if O.size else None, a.shape[0], O.shape[0],
                                          ctypes.byref(ga), ctypes.byref(gw)))
    return int(ga.value), int(gw.value)


def calibrate_finalize_scored(amax_host: np.ndarray, score_host: np.ndarray, wmax_host: np.ndarray, alpha: float,
                              k: int):
    """Eq. (2) from amax, Eq. (4)'s top-k by score -> (s, inv_s, O) (osm_calibrate_finalize_scored)."""
    amax_host = np.ascontiguousarray(amax_host, dtype=np.float32)
    score_host = np.ascontiguousarray(score_host, dtype=np.float32)
    wmax_host = np.ascontiguousarray(wmax_host, dtype=np.float32)
    K = amax_host.shape[0]
    s = np.empty(K, np.float32)
    inv_s = np.empty(K, np.float32)
    O = np.empty(max(k, 1), np.int32)
    _check(lib().osm_calibrate_finalize_scored(_host_ptr(amax_host), _host_ptr(score_host), _host_ptr(wmax_host), K,
                                               float(alpha), int(k), _host_ptr(s), _host_ptr(inv_s), _host_ptr(O)))
    return s, inv_s, O[:k].copy()


# ----------------------------------------------------------------- layer path

def pack_weights(plan: Plan, W, w_codes, w_scales, w_hp, stream=None):
    """Fold s into W and pack it (osm_pack_weights). W: [K][N] BF16."""
    cb, sb, hb = plan.sizes(plan.N)
    if tuple(W.shape) != (plan.K, plan.N):
        raise ValueError("W must have shape (K, N)")
    _check(lib().osm_pack_weights(plan.handle, _ptr(W, "W", _bf16_types()),
                                  _ptr(w_codes, "w_codes", _u8_types(), cb, allow_none=cb == 0),
                                  _ptr(w_scales, "w_scales", _u8_types(), sb, allow_none=sb == 0),
                                  _ptr(w_hp, "w_hp", _bf16_types(), hb, allow_none=hb == 0), _stream(stream)))


def pack_weights_for_next(plan: Plan, next_plan: Plan, W, w_codes, w_scales, w_hp, stream=None):
    """Pack W with its output columns in next_plan's channel order
    (osm_pack_weights_for_next), for OSM_EPI_GELU_REQUANT."""
    cb, sb, hb = plan.sizes(plan.N)
    if tuple(W.shape) != (plan.K, plan.N):
        raise ValueError("W must have shape (K, N)")
    _check(lib().osm_pack_weights_for_next(plan.handle, next_plan.handle, _ptr(W, "W", _bf16_types()),
                                           _ptr(w_codes, "w_codes", _u8_types(), cb, allow_none=cb == 0),
                                           _ptr(w_scales, "w_scales", _u8_types(), sb, allow_none=sb == 0),
                                           _ptr(w_hp, "w_hp", _bf16_types(), hb, allow_none=hb == 0), _stream(stream)))


def quantize_act(plan: Plan, X, a_codes, a_scales, a_hp, stream=None):
    """Smooth, split and MXFP4-encode activations (osm_quantize_act). X: [M][K] BF16."""
    M, K = X.shape
    if K != plan.K:
        raise ValueError("X must have K columns")
    cb, sb, hb = plan.sizes(M)
    _check(lib().osm_quantize_act(plan.handle, _ptr(X, "X", _bf16_types()), M,
                                  _ptr(a_codes, "a_codes", _u8_types(), cb, allow_none=cb == 0),
                                  _ptr(a_scales, "a_scales", _u8_types(), sb, allow_none=sb == 0),
                                  _ptr(a_hp, "a_hp", _bf16_types(), hb, allow_none=hb == 0), _stream(stream)))


def dual_gemm(plan: Plan, a_codes, a_scales, a_hp, M: int, w_codes, w_scales, w_hp, Y, bias=None,
              epi: int = EPI_F32, stream=None, next_plan: Plan | None = None, next_buffers=None):
    """Eq. (5) on packed operands (osm_dual_gemm). Y: [M][N] float32 or BF16.
    With epi=EPI_GELU_REQUANT, Y and bias are None and next_buffers are the
    (codes, scales, hp) of next_plan for M rows."""
    import torch
    cbm, sbm, hbm = plan.sizes(M)
    cbn, sbn, hbn = plan.sizes(plan.N)
    if epi == EPI_GELU_REQUANT:
        if next_plan is None or next_buffers is None or Y is not None or bias is not None:
            raise ValueError("GELU_REQUANT needs next_plan and next_buffers, and no Y or bias")
        ncb, nsb, nhb = next_plan.sizes(M)
        nc, ns, nh = next_buffers
        _check(lib().osm_dual_gemm(plan.handle,
                                   _ptr(a_codes, "a_codes", _u8_types(), cbm, allow_none=cbm == 0),
                                   _ptr(a_scales, "a_scales", _u8_types(), sbm, allow_none=sbm == 0),
                                   _ptr(a_hp, "a_hp", _bf16_types(), hbm, allow_none=hbm == 0), M,
                                   _ptr(w_codes, "w_codes", _u8_types(), cbn, allow_none=cbn == 0),
                                   _ptr(w_scales, "w_scales", _u8_types(), sbn, allow_none=sbn == 0),
                                   _ptr(w_hp, "w_hp", _bf16_types(), hbn, allow_none=hbn == 0),
                                   None, int(epi), None, next_plan.handle,
                                   _ptr(nc, "next_codes", _u8_types(), ncb, allow_none=ncb == 0),
                                   _ptr(ns, "next_scales", _u8_types(), nsb, allow_none=nsb == 0),
                                   _ptr(nh, "next_hp", _bf16_types(), nhb, allow_none=nhb == 0), _stream(stream)))
        return
    ybytes = M * plan.N * (4 if epi == EPI_F32 else 2)
    ytypes = (torch.float32,) if epi == EPI_F32 else _bf16_types()
    _check(lib().osm_dual_gemm(plan.handle,
                               _ptr(a_codes, "a_codes", _u8_types(), cbm, allow_none=cbm == 0),
                               _ptr(a_scales, "a_scales", _u8_types(), sbm, allow_none=sbm == 0),
                               _ptr(a_hp, "a_hp", _bf16_types(), hbm, allow_none=hbm == 0), M,
                               _ptr(w_codes, "w_codes", _u8_types(), cbn, allow_none=cbn == 0),
                               _ptr(w_scales, "w_scales", _u8_types(), sbn, allow_none=sbn == 0),
                               _ptr(w_hp, "w_hp", _bf16_types(), hbn, allow_none=hbn == 0),
                               _ptr(bias, "bias", (torch.float32,), plan.N * 4, allow_none=True), int(epi),
                               _ptr(Y, "Y", ytypes, ybytes), None, None, None, None, _stream(stream)))


def linear_workspace_size(plan: Plan, M: int, epi: int = EPI_F32) -> int:
    return int(lib().osm_linear_workspace_size(plan.handle, M, int(epi)))


def linear_host(plan: Plan, X_host, M: int, w_codes, w_scales, w_hp, Y_host, workspace, bias=None,
                epi: int = EPI_F32, stream=None):
    """Host X -> device quantize + dual GEMM -> host Y (osm_linear_host).
    X_host / Y_host: pinned CPU torch tensors; the caller synchronises."""
    import torch
    for t, n in ((X_host, "X_host"), (Y_host, "Y_host")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous host tensor")
    cbn, sbn, hbn = plan.sizes(plan.N)
    _check(lib().osm_linear_host(plan.handle, ctypes.c_void_p(X_host.data_ptr()), M,
                                 _ptr(w_codes, "w_codes", _u8_types(), cbn, allow_none=cbn == 0),
                                 _ptr(w_scales, "w_scales", _u8_types(), sbn, allow_none=sbn == 0),
                                 _ptr(w_hp, "w_hp", _bf16_types(), hbn, allow_none=hbn == 0),
                                 _ptr(bias, "bias", (torch.float32,), plan.N * 4, allow_none=True), int(epi),
                                 ctypes.c_void_p(Y_host.data_ptr()), _ptr(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))


def ffn_workspace_size(up: Plan, down: Plan, M: int) -> int:
    """Device bytes osm_ffn_block needs for M tokens (both layers' packed activations)."""
    return int(lib().osm_ffn_workspace_size(up.handle, down.handle, M))


def ffn_host_workspace_size(up: Plan, down: Plan, M: int) -> int:
    """Device bytes osm_ffn_block_host needs for M tokens."""
    return int(lib().osm_ffn_host_workspace_size(up.handle, down.handle, M))


def _ffn_weight_ptrs(up: Plan, down: Plan, wu, wd):
    cu, su, hu = up.sizes(up.N)
    cd, sd, hd = down.sizes(down.N)
    return (_ptr(wu[0], "wu_codes", _u8_types(), cu, allow_none=cu == 0),
            _ptr(wu[1], "wu_scales", _u8_types(), su, allow_none=su == 0),
            _ptr(wu[2], "wu_hp", _bf16_types(), hu, allow_none=hu == 0),
            _ptr(wd[0], "wd_codes", _u8_types(), cd, allow_none=cd == 0),
            _ptr(wd[1], "wd_scales", _u8_types(), sd, allow_none=sd == 0),
            _ptr(wd[2], "wd_hp", _bf16_types(), hd, allow_none=hd == 0))


def ffn_block(up: Plan, down: Plan, X, wu, wd, Y, workspace, bias_down=None, stream=None):
    """One FFN block on the device (osm_ffn_block): quantize_act(up), the
    up-projection with the fused GELU + smoothing + requantisation epilogue,
    the down-projection to BF16. wu = (codes, scales, hp) packed by
    pack_weights_for_next(up, down), wd packed by pack_weights(down).
    X: [M][up.K] BF16, Y: [M][down.N] BF16, both CUDA tensors."""
    import torch
    M, K = X.shape
    if K != up.K or tuple(Y.shape) != (M, down.N):
        raise ValueError("X must be [M][up.K] and Y [M][down.N]")
    _check(lib().osm_ffn_block(up.handle, down.handle, _ptr(X, "X", _bf16_types()), M,
                               *_ffn_weight_ptrs(up, down, wu, wd),
                               _ptr(bias_down, "bias_down", (torch.float32,), down.N * 4, allow_none=True),
                               _ptr(Y, "Y", _bf16_types(), M * down.N * 2), _ptr(workspace, "workspace"),
                               workspace.numel() * workspace.element_size(), _stream(stream)))


def ffn_block_host(up: Plan, down: Plan, X_host, wu, wd, Y_host, workspace, bias_down=None, stream=None):
    """osm_ffn_block_host: host (pinned) X in, the block on the device, host
    Y out, all enqueued on `stream`; the caller synchronises."""
    import torch
    for t, n in ((X_host, "X_host"), (Y_host, "Y_host")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous host tensor")
    M, K = X_host.shape
    if K != up.K or tuple(Y_host.shape) != (M, down.N):
        raise ValueError("X_host must be [M][up.K] and Y_host [M][down.N]")
    _check(lib().osm_ffn_block_host(up.handle, down.handle, ctypes.c_void_p(X_host.data_ptr()), M,
                                    *_ffn_weight_ptrs(up, down, wu, wd),
                                    _ptr(bias_down, "bias_down", (torch.float32,), down.N * 4, allow_none=True),
                                    ctypes.c_void_p(Y_host.data_ptr()), _ptr(workspace, "workspace"),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 16 << 20


def linear_noalloc(plan: Plan, X, w_codes, w_scales, w_hp, Y, bias=None, epi: int = EPI_F32, stream=None):
    """quantize_act + dual_gemm with the packed activations in the library's
    static scratch (osm_linear_noalloc): nothing is allocated, for callers
    that cannot allocate device memory at run time (a runtime whose pool
    owns the GPU's memory, a plug-in handed only tensors and a stream).
    Calls that overlap on the GPU race on the shared scratch; the first call
    on a device looks up the scratch address and should precede any stream
    capture."""
    import torch
    M, K = X.shape
    if K != plan.K:
        raise ValueError("X must have K columns")
    cbn, sbn, hbn = plan.sizes(plan.N)
    ybytes = M * plan.N * (4 if epi == EPI_F32 else 2)
    ytypes = (torch.float32,) if epi == EPI_F32 else _bf16_types()
    _check(lib().osm_linear_noalloc(plan.handle, _ptr(X, "X", _bf16_types()), M,
                                    _ptr(w_codes, "w_codes", _u8_types(), cbn, allow_none=cbn == 0),
                                    _ptr(w_scales, "w_scales", _u8_types(), sbn, allow_none=sbn == 0),
                                    _ptr(w_hp, "w_hp", _bf16_types(), hbn, allow_none=hbn == 0),
                                    _ptr(bias, "bias", (torch.float32,), plan.N * 4, allow_none=True), int(epi),
                                    _ptr(Y, "Y", ytypes, ybytes), _stream(stream)))


def scales_to_logical(swizzled: np.ndarray, rows: int, nblocks: int) -> np.ndarray:
    """Un-swizzle a scales buffer into [rows][nblocks] (osm_scales_to_logical)."""
    swizzled = np.ascontiguousarray(swizzled, dtype=np.uint8)
    out = np.zeros((rows, nblocks), np.uint8)
    if rows and nblocks:
        _check(lib().osm_scales_to_logical(_host_ptr(swizzled), rows, nblocks, _host_ptr(out)))
    return out


# ----------------------------------------------------------------- composition

def calibrate(X_batches, W, alpha: float, k: int, stream=None):
    """Per-channel statistics over calibration batches (device kernels),
    then Eq. (2)/(4) on the host: returns (s, inv_s, O, amax, wmax)."""
    import torch
    K = W.shape[0]
    amax = torch.zeros(K, dtype=torch.float32, device=W.device)
    wmax = torch.empty(K, dtype=torch.float32, device=W.device)
    for X in X_batches:
        act_amax_accumulate(X, amax, stream)
    weight_amax(W, wmax, stream)
    a, w = amax.cpu().numpy(), wmax.cpu().numpy()
    s, inv_s, O = calibrate_finalize(a, w, alpha, k)
    return s, inv_s, O, a, w


class QuantLinear:
    """A packed layer: plan + resident packed weights. `forward(X)` runs
    quantize_act and dual_gemm on the current stream."""

    def __init__(self, plan: Plan, W, bias=None, device="cuda"):
        self.plan = plan
        self.w_codes, self.w_scales, self.w_hp = plan.alloc_packed(plan.N, device)
        pack_weights(plan, W, self.w_codes, self.w_scales, self.w_hp)
        self.bias = bias

    def forward(self, X, epi: int = EPI_F32, out=None, act_buffers=None, stream=None):
        import torch
        M = X.shape[0]
        a = act_buffers if act_buffers is not None else self.plan.alloc_packed(M, X.device)
        quantize_act(self.plan, X, *a, stream=stream)
        if out is None:
            out = torch.empty((M, self.plan.N), dtype=torch.float32 if epi == EPI_F32 else torch.bfloat16,
                              device=X.device)
        dual_gemm(self.plan, *a, M, self.w_codes, self.w_scales, self.w_hp, out, bias=self.bias, epi=epi,
                  stream=stream)
        return out
