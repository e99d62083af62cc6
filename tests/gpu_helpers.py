"""Shared helpers for the GPU parity tests: run the CUDA path through the C
ABI and the oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import outlier_split_mixed_b200 as osm


def to_dev_bf16(h: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(h).view(np.int16)).cuda().view(torch.bfloat16)


def to_np_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def unswizzle(buf: np.ndarray, rows: int, nb: int) -> np.ndarray:
    """tcgen05 scale layout -> logical [round_up(rows,128)][nb], written from
    the layout's definition: 512-byte atoms (128 rows x 4 blocks), K-atoms
    contiguous, inside the atom (r%32)*16 + ((r%128)//32)*4 + b%4."""
    rows_p = (rows + 127) // 128 * 128
    if nb == 0:
        return np.zeros((rows_p, 0), np.uint8)
    a = np.asarray(buf, np.uint8).reshape(rows_p // 128, nb // 4, 32, 4, 4)
    return a.transpose(0, 3, 2, 1, 4).reshape(rows_p, nb)


def gpu_calibrate(X: np.ndarray, W: np.ndarray, alpha: float, k: int, batches: int = 1):
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    chunks = [c for c in torch.tensor_split(Xd, batches, dim=0) if c.shape[0] > 0]
    s, inv_s, O, amax, wmax = osm.calibrate([c.contiguous() for c in chunks], Wd, alpha, k)
    return Xd, Wd, s, inv_s, O, amax, wmax


def gpu_layer(X, W, alpha, k, mode, epi=osm.EPI_F32, bias=None, batches=1, plan_sO=None, rows=None,
              hp_fp16=False, nv=False):
    """Full CUDA path. Returns a dict of host arrays (rows of the activation
    outputs and of Y restricted to `rows` when given)."""
    M, K = X.shape
    N = W.shape[1]
    Xd, Wd, s, inv_s, O, amax, wmax = gpu_calibrate(X, W, alpha, k, batches)
    if plan_sO is not None:
        s, O = plan_sO
    g_act = g_w = 0
    if nv:
        g_act, g_w = osm.nvfp4_plan_exponents(amax, wmax, s, inv_s, O)
    plan = osm.Plan(K, N, k, s, O, mode, hp_fp16=hp_fp16, fmt=osm.FMT_NVFP4 if nv else osm.FMT_MXFP4,
                    g_act=g_act, g_w=g_w)
    wc, wsc, wh = plan.alloc_packed(N)
    osm.pack_weights(plan, Wd, wc, wsc, wh)
    ac, asc, ah = plan.alloc_packed(M)
    osm.quantize_act(plan, Xd, ac, asc, ah)
    Y = torch.empty((M, N), dtype=torch.float32 if epi == osm.EPI_F32 else torch.bfloat16, device="cuda")
    bd = None if bias is None else torch.from_numpy(bias).cuda()
    osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y, bias=bd, epi=epi)
    torch.cuda.synchronize()
    status = plan.status()
    nb = plan.nblocks
    sel = slice(None) if rows is None else torch.from_numpy(np.asarray(rows)).cuda()
    out = dict(
        s=s, inv_s=inv_s, O=O, amax=amax, wmax=wmax, status=status, plan=plan, M=M, g=(g_act, g_w),
        w_codes=wc.cpu().numpy().reshape(N, plan.Kbp // 2),
        w_scales=unswizzle(wsc.cpu().numpy(), N, nb),
        w_hp=to_np_u16(wh).reshape(N, plan.kp),
        a_codes=ac.view(M, plan.Kbp // 2)[sel].cpu().numpy(),
        a_scales_full=unswizzle(asc.cpu().numpy(), M, nb),
        a_hp=to_np_u16(ah.view(M, plan.kp)[sel]),
        Y=(Y[sel].cpu().numpy() if epi == osm.EPI_F32 else Y[sel].float().cpu().numpy()),
    )
    return out


def oracle_layer(X, W, alpha, k, mode, rows=None, bias=None, hp_fp16=False, nv=False):
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, O = oracle.calibrate(amax, wmax, alpha, k)
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    g = None
    if nv:
        g = oracle.nvfp4_plan_exponents(amax, wmax, s, inv_s, O)
        wc, wsc, wh = oracle.pack_weights_nv(W, s, O, g[1])
        ac, asc, ah = oracle.quantize_act_nv(X[rows], inv_s, O, g[0])
        y, T = oracle.dual_gemm_rows_nv(ac, asc, ah, np.arange(len(rows)), wc, wsc, wh, g[0], g[1], bias)
    else:
        wc, wsc, wh = oracle.pack_weights(W, s, O, mode, hp_fp16=hp_fp16)
        ac, asc, ah = oracle.quantize_act(X[rows], inv_s, O, hp_fp16=hp_fp16)
        y, T = oracle.dual_gemm_rows(ac, asc, ah, np.arange(len(rows)), wc, wsc, wh, bias, hp_fp16=hp_fp16)
    return dict(amax=amax, wmax=wmax, s=s, inv_s=inv_s, O=O, w_codes=wc, w_scales=wsc, w_hp=wh,
                a_codes=ac, a_scales=asc, a_hp=ah, y=y, T=T, rows=rows, g=g)


def bits(a):
    return np.asarray(a).view(np.uint32) if np.asarray(a).dtype == np.float32 else np.asarray(a)


def assert_bitexact(name, got, want):
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    if not np.array_equal(bits(got), bits(want)):
        bad = np.argwhere(bits(got) != bits(want))
        raise AssertionError(f"{name}: {len(bad)} mismatches, first at {bad[:5].tolist()}: "
                             f"got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}")


def assert_y_close(Y, y_ref, T, bf16: bool):
    """|y_gpu - y_ref| <= 1e-5 * sum_k |a_k w_k| + 1e-6 (FP32 accumulation
    bound); BF16 output adds one BF16 rounding, 2^-8 |y_ref|."""
    tol = 1e-5 * T + 1e-6
    if bf16:
        tol = tol + 2.0 ** -8 * np.abs(y_ref)
    err = np.abs(Y.astype(np.float64) - y_ref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"Y out of tolerance at {int(bad.sum())} elements; first {i.tolist()}: "
                             f"gpu {Y[tuple(i)]} ref {y_ref[tuple(i)]} tol {tol[tuple(i)]} "
                             f"max err/T {np.max(err / np.maximum(T, 1e-30)):.3e}")
    return float(np.max(err / np.maximum(T, 1e-30)))


def compare_layer(g, o, rows=None, check_weights_rows=None):
    """Bit-exact on everything integer-valued, tolerance on Y."""
    assert g["status"] == 0
    assert_bitexact("amax", g["amax"], o["amax"])
    assert_bitexact("wmax", g["wmax"], o["wmax"])
    assert_bitexact("s", g["s"], o["s"])
    assert_bitexact("inv_s", g["inv_s"], o["inv_s"])
    assert_bitexact("O", g["O"], o["O"])
    if o.get("g") is not None:
        assert tuple(g["g"]) == tuple(o["g"]), ("NVFP4 tensor exponents", g["g"], o["g"])
    N = o["w_codes"].shape[0]
    wr = np.arange(N) if check_weights_rows is None else check_weights_rows
    assert_bitexact("w_codes", g["w_codes"][wr], o["w_codes"][wr])
    assert_bitexact("w_scales", g["w_scales"][:N][wr], o["w_scales"][wr])
    assert np.all(g["w_scales"][N:] == 0), "padding rows of w_scales must be 0"
    assert_bitexact("w_hp", g["w_hp"][wr], o["w_hp"][wr])
    r = o["rows"]
    M = g["M"]
    assert_bitexact("a_codes", g["a_codes"], o["a_codes"])
    assert_bitexact("a_scales", g["a_scales_full"][:M][r], o["a_scales"])
    assert np.all(g["a_scales_full"][M:] == 0), "padding rows of a_scales must be 0"
    assert_bitexact("a_hp", g["a_hp"], o["a_hp"])


def gelu_tolerance(y, T, g):
    """Bound on |h_gpu - GELU(y)| for h_gpu = bf16(GELU_f32(acc)), with y the
    oracle's FP64 sum, T = sum |a w| and g = GELU(y) in FP64:
      1.13 (1e-5 T + 1e-6)        the FP32 accumulation bound through GELU
                                  (|GELU'| <= 1.129);
      5e-7 |g| + 2e-8 |y|         the epilogue's FP32 routine against the
                                  definition (the relative error of
                                  exp(-2|u|) grows with |u| in the left tail);
      2^-8 |g| (1 + 1e-6)         one rounding to BF16 (half an ulp)."""
    return (1.13 * (1e-5 * T + 1e-6) + 5e-7 * np.abs(g) + 2e-8 * np.abs(y)
            + 2.0 ** -8 * (1.0 + 1e-6) * np.abs(g) + 1e-30)
