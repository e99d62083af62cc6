"""Per-layer alpha / k search.

"W4A4 Quantization for Inference on Wan2.2-I2V-A14B" observes the largest
activation tails in early high-noise FFN blocks and suggests tuning alpha
(Eq. (2)) and k (Eq. (4)) per layer. This harness scores every candidate
(alpha, k) on a calibration batch with the library's own CUDA path --
calibration, plan, weight packing, quantize_act, dual_gemm -- by the
relative Frobenius error of the layer output against the unquantised
product of the same BF16 operands (a k = K, s = 1 plan: every channel on
the BF16 branch, FP32 accumulation), and returns the best candidate.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Iterable, List, Optional, Tuple

import numpy as np

from . import (WSCALE_1x32, EPI_F32, Plan, act_amax_accumulate, calibrate_finalize, calibrate_finalize_scored,
               dual_gemm, error_norms, pack_weights, quantize_act, weight_amax)


@dataclass
class SearchResult:
    alpha: float
    k: int
    rel_err: float
    table: List[Tuple[float, int, float]] = field(default_factory=list)  # (alpha, k, rel_err) in search order


def pick_best(table: Iterable[Tuple[float, int, float]]) -> Tuple[float, int, float]:
    """The entry with the smallest error; ties go to the earlier entry."""
    best = None
    for entry in table:
        if best is None or entry[2] < best[2]:
            best = entry
    if best is None:
        raise ValueError("empty search")
    return best


def _dense_output(X, W, wmode):
    import torch
    M, K = X.shape
    N = W.shape[1]
    plan = Plan(K, N, K, np.ones(K, np.float32), np.arange(K, dtype=np.int32), wmode)
    try:
        wc, wsc, wh = plan.alloc_packed(N, X.device)
        pack_weights(plan, W, wc, wsc, wh)
        ac, asc, ah = plan.alloc_packed(M, X.device)
        quantize_act(plan, X, ac, asc, ah)
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
        dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y, epi=EPI_F32)
        return Y
    finally:
        plan.close()


def search_alpha_k(X, W, alphas: Iterable[float], ks: Iterable[int], wmode: int = WSCALE_1x32,
                   score: Optional[np.ndarray] = None,
                   evaluate: Optional[Callable[[float, int], float]] = None) -> SearchResult:
    """Search alpha x k (k in the order given, alpha inner) on the
    calibration batch X [M][K] BF16 (device) for the layer W [K][N] BF16
    (device). `score` (host float[K]) replaces the maximum as Eq. (4)'s
    channel score (e.g. osm_act_percentile). `evaluate(alpha, k) -> rel_err`
    replaces the CUDA evaluation (for testing the search logic)."""
    alphas = [float(a) for a in alphas]
    ks = [int(k) for k in ks]
    if evaluate is None:
        evaluate = _cuda_evaluator(X, W, wmode, score)
    table = [(a, k, float(evaluate(a, k))) for k in ks for a in alphas]
    a, k, e = pick_best(table)
    return SearchResult(alpha=a, k=k, rel_err=e, table=table)


def _cuda_evaluator(X, W, wmode, score):
    import torch
    M, K = X.shape
    N = W.shape[1]
    amax = torch.zeros(K, dtype=torch.float32, device=X.device)
    wmax = torch.empty(K, dtype=torch.float32, device=X.device)
    act_amax_accumulate(X, amax)
    weight_amax(W, wmax)
    amax_h, wmax_h = amax.cpu().numpy(), wmax.cpu().numpy()
    Y_ref = _dense_output(X, W, wmode)
    Y = torch.empty((M, N), dtype=torch.float32, device=X.device)

    def evaluate(alpha: float, k: int) -> float:
        if score is None:
            s, _, O = calibrate_finalize(amax_h, wmax_h, alpha, k)
        else:
            s, _, O = calibrate_finalize_scored(amax_h, score, wmax_h, alpha, k)
        plan = Plan(K, N, k, s, O, wmode)
        try:
            wc, wsc, wh = plan.alloc_packed(N, X.device)
            pack_weights(plan, W, wc, wsc, wh)
            ac, asc, ah = plan.alloc_packed(M, X.device)
            quantize_act(plan, X, ac, asc, ah)
            dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y, epi=EPI_F32)
            e, n = error_norms(Y, Y_ref)
        finally:
            plan.close()
        return float(np.sqrt(e / n)) if n > 0 else float(np.sqrt(e))

    return evaluate
