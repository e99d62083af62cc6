"""Data-parallel plumbing for the layer over several GPUs (one process per GPU).

The hot path is data-parallel over tokens: every rank holds the packed
weights and processes its own token shard with no collective on the data
path. Calibration is the only exchange: the per-channel activation maxima
of Eq. (4) / Eq. (2) are combined across ranks with an all-reduce (MAX)
before the host-side finalisation (osm_calibrate_finalize), so every rank
derives the same s and O.
"""
from __future__ import annotations

import numpy as np


def shard_rows(M: int, world: int, rank: int, align: int = 128):
    """Contiguous token range [lo, hi) of `rank` when M tokens are split over
    `world` ranks in multiples of `align` rows (the last rank takes the rest)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    blocks = -(-M // align)
    per = blocks // world
    extra = blocks % world
    b0 = rank * per + min(rank, extra)
    b1 = b0 + per + (1 if rank < extra else 0)
    return min(M, b0 * align), min(M, b1 * align)


def allreduce_max_(t, group=None):
    """In-place all-reduce (MAX) of a tensor of per-channel maxima."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t


def calibrate_from_local_stats(amax_local, wmax, alpha: float, k: int, group=None):
    """Combine per-rank activation maxima (torch tensor, any device) across
    ranks, then run Eq. (2) / Eq. (4) on the host. Returns (s, inv_s, O)."""
    import outlier_split_mixed_b200 as osm
    amax = allreduce_max_(amax_local.clone(), group)
    return osm.calibrate_finalize(amax.cpu().numpy().astype(np.float32),
                                  np.asarray(wmax.cpu().numpy() if hasattr(wmax, "cpu") else wmax, np.float32),
                                  alpha, k)


def nvfp4_exponents_from_local_stats(amax_local, wmax, s, inv_s, O, group=None):
    """The NVFP4 per-tensor exponents (g_act, g_w) of a plan from per-rank
    activation maxima combined across ranks (all-reduce MAX), so that every
    rank encodes with the same factors (osm_nvfp4_plan_exponents)."""
    import outlier_split_mixed_b200 as osm
    amax = allreduce_max_(amax_local.clone(), group)
    return osm.nvfp4_plan_exponents(amax.cpu().numpy().astype(np.float32),
                                    np.asarray(wmax.cpu().numpy() if hasattr(wmax, "cpu") else wmax, np.float32),
                                    s, inv_s, O)
