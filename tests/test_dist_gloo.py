"""Multi-rank host logic on CPU (gloo, world size 2): token sharding and the
calibration all-reduce. Each rank computes the activation maxima of its own
token shard (oracle, CPU), the ranks combine them with an all-reduce (MAX),
and the library's host-side Eq. (2)/(4) finalisation must then reproduce,
bit for bit, the calibration of the whole batch on one process (and the
same NVFP4 per-tensor exponents)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from outlier_split_mixed_b200 import dist as odist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_rows_covers_everything_once():
    for M in (1, 127, 128, 300, 4096, 32760):
        for world in (1, 2, 3, 4, 8):
            seen = []
            for r in range(world):
                lo, hi = odist.shard_rows(M, world, r)
                assert (lo % 128 == 0 or lo == M) and lo <= hi
                seen.extend(range(lo, hi))
            assert seen == list(range(M))


def _worker(rank, world, port, out_q):
    import torch.distributed as dist

    import oracle
    from outlier_split_mixed_b200 import build, synth
    from outlier_split_mixed_b200 import dist as odist2
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        build.build()
        X = synth.acts_heavy_tailed(520, 256, seed=90, frac=0.03)
        W = synth.weights_gaussian(256, 64, seed=91, sigma=0.05)
        lo, hi = odist2.shard_rows(X.shape[0], world, rank)
        amax_local = torch.from_numpy(oracle.act_amax(X[lo:hi]) if hi > lo else np.zeros(256, np.float32))
        wmax = oracle.weight_amax(W)
        s, inv_s, O = odist2.calibrate_from_local_stats(amax_local, wmax, 0.6, 24)
        g = odist2.nvfp4_exponents_from_local_stats(amax_local, wmax, s, inv_s, O)
        out_q.put((rank, s.view(np.uint32).tolist(), O.tolist(), g))
    finally:
        dist.destroy_process_group()


def test_two_rank_calibration_matches_single_process():
    import oracle
    from outlier_split_mixed_b200 import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X = synth.acts_heavy_tailed(520, 256, seed=90, frac=0.03)
    W = synth.weights_gaussian(256, 64, seed=91, sigma=0.05)
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, O = oracle.calibrate(amax, wmax, 0.6, 24)
    g = oracle.nvfp4_plan_exponents(amax, wmax, s, inv_s, O)
    for rank, s_bits, O_r, g_r in results:
        assert s_bits == s.view(np.uint32).tolist(), rank
        assert O_r == O.tolist(), rank
        assert tuple(g_r) == tuple(g), rank     # NVFP4 exponents of the whole batch on every rank
