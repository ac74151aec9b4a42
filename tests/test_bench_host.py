"""Host-side logic of bench.py: FLOP/pair accounting and the N > 1 timing rule.

The multi-rank part runs two gloo ranks on the CPU (no GPU involved).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle


@pytest.mark.parametrize("n,L,W", [(4, 16, 3), (3, 10, 2), (1, 12, 5), (4, 8, 100)])
@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("fin", [0, 1])
def test_pair_counts_match_the_oracle_mask(n, L, W, mode, fin):
    S = n * L
    want = oracle.mask_matrix(oracle.query_positions(S, n, bool(fin)), S, n, mode, W).sum()
    assert bench.pairs(S, n, mode, W, fin) == want


@pytest.mark.parametrize("mode", [0, 1])
def test_decode_pair_counts_match_the_oracle_mask(mode):
    n, T = 4, 9
    S = (T + 1) * n
    qpos = T * n + np.arange(n)
    want = oracle.mask_matrix(qpos, S, n, mode, 1).sum()
    assert bench.decode_pairs(n, T, mode) == want


def test_step_plan_covers_every_hot_path_row():
    ops = bench.step_plan(dict(bench.WL))
    names = {o["name"] for o in ops}
    for m in ("intra", "cross_full", "cross_window", "final_only"):
        assert f"fwd_{m}" in names and f"bwd_{m}" in names
    assert {"expand", "decode_cross_full", "decode_intra"} <= names
    fwd = next(o for o in ops if o["name"] == "fwd_intra")
    # B4 n4 L2048 Hq16 D128: 4 * 2048*2049/2 pairs per (b, h), 64 (b, h)
    assert fwd["pairs"] == 64 * 4 * 2048 * 2049 // 2
    assert fwd["flops"] == 4 * 128 * fwd["pairs"]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_max([10.0 + rank, 5.0 - rank], torch.device("cpu"))
        val = bench.whole_job_value(1e12, world, got[0])
        out.put((rank, got, val))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_count_every_replica():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, val in res:
        assert got == [11.0, 5.0]
        assert abs(val - 2 * 1e12 / 11e-3 / 1e12) < 1e-9
