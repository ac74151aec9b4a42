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


def test_default_step_runs_every_configuration_at_its_sizes():
    parts = bench.plan_for("step")
    names = {o["name"] for _, _, ops in parts for o in ops}
    assert {"c2.fwd_intra", "c2.bwd_intra", "c3.fwd_cross_window", "c3.bwd_cross_window",
            "c4.fwd_cross_full", "c4.fwd_final_only", "c4.bwd_final_only", "c5b8.decode_cross_full",
            "c5b8.decode_intra", "c5b64.decode_cross_full", "c5b64.decode_intra", "x.expand"} == names
    sizes = {label: wl for label, wl, _ in parts}
    assert (sizes["c2"]["B"], sizes["c2"]["L"], sizes["c2"]["Hq"], sizes["c2"]["Hkv"]) == (4, 2048, 16, 4)
    assert (sizes["c3"]["B"], sizes["c3"]["L"], sizes["c3"]["W"], sizes["c3"]["Hq"]) == (2, 8192, 1024, 32)
    assert (sizes["c4"]["B"], sizes["c4"]["n"] * sizes["c4"]["L"]) == (1, 131072)
    assert (sizes["c5b8"]["B"], sizes["c5b64"]["B"], sizes["c5b8"]["T"]) == (8, 64, 16384)
    op = {o["name"]: o for _, _, ops in parts for o in ops}
    # 4a: 131072 (131072 + 1) / 2 pairs per head, 32 heads, 4 * D FLOPs each (140.7 TFLOP, the
    # published count for this configuration)
    assert op["c4.fwd_cross_full"]["flops"] == 4 * 128 * 32 * 131072 * 131073 // 2
    assert abs(op["c4.fwd_cross_full"]["flops"] / 1e12 - 140.7) < 0.1
    # decode B8: K and V of 65540 cache rows, 8 heads, D128, bf16 (2.148 GB)
    assert abs(op["c5b8.decode_cross_full"]["bytes"] / 1e9 - 2.148) < 0.01


def test_roofline_fraction_uses_the_burst_peak():
    op = dict(kind="fwd", flops=2e12)
    r = bench.roofline_of(op, 2.0, {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0})
    assert r["achieved"] == 1000.0 and r["frac"] == 0.625 and r["frac_of_sustained"] == round(1000 / 1400, 4)
    d = bench.roofline_of(dict(kind="decode", bytes=6e9), 1.0, {"hbm_gbs": 6000.0})
    assert d["bound"] == "hbm" and d["frac"] == 1.0


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
