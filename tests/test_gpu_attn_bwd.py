"""Backward parity: hd_attn_bwd (CUDA, through the C ABI) vs the float64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import synthetic as syn
from tests.gpu_util import G_MAX, G_MEAN, check, dev, host64, need_gpu, sample_rows

pytestmark = pytest.mark.gpu

MODES = [hd.INTRA, hd.CROSS_FULL, hd.CROSS_WINDOW]


def run_bwd(inp, n, mode, W, fin, scale):
    q, k, v, do = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["do"])
    out, lse = hd.attn_fwd(q, k, v, n, mode, W, fin, scale)
    dq, dk, dv = hd.attn_bwd(q, k, v, out, lse, do, n, mode, W, fin, scale)
    torch.cuda.synchronize()
    assert hd.hd_device_status() == hd.HD_OK
    return dq, dk, dv


SMALL = [
    (1, 64, 4, 4, 4, 64, 3),
    (2, 37, 3, 4, 2, 128, 5),
    (1, 50, 1, 2, 1, 64, 17),
    (1, 9, 8, 2, 2, 128, 2),
    (1, 1, 4, 2, 1, 64, 1),
    (1, 130, 2, 6, 3, 64, 64),
    (1, 100, 4, 2, 2, 128, 300),
    (1, 1200, 2, 2, 1, 64, 100),  # 10 key tiles per INTRA stream: a partial grid bucket
]


@pytest.mark.parametrize("shape", SMALL, ids=[str(s) for s in SMALL])
@pytest.mark.parametrize("mode", MODES, ids=["INTRA", "CROSS_FULL", "CROSS_WINDOW"])
@pytest.mark.parametrize("fin", [0, 1], ids=["all", "final"])
def test_bwd_small_full_compare(shape, mode, fin):
    need_gpu()
    B, L, n, Hq, Hkv, D, W = shape
    scale = 1.0 / math.sqrt(D)
    inp = syn.attention_inputs(B, L, n, Hq, Hkv, D, final_only=bool(fin), seed=L + 3 * n + D,
                               with_grad=True)
    dq, dk, dv = run_bwd(inp, n, mode, W, fin, scale)
    rq, rk, rv = oracle.attn_bwd(inp["q"], inp["k"], inp["v"], inp["do"], n, mode, W, bool(fin), scale)
    check(host64(dq), rq, G_MAX, G_MEAN, "dQ")
    check(host64(dk), rk, G_MAX, G_MEAN, "dK")
    check(host64(dv), rv, G_MAX, G_MEAN, "dV")


def test_bwd_tiny_workload_exact_shapes():
    need_gpu()
    w = syn.WORKLOADS["tiny"]
    inp = syn.attention_inputs(w["B"], w["L"], w["n"], w["Hq"], w["Hkv"], w["D"], seed=1, with_grad=True)
    for mode in (hd.INTRA, hd.CROSS_FULL):
        dq, dk, dv = run_bwd(inp, w["n"], mode, 0, 0, w["scale"])
        rq, rk, rv = oracle.attn_bwd(inp["q"], inp["k"], inp["v"], inp["do"], w["n"], mode, 1, False,
                                     w["scale"])
        check(host64(dq), rq, G_MAX, G_MEAN, "dQ")
        check(host64(dk), rk, G_MAX, G_MEAN, "dK")
        check(host64(dv), rv, G_MAX, G_MEAN, "dV")


def _sampled(name, mode, seed, qpairs, kvpairs, rows_per_head=256, key_runs=2):
    need_gpu()
    w = syn.WORKLOADS[name]
    B, L, n, Hq, Hkv, D = w["B"], w["L"], w["n"], w["Hq"], w["Hkv"], w["D"]
    W = w.get("W", 0)
    inp = syn.attention_inputs(B, L, n, Hq, Hkv, D, seed=seed, with_grad=True)
    dq, dk, dv = run_bwd(inp, n, mode, W, 0, w["scale"])
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    torch.cuda.empty_cache()
    S = n * L
    t64 = {k: inp[k].float().numpy().astype(np.float64) for k in ("q", "k", "v", "do")}
    errs = []
    for (b, h) in qpairs:
        rows = sample_rows(S, n, W, False, rows_per_head, seed * 1000 + b * 31 + h)
        ref = oracle.attn_bwd_dq_rows(t64["q"], t64["k"], t64["v"], t64["do"], n, mode, max(W, 1), False,
                                      w["scale"], b, h, rows)
        got = dq[b, rows, h].float().numpy()
        assert np.abs(got - ref).max() <= G_MAX, ("dQ", b, h, np.abs(got - ref).max())
        errs.append(np.abs(got - ref).ravel())
    rng = np.random.default_rng(seed)
    for (b, kh) in kvpairs:
        starts = [0, S - 64] + list(rng.integers(64, S - 128, size=max(0, key_runs - 2)))
        cols = np.unique(np.concatenate([np.arange(s0, s0 + 64) for s0 in starts[:key_runs]]))
        rk, rv = oracle.attn_bwd_kv_cols(t64["q"], t64["k"], t64["v"], t64["do"], n, mode, max(W, 1),
                                         False, w["scale"], b, kh, cols)
        gk, gv = dk[b, cols, kh].float().numpy(), dv[b, cols, kh].float().numpy()
        assert np.abs(gk - rk).max() <= G_MAX, ("dK", b, kh, np.abs(gk - rk).max())
        assert np.abs(gv - rv).max() <= G_MAX, ("dV", b, kh, np.abs(gv - rv).max())
        errs += [np.abs(gk - rk).ravel(), np.abs(gv - rv).ravel()]
    allerr = np.concatenate(errs)
    assert allerr.mean() <= G_MEAN, allerr.mean()


def test_bwd_intra_train_workload_sampled():
    """B4 n4 L2048, 16/4 heads, D128, INTRA: dQ on 256 rows per head, dK/dV on key runs."""
    w = syn.WORKLOADS["intra_train"]
    qpairs = [(b, h) for b in range(w["B"]) for h in range(w["Hq"])]
    _sampled("intra_train", hd.INTRA, 6, qpairs, [(0, 0), (3, 3)], key_runs=2)


def test_bwd_cross_window_workload_sampled():
    """B2 n4 L8192 W1024, 32/8 heads, D128, CROSS_WINDOW: dQ on 256 rows per head, dK/dV runs."""
    w = syn.WORKLOADS["cross_window"]
    qpairs = [(b, h) for b in range(w["B"]) for h in range(w["Hq"])]
    _sampled("cross_window", hd.CROSS_WINDOW, 7, qpairs, [(0, 0), (1, 7)], key_runs=2)
