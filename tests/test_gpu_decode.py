"""Decode parity: hd_decode_attn (CUDA, through the C ABI) vs the float64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import synthetic as syn
from tests.gpu_util import LSE_MAX, O_MAX, O_MEAN, check, host64, need_gpu

pytestmark = pytest.mark.gpu

MODES = [hd.INTRA, hd.CROSS_FULL, hd.CROSS_WINDOW]


def run_decode(inp, mode, W, scale):
    out, lse = hd.decode_attn(inp["q"].cuda(), inp["k_cache"].cuda(), inp["v_cache"].cuda(),
                              inp["seqlen"].cuda(), mode, W, scale)
    torch.cuda.synchronize()
    return out, lse


SMALL = [
    # B, n, T, Tcap, Hq, Hkv, D, W, ragged
    (3, 3, 20, 30, 6, 2, 64, 4, True),     # 9 query rows, ragged lengths
    (2, 4, 700, 701, 16, 4, 128, 37, False),
    (4, 4, 100, 128, 32, 4, 128, 9, True),  # 32 rows: two 16-row tiles
    (1, 8, 3, 5, 2, 1, 64, 2, False),
    (2, 1, 333, 400, 4, 4, 128, 50, True),  # n = 1: ordinary decode
    (2, 4, 0, 4, 8, 8, 64, 1, False),       # first token: only the new rows
]


@pytest.mark.parametrize("shape", SMALL, ids=[str(s) for s in SMALL])
@pytest.mark.parametrize("mode", MODES, ids=["INTRA", "CROSS_FULL", "CROSS_WINDOW"])
def test_decode_small_full_compare(shape, mode):
    need_gpu()
    B, n, T, Tcap, Hq, Hkv, D, W, ragged = shape
    inp = syn.decode_inputs(B, n, T, Tcap, Hq, Hkv, D, seed=T + n, ragged=ragged)
    scale = 1.0 / math.sqrt(D)
    out, lse = run_decode(inp, mode, W, scale)
    assert hd.hd_device_status() == hd.HD_OK
    o_ref, l_ref = oracle.decode_attn(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlen"], n, mode,
                                      W, scale)
    check(host64(out), o_ref, O_MAX, O_MEAN, "O")
    check(host64(lse), l_ref, LSE_MAX, LSE_MAX, "LSE")


def test_decode_equals_prefill_rows_on_device():
    """Property: decode row (T, s) equals prefill row p = T*n + s over the same cache."""
    need_gpu()
    n, T, Hq, Hkv, D = 4, 77, 8, 2, 128
    S = (T + 1) * n
    att = syn.attention_inputs(1, T + 1, n, Hq, Hkv, D, seed=21)
    for mode in MODES:
        o_all, l_all = hd.attn_fwd(att["q"].cuda(), att["k"].cuda(), att["v"].cuda(), n, mode, 9, 0, 0.1)
        q = att["q"][:, T * n:].contiguous()
        seq = torch.tensor([T + 1], dtype=torch.int32)
        out, lse = hd.decode_attn(q.cuda(), att["k"].cuda(), att["v"].cuda(), seq.cuda(), mode, 9, 0.1)
        torch.cuda.synchronize()
        check(host64(out), host64(o_all[:, T * n:]), 1.6e-2, 1e-3, "decode vs prefill")
        check(host64(lse), host64(l_all[:, :, T * n:]), 1e-4, 1e-4, "decode lse vs prefill")
        assert S == att["k"].shape[1]


@pytest.mark.parametrize("B", [8, 64])
@pytest.mark.parametrize("mode", [hd.CROSS_FULL, hd.INTRA], ids=["CROSS_FULL", "INTRA"])
def test_decode_workload(B, mode):
    """n4, 16384 prior tokens (65540 cache rows incl. the new token), 32/8 heads, D128."""
    need_gpu()
    w = syn.WORKLOADS["decode"]
    n, T, Hq, Hkv, D = w["n"], w["T"], w["Hq"], w["Hkv"], w["D"]
    inp = syn.decode_inputs(B, n, T, T + 1, Hq, Hkv, D, seed=5 + B)
    out, lse = run_decode(inp, mode, 0, w["scale"])
    assert hd.hd_device_status() == hd.HD_OK
    # every query row for B = 8; a seeded subset of sequences for B = 64
    bs = list(range(B)) if B <= 8 else sorted({0, B - 1, *np.random.default_rng(B).choice(B, 6, replace=False)})
    sub = {k: inp[k][bs] for k in ("q", "k_cache", "v_cache", "seqlen")}
    o_ref, l_ref = oracle.decode_attn(sub["q"], sub["k_cache"], sub["v_cache"], sub["seqlen"], n, mode, 1,
                                      w["scale"])
    check(host64(out[bs]), o_ref, O_MAX, O_MEAN, "O")
    check(host64(lse[bs]), l_ref, LSE_MAX, LSE_MAX, "LSE")


def test_decode_rejects_bad_seqlen_on_device():
    """A seqlen outside [1, Tcap] leaves its rows zero and records HD_ERR_DEVICE_INDEX."""
    need_gpu()
    inp = syn.decode_inputs(3, 2, 10, 12, 4, 2, 64, seed=3)
    inp["seqlen"][1] = 13
    hd.hd_device_status(clear=True)
    out, lse = run_decode(inp, hd.CROSS_FULL, 0, 0.125)
    assert hd.hd_device_status(clear=True) == hd.HD_ERR_DEVICE_INDEX
    assert hd.hd_device_status(clear=True) == hd.HD_OK
    assert (out[1] == 0).all() and torch.isinf(lse[1]).all()
    o_ref, _ = oracle.decode_attn(inp["q"][[0, 2]], inp["k_cache"][[0, 2]], inp["v_cache"][[0, 2]],
                                  inp["seqlen"][[0, 2]], 2, hd.CROSS_FULL, 1, 0.125)
    check(host64(out[[0, 2]]), o_ref, O_MAX, O_MEAN, "valid rows")
