"""Final-stream-only decode parity: hd_decode_attn_final (CUDA, through the C ABI) vs the
float64 oracle, plus its agreement with the last row of the all-stream decode."""
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
IDS = ["INTRA", "CROSS_FULL", "CROSS_WINDOW"]


def _final_inputs(B, n, T, Tcap, Hq, Hkv, D, seed, ragged):
    inp = syn.decode_inputs(B, n, T, Tcap, Hq, Hkv, D, seed=seed, ragged=ragged)
    inp["qf"] = inp["q"][:, n - 1:n].contiguous()  # the final stream's query
    return inp


def _run(inp, n, mode, W, scale):
    out, lse = hd.decode_attn_final(inp["qf"].cuda(), inp["k_cache"].cuda(), inp["v_cache"].cuda(),
                                    inp["seqlen"].cuda(), n, mode, W, scale)
    torch.cuda.synchronize()
    return out, lse


SMALL = [
    # B, n, T, Tcap, Hq, Hkv, D, W, ragged
    (3, 3, 20, 30, 6, 2, 64, 4, True),
    (2, 4, 700, 701, 16, 4, 128, 37, False),
    (4, 4, 100, 128, 32, 4, 128, 9, True),   # 8 query rows per KV head
    (1, 8, 3, 5, 2, 1, 64, 2, False),
    (2, 1, 333, 400, 4, 4, 128, 50, True),   # n = 1: ordinary decode
    (2, 4, 0, 4, 8, 8, 64, 1, False),        # first token
    (3, 2, 1000, 1100, 4, 1, 128, 300, True),  # INTRA key space spans several chunks
]


@pytest.mark.parametrize("shape", SMALL, ids=[str(s) for s in SMALL])
@pytest.mark.parametrize("mode", MODES, ids=IDS)
def test_final_decode_small_full_compare(shape, mode):
    need_gpu()
    B, n, T, Tcap, Hq, Hkv, D, W, ragged = shape
    inp = _final_inputs(B, n, T, Tcap, Hq, Hkv, D, seed=T + n + 1, ragged=ragged)
    scale = 1.0 / math.sqrt(D)
    out, lse = _run(inp, n, mode, W, scale)
    assert hd.hd_device_status() == hd.HD_OK
    assert out.shape == (B, 1, Hq, D) and lse.shape == (B, Hq, 1)
    o_ref, l_ref = oracle.decode_attn(inp["qf"], inp["k_cache"], inp["v_cache"], inp["seqlen"], n, mode,
                                      W, scale, final_only=True)
    check(host64(out), o_ref, O_MAX, O_MEAN, "O")
    check(host64(lse), l_ref, LSE_MAX, LSE_MAX, "LSE")


@pytest.mark.parametrize("mode", MODES, ids=IDS)
def test_final_decode_equals_last_row_of_all_stream_decode(mode):
    need_gpu()
    B, n, T, Hq, Hkv, D, W = 3, 4, 300, 16, 4, 128, 20
    inp = _final_inputs(B, n, T, T + 1, Hq, Hkv, D, seed=8, ragged=True)
    out_all, lse_all = hd.decode_attn(inp["q"].cuda(), inp["k_cache"].cuda(), inp["v_cache"].cuda(),
                                      inp["seqlen"].cuda(), mode, W, 0.09)
    out, lse = _run(inp, n, mode, W, 0.09)
    check(host64(out), host64(out_all[:, n - 1:n]), 1.6e-2, 1e-3, "final vs all-stream row")
    check(host64(lse), host64(lse_all[:, :, n - 1:n]), 1e-4, 1e-4, "final lse vs all-stream row")


def test_final_intra_ignores_other_streams_rows():
    """INTRA reads only the final stream's cache rows: poisoning the others changes nothing."""
    need_gpu()
    B, n, T, Hq, Hkv, D = 2, 4, 200, 8, 2, 64
    inp = _final_inputs(B, n, T, T + 1, Hq, Hkv, D, seed=9, ragged=False)
    out1, lse1 = _run(inp, n, hd.INTRA, 0, 0.125)
    other = torch.arange(inp["k_cache"].shape[1]) % n != n - 1
    inp["k_cache"][:, other] = float("nan")
    inp["v_cache"][:, other] = float("inf")
    out2, lse2 = _run(inp, n, hd.INTRA, 0, 0.125)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


@pytest.mark.parametrize("mode", MODES, ids=IDS)
def test_final_decode_workload(mode):
    """B8, n4, 16384 prior tokens (65540 cache rows), 32/8 heads, D128; every row vs the oracle."""
    need_gpu()
    w = syn.WORKLOADS["decode"]
    B, n, T, Hq, Hkv, D = 8, w["n"], w["T"], w["Hq"], w["Hkv"], w["D"]
    inp = _final_inputs(B, n, T, T + 1, Hq, Hkv, D, seed=13, ragged=False)
    out, lse = _run(inp, n, mode, 1024, w["scale"])
    assert hd.hd_device_status() == hd.HD_OK
    o_ref, l_ref = oracle.decode_attn(inp["qf"], inp["k_cache"], inp["v_cache"], inp["seqlen"], n, mode,
                                      1024, w["scale"], final_only=True)
    check(host64(out), o_ref, O_MAX, O_MEAN, "O")
    check(host64(lse), l_ref, LSE_MAX, LSE_MAX, "LSE")


def test_final_decode_bad_seqlen_on_device():
    need_gpu()
    inp = _final_inputs(3, 2, 10, 12, 4, 2, 64, seed=3, ragged=False)
    inp["seqlen"][2] = 0
    hd.hd_device_status(clear=True)
    out, lse = _run(inp, 2, hd.INTRA, 0, 0.125)
    assert hd.hd_device_status(clear=True) == hd.HD_ERR_DEVICE_INDEX
    assert (out[2] == 0).all() and torch.isinf(lse[2]).all()
    o_ref, _ = oracle.decode_attn(inp["qf"][:2], inp["k_cache"][:2], inp["v_cache"][:2],
                                  inp["seqlen"][:2], 2, hd.INTRA, 1, 0.125, final_only=True)
    check(host64(out[:2]), o_ref, O_MAX, O_MEAN, "valid rows")
