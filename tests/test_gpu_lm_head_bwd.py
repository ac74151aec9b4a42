"""LM-head cross-entropy gradients: hd_lm_head_ce_bwd (CUDA, through the C ABI) vs the
float64 oracle.

Tolerance: G is stored in bf16 (relative rounding 2^-9) and the two products sum
in fp32, dh is rounded once to bf16. So errors are a few 2^-9 of the gradients'
scale: max |err| <= 2e-2 * max|ref|, mean <= 2e-3 * max|ref|.
"""
import numpy as np
import pytest
import torch

import oracle
import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import synthetic as syn
from tests.gpu_util import host64, need_gpu

pytestmark = pytest.mark.gpu


def _rel_check(got, want, what):
    got = host64(got) if torch.is_tensor(got) else np.asarray(got)
    want = np.asarray(want)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    scale = float(np.abs(want).max()) or 1.0
    err = np.abs(got - want)
    assert err.max() <= 2e-2 * scale and err.mean() <= 2e-3 * scale, \
        f"{what}: max {err.max():.3e} mean {err.mean():.3e} scale {scale:.3e}"


SHAPES = [
    # B, L, n, d, V
    (1, 64, 4, 256, 1000),    # the tiny workload's sizes
    (2, 37, 3, 128, 515),     # ragged rows and vocabulary
    (1, 300, 1, 192, 257),    # n = 1
    (2, 129, 4, 512, 2048),
    (1, 1024, 2, 512, 4096),  # mid size: several tiles of every kind
]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_lm_head_bwd_matches_oracle(shape):
    need_gpu()
    B, L, n, d, V = shape
    inp = syn.lm_head_inputs(B, L, n, d, V, seed=B * 7 + L, ignore_every=5)
    x, w, lab = inp["x"].cuda(), inp["w"].cuda(), inp["labels"].cuda()
    loss, lse = hd.lm_head_ce(x, w, lab, n)
    dh, dw = hd.lm_head_ce_bwd(x, w, lab, lse, n, grad_scale=0.5)
    torch.cuda.synchronize()
    assert hd.hd_device_status() == hd.HD_OK
    _, dh_ref, dw_ref = oracle.lm_head_ce_grad(inp["x"], inp["w"], inp["labels"], n)
    _rel_check(dh, 0.5 * dh_ref, "dh")
    _rel_check(dw, 0.5 * dw_ref, "dW")
    ign = inp["labels"].view(-1) < 0
    assert (dh.view(-1, d)[ign.cuda()] == 0).all()  # tokens without a target


def test_lm_head_bwd_workload_sampled_rows_and_zero_column_sums():
    """B2 L8192 n4 d4096 V32000: dh on sampled rows vs the oracle; every column sum of dW
    is ~0 because each row of G = softmax - onehot sums to zero."""
    need_gpu()
    w_ = syn.WORKLOADS["lm_head"]
    B, L, n, d, V = w_["B"], w_["L"], w_["n"], w_["d"], w_["V"]
    inp = syn.lm_head_inputs(B, L, n, d, V, seed=4)
    x, w, lab = inp["x"].cuda(), inp["w"].cuda(), inp["labels"].cuda()
    loss, lse = hd.lm_head_ce(x, w, lab, n)
    dh, dw = hd.lm_head_ce_bwd(x, w, lab, lse, n)
    torch.cuda.synchronize()
    assert hd.hd_device_status() == hd.HD_OK
    R = B * L
    rows = np.unique(np.concatenate([[0, 1, 255, 256, R // 2, R - 1],
                                     np.random.default_rng(23).choice(R, 26, replace=False)]))
    hrows = inp["x"][rows // L, (rows % L) * n + n - 1, :]
    g, dh_ref, _ = oracle.lm_head_ce_grad(hrows[None], inp["w"], inp["labels"].view(-1)[rows][None], 1)
    _rel_check(dh.view(R, d).cpu()[rows], dh_ref[0], "dh rows")
    colsum = host64(dw).sum(axis=0)
    # sum_v dW[v, :] = sum_r (sum_v G[r, v]) h_r: 0 exactly; the bf16 rounding of G leaves
    # ~2^-9 per row, a random walk of ~2^-9 sqrt(R) |h| (without the one-hot it would be ~sqrt(R))
    assert np.abs(colsum).max() < 0.05 * np.sqrt(R), np.abs(colsum).max()
    assert np.isfinite(host64(dw)).all()
