"""RoPE parity: hd_rope_expanded (CUDA, through the C ABI) vs the float64 oracle.

Tolerance: the kernel reads bf16, computes x1 cos - x2 sin in fp32 with sin/cos
good to 4e-7 absolute, and rounds once to bf16 (relative error <= 2^-9). So
|gpu - oracle| <= 2^-8 |oracle| + 1e-5 elementwise for N(0,1) inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import synthetic as syn
from tests.gpu_util import host64, need_gpu

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2.0 ** -8, 1e-5


def _close(got, want, what):
    got = host64(got) if torch.is_tensor(got) else got
    err = np.abs(got - want)
    bound = RTOL * np.abs(want) + ATOL
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of bound, worst {float((err - bound).max()):.3e}"


def _inputs(B, L, n, Hq, Hkv, D, final_only, seed):
    Sq = L if final_only else n * L
    q = syn.normal_bf16((B, Sq, Hq, D), seed) if Hq else None
    k = syn.normal_bf16((B, n * L, Hkv, D), seed + 1) if Hkv else None
    return q, k


@pytest.mark.parametrize("B,L,n,Hq,Hkv,D,fin,base", [
    (1, 64, 4, 4, 4, 64, 0, 10000.0),      # the tiny workload's shapes
    (2, 37, 3, 6, 2, 128, 0, 10000.0),     # ragged, heads not a multiple of the unroll
    (2, 37, 3, 6, 2, 128, 1, 10000.0),     # final-stream-only queries
    (1, 50, 1, 5, 5, 32, 0, 500000.0),     # n = 1: plain RoPE, another base
    (3, 9, 8, 3, 1, 16, 1, 10000.0),       # smallest head size
    (1, 21, 2, 2, 2, 256, 0, 10000.0),     # largest head size
])
def test_rope_matches_oracle(B, L, n, Hq, Hkv, D, fin, base):
    need_gpu()
    q, k = _inputs(B, L, n, Hq, Hkv, D, bool(fin), seed=B * 100 + L)
    want_q, want_k = oracle.rope_expanded(q, k, n, bool(fin), base)
    gq, gk = q.cuda(), k.cuda()
    hd.rope_(gq, gk, n, final_only=bool(fin), base=base)
    torch.cuda.synchronize()
    _close(gq, want_q, "q")
    _close(gk, want_k, "k")
    assert hd.hd_device_status() == hd.HD_OK


def test_rope_q_only_and_k_only():
    need_gpu()
    q, k = _inputs(2, 19, 4, 8, 2, 64, False, seed=5)
    want_q, want_k = oracle.rope_expanded(q, k, 4, False, 10000.0)
    gq = q.cuda()
    hd.rope_(gq, None, 4)
    gk = k.cuda()
    hd.rope_(None, gk, 4)
    torch.cuda.synchronize()
    _close(gq, want_q, "q only")
    _close(gk, want_k, "k only")


def test_rope_token_offset_decode_step():
    """L = 1 with per-sequence cached-token counts, as one decode step uses it."""
    need_gpu()
    B, n, Hq, Hkv, D = 5, 4, 8, 2, 128
    offs = np.array([0, 1, 16383, 100000, 7], dtype=np.int32)
    q, k = _inputs(B, 1, n, Hq, Hkv, D, False, seed=11)
    want_q, want_k = oracle.rope_expanded(q, k, n, False, 10000.0, token_offset=offs)
    gq, gk = q.cuda(), k.cuda()
    hd.rope_(gq, gk, n, token_offset=torch.from_numpy(offs).cuda())
    torch.cuda.synchronize()
    _close(gq, want_q, "q")
    _close(gk, want_k, "k")
    assert hd.hd_device_status() == hd.HD_OK


def test_rope_negative_offset_leaves_rows_and_records_status():
    need_gpu()
    q, k = _inputs(3, 2, 2, 2, 2, 64, False, seed=12)
    offs = torch.tensor([3, -1, 0], dtype=torch.int32)
    want_q, want_k = oracle.rope_expanded(q, k, 2, False, 10000.0, token_offset=[3, 0, 0])
    gq, gk = q.cuda(), k.cuda()
    hd.hd_device_status(clear=True)
    hd.rope_(gq, gk, 2, token_offset=offs.cuda())
    assert hd.hd_device_status(clear=True) == hd.HD_ERR_DEVICE_INDEX
    assert torch.equal(gq[1].cpu(), q[1]) and torch.equal(gk[1].cpu(), k[1])
    for b in (0, 2):
        _close(gq[b:b + 1], want_q[b:b + 1], f"q[{b}]")
        _close(gk[b:b + 1], want_k[b:b + 1], f"k[{b}]")


@pytest.mark.parametrize("fin", [0, 1])
def test_rope_long_sequence_sampled_rows(fin):
    """B1 S131072 Hq32 Hkv8 D128 (positions up to 131071): sampled rows vs the oracle."""
    need_gpu()
    B, L, n, Hq, Hkv, D = 1, 32768, 4, 32, 8, 128
    Sq = L if fin else n * L
    g = torch.Generator(device="cuda")
    g.manual_seed(21 + fin)
    gq = torch.empty((B, Sq, Hq, D), dtype=torch.bfloat16, device="cuda").normal_(generator=g)
    gk = torch.empty((B, n * L, Hkv, D), dtype=torch.bfloat16, device="cuda").normal_(generator=g)
    q0, k0 = gq.clone(), gk.clone()
    hd.rope_(gq, gk, n, final_only=bool(fin))
    torch.cuda.synchronize()
    rng = np.random.default_rng(31)
    rows_q = np.unique(np.concatenate([[0, 1, Sq - 1], rng.choice(Sq, 200, replace=False)]))
    rows_k = np.unique(np.concatenate([[0, n - 1, n * L - 1], rng.choice(n * L, 200, replace=False)]))
    pos_q = (rows_q * n + n - 1) if fin else rows_q
    _close(gq[:, rows_q], oracle.rope(q0[:, rows_q].cpu(), pos_q, 10000.0), "q rows")
    _close(gk[:, rows_k], oracle.rope(k0[:, rows_k].cpu(), rows_k, 10000.0), "k rows")
    assert torch.equal(gk[:, 0], k0[:, 0])  # position 0 is the identity rotation


def test_rope_then_attention_scores_shift_invariant():
    """Rotated q.k depends on p - p' only: shifting all positions by a token offset keeps
    the attention output (a property that holds at any size)."""
    need_gpu()
    B, L, n, Hq, Hkv, D = 1, 64, 4, 4, 2, 64
    q, k = _inputs(B, L, n, Hq, Hkv, D, False, seed=41)
    v = syn.normal_bf16((B, n * L, Hkv, D), 42).cuda()
    outs = []
    for off in (0, 5000):
        gq, gk = q.cuda(), k.cuda()
        hd.rope_(gq, gk, n, token_offset=torch.full((B,), off, dtype=torch.int32, device="cuda"))
        o, _ = hd.attn_fwd(gq, gk, v, n, hd.CROSS_FULL)
        outs.append(host64(o))
    assert np.abs(outs[0] - outs[1]).max() < 3e-2
