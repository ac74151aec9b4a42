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


def _key_runs(S, n, mode, W, final_only, seed, extra=()):
    """Seeded runs of 64 key positions (memory rows of K) for the dK / dV checks.

    Always the first and the last 64 keys, a run straddling a grid bucket of
    eight 128-key tiles (INTRA buckets tokens of one stream, whose rows sit n
    apart), a run straddling a 128-key tile boundary inside a bucket, one at a
    random place, plus any ``extra`` starts (window edges).
    """
    rng = np.random.default_rng(seed)
    step = n if mode == hd.INTRA and not final_only else 1   # memory rows per problem key
    nkey = S // step                                          # keys per problem
    starts = [0, S - 64]
    if nkey > 1024:
        kb = int(rng.integers(1, nkey // 1024)) * 1024          # bucket boundary (problem keys)
        starts.append(kb * step - 32)
    if nkey > 256:
        kt = int(rng.integers(1, nkey // 128))
        kt += (kt % 8 == 0)                                    # a tile boundary inside a bucket
        starts.append(min(kt * 128, nkey - 1) * step - 32)
    starts.append(int(rng.integers(64, S - 128)))
    starts += list(extra)
    starts = [min(max(0, s0), S - 64) for s0 in starts]
    return np.unique(np.concatenate([np.arange(s0, s0 + 64) for s0 in starts]))


def _sampled(name, mode, seed, qpairs, kvpairs, rows_per_head=256, final_only=False, key_starts=None,
             extra_starts=()):
    """Full-size backward against the oracle on samples: dQ on ``rows_per_head``
    seeded rows of every (b, h) in ``qpairs``; dK / dV on key runs of every
    (b, h_kv) in ``kvpairs``, element by element; and, for every (b, h_kv), the
    closed form sum_keys dV = sum over the group's query heads and rows of dO
    (each row's P sums to one)."""
    need_gpu()
    w = syn.WORKLOADS[name] if isinstance(name, str) else name
    B, L, n, Hq, Hkv, D = w["B"], w["L"], w["n"], w["Hq"], w["Hkv"], w["D"]
    W = w.get("W", 0)
    inp = syn.attention_inputs(B, L, n, Hq, Hkv, D, final_only=final_only, seed=seed, with_grad=True)
    dq, dk, dv = run_bwd(inp, n, mode, W, int(final_only), w["scale"])
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    torch.cuda.empty_cache()
    S = n * L
    Sq = L if final_only else S
    g = Hq // Hkv
    # closed form at full size: sum over keys of dV = sum over queries of dO
    dv_sum = dv.double().sum(dim=1)                                     # [B, Hkv, D]
    do_sum = inp["do"].double().sum(dim=1).view(B, Hkv, g, D).sum(dim=2)
    # bf16 rounding of every dV element and of P (2^-9 relative each), summed
    # as independent errors, with a 6-sigma margin
    tol = 6 * 2.0 ** -8 * (dv.double().pow(2).sum(dim=1).sqrt() +
                           inp["do"].double().pow(2).sum(dim=1).view(B, Hkv, g, D).sum(dim=2).sqrt())
    assert ((dv_sum - do_sum).abs() <= tol + 1e-3).all(), float((dv_sum - do_sum).abs().max())
    t64 = {k: inp[k].to(torch.float64).numpy() for k in ("q", "k", "v", "do")}
    errs = []
    for (b, h) in qpairs:
        rows = sample_rows(Sq, n, W, final_only, rows_per_head, seed * 1000 + b * 31 + h)
        ref = oracle.attn_bwd_dq_rows(t64["q"], t64["k"], t64["v"], t64["do"], n, mode, max(W, 1), final_only,
                                      w["scale"], b, h, rows)
        got = dq[b, rows, h].float().numpy()
        assert np.abs(got - ref).max() <= G_MAX, ("dQ", b, h, np.abs(got - ref).max())
        errs.append(np.abs(got - ref).ravel())
    for (b, kh) in kvpairs:
        cols = key_starts(b, kh) if key_starts else _key_runs(S, n, mode, W, final_only, seed * 7919 + b * 97 + kh,
                                                               extra_starts)
        rk, rv = oracle.attn_bwd_kv_cols(t64["q"], t64["k"], t64["v"], t64["do"], n, mode, max(W, 1),
                                         final_only, w["scale"], b, kh, cols)
        gk, gv = dk[b, cols, kh].float().numpy(), dv[b, cols, kh].float().numpy()
        assert np.abs(gk - rk).max() <= G_MAX, ("dK", b, kh, np.abs(gk - rk).max())
        assert np.abs(gv - rv).max() <= G_MAX, ("dV", b, kh, np.abs(gv - rv).max())
        errs += [np.abs(gk - rk).ravel(), np.abs(gv - rv).ravel()]
    allerr = np.concatenate(errs)
    assert allerr.mean() <= G_MEAN, allerr.mean()


def test_bwd_intra_train_workload_sampled():
    """B4 n4 L2048, 16/4 heads, D128, INTRA: dQ on 256 rows of every head; dK/dV
    on five 64-key runs (ends, a grid-bucket boundary, a tile boundary, random)
    of every (batch, KV head)."""
    w = syn.WORKLOADS["intra_train"]
    qpairs = [(b, h) for b in range(w["B"]) for h in range(w["Hq"])]
    kvpairs = [(b, kh) for b in range(w["B"]) for kh in range(w["Hkv"])]
    _sampled("intra_train", hd.INTRA, 6, qpairs, kvpairs)


def test_bwd_cross_window_workload_sampled():
    """B2 n4 L8192 W1024 (window 4096 positions), 32/8 heads, D128, CROSS_WINDOW:
    dQ on 256 rows of every head; dK/dV on 64-key runs (ends, bucket and tile
    boundaries, random, and both window edges n*W and S - n*W) of four seeded
    KV heads per batch."""
    w = syn.WORKLOADS["cross_window"]
    S, nW = w["n"] * w["L"], w["n"] * w["W"]
    qpairs = [(b, h) for b in range(w["B"]) for h in range(w["Hq"])]
    rng = np.random.default_rng(77)
    kvpairs = [(b, int(kh)) for b in range(w["B"]) for kh in sorted(rng.choice(w["Hkv"], 4, replace=False))]
    _sampled("cross_window", hd.CROSS_WINDOW, 7, qpairs, kvpairs, extra_starts=(nW - 32, S - nW - 32))


def test_bwd_long_cross_final_only_workload_sampled():
    """KV-mirror backward at full size: B1 n4 L32768, final-stream queries only
    (32768 rows at positions 4t+3) against 131072 keys, 32/8 heads, D128,
    CROSS_FULL. dQ on 256 rows of every head; dK/dV on 64-key runs in the last
    8192 positions (the end, a tile boundary, random) of two KV heads; the dV
    column sums of every KV head against the closed form."""
    w = syn.WORKLOADS["long_cross"]
    S = w["n"] * w["L"]
    qpairs = [(0, h) for h in range(w["Hq"])]

    def starts(b, kh):
        rng = np.random.default_rng(500 + kh)
        st = [S - 64, S - 4096 - 32, int(rng.integers(S - 8192, S - 128))]
        return np.unique(np.concatenate([np.arange(s0, s0 + 64) for s0 in st]))

    _sampled("long_cross", hd.CROSS_FULL, 8, qpairs, [(0, 0), (0, 5)], final_only=True, key_starts=starts)


def test_bwd_long_problem_one_bucket_sampled():
    """A causal problem of 516 key tiles (66000 positions, a tile count that is
    no power of two): the grid makes a problem of at least 512 key tiles one
    bucket, its key tiles adjacent, heaviest first. dQ on 256 rows per head;
    dK/dV on runs at the last tiles, across key 65536 and at the end."""
    w = dict(B=1, L=16500, n=4, Hq=2, Hkv=1, D=64, scale=0.125)
    S = w["n"] * w["L"]

    def starts(b, kh):
        st = [S - 64, 65536 - 32, 65536 + 200, S - 300]
        return np.unique(np.concatenate([np.arange(s0, s0 + 64) for s0 in st]))

    _sampled(w, hd.CROSS_FULL, 9, [(0, 0), (0, 1)], [(0, 0)], key_starts=starts)
