"""Pins for the float64 oracle: checked against things other than itself.

* hand-worked values (tests/golden/worked_examples.json, each cited there);
* masks enumerated from (token, stream) coordinates rather than positions;
* closed forms (visible-key counts, Q = 0 gives the mean of the visible V);
* textbook special cases computed by a library routine (torch SDPA in float64):
  n = 1, INTRA on de-interleaved streams, CROSS_FULL on the nL sequence;
* brute-force per-row sliding windows built by slicing;
* central finite differences for the backward;
* the sampled-row/column helpers against the full functions.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import CROSS_FULL, CROSS_WINDOW, INTRA

MODES = {"INTRA": INTRA, "CROSS_FULL": CROSS_FULL, "CROSS_WINDOW": CROSS_WINDOW}


def _val(s):
    if isinstance(s, (int, float)):
        return float(s)
    s = s.strip()
    if s.startswith("log(") and s.endswith(")"):
        return math.log(float(Fraction(s[4:-1])))
    return float(Fraction(s))


def _vals(xs):
    return np.array([_val(x) for x in xs])


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- masks

def test_golden_masks(golden):
    g = golden["masks_n2_L3_W1"]
    for name, mode in MODES.items():
        want = np.array([[c == "1" for c in row] for row in g[name]])
        got = oracle.mask_matrix(np.arange(6), 6, 2, mode, 1)
        assert (got == want).all(), name
        fin = oracle.mask_matrix(oracle.query_positions(6, 2, True), 6, 2, mode, 1)
        assert (fin == want[g["final_rows"]]).all(), name
    assert list(oracle.query_positions(6, 2, True)) == g["final_rows"]


@pytest.mark.parametrize("n,L,W", [(1, 7, 3), (2, 5, 2), (3, 6, 1), (4, 5, 3), (8, 3, 2)])
def test_masks_from_token_stream_coordinates(n, L, W):
    """Enumerate visibility from (token, stream) pairs, as step 1 describes them."""
    S = n * L
    want = {m: np.zeros((S, S), bool) for m in MODES.values()}
    for t in range(L):
        for s in range(n):
            p = t * n + s
            for t2 in range(L):
                for s2 in range(n):
                    p2 = t2 * n + s2
                    if t2 <= t and s2 == s:
                        want[INTRA][p, p2] = True
                    if p2 <= p:
                        want[CROSS_FULL][p, p2] = True
                    if p2 <= p and p - p2 <= n * W - 1:
                        want[CROSS_WINDOW][p, p2] = True
    for m in MODES.values():
        assert (oracle.mask_matrix(np.arange(S), S, n, m, W) == want[m]).all()


@pytest.mark.parametrize("n,L,W", [(1, 9, 4), (3, 7, 2), (4, 16, 5)])
def test_visible_counts_closed_form(n, L, W):
    S = n * L
    p = np.arange(S)
    c = {m: oracle.mask_matrix(p, S, n, m, W).sum(1) for m in MODES.values()}
    assert (c[INTRA] == p // n + 1).all()
    assert (c[CROSS_FULL] == p + 1).all()
    assert (c[CROSS_WINDOW] == np.minimum(p + 1, n * W)).all()


# ------------------------------------------------------- worked examples

def _as4(x):  # [S] -> [1, S, 1, 1]
    return np.asarray(x, dtype=np.float64).reshape(1, -1, 1, 1)


def test_golden_uniform(golden):
    g = golden["uniform_n2_L2"]
    q = np.zeros((1, 4, 1, 1))
    k, v = _as4(g["K"]), _as4(g["V"])
    for name, mode in MODES.items():
        o, lse = oracle.attn_fwd(q, k, v, 2, mode, 1, False, 1.0)
        np.testing.assert_allclose(o[0, :, 0, 0], _vals(g[name]["O"]), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, 0], _vals(g[name]["LSE"]), rtol=0, atol=1e-12)
    f = g["CROSS_FULL_final_only"]
    o, lse = oracle.attn_fwd(q[:, :2], k, v, 2, CROSS_FULL, 1, True, 1.0)
    np.testing.assert_allclose(o[0, :, 0, 0], _vals(f["O"]), atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], _vals(f["LSE"]), atol=1e-12)
    # backward: dO = 1
    do = np.ones((1, 4, 1, 1))
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 2, CROSS_FULL, 1, False, 1.0)
    np.testing.assert_allclose(dv[0, :, 0, 0], _vals(g["CROSS_FULL"]["dV"]), atol=1e-12)
    np.testing.assert_allclose(dq[0, :, 0, 0], _vals(g["CROSS_FULL"]["dQ"]), atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)


def test_golden_weighted(golden):
    g = golden["weighted_n2_L2"]
    q = np.ones((1, 4, 1, 1))
    k, v = _as4(_vals(g["K"])), _as4(g["V"])
    for name, mode in MODES.items():
        o, lse = oracle.attn_fwd(q, k, v, 2, mode, 1, False, 1.0)
        np.testing.assert_allclose(o[0, :, 0, 0], _vals(g[name]["O"]), atol=1e-12)
        np.testing.assert_allclose(lse[0, 0], _vals(g[name]["LSE"]), atol=1e-12)


def test_golden_decode(golden):
    g = golden["decode_n2_T1"]
    w = golden["weighted_n2_L2"]
    k, v = _as4(_vals(w["K"])), _as4(w["V"])
    q = np.ones((1, 2, 1, 1))
    for name in ("INTRA", "CROSS_FULL"):
        o, lse = oracle.decode_attn(q, k, v, np.array([2]), 2, MODES[name], 1, 1.0)
        np.testing.assert_allclose(o[0, :, 0, 0], _vals(g[name]["O"]), atol=1e-12)
        np.testing.assert_allclose(lse[0, 0], _vals(g[name]["LSE"]), atol=1e-12)


def test_golden_expand(golden):
    g = golden["expand_n2_V3_d1"]
    x = oracle.expand_embed(np.array(g["ids"]), np.array(g["tables"], dtype=np.float32))
    assert (x == np.array(g["X"], dtype=np.float32)).all()


# ------------------------------------------------ closed forms / invariants

@pytest.mark.parametrize("name", list(MODES))
def test_zero_query_is_mean_of_visible_values(name):
    """With Q = 0 every visible key has equal weight; V = one-hot rows exposes P."""
    n, L, W = 3, 5, 2
    S = n * L
    mode = MODES[name]
    q = np.zeros((1, S, 1, S))
    k = _rand((1, S, 1, S), 1)
    v = np.eye(S).reshape(1, S, 1, S)
    o, lse = oracle.attn_fwd(q, k, v, n, mode, W, False, 0.37)
    m = oracle.mask_matrix(np.arange(S), S, n, mode, W)
    cnt = m.sum(1)
    np.testing.assert_allclose(o[0, :, 0, :], m / cnt[:, None], atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.log(cnt), atol=1e-14)


def _sdpa_causal(q, k, v, scale, window=None):
    """Textbook causal (or sliding-window) attention via torch SDPA, float64.

    q [Sq, H, D], k/v [S, H, D] with the same H; returns [Sq, H, D].
    """
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(k).permute(1, 0, 2)
    vt = torch.from_numpy(v).permute(1, 0, 2)
    if window is None:
        o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    else:
        raise AssertionError
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("name", list(MODES))
def test_n1_reduces_to_textbook_causal(name):
    L, H, D = 23, 2, 8
    q, k, v = _rand((1, L, H, D), 2), _rand((1, L, H, D), 3), _rand((1, L, H, D), 4)
    mode = MODES[name]
    W = L  # window covering everything: sliding window = causal
    o, _ = oracle.attn_fwd(q, k, v, 1, mode, W, False, 0.3)
    ref = _sdpa_causal(q[0], k[0], v[0], 0.3)
    np.testing.assert_allclose(o[0], ref, atol=1e-12)


def test_n1_window_is_textbook_sliding_window():
    """Row loop over explicit slices k[p-W+1 : p+1] (no mask matrix involved)."""
    L, D, W = 19, 5, 4
    q, k, v = _rand((1, L, 1, D), 5), _rand((1, L, 1, D), 6), _rand((1, L, 1, D), 7)
    o, lse = oracle.attn_fwd(q, k, v, 1, CROSS_WINDOW, W, False, 0.5)
    for p in range(L):
        lo = max(0, p - W + 1)
        s = 0.5 * k[0, lo:p + 1, 0] @ q[0, p, 0]
        w = np.exp(s - s.max())
        np.testing.assert_allclose(o[0, p, 0], (w / w.sum()) @ v[0, lo:p + 1, 0], atol=1e-12)
        np.testing.assert_allclose(lse[0, 0, p], s.max() + np.log(w.sum()), atol=1e-12)


@pytest.mark.parametrize("n", [2, 3, 4])
def test_intra_is_causal_per_deinterleaved_stream(n):
    L, H, D = 11, 2, 8
    S = n * L
    q, k, v = _rand((1, S, H, D), 8), _rand((1, S, H, D), 9), _rand((1, S, H, D), 10)
    o, _ = oracle.attn_fwd(q, k, v, n, INTRA, 1, False, 0.25)
    for s in range(n):
        ref = _sdpa_causal(q[0, s::n], k[0, s::n], v[0, s::n], 0.25)
        np.testing.assert_allclose(o[0, s::n], ref, atol=1e-12)


@pytest.mark.parametrize("n", [2, 4])
def test_cross_full_is_causal_on_expanded_sequence(n):
    L, H, D = 9, 3, 8
    S = n * L
    q, k, v = _rand((2, S, H, D), 11), _rand((2, S, H, D), 12), _rand((2, S, H, D), 13)
    o, _ = oracle.attn_fwd(q, k, v, n, CROSS_FULL, 1, False, 0.2)
    for b in range(2):
        np.testing.assert_allclose(o[b], _sdpa_causal(q[b], k[b], v[b], 0.2), atol=1e-12)


def test_cross_window_sliced_rows_on_expanded_sequence():
    """CROSS_WINDOW with n > 1: each row is softmax over k[p-nW+1 : p+1] by slicing."""
    n, L, W, D = 3, 10, 2, 6
    S = n * L
    q, k, v = _rand((1, S, 1, D), 14), _rand((1, S, 1, D), 15), _rand((1, S, 1, D), 16)
    o, _ = oracle.attn_fwd(q, k, v, n, CROSS_WINDOW, W, False, 0.4)
    for p in range(S):
        lo = max(0, p - n * W + 1)
        s = 0.4 * k[0, lo:p + 1, 0] @ q[0, p, 0]
        w = np.exp(s - s.max())
        np.testing.assert_allclose(o[0, p, 0], (w / w.sum()) @ v[0, lo:p + 1, 0], atol=1e-12)


@pytest.mark.parametrize("n,L,W", [(4, 6, 6), (4, 6, 9), (2, 5, 100)])
def test_window_at_least_L_equals_cross_full(n, L, W):
    S = n * L
    q, k, v = _rand((1, S, 2, 4), 17), _rand((1, S, 2, 4), 18), _rand((1, S, 2, 4), 19)
    a = oracle.attn_fwd(q, k, v, n, CROSS_WINDOW, W, False, 0.5)
    b = oracle.attn_fwd(q, k, v, n, CROSS_FULL, 1, False, 0.5)
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], atol=1e-13)


@pytest.mark.parametrize("name", list(MODES))
def test_final_only_equals_final_stream_rows(name):
    n, L, H, D, W = 4, 7, 2, 8, 2
    S = n * L
    mode = MODES[name]
    q, k, v = _rand((1, S, H, D), 20), _rand((1, S, H, D), 21), _rand((1, S, H, D), 22)
    full_o, full_l = oracle.attn_fwd(q, k, v, n, mode, W, False, 0.3)
    fo, fl = oracle.attn_fwd(q[:, n - 1::n], k, v, n, mode, W, True, 0.3)
    np.testing.assert_allclose(fo, full_o[:, n - 1::n], atol=1e-13)
    np.testing.assert_allclose(fl, full_l[:, :, n - 1::n], atol=1e-13)


@pytest.mark.parametrize("name", list(MODES))
def test_gqa_equals_mha_with_repeated_kv(name):
    n, L, Hq, Hkv, D, W = 2, 6, 6, 2, 4, 2
    S = n * L
    mode = MODES[name]
    q, k, v = _rand((1, S, Hq, D), 23), _rand((1, S, Hkv, D), 24), _rand((1, S, Hkv, D), 25)
    g = Hq // Hkv
    kr, vr = np.repeat(k, g, axis=2), np.repeat(v, g, axis=2)
    a = oracle.attn_fwd(q, k, v, n, mode, W, False, 0.5)
    b = oracle.attn_fwd(q, kr, vr, n, mode, W, False, 0.5)
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)
    do = _rand(q.shape, 26)
    ga = oracle.attn_bwd(q, k, v, do, n, mode, W, False, 0.5)
    gb = oracle.attn_bwd(q, kr, vr, do, n, mode, W, False, 0.5)
    np.testing.assert_allclose(ga[0], gb[0], atol=1e-12)
    np.testing.assert_allclose(ga[1], gb[1].reshape(1, S, Hkv, g, D).sum(3), atol=1e-12)
    np.testing.assert_allclose(ga[2], gb[2].reshape(1, S, Hkv, g, D).sum(3), atol=1e-12)


def test_brute_force_row_loop():
    """Per-(row, key) scalar loop with math.exp on a tiny input."""
    n, L, H, D, W = 3, 4, 1, 3, 2
    S = n * L
    q, k, v = _rand((1, S, H, D), 27), _rand((1, S, H, D), 28), _rand((1, S, H, D), 29)
    for mode in MODES.values():
        o, lse = oracle.attn_fwd(q, k, v, n, mode, W, False, 0.7)
        for p in range(S):
            ws, acc = [], np.zeros(D)
            for pk in range(S):
                ok = pk <= p and (
                    (mode == INTRA and pk % n == p % n)
                    or mode == CROSS_FULL
                    or (mode == CROSS_WINDOW and p - pk < n * W)
                )
                if ok:
                    ws.append((0.7 * float(np.dot(q[0, p, 0], k[0, pk, 0])), pk))
            m = max(w for w, _ in ws)
            tot = sum(math.exp(w - m) for w, _ in ws)
            for w, pk in ws:
                acc += math.exp(w - m) / tot * v[0, pk, 0]
            np.testing.assert_allclose(o[0, p, 0], acc, atol=1e-12)
            assert abs(lse[0, 0, p] - (m + math.log(tot))) < 1e-12


# ---------------------------------------------------------------- backward

def _loss(q, k, v, do, n, mode, W, fin, scale):
    return float((oracle.attn_fwd(q, k, v, n, mode, W, fin, scale)[0] * do).sum())


@pytest.mark.parametrize("name,fin", [("INTRA", False), ("CROSS_FULL", False),
                                      ("CROSS_WINDOW", False), ("CROSS_FULL", True),
                                      ("INTRA", True), ("CROSS_WINDOW", True)])
def test_backward_central_differences(name, fin):
    n, L, Hq, Hkv, D, W = 2, 4, 2, 1, 3, 2
    S = n * L
    Sq = L if fin else S
    mode = MODES[name]
    q, k, v = _rand((1, Sq, Hq, D), 30), _rand((1, S, Hkv, D), 31), _rand((1, S, Hkv, D), 32)
    do = _rand((1, Sq, Hq, D), 33)
    sc = 0.6
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, n, mode, W, fin, sc)
    eps = 1e-6
    for name_t, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + eps
            fp = _loss(q, k, v, do, n, mode, W, fin, sc)
            x[idx] = old - eps
            fm = _loss(q, k, v, do, n, mode, W, fin, sc)
            x[idx] = old
            num[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7, rtol=1e-6, err_msg=name_t)


@pytest.mark.parametrize("n", [1, 3])
def test_backward_matches_library_autograd_textbook(n):
    """CROSS_FULL backward == autograd through torch SDPA (causal) in float64."""
    L, H, D = 7, 2, 4
    S = n * L
    q, k, v, do = (_rand((1, S, H, D), s) for s in (34, 35, 36, 37))
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, n, CROSS_FULL, 1, False, 0.45)
    qt, kt, vt = (torch.from_numpy(x[0]).permute(1, 0, 2).requires_grad_() for x in (q, k, v))
    o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.45)
    o.backward(torch.from_numpy(do[0]).permute(1, 0, 2))
    np.testing.assert_allclose(dq[0], qt.grad.permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dk[0], kt.grad.permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dv[0], vt.grad.permute(1, 0, 2).numpy(), atol=1e-12)


# -------------------------------------------------- sampled helpers

@pytest.mark.parametrize("name,fin", [("INTRA", False), ("CROSS_FULL", False),
                                      ("CROSS_WINDOW", False), ("CROSS_FULL", True),
                                      ("CROSS_WINDOW", True), ("INTRA", True)])
def test_sampled_helpers_match_full(name, fin):
    n, L, Hq, Hkv, D, W = 4, 9, 4, 2, 8, 3
    S = n * L
    Sq = L if fin else S
    mode = MODES[name]
    q, k, v = _rand((2, Sq, Hq, D), 38), _rand((2, S, Hkv, D), 39), _rand((2, S, Hkv, D), 40)
    do = _rand((2, Sq, Hq, D), 41)
    o, lse = oracle.attn_fwd(q, k, v, n, mode, W, fin, 0.3)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, n, mode, W, fin, 0.3)
    rows = [0, 1, Sq // 2, Sq - 1]
    for b in range(2):
        for h in range(Hq):
            ro, rl = oracle.attn_fwd_rows(q, k, v, n, mode, W, fin, 0.3, b, h, rows)
            np.testing.assert_allclose(ro, o[b, rows, h], atol=1e-12)
            np.testing.assert_allclose(rl, lse[b, h, rows], atol=1e-12)
            rq = oracle.attn_bwd_dq_rows(q, k, v, do, n, mode, W, fin, 0.3, b, h, rows)
            np.testing.assert_allclose(rq, dq[b, rows, h], atol=1e-12)
        cols = [0, 5, 6, 7, S - 2, S - 1]
        for kh in range(Hkv):
            ck, cv = oracle.attn_bwd_kv_cols(q, k, v, do, n, mode, W, fin, 0.3, b, kh, cols)
            np.testing.assert_allclose(ck, dk[b, cols, kh], atol=1e-12)
            np.testing.assert_allclose(cv, dv[b, cols, kh], atol=1e-12)


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("name", list(MODES))
def test_decode_equals_prefill_rows(name):
    n, T, Tcap, Hq, Hkv, D, W = 3, 6, 9, 4, 2, 8, 2
    mode = MODES[name]
    B = 3
    kc, vc = _rand((B, Tcap * n, Hkv, D), 42), _rand((B, Tcap * n, Hkv, D), 43)
    q = _rand((B, n, Hq, D), 44)
    seqlen = np.array([T + 1, 1, 4])
    o, lse = oracle.decode_attn(q, kc, vc, seqlen, n, mode, W, 0.35)
    for b in range(B):
        Tb = seqlen[b] - 1
        S = (Tb + 1) * n
        qf = np.zeros((1, S, Hq, D))
        qf[0, Tb * n:] = q[b]
        fo, fl = oracle.attn_fwd(qf, kc[b:b + 1, :S], vc[b:b + 1, :S], n, mode, W, False, 0.35)
        np.testing.assert_allclose(o[b], fo[0, Tb * n:], atol=1e-12)
        np.testing.assert_allclose(lse[b], fl[0, :, Tb * n:], atol=1e-12)


@pytest.mark.parametrize("name", list(MODES))
def test_final_only_decode_equals_final_only_prefill_last_row(name):
    """One query per sequence at T*n + n-1 = the last row of a final-stream-only prefill."""
    n, Tcap, Hq, Hkv, D, W = 4, 7, 6, 3, 8, 2
    mode = MODES[name]
    B = 3
    kc, vc = _rand((B, Tcap * n, Hkv, D), 46), _rand((B, Tcap * n, Hkv, D), 47)
    q = _rand((B, 1, Hq, D), 48)
    seqlen = np.array([Tcap, 1, 3])
    o, lse = oracle.decode_attn(q, kc, vc, seqlen, n, mode, W, 0.4, final_only=True)
    assert o.shape == (B, 1, Hq, D) and lse.shape == (B, Hq, 1)
    for b in range(B):
        T1 = int(seqlen[b])
        qf = np.zeros((1, T1, Hq, D))
        qf[0, T1 - 1] = q[b, 0]
        fo, fl = oracle.attn_fwd(qf, kc[b:b + 1, :T1 * n], vc[b:b + 1, :T1 * n], n, mode, W, True, 0.4)
        np.testing.assert_allclose(o[b, 0], fo[0, T1 - 1], atol=1e-12)
        np.testing.assert_allclose(lse[b, :, 0], fl[0, :, T1 - 1], atol=1e-12)


def test_final_only_intra_decode_reads_only_the_final_stream():
    """INTRA, final stream: the other streams' cache rows do not change the result."""
    n, Tcap, Hq, Hkv, D = 3, 5, 2, 1, 8
    kc, vc = _rand((1, Tcap * n, Hkv, D), 49), _rand((1, Tcap * n, Hkv, D), 50)
    q = _rand((1, 1, Hq, D), 51)
    o1, l1 = oracle.decode_attn(q, kc, vc, [Tcap], n, MODES["INTRA"], 1, 0.5, final_only=True)
    kc2, vc2 = kc.copy(), vc.copy()
    other = np.arange(Tcap * n) % n != n - 1
    kc2[:, other] = 7.0
    vc2[:, other] = -3.0
    o2, l2 = oracle.decode_attn(q, kc2, vc2, [Tcap], n, MODES["INTRA"], 1, 0.5, final_only=True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # and equals plain softmax attention over the final stream's rows
    kk, vv = kc[0, n - 1::n, 0], vc[0, n - 1::n, 0]
    for h in range(Hq):
        sc = 0.5 * kk @ q[0, 0, h]
        w = np.exp(sc - sc.max())
        np.testing.assert_allclose(o1[0, 0, h], (w / w.sum()) @ vv, atol=1e-12)


# ---------------------------------------------------------------- expansion

@pytest.mark.parametrize("B,L,n,V,d", [(1, 5, 3, 7, 4), (2, 3, 1, 5, 6), (3, 4, 4, 9, 1)])
def test_expand_triple_loop(B, L, n, V, d):
    rng = np.random.default_rng(45)
    ids = rng.integers(0, V, (B, L))
    tab = rng.standard_normal((n, V, d)).astype(np.float32)
    x = oracle.expand_embed(ids, tab)
    for b in range(B):
        for i in range(L):
            for kk in range(n):
                assert (x[b, i * n + kk] == tab[kk, ids[b, i]]).all()


def test_expand_n1_is_plain_lookup():
    rng = np.random.default_rng(46)
    ids = rng.integers(0, 11, (2, 9))
    tab = rng.standard_normal((1, 11, 5)).astype(np.float32)
    assert (oracle.expand_embed(ids, tab) == np.take(tab[0], ids, axis=0)).all()


def test_expand_rejects_out_of_range_ids():
    with pytest.raises(IndexError):
        oracle.expand_embed(np.array([[3]]), np.zeros((2, 3, 1), np.float32))
