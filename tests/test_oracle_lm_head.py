"""Pins for the final-stream readout and LM-head cross-entropy oracle."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


@pytest.mark.parametrize("n", [1, 2, 4])
def test_readout_is_the_last_stream_of_each_token(n):
    """Enumerated from (token, stream) coordinates: token t, stream n-1."""
    B, L, d = 2, 5, 3
    x = np.zeros((B, n * L, d))
    for b in range(B):
        for t in range(L):
            for s in range(n):
                x[b, t * n + s] = 100 * b + 10 * t + s  # encodes (b, t, s)
    h = oracle.final_readout(x, n)
    assert h.shape == (B, L, d)
    for b in range(B):
        for t in range(L):
            assert (h[b, t] == 100 * b + 10 * t + (n - 1)).all()


def test_ce_matches_torch_cross_entropy():
    """Library routine in float64, including ignored (negative) labels."""
    B, L, n, d, V = 2, 7, 3, 16, 50
    x, w = _rand((B, n * L, d), 1), _rand((V, d), 2, 0.3)
    labels = np.random.default_rng(3).integers(0, V, (B, L))
    labels[0, 2] = labels[1, 6] = -100
    loss, lse = oracle.lm_head_ce(x, w, labels, n)
    h = torch.from_numpy(x[:, n - 1::n].reshape(-1, d))
    logits = h @ torch.from_numpy(w).T
    ref = F.cross_entropy(logits, torch.from_numpy(labels.reshape(-1)), ignore_index=-100,
                          reduction="none").numpy()
    np.testing.assert_allclose(loss.reshape(-1), ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), torch.logsumexp(logits, -1).numpy(), rtol=1e-12)
    assert loss[0, 2] == 0.0 and loss[1, 6] == 0.0


def test_zero_head_gives_log_vocab():
    x, V = _rand((1, 12, 8), 4), 37
    loss, lse = oracle.lm_head_ce(x, np.zeros((V, 8)), (np.arange(4) % V)[None], 3)
    np.testing.assert_allclose(loss, math.log(V), rtol=1e-14)
    np.testing.assert_allclose(lse, math.log(V), rtol=1e-14)


def test_large_logits_stay_finite():
    """Logits of order 1e3: the loss of a dominant correct label is ~0, a wrong one ~ the gap."""
    d, V = 4, 6
    w = np.zeros((V, d))
    w[2, 0] = 1.0
    w[5, 0] = 0.5
    x = np.zeros((1, 2, d))
    x[0, 1, 0] = 2000.0  # n = 2: token 0's final stream
    loss, lse = oracle.lm_head_ce(x, w, np.array([[2]]), 2)
    assert np.isfinite(lse).all()
    np.testing.assert_allclose(lse[0, 0], 2000.0, atol=1e-12)
    assert loss[0, 0] < 1e-12
    loss5, _ = oracle.lm_head_ce(x, w, np.array([[5]]), 2)
    np.testing.assert_allclose(loss5[0, 0], 1000.0, atol=1e-9)


def test_unsupervised_streams_do_not_matter():
    """Streams 0..n-2 get no direct supervision: changing them leaves the loss unchanged."""
    B, L, n, d, V = 2, 4, 4, 8, 20
    x, w = _rand((B, n * L, d), 5), _rand((V, d), 6)
    labels = np.random.default_rng(7).integers(0, V, (B, L))
    loss1, _ = oracle.lm_head_ce(x, w, labels, n)
    x2 = x.copy()
    x2[:, np.arange(n * L) % n != n - 1] = 123.0
    loss2, _ = oracle.lm_head_ce(x2, w, labels, n)
    np.testing.assert_array_equal(loss1, loss2)


def test_rows_helper_matches_full():
    B, L, n, d, V = 2, 9, 2, 8, 30
    x, w = _rand((B, n * L, d), 8), _rand((V, d), 9)
    labels = np.random.default_rng(10).integers(-1, V, (B, L))
    loss, lse = oracle.lm_head_ce(x, w, labels, n)
    rows = np.array([0, 4, 9, 17])
    rl, rs = oracle.lm_head_ce_rows(x, w, labels, n, rows)
    np.testing.assert_allclose(rl, loss.reshape(-1)[rows], atol=1e-13)
    np.testing.assert_allclose(rs, lse.reshape(-1)[rows], atol=1e-13)


def test_grad_matches_central_differences():
    """dh and dW of the summed loss against float64 central differences."""
    B, L, n, d, V = 1, 3, 2, 5, 7
    x, w = _rand((B, n * L, d), 11), _rand((V, d), 12)
    labels = np.array([[2, -1, 6]])
    _, dh, dw = oracle.lm_head_ce_grad(x, w, labels, n)
    eps = 1e-6

    def total(xx, ww):
        return oracle.lm_head_ce(xx, ww, labels, n)[0].sum()
    for (t, k) in [(0, 0), (0, 4), (1, 2), (2, 3)]:
        xp, xm = x.copy(), x.copy()
        xp[0, t * n + n - 1, k] += eps
        xm[0, t * n + n - 1, k] -= eps
        num = (total(xp, w) - total(xm, w)) / (2 * eps)
        assert abs(num - dh[0, t, k]) < 1e-7, (t, k, num, dh[0, t, k])
    for (v, k) in [(0, 0), (2, 1), (6, 4), (3, 2)]:
        wp, wm = w.copy(), w.copy()
        wp[v, k] += eps
        wm[v, k] -= eps
        num = (total(x, wp) - total(x, wm)) / (2 * eps)
        assert abs(num - dw[v, k]) < 1e-7, (v, k, num, dw[v, k])
    # the unsupervised streams' rows get no gradient: a change there changes nothing
    xs = x.copy()
    xs[0, 0, :] += 1.0
    assert total(xs, w) == total(x, w)


def test_grad_rows_sum_to_zero_and_zero_head_closed_form():
    B, L, n, d, V = 2, 4, 3, 6, 9
    x = _rand((B, n * L, d), 13)
    labels = np.array([[0, 8, -100, 4], [1, 1, 2, 3]])
    g, _, _ = oracle.lm_head_ce_grad(x, _rand((V, d), 14), labels, n)
    sup = labels >= 0
    np.testing.assert_allclose(g[sup].sum(axis=-1), 0.0, atol=1e-14)
    assert (g[~sup] == 0).all()
    g0, dh0, dw0 = oracle.lm_head_ce_grad(x, np.zeros((V, d)), labels, n)
    want = np.full((B, L, V), 1.0 / V)
    want[~sup] = 0
    for b in range(B):
        for t in range(L):
            if labels[b, t] >= 0:
                want[b, t, labels[b, t]] -= 1.0
    np.testing.assert_allclose(g0, want, atol=1e-15)
    assert (dh0 == 0).all()
