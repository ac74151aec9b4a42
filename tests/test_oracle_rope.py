"""Pins for the RoPE oracle (closed forms and invariants, not its own formula)."""
import math

import numpy as np
import pytest

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_position_zero_is_identity():
    x = _rand((2, 1, 3, 8), 1)
    np.testing.assert_array_equal(oracle.rope(x, [0], 10000.0), x)


def test_first_pair_turns_by_exactly_p_radians():
    """Frequency 0 is base^0 = 1: the pair (x_0, x_{D/2}) is rotated by p radians."""
    D = 6
    x = np.zeros((1, 4, 1, D))
    x[..., 0] = 1.0  # unit vector along the first element of pair 0
    out = oracle.rope(x, [0, 1, 2, 7], 500.0)
    for r, p in enumerate([0, 1, 2, 7]):
        assert abs(out[0, r, 0, 0] - math.cos(p)) < 1e-15
        assert abs(out[0, r, 0, D // 2] - math.sin(p)) < 1e-15


def test_last_frequency_matches_its_closed_form():
    D, base, p = 8, 100.0, 5
    x = np.zeros((1, 1, 1, D))
    x[..., D // 2 - 1] = 1.0  # pair i = D/2 - 1, frequency base^(-(D-2)/D)
    out = oracle.rope(x, [p], base)
    wv = base ** (-(D - 2) / D)
    assert abs(out[0, 0, 0, D // 2 - 1] - math.cos(p * wv)) < 1e-14
    assert abs(out[0, 0, 0, D - 1] - math.sin(p * wv)) < 1e-14


def test_rotation_preserves_pair_norms():
    x = _rand((2, 7, 3, 16), 2)
    out = oracle.rope(x, np.arange(7) * 13, 10000.0)
    n_in = x[..., :8] ** 2 + x[..., 8:] ** 2
    n_out = out[..., :8] ** 2 + out[..., 8:] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12)


def test_scores_depend_only_on_relative_position():
    """<rope(q, p), rope(k, p')> is unchanged when both positions shift together."""
    D = 32
    q, k = _rand((1, 1, 1, D), 3), _rand((1, 1, 1, D), 4)
    def score(p, pk):
        return float((oracle.rope(q, [p], 10000.0) * oracle.rope(k, [pk], 10000.0)).sum())
    for p, pk in [(10, 3), (100, 50), (7, 7)]:
        assert abs(score(p, pk) - score(p + 1000, pk + 1000)) < 1e-9


@pytest.mark.parametrize("n", [1, 3, 4])
def test_expanded_positions_are_physical(n):
    """Stream s of token t is encoded at p = t*n + s; final-only rows at t*n + n-1."""
    L, H, D = 5, 2, 8
    S = n * L
    q, k = _rand((1, S, H, D), 5), _rand((1, S, 1, D), 6)
    oq, ok = oracle.rope_expanded(q, k, n, False, 10000.0)
    for t in range(L):
        for s in range(n):
            p = t * n + s
            np.testing.assert_allclose(oq[0, p], oracle.rope(q[:, p:p + 1], [p], 10000.0)[0, 0], atol=0)
            np.testing.assert_allclose(ok[0, p], oracle.rope(k[:, p:p + 1], [p], 10000.0)[0, 0], atol=0)
    fq, _ = oracle.rope_expanded(q[:, n - 1::n], None, n, True, 10000.0)
    np.testing.assert_allclose(fq, oq[:, n - 1::n], atol=1e-15)
    if n > 1:  # a token index instead of the physical position would differ
        tok = oracle.rope(q[:, 1:2], [0], 10000.0)
        assert np.abs(tok - oq[:, 1:2]).max() > 1e-3


def test_token_offset_matches_the_tail_of_a_longer_sequence():
    """A decode step at offset T sees the positions of token T of a T+1-token prefill."""
    n, T, H, D = 3, 6, 2, 16
    k = _rand((2, (T + 1) * n, H, D), 7)
    q = _rand((2, T + 1, H, D), 8)
    fq, fk = oracle.rope_expanded(q, k, n, True, 10000.0)
    dq, dk = oracle.rope_expanded(q[:, T:], k[:, T * n:], n, True, 10000.0, token_offset=[T, T])
    np.testing.assert_array_equal(dk, fk[:, T * n:])
    np.testing.assert_array_equal(dq, fq[:, T:])
    # per-sequence offsets are independent
    mixed = np.stack([q[0, T:T + 1], q[1, 0:1]])
    mq, _ = oracle.rope_expanded(mixed, None, n, True, 10000.0, token_offset=[T, 0])
    np.testing.assert_array_equal(mq[0, 0], fq[0, T])
    np.testing.assert_array_equal(mq[1, 0], fq[1, 0])
