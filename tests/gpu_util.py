"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import pytest
import torch

# Tolerances of the parity bar: bf16 inputs, fp32 accumulation, bf16 outputs.
O_MAX, O_MEAN = 2e-2, 2e-3        # attention outputs
G_MAX, G_MEAN = 5e-2, 5e-3        # gradients
LSE_MAX = 5e-3                     # fp32 LSE: scores are exact fp32 sums of exact bf16 products


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from structured_causal_attention_b200.build import build

    build()


def dev(x):
    return x.cuda()


def host64(x):
    return x.detach().float().cpu().numpy().astype(np.float64)


def check(got, want, max_tol, mean_tol, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - want)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= max_tol and mean <= mean_tol, f"{what}: max {mx:.3e} (<= {max_tol}), mean {mean:.3e} (<= {mean_tol})"
    return mx, mean


def sample_rows(Sq, n, W, final_only, k, seed, tile=128):
    """Seeded query rows: boundaries of streams, tiles and the window, plus random."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, Sq - 1, Sq - 2, tile - 1, tile, Sq // 2}
    if not final_only:
        fixed |= {s for s in range(n)} | {Sq - n + s for s in range(n)}
        if W:
            fixed |= {n * W - 1, n * W, n * W + 1}
    fixed = sorted(r for r in fixed if 0 <= r < Sq)
    rest = rng.choice(Sq, size=max(0, min(Sq, k) - len(fixed)), replace=False)
    return np.unique(np.concatenate([np.array(fixed, dtype=np.int64), rest.astype(np.int64)]))[:max(k, len(fixed))]
