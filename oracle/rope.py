"""CPU oracle: rotary position embedding at the physical expanded positions.

TEST INFRASTRUCTURE ONLY; the library never calls it.

Source: page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), section
"隐式序列缩放的技术细节", step 2: the expanded sequence goes through the same
Transformer with standard causal attention and *continuous* position encoding,
i.e. the representation at physical position p = t*n + s is encoded with the
position p itself (0-based), not with its token index t.

Reading (the page names no encoding): the base model's rotary embedding,
rotate-half pairing (element i pairs with i + D/2), frequencies
base^(-2i/D) for i = 0..D/2-1:
    out[i]       = x[i] cos(p w_i) - x[i + D/2] sin(p w_i)
    out[i + D/2] = x[i + D/2] cos(p w_i) + x[i] sin(p w_i)
Final-stream-only queries sit at p = t*n + n-1.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64, query_positions


def rope(x, positions, base):
    """x [B, R, H, D] (any float), positions int [R] -> float64 [B, R, H, D]."""
    x = _f64(x)
    D = x.shape[-1]
    half = D // 2
    w = base ** (-np.arange(half, dtype=np.float64) * 2.0 / D)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * w[None, :]  # [R, D/2]
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_expanded(q, k, n, final_only, base, token_offset=None):
    """RoPE of q (all positions, or final-stream rows) and k at physical positions.

    token_offset[b] tokens precede the rows of sequence b, shifting every
    position of that sequence by token_offset[b] * n (a decode step).
    """
    ref = k if k is not None else q
    B = ref.shape[0]
    S = k.shape[1] if k is not None else (q.shape[1] * (n if final_only else 1))
    offs = np.zeros(B, dtype=np.int64) if token_offset is None else np.asarray(token_offset, np.int64)
    out_q = np.empty(q.shape) if q is not None else None
    out_k = np.empty(k.shape) if k is not None else None
    for b in range(B):
        shift = int(offs[b]) * n
        if q is not None:
            out_q[b:b + 1] = rope(q[b:b + 1], query_positions(S, n, final_only) + shift, base)
        if k is not None:
            out_k[b:b + 1] = rope(k[b:b + 1], np.arange(S) + shift, base)
    return out_q, out_k
