"""CPU oracle: interleaved n-table embedding expansion.

TEST INFRASTRUCTURE ONLY; the library never calls it.

Source: page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), section
"隐式序列缩放的技术细节", step 1: given the input sequence and n embedding tables,
the representation of stream k of token i is put at physical position (i-1)n+k,
giving an nL-long sequence; page "WeLM ... Latent computation scaling and Hidden
Decoding" (aiflownews.com): each stream has its own embedding table.
0-based: X[b, t*n + s, :] = E[s][ids[b, t], :].

The copy is exact, so the result is compared bit for bit.
"""
from __future__ import annotations

import numpy as np


def expand_embed(ids, tables):
    """ids int [B, L], tables [n, V, d] (any dtype) -> X [B, L*n, d], same dtype.

    Written as the definition: for each stream s, the rows t*n + s take table s
    at the token's id.
    """
    ids = np.asarray(ids)
    tables = np.asarray(tables)
    B, L = ids.shape
    n, V, d = tables.shape
    if ids.size and (ids.min() < 0 or ids.max() >= V):
        raise IndexError("token id outside the table")
    out = np.empty((B, L * n, d), dtype=tables.dtype)
    for s in range(n):
        out[:, s::n, :] = tables[s][ids]
    return out
