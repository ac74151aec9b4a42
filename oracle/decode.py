"""CPU oracle: one multi-stream decode step against an interleaved KV cache.

TEST INFRASTRUCTURE ONLY; the library never calls it.

Sources (page "微信WeLM提出Hidden Decoding：大模型推理新范式", tahou.com):
  * section "实验效果与成本分析": the n streams of a new token are computed in one
    parallel forward, not one after another;
  * section "中间流的作用验证": each stream keeps its own KV state;
  * the mask is the prefill mask of the same layer type (section
    "规模化落地的工程优化").

Reading (pages silent on the cache layout): the cache holds the expanded
sequence in position order, [B, Tcap*n, Hkv, D]; seqlen[b] counts tokens
including the new one, whose n rows are already written at positions
T*n .. T*n+n-1 (T = seqlen[b]-1). Query (s, h) of sequence b sits at p = T*n+s
and reads cache positions p' < seqlen[b]*n that the layer's mask allows.

Final-stream-only decode (section "规模化落地的工程优化", KV-mirror paragraph:
only the last stream passes through the mirror layers): one query per
sequence, at p = T*n + n-1, against the same cache and mask.
"""
from __future__ import annotations

import numpy as np

from .attention import CROSS_WINDOW, _f64, visible


def decode_attn(q, k_cache, v_cache, seqlen, n, mode, W, scale, final_only=False):
    """q [B, n, Hq, D] ([B, 1, Hq, D] with final_only); caches [B, Tcap*n, Hkv, D]; seqlen int [B].

    Returns (o like q, lse [B, Hq, n or 1]) in float64.
    """
    q = _f64(q)
    seqlen = np.asarray(seqlen.cpu() if hasattr(seqlen, "cpu") else seqlen, dtype=np.int64)
    B, nn, Hq, D = q.shape
    streams = np.array([n - 1]) if final_only else np.arange(n)
    assert nn == len(streams)
    Hkv = k_cache.shape[2]
    g = Hq // Hkv
    o = np.zeros((B, nn, Hq, D))
    lse = np.zeros((B, Hq, nn))
    for b in range(B):
        T = int(seqlen[b]) - 1
        qpos = T * n + streams
        lo = max(0, T * n - n * W + 1) if mode == CROSS_WINDOW else 0
        keys = np.arange(lo, (T + 1) * n)
        mask = visible(qpos[:, None], keys[None, :], n, mode, W)  # [queries, keys]
        for kh in range(Hkv):
            kk = _f64(k_cache[b, lo:(T + 1) * n, kh, :])
            vv = _f64(v_cache[b, lo:(T + 1) * n, kh, :])
            for h in range(kh * g, (kh + 1) * g):
                sc = scale * (q[b, :, h, :] @ kk.T)  # [queries, keys]
                sc = np.where(mask, sc, -np.inf)
                mx = sc.max(axis=1, keepdims=True)
                e = np.exp(sc - mx)
                tot = e.sum(axis=1, keepdims=True)
                lse[b, h, :] = (mx + np.log(tot))[:, 0]
                o[b, :, h, :] = (e / tot) @ vv
    return o, lse
