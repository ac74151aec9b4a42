"""Seeded synthetic inputs for the Hidden Decoding hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic. Tests feed the same tensors to the CUDA library and to the
float64 oracle, so both sides always see identical bits.

All draws use torch's CPU generator (mt19937, seeded per tensor), then the bf16 tensors are rounded with torch's round-to-nearest-even
conversion. Drawing on the CPU keeps the values identical whichever device the
caller later copies them to.

Workload recipes (the shapes of the five attention workloads and the expansion
workload) live in ``WORKLOADS``; each entry is a plain dict of sizes.
"""
from __future__ import annotations

import math

import torch

INTRA, CROSS_FULL, CROSS_WINDOW = 0, 1, 2
MODE_NAMES = {INTRA: "INTRA", CROSS_FULL: "CROSS_FULL", CROSS_WINDOW: "CROSS_WINDOW"}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 on the CPU, rounded to bf16 (RNE)."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def normal_f32(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def token_ids(B: int, L: int, V: int, seed: int) -> torch.Tensor:
    """Token ids uniform in [0, V), int32 [B, L]."""
    return torch.randint(0, V, (B, L), generator=_gen(seed), dtype=torch.int64).to(torch.int32)


def attention_inputs(B, L, n, Hq, Hkv, D, final_only=False, seed=0, with_grad=False):
    """Q, K, V (and dO) bf16 ~N(0,1) in the expanded-sequence layout.

    Q / dO are [B, S, Hq, D] (S = n*L), or [B, L, Hq, D] with ``final_only``;
    K / V are [B, S, Hkv, D]. Row p of the expanded sequence is stream p mod n
    of token p div n.
    """
    S = n * L
    Sq = L if final_only else S
    out = {
        "q": normal_bf16((B, Sq, Hq, D), seed * 16 + 1),
        "k": normal_bf16((B, S, Hkv, D), seed * 16 + 2),
        "v": normal_bf16((B, S, Hkv, D), seed * 16 + 3),
    }
    if with_grad:
        out["do"] = normal_bf16((B, Sq, Hq, D), seed * 16 + 4)
    return out


def decode_inputs(B, n, T, Tcap, Hq, Hkv, D, seed=0, ragged=False):
    """One decode step: q [B, n, Hq, D], caches [B, Tcap*n, Hkv, D], seqlen [B].

    seqlen[b] counts tokens including the new one, so (seqlen[b]) * n cache rows
    are valid and the new token's n rows already sit at the end of them. With
    ``ragged`` the sequences get different lengths in [1, T+1].
    """
    q = normal_bf16((B, n, Hq, D), seed * 16 + 5)
    kc = normal_bf16((B, Tcap * n, Hkv, D), seed * 16 + 6)
    vc = normal_bf16((B, Tcap * n, Hkv, D), seed * 16 + 7)
    if ragged:
        seqlen = torch.randint(1, T + 2, (B,), generator=_gen(seed * 16 + 8), dtype=torch.int64)
        seqlen[0] = T + 1
        seqlen = seqlen.to(torch.int32)
    else:
        seqlen = torch.full((B,), T + 1, dtype=torch.int32)
    return {"q": q, "k_cache": kc, "v_cache": vc, "seqlen": seqlen}


def expand_inputs(B, L, n, V, d, seed=0, dtype=torch.float32, std=0.02):
    """Token ids U[0, V) and n embedding tables [n, V, d] ~N(0, std^2)."""
    ids = token_ids(B, L, V, seed * 16 + 9)
    if dtype == torch.float32:
        tables = normal_f32((n, V, d), seed * 16 + 10, std)
    else:
        tables = normal_f32((n, V, d), seed * 16 + 10, std).to(dtype)
    return {"ids": ids, "tables": tables}


def lm_head_inputs(B, L, n, d, V, seed=0, ignore_every=0):
    """Hidden states x bf16 [B, n*L, d] ~N(0, 1), LM head w bf16 [V, d] ~N(0, (3/sqrt(d))^2)
    (logits of standard deviation about 3), labels int32 [B, L] uniform in [0, V); with
    ``ignore_every`` = k > 0 every k-th label is -100 (a token without a target)."""
    x = normal_bf16((B, n * L, d), seed * 16 + 11)
    w = normal_bf16((V, d), seed * 16 + 12, std=3.0 / math.sqrt(d))
    labels = token_ids(B, L, V, seed * 16 + 13)
    if ignore_every:
        labels.view(-1)[::ignore_every] = -100
    return {"x": x, "w": w, "labels": labels}


# Sizes of the workloads this library is exercised on.
WORKLOADS = {
    # tiny end-to-end case: expansion + INTRA / CROSS_FULL fwd and bwd
    "tiny": dict(B=1, L=64, n=4, V=1000, d=256, Hq=4, Hkv=4, D=64, scale=1.0 / 8.0),
    # intra-stream training layer
    "intra_train": dict(B=4, L=2048, n=4, Hq=16, Hkv=4, D=128, scale=1.0 / math.sqrt(128)),
    # cross-stream sliding-window training layer, window in tokens
    "cross_window": dict(B=2, L=8192, n=4, Hq=32, Hkv=8, D=128, W=1024, scale=1.0 / math.sqrt(128)),
    # long-context full cross-stream layer (+ final-stream-only queries)
    "long_cross": dict(B=1, L=32768, n=4, Hq=32, Hkv=8, D=128, scale=1.0 / math.sqrt(128)),
    # final-stream LM-head loss over the cross_window layer's tokens (d = 32 heads x 128)
    "lm_head": dict(B=2, L=8192, n=4, d=4096, V=32000),
    # multi-stream decode step against a 16384-token cache
    "decode": dict(B=8, n=4, T=16384, Hq=32, Hkv=8, D=128, scale=1.0 / math.sqrt(128)),
}
