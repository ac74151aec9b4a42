"""Hidden Decoding hot path on B200: a C-ABI CUDA library and its Python binding.

The library (``libhd.so``, built from ``csrc/`` by ``build.py``) implements the
data-parallel hot path of Hidden Decoding with Stream-Factorized Attention
(page "微信WeLM提出Hidden Decoding：大模型推理新范式", tahou.com):

* ``hd_expand_embed``  interleaved n-table embedding gather (stream k of token i
  at position (i-1)n+k);
* ``hd_rope_expanded``  rotary position embedding of q and k at the physical
  positions p = t*n + s (continuous positions over the expanded sequence);
* ``hd_final_readout`` / ``hd_lm_head_ce``  the final stream's hidden rows and the
  LM-head cross-entropy on them (the only supervised stream), logits never
  materialised;
* ``hd_attn_fwd`` / ``hd_attn_bwd``  attention over the expanded sequence with
  intra-stream, cross-stream full-causal and cross-stream sliding-window masks,
  optionally with final-stream-only queries (KV-mirror);
* ``hd_decode_attn_final``  the final stream's query alone (KV-mirror layers);
* ``hd_decode_attn``  the n stream queries of a new token against the
  interleaved per-stream KV cache.

The C names are re-exported from ``_lib`` (pointer + size arguments). The
tensor helpers below (``expand_embed``, ``rope_``, ``attn_fwd``, ``attn_bwd``,
``decode_attn``, ``decode_attn_final``) allocate outputs and workspace with torch and call the same C
entry points; torch is used for device memory and streams only.
"""
from __future__ import annotations

from ._lib import (  # noqa: F401
    HD_ERR_CUDA,
    HD_ERR_DEVICE_INDEX,
    HD_ERR_INVALID_ARG,
    HD_ERR_TIMEOUT,
    HD_ERR_UNSUPPORTED,
    HD_OK,
    HDError,
    hd_attn_bwd,
    hd_attn_bwd_workspace_bytes,
    hd_attn_fwd,
    hd_decode_attn,
    hd_decode_attn_final,
    hd_decode_attn_noalloc,
    hd_decode_final_workspace_bytes,
    hd_decode_workspace_bytes,
    hd_device_status,
    hd_expand_embed,
    hd_final_readout,
    hd_lm_head_ce,
    hd_lm_head_ce_bwd,
    hd_lm_head_ce_bwd_workspace_bytes,
    hd_lm_head_ce_workspace_bytes,
    hd_rope_expanded,
    hd_selftest_wait_timeout,
    lib,
    status_string,
)

INTRA, CROSS_FULL, CROSS_WINDOW = 0, 1, 2


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device (the library has no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def expand_embed(ids, tables, stream=None):
    """ids int32 [B, L], tables [n, V, d] -> out [B, L*n, d] (tables' dtype)."""
    import torch

    _need_cuda(ids, tables)
    B, L = ids.shape
    n, V, d = tables.shape
    out = torch.empty((B, L * n, d), dtype=tables.dtype, device=tables.device)
    hd_expand_embed(ids, tables, out, B, L, n, V, d, tables.element_size(), stream)
    return out


def rope_(q, k, n, final_only=False, base=10000.0, token_offset=None, stream=None):
    """Rotate q [B, Sq, Hq, D] and k [B, n*L, Hkv, D] bf16 in place at their physical positions.

    Either may be None. ``token_offset`` (int32 [B] on the device) gives the
    tokens that precede the rows of each sequence. Returns (q, k).
    """
    ts = [t for t in (q, k, token_offset) if t is not None]
    _need_cuda(*ts)
    ref = k if k is not None else q
    B, D = ref.shape[0], ref.shape[-1]
    if k is not None:
        L = k.shape[1] // n
    else:
        L = q.shape[1] if final_only else q.shape[1] // n
    Hq = q.shape[2] if q is not None else 0
    Hkv = k.shape[2] if k is not None else 0
    hd_rope_expanded(q, k, token_offset, B, L, n, Hq, Hkv, D, final_only, base, stream)
    return q, k


def attn_fwd(q, k, v, n, mode, W=0, final_only=False, scale=None, stream=None):
    """q [B, Sq, Hq, D], k/v [B, n*L, Hkv, D] bf16 -> (out bf16 like q, lse fp32 [B, Hq, Sq])."""
    import torch

    _need_cuda(q, k, v)
    B, S, Hkv, D = k.shape
    L = S // n
    Hq = q.shape[2]
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, q.shape[1]), dtype=torch.float32, device=q.device)
    hd_attn_fwd(q, k, v, out, lse, B, L, n, Hq, Hkv, D, mode, W, final_only, scale, stream)
    return out, lse


def attn_bwd(q, k, v, out, lse, dout, n, mode, W=0, final_only=False, scale=None, stream=None,
             workspace=None):
    """Gradients (dq, dk, dv) in bf16; the fp32 workspace is allocated if not given."""
    import torch

    _need_cuda(q, k, v, out, lse, dout)
    B, S, Hkv, D = k.shape
    L = S // n
    Hq = q.shape[2]
    if scale is None:
        scale = D ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nbytes = hd_attn_bwd_workspace_bytes(B, L, n, Hq, Hkv, D, final_only)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    hd_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, L, n, Hq, Hkv, D, mode, W, final_only, scale,
                workspace, workspace.numel() * workspace.element_size(), stream)
    return dq, dk, dv


def decode_attn(q, k_cache, v_cache, seqlen, mode, W=0, scale=None, stream=None, workspace=None):
    """q [B, n, Hq, D]; caches [B, Tcap*n, Hkv, D]; seqlen int32 [B] (tokens incl. the new one)."""
    import torch

    _need_cuda(q, k_cache, v_cache, seqlen)
    B, n, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    Tcap = k_cache.shape[1] // n
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, n), dtype=torch.float32, device=q.device)
    nbytes = hd_decode_workspace_bytes(B, n, Tcap, Hq, Hkv, D)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    hd_decode_attn(q, k_cache, v_cache, seqlen, out, lse, B, n, Tcap, Hq, Hkv, D, mode, W, scale,
                   workspace, workspace.numel() * workspace.element_size(), stream)
    return out, lse


def decode_attn_final(q, k_cache, v_cache, seqlen, n, mode, W=0, scale=None, stream=None,
                      workspace=None):
    """q [B, 1, Hq, D] (stream n-1 of the new token); caches [B, Tcap*n, Hkv, D]; seqlen int32 [B].

    Returns (out [B, 1, Hq, D] bf16, lse [B, Hq, 1] fp32).
    """
    import torch

    _need_cuda(q, k_cache, v_cache, seqlen)
    B, one, Hq, D = q.shape
    if one != 1:
        raise ValueError("q must be [B, 1, Hq, D]")
    Hkv = k_cache.shape[2]
    Tcap = k_cache.shape[1] // n
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device)
    nbytes = hd_decode_final_workspace_bytes(B, n, Tcap, Hq, Hkv, D)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    hd_decode_attn_final(q, k_cache, v_cache, seqlen, out, lse, B, n, Tcap, Hq, Hkv, D, mode, W,
                         scale, workspace, workspace.numel() * workspace.element_size(), stream)
    return out, lse


def final_readout(x, n, stream=None):
    """x [B, n*L, d] -> the final stream's rows [B, L, d] (positions t*n + n-1)."""
    import torch

    _need_cuda(x)
    B, S, d = x.shape
    L = S // n
    out = torch.empty((B, L, d), dtype=x.dtype, device=x.device)
    hd_final_readout(x, out, B, L, n, d, x.element_size(), stream)
    return out


def lm_head_ce(x, w, labels, n, stream=None, workspace=None):
    """x bf16 [B, n*L, d], w bf16 [V, d], labels int32 [B, L] -> (loss, lse) fp32 [B, L]."""
    import torch

    _need_cuda(x, w, labels)
    B, S, d = x.shape
    L = S // n
    V = w.shape[0]
    loss = torch.empty((B, L), dtype=torch.float32, device=x.device)
    lse = torch.empty((B, L), dtype=torch.float32, device=x.device)
    nbytes = hd_lm_head_ce_workspace_bytes(B, L, V)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    hd_lm_head_ce(x, w, labels, loss, lse, B, L, n, d, V, workspace,
                  workspace.numel() * workspace.element_size(), stream)
    return loss, lse


def lm_head_ce_bwd(x, w, labels, lse, n, grad_scale=1.0, stream=None, workspace=None):
    """Gradients of sum(loss) * grad_scale: (dh bf16 [B, L, d], dw fp32 [V, d])."""
    import torch

    _need_cuda(x, w, labels, lse)
    B, S, d = x.shape
    L = S // n
    V = w.shape[0]
    dh = torch.empty((B, L, d), dtype=torch.bfloat16, device=x.device)
    dw = torch.empty((V, d), dtype=torch.float32, device=x.device)
    nbytes = hd_lm_head_ce_bwd_workspace_bytes(B, L, V)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    hd_lm_head_ce_bwd(x, w, labels, lse, grad_scale, dh, dw, B, L, n, d, V, workspace,
                      workspace.numel() * workspace.element_size(), stream)
    return dh, dw
