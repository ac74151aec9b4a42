"""CPU oracle: final-stream readout and the LM-head cross-entropy on it.

TEST INFRASTRUCTURE ONLY; the library never calls it.

Source: page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), section
"隐式序列缩放的技术细节", step 3: in training, the next-token prediction loss is
taken only on the last stream of every token; the first n-1 streams get no
direct supervision. The hidden state that is read out for token t is therefore
the one at physical position t*n + n-1.

Readings (the page gives no formula): the LM head is a plain linear map
logits = h W^T (W [V, d], no bias), the loss per token is the softmax
cross-entropy  loss = logsumexp(logits) - logits[label],  labels are already
shifted by the caller (label[b, t] is the target of token t), and a negative
label marks a token without a target (loss 0; its logsumexp is still returned).
"""
from __future__ import annotations

import numpy as np

from .attention import _f64


def final_readout(x, n):
    """x [B, n*L, d] -> the final stream's rows [B, L, d] (positions t*n + n-1)."""
    x = np.asarray(x) if not hasattr(x, "detach") else x.detach().cpu()
    return x[:, n - 1::n, :]


def lm_head_ce(x, w, labels, n):
    """Cross-entropy of the final-stream rows of x under the LM head w.

    x [B, n*L, d], w [V, d], labels int [B, L]. Returns (loss [B, L], lse [B, L])
    in float64; loss is 0 where label < 0.
    """
    h = _f64(final_readout(x, n))                     # [B, L, d]
    w = _f64(w)
    labels = np.asarray(labels.cpu() if hasattr(labels, "cpu") else labels, dtype=np.int64)
    logits = h @ w.T                                  # [B, L, V]
    mx = logits.max(axis=-1, keepdims=True)
    lse = (mx + np.log(np.exp(logits - mx).sum(axis=-1, keepdims=True)))[..., 0]
    safe = np.clip(labels, 0, w.shape[0] - 1)
    picked = np.take_along_axis(logits, safe[..., None], axis=-1)[..., 0]
    loss = np.where(labels >= 0, lse - picked, 0.0)
    return loss, lse


def lm_head_ce_rows(x, w, labels, n, rows):
    """lm_head_ce for the flattened token indices `rows` (b*L + t) only."""
    B, S, d = x.shape
    L = S // n
    rows = np.asarray(rows, dtype=np.int64)
    h = _f64(x[rows // L, (rows % L) * n + n - 1, :])  # token t of sequence b: position t*n + n-1
    w = _f64(w)
    lab = np.asarray(labels.cpu() if hasattr(labels, "cpu") else labels, dtype=np.int64).reshape(-1)[rows]
    logits = h @ w.T
    mx = logits.max(axis=-1, keepdims=True)
    lse = (mx + np.log(np.exp(logits - mx).sum(axis=-1, keepdims=True)))[:, 0]
    picked = logits[np.arange(len(rows)), np.clip(lab, 0, w.shape[0] - 1)]
    return np.where(lab >= 0, lse - picked, 0.0), lse


def lm_head_ce_grad(x, w, labels, n):
    """Gradients of the summed loss, sum_r loss_r (ignored tokens add nothing).

    With G = softmax(logits) - onehot(label) per supervised row (G = 0 for a
    negative label), the chain rule gives dh = G W and dW = G^T h. Returns
    (G [B, L, V], dh [B, L, d], dW [V, d]) in float64; dh is the gradient with
    respect to the final-stream rows, i.e. dX[b, t*n + n-1] = dh[b, t] and the
    other streams' rows of dX are zero.
    """
    h = _f64(final_readout(x, n))                     # [B, L, d]
    w = _f64(w)
    labels = np.asarray(labels.cpu() if hasattr(labels, "cpu") else labels, dtype=np.int64)
    logits = h @ w.T
    mx = logits.max(axis=-1, keepdims=True)
    p = np.exp(logits - mx)
    p /= p.sum(axis=-1, keepdims=True)
    g = p.copy()
    rows = np.argwhere(labels >= 0)
    g[rows[:, 0], rows[:, 1], labels[labels >= 0]] -= 1.0
    g[labels < 0] = 0.0
    dh = g @ w
    dw = np.einsum("blv,bld->vd", g, h)
    return g, dh, dw
