"""Float64 CPU oracle: Stream-Factorized attention, forward and backward.

TEST INFRASTRUCTURE ONLY. Nothing in the library imports or calls this module;
only the tests, the smoke check and the bench's CPU-baseline leg do. It is a
plain, slow restatement of the method's definition in NumPy float64.

Sources (page "微信WeLM提出Hidden Decoding：大模型推理新范式", tahou.com):
  * section "隐式序列缩放的技术细节", step 1: stream k of token i sits at
    physical position (i-1)n+k of an nL-long sequence. 0-based here:
    p = t*n + s, token(p) = p // n, stream(p) = p % n.
  * same section, step 2: that sequence goes through standard causal attention.
  * section "规模化落地的工程优化", the two bullets: intra-stream layers see only
    earlier positions of their own stream; cross-stream layers keep the base
    model's shape, full causal or sliding window.
  * same section, KV-mirror paragraph: only the final stream passes through the
    mirror layers, so there only the final stream's queries exist and they read
    K/V built for all n streams.

Readings where the page is not explicit:
  * a position is one of the "earlier positions" it may see (self included):
    the backbone is standard causal attention, and without self the first row of
    every stream would see nothing;
  * the window W is counted in tokens, so it spans n*W expanded positions,
    self included: visible iff 0 <= p - p' < n*W;
  * intra-stream layers have no window;
  * LSE is the natural-log log-sum-exp of the scaled scores.

Layouts: q / dO [B, Sq, Hq, D], k / v [B, S, Hkv, D], lse [B, Hq, Sq] with
Sq = S, or Sq = L = S/n when only final-stream queries exist (their positions are
t*n + n-1). Query head h reads KV head h // (Hq // Hkv) (grouped-query attention).
"""
from __future__ import annotations

import numpy as np

INTRA, CROSS_FULL, CROSS_WINDOW = 0, 1, 2


def stream_of(p, n):
    """Stream index of expanded position p (step 1 of the method, 0-based)."""
    return p % n


def token_of(p, n):
    """Token index of expanded position p (step 1 of the method, 0-based)."""
    return p // n


def query_positions(S, n, final_only):
    """Physical positions of the query rows: all S, or t*n + n-1 for KV-mirror."""
    if final_only:
        return np.arange(S // n, dtype=np.int64) * n + (n - 1)
    return np.arange(S, dtype=np.int64)


def visible(p, pk, n, mode, W):
    """Boolean mask: may the query at position p read the key at position pk?

    Broadcasts over array arguments. Causal in every mode (pk <= p); INTRA adds
    "same stream"; CROSS_WINDOW adds "fewer than n*W positions back".
    """
    p = np.asarray(p)
    pk = np.asarray(pk)
    m = pk <= p
    if mode == INTRA:
        m = m & (stream_of(pk, n) == stream_of(p, n))
    elif mode == CROSS_FULL:
        pass
    elif mode == CROSS_WINDOW:
        if W < 1:
            raise ValueError("window must hold at least one token")
        m = m & ((p - pk) < n * W)
    else:
        raise ValueError(f"unknown mode {mode}")
    return m


def mask_matrix(qpos, S, n, mode, W):
    """Explicit [len(qpos), S] mask of visible (query, key) pairs."""
    return visible(np.asarray(qpos)[:, None], np.arange(S)[None, :], n, mode, W)


def _f64(x):
    """Exact upcast of a bf16/fp32 torch tensor or array to float64 NumPy."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


def _rows_softmax(scores, mask):
    """Masked row softmax: returns (P, lse); every row has >= 1 visible key."""
    s = np.where(mask, scores, -np.inf)
    mx = s.max(axis=-1, keepdims=True)
    e = np.exp(s - mx)
    tot = e.sum(axis=-1, keepdims=True)
    lse = (mx + np.log(tot))[..., 0]
    return e / tot, lse


def attn_fwd(q, k, v, n, mode, W, final_only, scale):
    """O = softmax(scale * Q K^T restricted to visible keys) V, and LSE.

    Returns (o [B, Sq, Hq, D] float64, lse [B, Hq, Sq] float64).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, Hq, D = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    qpos = query_positions(S, n, final_only)
    assert len(qpos) == Sq
    mask = mask_matrix(qpos, S, n, mode, W)
    o = np.zeros((B, Sq, Hq, D))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            scores = scale * (q[b, :, h, :] @ k[b, :, kh, :].T)
            P, lse[b, h] = _rows_softmax(scores, mask)
            o[b, :, h, :] = P @ v[b, :, kh, :]
    return o, lse


def _row_block(q, k, v, n, mode, W, final_only, scale, b, h, rows):
    """Scores of selected query rows against the keys they can reach.

    Returns (Q rows, K, V, P, lse) in float64 for the key window
    [lo, hi) that covers every selected row; P is the masked softmax.
    """
    S, Hkv = k.shape[1], k.shape[2]
    Hq = q.shape[2]
    kh = h // (Hq // Hkv)
    rows = np.asarray(rows, dtype=np.int64)
    qpos = query_positions(S, n, final_only)[rows]
    lo = max(0, int(qpos.min()) - n * W + 1) if mode == CROSS_WINDOW else 0
    hi = int(qpos.max()) + 1
    keys = np.arange(lo, hi)
    mask = visible(qpos[:, None], keys[None, :], n, mode, W)
    Q = _f64(q[b, rows, h, :])
    K = _f64(k[b, lo:hi, kh, :])
    V = _f64(v[b, lo:hi, kh, :])
    P, lse = _rows_softmax(scale * (Q @ K.T), mask)
    return Q, K, V, P, lse, lo


def attn_fwd_rows(q, k, v, n, mode, W, final_only, scale, b, h, rows, block=64):
    """Forward for selected query rows of one (batch, query head).

    ``rows`` index the query dimension of q (0..Sq-1). Returns
    (o [len(rows), D], lse [len(rows)]), both float64. Rows are taken in blocks
    so the score matrix stays small at any sequence length.
    """
    rows = np.asarray(rows, dtype=np.int64)
    D = q.shape[-1]
    o = np.zeros((len(rows), D))
    lse = np.zeros(len(rows))
    for i in range(0, len(rows), block):
        sel = rows[i:i + block]
        _, _, V, P, l, _ = _row_block(q, k, v, n, mode, W, final_only, scale, b, h, sel)
        o[i:i + block] = P @ V
        lse[i:i + block] = l
    return o, lse


def attn_bwd(q, k, v, do, n, mode, W, final_only, scale):
    """Gradients of sum(dO * O) for O = attn_fwd(q, k, v, ...).

    D_i = sum_d dO_id O_id; dP = dO V^T; dS = P * (dP - D); dQ = scale dS K;
    dK = scale sum_group dS^T Q; dV = sum_group P^T dO. Returns float64
    (dq like q, dk like k, dv like v). O and P are the oracle's own, not the
    kernel's.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Sq, Hq, D = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    mask = mask_matrix(query_positions(S, n, final_only), S, n, mode, W)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            K, V, Q, dO = k[b, :, kh], v[b, :, kh], q[b, :, h], do[b, :, h]
            P, _ = _rows_softmax(scale * (Q @ K.T), mask)
            O = P @ V
            Dvec = (dO * O).sum(axis=-1)
            dP = dO @ V.T
            dS = P * (dP - Dvec[:, None])
            dq[b, :, h] = scale * (dS @ K)
            dk[b, :, kh] += scale * (dS.T @ Q)
            dv[b, :, kh] += P.T @ dO
    return dq, dk, dv


def attn_bwd_dq_rows(q, k, v, do, n, mode, W, final_only, scale, b, h, rows, block=64):
    """dQ for selected query rows of one (batch, query head); row-local:
    dQ_i = scale sum_j P_ij (dO_i . V_j - dO_i . O_i) K_j."""
    rows = np.asarray(rows, dtype=np.int64)
    D = q.shape[-1]
    out = np.zeros((len(rows), D))
    for i in range(0, len(rows), block):
        sel = rows[i:i + block]
        _, K, V, P, _, _ = _row_block(q, k, v, n, mode, W, final_only, scale, b, h, sel)
        dO = _f64(do[b, sel, h, :])
        O = P @ V
        dS = P * (dO @ V.T - (dO * O).sum(-1, keepdims=True))
        out[i:i + block] = scale * (dS @ K)
    return out


def attn_bwd_kv_cols(q, k, v, do, n, mode, W, final_only, scale, b, kh, cols, block=64):
    """dK, dV for selected key positions of one (batch, KV head).

    Every query that sees one of the keys gets its full row recomputed (LSE, O
    and D need all of that row's keys), then dK_j = scale sum_i dS_ij Q_i and
    dV_j = sum_i P_ij dO_i, summed over the query heads of the group.
    Returns (dk [len(cols), D], dv [len(cols), D]).
    """
    S, Hkv = k.shape[1], k.shape[2]
    Hq = q.shape[2]
    g = Hq // Hkv
    D = q.shape[-1]
    cols = np.asarray(cols, dtype=np.int64)
    qpos_all = query_positions(S, n, final_only)
    sees = visible(qpos_all[:, None], cols[None, :], n, mode, W)
    qrows = np.nonzero(sees.any(axis=1))[0]
    dk = np.zeros((len(cols), D))
    dv = np.zeros((len(cols), D))
    for h in range(kh * g, (kh + 1) * g):
        for i in range(0, len(qrows), block):
            sel = qrows[i:i + block]
            Q, K, V, P, _, lo = _row_block(q, k, v, n, mode, W, final_only, scale, b, h, sel)
            dO = _f64(do[b, sel, h, :])
            O = P @ V
            Dvec = (dO * O).sum(-1)
            # the selected keys inside this block's key window
            inwin = (cols >= lo) & (cols < lo + K.shape[0])
            idx = cols[inwin] - lo
            Pc = P[:, idx]
            dSc = Pc * (dO @ V[idx].T - Dvec[:, None])
            dk[inwin] += scale * (dSc.T @ Q)
            dv[inwin] += Pc.T @ dO
    return dk, dv
