"""Float64 CPU oracle for the Hidden Decoding hot path.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg import this package; the CUDA library and its Python
binding never do, and the two share no code. Every function restates a passage
of the page "微信WeLM提出Hidden Decoding：大模型推理新范式" (tahou.com), cited in
each module's header.

Parity status: every function here is pinned by `-m "not gpu"` tests against
hand-worked values, closed forms, textbook/library special cases, brute force
and finite differences (tests/test_oracle_*.py).
"""
from .attention import (  # noqa: F401
    CROSS_FULL,
    CROSS_WINDOW,
    INTRA,
    attn_bwd,
    attn_bwd_dq_rows,
    attn_bwd_kv_cols,
    attn_fwd,
    attn_fwd_rows,
    mask_matrix,
    query_positions,
    stream_of,
    token_of,
    visible,
)
from .decode import decode_attn  # noqa: F401
from .expand import expand_embed  # noqa: F401
from .rope import rope, rope_expanded  # noqa: F401
from .lm_head import final_readout, lm_head_ce, lm_head_ce_grad, lm_head_ce_rows  # noqa: F401
