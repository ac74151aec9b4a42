"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

Each case rewrites one expression of an oracle module's source, executes the
rewritten module, swaps its functions into the ``oracle`` package, and runs the
pins that should fail. A mutant that every pin accepts would mean the pins do
not constrain that part of the oracle.
"""
import importlib
import inspect
import types

import pytest

import oracle
import oracle.attention
import oracle.decode
import oracle.expand
import oracle.lm_head
from tests import test_oracle_lm_head as lm_pins
from tests import test_oracle_pins as pins
from tests import test_oracle_rope as rope_pins

# the package re-exports a function named `rope`, which hides the submodule attribute
rope_mod = importlib.import_module("oracle.rope")

EXPORTS = {
    oracle.attention: ["attn_bwd", "attn_bwd_dq_rows", "attn_bwd_kv_cols", "attn_fwd",
                       "attn_fwd_rows", "mask_matrix", "query_positions", "visible"],
    oracle.decode: ["decode_attn"],
    oracle.expand: ["expand_embed"],
    oracle.lm_head: ["final_readout", "lm_head_ce", "lm_head_ce_grad", "lm_head_ce_rows"],
    rope_mod: ["rope", "rope_expanded"],
}


def _mutant(module, old, new):
    src = inspect.getsource(module)
    assert src.count(old) >= 1, old
    src = src.replace(old, new)
    mod = types.ModuleType(module.__name__ + "_mutant")
    mod.__dict__["__package__"] = "oracle"
    exec(compile(src, module.__name__ + "_mutant", "exec"), mod.__dict__)
    return mod


def _run_pins(golden, checks):
    """True if at least one pin raises AssertionError."""
    for fn, args in checks:
        try:
            fn(*args)
        except AssertionError:
            return True
    return False


MUTANTS = [
    ("self excluded", oracle.attention, "m = pk <= p", "m = pk < p",
     [(pins.test_golden_masks, "G")]),
    ("token instead of stream", oracle.attention,
     "(stream_of(pk, n) == stream_of(p, n))", "(token_of(pk, n) == token_of(p, n))",
     [(pins.test_golden_masks, "G")]),
    ("window off by one", oracle.attention, "((p - pk) < n * W)", "((p - pk) <= n * W)",
     [(pins.test_golden_masks, "G")]),
    ("window counted in positions", oracle.attention, "((p - pk) < n * W)", "((p - pk) < W)",
     [(pins.test_golden_masks, "G")]),
    ("final stream is stream 0", oracle.attention,
     "np.arange(S // n, dtype=np.int64) * n + (n - 1)", "np.arange(S // n, dtype=np.int64) * n",
     [(pins.test_golden_masks, "G")]),
    ("dropped D term", oracle.attention, "dS = P * (dP - Dvec[:, None])", "dS = P * dP",
     [(pins.test_golden_uniform, "G")]),
    ("dV not transposed", oracle.attention, "dv[b, :, kh] += P.T @ dO", "dv[b, :, kh] += P @ dO",
     [(pins.test_golden_uniform, "G")]),
    ("dK sign flipped", oracle.attention, "dk[b, :, kh] += scale * (dS.T @ Q)",
     "dk[b, :, kh] -= scale * (dS.T @ Q)",
     [(pins.test_backward_matches_library_autograd_textbook, 1)]),
    ("GQA head map", oracle.attention, "            kh = h // g\n            scores",
     "            kh = h % Hkv\n            scores",
     [(pins.test_gqa_equals_mha_with_repeated_kv, "INTRA")]),
    ("LSE without max", oracle.attention, "lse = (mx + np.log(tot))[..., 0]",
     "lse = np.log(tot)[..., 0]", [(pins.test_golden_weighted, "G")]),
    ("scale dropped", oracle.attention, "scores = scale * (q[b, :, h, :] @ k[b, :, kh, :].T)",
     "scores = (q[b, :, h, :] @ k[b, :, kh, :].T)",
     [(pins.test_n1_reduces_to_textbook_causal, "CROSS_FULL")]),
    ("stream-major expansion", oracle.expand, "out[:, s::n, :] = tables[s][ids]",
     "out[:, s * L:(s + 1) * L, :] = tables[s][ids]", [(pins.test_golden_expand, "G")]),
    ("decode query at stream 0", oracle.decode, "qpos = T * n + streams",
     "qpos = T * n + 0 * streams",
     [(pins.test_golden_decode, "G")]),
    ("readout of stream 0", oracle.lm_head, "return x[:, n - 1::n, :]", "return x[:, 0::n, :]",
     [(lm_pins.test_readout_is_the_last_stream_of_each_token, 4)]),
    ("loss sign flipped", oracle.lm_head, "loss = np.where(labels >= 0, lse - picked, 0.0)",
     "loss = np.where(labels >= 0, picked - lse, 0.0)", [(lm_pins.test_ce_matches_torch_cross_entropy, None)]),
    ("logsumexp without max", oracle.lm_head,
     "lse = (mx + np.log(np.exp(logits - mx).sum(axis=-1, keepdims=True)))[..., 0]",
     "lse = np.log(np.exp(logits).sum(axis=-1, keepdims=True))[..., 0]",
     [(lm_pins.test_large_logits_stay_finite, None)]),
    ("ignored label not zeroed", oracle.lm_head, "loss = np.where(labels >= 0, lse - picked, 0.0)",
     "loss = lse - picked", [(lm_pins.test_ce_matches_torch_cross_entropy, None)]),
    ("CE gradient without the one-hot", oracle.lm_head, "g[rows[:, 0], rows[:, 1], labels[labels >= 0]] -= 1.0",
     "pass", [(lm_pins.test_grad_matches_central_differences, None)]),
    ("dW from the probabilities", oracle.lm_head, 'dw = np.einsum("blv,bld->vd", g, h)',
     'dw = np.einsum("blv,bld->vd", p, h)', [(lm_pins.test_grad_matches_central_differences, None)]),
    ("rope interleaved pairs", rope_mod,
     "return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)",
     "return np.stack([x[..., 0::2] * c - x[..., 1::2] * s, x[..., 1::2] * c + x[..., 0::2] * s], "
     "axis=-1).reshape(x.shape)", [(rope_pins.test_first_pair_turns_by_exactly_p_radians, None)]),
    ("rope sine sign", rope_mod, "x1 * c - x2 * s, x2 * c + x1 * s", "x1 * c + x2 * s, x2 * c - x1 * s",
     [(rope_pins.test_first_pair_turns_by_exactly_p_radians, None)]),
    ("rope frequency exponent i/D", rope_mod, "* 2.0 / D)", "* 1.0 / D)",
     [(rope_pins.test_last_frequency_matches_its_closed_form, None)]),
    ("rope at token index", rope_mod, "rope(k[b:b + 1], np.arange(S) + shift, base)",
     "rope(k[b:b + 1], np.arange(S) // n + shift, base)", [(rope_pins.test_expanded_positions_are_physical, 4)]),
]


# a planted mistake may overflow on the way to failing its pin (that is the point)
@pytest.mark.filterwarnings("ignore:overflow encountered:RuntimeWarning")
@pytest.mark.parametrize("case", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(case, golden, monkeypatch):
    _, module, old, new, checks = case
    mut = _mutant(module, old, new)
    for name in EXPORTS[module]:
        monkeypatch.setattr(oracle, name, getattr(mut, name))
        monkeypatch.setattr(module, name, getattr(mut, name))
    if module is oracle.attention:
        # decode reads the mask predicate from the attention module
        monkeypatch.setattr(oracle.decode, "visible", mut.visible)
    resolved = [(fn, (golden,) if a == "G" else () if a is None else (a,)) for fn, a in checks]
    assert _run_pins(golden, resolved), "planted mistake went unnoticed"


def test_unmutated_oracle_passes_the_same_pins(golden):
    for case in MUTANTS:
        for fn, a in case[4]:
            fn(*((golden,) if a == "G" else () if a is None else (a,)))
