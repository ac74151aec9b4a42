"""The C-ABI library builds, loads, exports every declared symbol and rejects bad
arguments on the host, before any CUDA call (so this runs without a GPU)."""
import os
import re

import pytest

import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import _lib
from structured_causal_attention_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # an aligned, never-dereferenced address: validation fails first


@pytest.fixture(scope="module")
def lib():
    build()
    return hd.lib()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(hd_\w+)\s*\(", src, re.M))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"hd_expand_embed", "hd_attn_fwd", "hd_attn_bwd", "hd_decode_attn"} <= names
    for name in names:
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, name


def test_checked_build_exports_the_same_abi():
    """libhd_checked.so (HD_CHECK_BOUNDS) loads, exports every declared symbol and
    reports its flag; the normal library reports none."""
    build(checked=True)
    checked = _lib.lib_checked()
    for name in _declared():
        assert hasattr(checked, name), name
    assert checked.hd_build_flags() == 1
    assert hd.lib().hd_build_flags() == 0
    assert checked.hd_version() == hd.lib().hd_version()


def test_version_and_status_strings(lib):
    assert hd.lib().hd_version() >> 16 == 1
    for code in range(6):
        assert hd.status_string(code).startswith("HD_")
    assert "unknown" in hd.status_string(99)


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, L=8, n=4, Hq=4, Hkv=2, D=64,
             mode=hd.CROSS_FULL, W=1, fin=0, scale=0.125)
    a.update(kw)
    return hd.lib().hd_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["L"], a["n"],
                                a["Hq"], a["Hkv"], a["D"], a["mode"], a["W"], a["fin"], a["scale"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), hd.HD_ERR_INVALID_ARG), (dict(out=0), hd.HD_ERR_INVALID_ARG),
    (dict(B=0), hd.HD_ERR_INVALID_ARG), (dict(L=-1), hd.HD_ERR_INVALID_ARG),
    (dict(n=0), hd.HD_ERR_INVALID_ARG), (dict(Hq=3), hd.HD_ERR_INVALID_ARG),
    (dict(mode=3), hd.HD_ERR_INVALID_ARG), (dict(mode=hd.CROSS_WINDOW, W=0), hd.HD_ERR_INVALID_ARG),
    (dict(fin=2), hd.HD_ERR_INVALID_ARG), (dict(scale=0.0), hd.HD_ERR_INVALID_ARG),
    (dict(scale=float("nan")), hd.HD_ERR_INVALID_ARG), (dict(D=96), hd.HD_ERR_UNSUPPORTED),
    (dict(D=256), hd.HD_ERR_UNSUPPORTED), (dict(q=FAKE + 2), hd.HD_ERR_INVALID_ARG),
    (dict(L=1 << 27, n=4), hd.HD_ERR_UNSUPPORTED),
])
def test_fwd_rejects(lib, kw, code):
    assert _fwd(**kw) == code


def test_bwd_workspace_and_rejects(lib):
    ws = hd.hd_attn_bwd_workspace_bytes(2, 16, 4, 8, 2, 128, 0)
    rows = 2 * 64 * 8
    # fp32 dQ accumulator + LSE and D rows packed per problem, padded to 64 rows
    assert ws == rows * 128 * 4 + 2 * (2 * 8 * 4 * 64 * 4)
    assert hd.hd_attn_bwd_workspace_bytes(2, 16, 4, 8, 2, 128, 1) == 2 * 16 * 8 * 128 * 4 + 2 * (2 * 8 * 64 * 4)
    assert hd.hd_attn_bwd_workspace_bytes(0, 16, 4, 8, 2, 128, 0) == 0
    L = hd.lib()
    args = [FAKE] * 9 + [2, 16, 4, 8, 2, 128, hd.INTRA, 1, 0, 0.1]
    assert L.hd_attn_bwd(*args, FAKE, ws - 1, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_attn_bwd(*args, 0, ws, None) == hd.HD_ERR_INVALID_ARG
    bad = list(args)
    bad[6] = 0  # dq
    assert L.hd_attn_bwd(*bad, FAKE, ws, None) == hd.HD_ERR_INVALID_ARG


def test_decode_rejects(lib):
    L = hd.lib()
    ws = hd.hd_decode_workspace_bytes(2, 4, 100, 16, 4, 128)
    assert ws > 0
    base = [FAKE] * 6
    ok = [2, 4, 100, 16, 4, 128, hd.CROSS_FULL, 1, 0.1]
    assert L.hd_decode_attn(*base, *ok, FAKE, ws - 1, None) == hd.HD_ERR_INVALID_ARG
    bad = list(ok)
    bad[5] = 80
    assert L.hd_decode_attn(*base, *bad, FAKE, ws, None) == hd.HD_ERR_UNSUPPORTED
    bad = list(ok)
    bad[4] = 3  # Hkv does not divide Hq
    assert L.hd_decode_attn(*base, *bad, FAKE, ws, None) == hd.HD_ERR_INVALID_ARG
    bad = list(ok)
    bad[6], bad[7] = hd.CROSS_WINDOW, 0
    assert L.hd_decode_attn(*base, *bad, FAKE, ws, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_decode_attn(0, *base[1:], *ok, FAKE, ws, None) == hd.HD_ERR_INVALID_ARG


def test_decode_final_workspace_and_rejects(lib):
    L = hd.lib()
    B, n, Tcap, Hq, Hkv, D = 2, 4, 100, 16, 4, 128
    ws = hd.hd_decode_final_workspace_bytes(B, n, Tcap, Hq, Hkv, D)
    assert ws > 0 and hd.hd_decode_final_workspace_bytes(B, n, Tcap, 15, Hkv, D) == 0
    base = [FAKE] * 6
    ok = [B, n, Tcap, Hq, Hkv, D, hd.INTRA, 1, 0.1]
    assert L.hd_decode_attn_final(*base, *ok, FAKE, ws - 1, None) == hd.HD_ERR_INVALID_ARG
    bad = list(ok)
    bad[5] = 96
    assert L.hd_decode_attn_final(*base, *bad, FAKE, ws, None) == hd.HD_ERR_UNSUPPORTED
    bad = list(ok)
    bad[6], bad[7] = hd.CROSS_WINDOW, 0
    assert L.hd_decode_attn_final(*base, *bad, FAKE, ws, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_decode_attn_final(*base[:4], 0, base[5], *ok, FAKE, ws, None) == hd.HD_ERR_INVALID_ARG


def test_lm_head_workspace_and_rejects(lib):
    L = hd.lib()
    ws = hd.hd_lm_head_ce_workspace_bytes(2, 100, 1000)
    # per 256-wide vocabulary tile a (max, sum) pair per row, plus the label logit per row
    assert ws == 4 * 2 * 200 * 4 + 1024
    assert hd.hd_lm_head_ce_workspace_bytes(0, 100, 1000) == 0
    ok = [FAKE, FAKE, FAKE, FAKE, 0, 2, 100, 4, 128, 1000, FAKE, ws, None]
    def call(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return L.hd_lm_head_ce(*a)
    assert call(a11=ws - 1) == hd.HD_ERR_INVALID_ARG
    assert call(a0=0) == hd.HD_ERR_INVALID_ARG
    assert call(a8=96) == hd.HD_ERR_UNSUPPORTED            # d not a multiple of 64
    assert call(a1=FAKE + 4) == hd.HD_ERR_INVALID_ARG       # misaligned head
    assert call(a9=0) == hd.HD_ERR_INVALID_ARG
    assert L.hd_final_readout(FAKE, FAKE, 1, 4, 2, 6, 2, None) == hd.HD_ERR_UNSUPPORTED
    assert L.hd_final_readout(0, FAKE, 1, 4, 2, 8, 2, None) == hd.HD_ERR_INVALID_ARG


def test_lm_head_bwd_workspace_and_rejects(lib):
    L = hd.lib()
    ws = hd.hd_lm_head_ce_bwd_workspace_bytes(2, 100, 1000)
    assert ws == 200 * 1024 * 2  # B*L rows of G, V rounded up to 256 columns, bf16
    ok = [FAKE, FAKE, FAKE, FAKE, 1.0, FAKE, FAKE, 2, 100, 4, 128, 1000, FAKE, ws, None]
    bad = list(ok); bad[12 + 1] = ws - 1
    assert L.hd_lm_head_ce_bwd(*bad) == hd.HD_ERR_INVALID_ARG
    bad = list(ok); bad[10] = 96
    assert L.hd_lm_head_ce_bwd(*bad) == hd.HD_ERR_UNSUPPORTED
    bad = list(ok); bad[4] = float("nan")
    assert L.hd_lm_head_ce_bwd(*bad) == hd.HD_ERR_INVALID_ARG
    bad = list(ok); bad[3] = 0
    assert L.hd_lm_head_ce_bwd(*bad) == hd.HD_ERR_INVALID_ARG


def test_expand_rejects(lib):
    L = hd.lib()
    assert L.hd_expand_embed(FAKE, FAKE, FAKE, 1, 4, 2, 0, 8, 4, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_expand_embed(FAKE, FAKE, FAKE, 1, 4, 2, 9, 8, 3, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_expand_embed(0, FAKE, FAKE, 1, 4, 2, 9, 8, 4, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_expand_embed(FAKE, FAKE + 1, FAKE, 1, 4, 2, 9, 8, 4, None) == hd.HD_ERR_INVALID_ARG


def test_rope_rejects(lib):
    L = hd.lib()
    ok = [FAKE, FAKE, 0, 2, 8, 4, 8, 2, 128, 0, 10000.0, None]
    def call(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return L.hd_rope_expanded(*a)
    assert call(a0=0, a1=0) == hd.HD_ERR_INVALID_ARG       # nothing to rotate
    assert call(a3=0) == hd.HD_ERR_INVALID_ARG             # B
    assert call(a6=0) == hd.HD_ERR_INVALID_ARG             # Hq with q given
    assert call(a9=2) == hd.HD_ERR_INVALID_ARG             # final flag
    assert call(a10=1.0) == hd.HD_ERR_INVALID_ARG          # base must exceed 1
    assert call(a10=float("inf")) == hd.HD_ERR_INVALID_ARG
    assert call(a0=FAKE + 8) == hd.HD_ERR_INVALID_ARG      # misaligned
    assert call(a8=96) == hd.HD_ERR_UNSUPPORTED
    assert call(a8=512) == hd.HD_ERR_UNSUPPORTED


def test_selftest_rejects_bad_limits(lib):
    L = hd.lib()
    assert L.hd_selftest_wait_timeout(0, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_selftest_wait_timeout((1 << 33) + 1, None) == hd.HD_ERR_INVALID_ARG


def test_python_binding_raises_on_error(lib):
    with pytest.raises(hd.HDError) as e:
        hd.hd_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 4, 4, 2, 96, 0, 1, 0, 0.1, stream=0)
    assert e.value.status == hd.HD_ERR_UNSUPPORTED


def test_tensor_helpers_refuse_cpu_tensors(lib):
    import torch

    q = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hd.attn_fwd(q, q, q, n=2, mode=hd.CROSS_FULL)
