"""Out-of-bounds write evidence without a sanitizer: guard bands and the checked build.

Every output and workspace buffer of a call is carved out of a larger device
allocation whose two ends (guard bands of 4 KiB) hold a byte pattern; after the
call both bands must be unchanged, so no kernel wrote before or after its
buffer, and every input must be unchanged too. The sizes are odd on purpose:
L not a multiple of 64 or 128, n in {1, 3, 8}, ragged decode lengths, a
vocabulary that leaves padding columns.

Each case runs through both libraries: libhd.so, and libhd_checked.so, the same
sources built with HD_CHECK_BOUNDS, whose kernels test every computed index of a
plain (non-TMA) load or store against the size of its buffer, record
HD_ERR_DEVICE_INDEX and skip the access instead of trapping. The device status
word of each library must stay HD_OK. The outputs are compared with the float64
oracle as well, so every element the call owns was written.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import _lib
from structured_causal_attention_b200 import synthetic as syn
from tests.gpu_util import G_MAX, G_MEAN, LSE_MAX, O_MAX, O_MEAN, check, host64, need_gpu

pytestmark = pytest.mark.gpu

GUARD = 4096        # bytes of pattern before and after every guarded buffer
PATTERN = 0xA5


def _libs():
    need_gpu()
    from structured_causal_attention_b200.build import build

    build(checked=True)
    return {"libhd": _lib.lib(), "libhd_checked": _lib.lib_checked()}


@pytest.fixture(scope="module")
def libs():
    return _libs()


class Guarded:
    """Device buffers carved out of allocations with patterned guard bands."""

    def __init__(self):
        self.raw = []

    def empty(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((2 * GUARD + nbytes,), PATTERN, dtype=torch.uint8, device="cuda")
        self.raw.append((raw, nbytes))
        return raw[GUARD:GUARD + nbytes].view(dtype).view(*shape)

    def like(self, t):
        g = self.empty(tuple(t.shape), t.dtype)
        g.copy_(t)
        return g

    def check_bands(self):
        torch.cuda.synchronize()
        for raw, nbytes in self.raw:
            head, tail = raw[:GUARD], raw[GUARD + nbytes:]
            assert bool((head == PATTERN).all()), "a kernel wrote before the start of its buffer"
            assert bool((tail == PATTERN).all()), "a kernel wrote past the end of its buffer"


def _run(L, name, *args):
    conv = [int(a.data_ptr()) if torch.is_tensor(a) else a for a in args]
    st = getattr(L, name)(*conv, int(torch.cuda.current_stream().cuda_stream))
    assert st == hd.HD_OK, (name, hd.status_string(st))


def _status_ok(L):
    st = L.hd_device_status(int(torch.cuda.current_stream().cuda_stream), 1)
    assert st == hd.HD_OK, hd.status_string(st)


def _unchanged(pairs):
    for dev_t, host_t in pairs:
        assert torch.equal(dev_t.cpu(), host_t), "an input buffer was modified"


def test_build_flags(libs):
    assert libs["libhd"].hd_build_flags() == 0
    assert libs["libhd_checked"].hd_build_flags() == 1  # HD_BUILD_CHECK_BOUNDS


@pytest.mark.parametrize("which", ["libhd", "libhd_checked"])
@pytest.mark.parametrize("case", [(2, 37, 3, 50, 40, torch.float32), (1, 21, 8, 30, 19, torch.bfloat16),
                                  (3, 5, 1, 7, 24, torch.float16)], ids=["fp32_d40", "bf16_d19", "fp16_n1"])
def test_expand_guarded(libs, which, case):
    L = libs[which]
    B, Lt, n, V, d, dt = case
    e = syn.expand_inputs(B, Lt, n, V, d, seed=B + Lt, dtype=dt)
    g = Guarded()
    ids, tables = g.like(e["ids"].cuda()), g.like(e["tables"].cuda())
    out = g.empty((B, Lt * n, d), dt)
    _run(L, "hd_expand_embed", ids, tables, out, B, Lt, n, V, d, tables.element_size())
    g.check_bands()
    _status_ok(L)
    _unchanged([(ids, e["ids"]), (tables, e["tables"])])
    want = oracle.expand_embed(e["ids"].numpy(), e["tables"].float().numpy())
    assert np.array_equal(out.float().cpu().numpy(), want)


@pytest.mark.parametrize("which", ["libhd", "libhd_checked"])
def test_final_readout_guarded(libs, which):
    L = libs[which]
    B, Lt, n, d = 2, 37, 3, 72
    x_h = syn.normal_bf16((B, n * Lt, d), 31)
    g = Guarded()
    x = g.like(x_h.cuda())
    out = g.empty((B, Lt, d), torch.bfloat16)
    _run(L, "hd_final_readout", x, out, B, Lt, n, d, 2)
    g.check_bands()
    _status_ok(L)
    _unchanged([(x, x_h)])
    assert torch.equal(out.cpu(), oracle.final_readout(x_h, n).contiguous())


ATTN = [  # B, L, n, Hq, Hkv, D, W
    (1, 37, 3, 4, 2, 64, 5),
    (2, 75, 8, 2, 1, 128, 3),
    (1, 131, 1, 2, 2, 64, 40),
    (1, 150, 3, 6, 2, 128, 17),
]


@pytest.mark.parametrize("which", ["libhd", "libhd_checked"])
@pytest.mark.parametrize("shape", ATTN, ids=[str(s) for s in ATTN])
@pytest.mark.parametrize("mode", [hd.INTRA, hd.CROSS_FULL, hd.CROSS_WINDOW], ids=["INTRA", "CROSS_FULL", "CROSS_WINDOW"])
@pytest.mark.parametrize("fin", [0, 1], ids=["all", "final"])
def test_attention_guarded(libs, which, shape, mode, fin):
    L = libs[which]
    B, Lt, n, Hq, Hkv, D, W = shape
    S = n * Lt
    Sq = Lt if fin else S
    scale = 1.0 / math.sqrt(D)
    a = syn.attention_inputs(B, Lt, n, Hq, Hkv, D, final_only=bool(fin), seed=Lt + n + D, with_grad=True)
    g = Guarded()
    q, k, v, do = (g.like(a[t].cuda()) for t in ("q", "k", "v", "do"))
    out = g.empty((B, Sq, Hq, D), torch.bfloat16)
    lse = g.empty((B, Hq, Sq), torch.float32)
    _run(L, "hd_attn_fwd", q, k, v, out, lse, B, Lt, n, Hq, Hkv, D, mode, W, fin, scale)
    ws_n = L.hd_attn_bwd_workspace_bytes(B, Lt, n, Hq, Hkv, D, fin)
    ws = g.empty((ws_n,), torch.uint8)
    dq = g.empty((B, Sq, Hq, D), torch.bfloat16)
    dk = g.empty((B, S, Hkv, D), torch.bfloat16)
    dv = g.empty((B, S, Hkv, D), torch.bfloat16)
    _run(L, "hd_attn_bwd", q, k, v, out, lse, do, dq, dk, dv, B, Lt, n, Hq, Hkv, D, mode, W, fin, scale, ws,
         ws_n)
    g.check_bands()
    _status_ok(L)
    _unchanged([(q, a["q"]), (k, a["k"]), (v, a["v"]), (do, a["do"])])
    ro, rl = oracle.attn_fwd(a["q"], a["k"], a["v"], n, mode, W, bool(fin), scale)
    check(host64(out), ro, O_MAX, O_MEAN, "O")
    check(host64(lse), rl, LSE_MAX, LSE_MAX, "LSE")
    rq, rk, rv = oracle.attn_bwd(a["q"], a["k"], a["v"], a["do"], n, mode, W, bool(fin), scale)
    check(host64(dq), rq, G_MAX, G_MEAN, "dQ")
    check(host64(dk), rk, G_MAX, G_MEAN, "dK")
    check(host64(dv), rv, G_MAX, G_MEAN, "dV")


@pytest.mark.parametrize("which", ["libhd", "libhd_checked"])
@pytest.mark.parametrize("mode", [hd.INTRA, hd.CROSS_FULL, hd.CROSS_WINDOW], ids=["INTRA", "CROSS_FULL", "CROSS_WINDOW"])
@pytest.mark.parametrize("final", [False, True], ids=["streams", "final"])
def test_decode_guarded(libs, which, mode, final):
    L = libs[which]
    B, n, T, Tcap, Hq, Hkv, D, W = 3, 3, 41, 45, 6, 2, 64, 4
    scale = 1.0 / math.sqrt(D)
    dd = syn.decode_inputs(B, n, T, Tcap, Hq, Hkv, D, seed=11, ragged=True)
    qh = dd["q"][:, n - 1:n].contiguous() if final else dd["q"]
    nq = qh.shape[1]
    g = Guarded()
    q, kc, vc, sl = g.like(qh.cuda()), g.like(dd["k_cache"].cuda()), g.like(dd["v_cache"].cuda()), \
        g.like(dd["seqlen"].cuda())
    out = g.empty((B, nq, Hq, D), torch.bfloat16)
    lse = g.empty((B, Hq, nq), torch.float32)
    if final:
        ws_n = L.hd_decode_final_workspace_bytes(B, n, Tcap, Hq, Hkv, D)
        ws = g.empty((ws_n,), torch.uint8)
        _run(L, "hd_decode_attn_final", q, kc, vc, sl, out, lse, B, n, Tcap, Hq, Hkv, D, mode, W, scale, ws,
             ws_n)
    else:
        ws_n = L.hd_decode_workspace_bytes(B, n, Tcap, Hq, Hkv, D)
        ws = g.empty((ws_n,), torch.uint8)
        _run(L, "hd_decode_attn", q, kc, vc, sl, out, lse, B, n, Tcap, Hq, Hkv, D, mode, W, scale, ws, ws_n)
    g.check_bands()
    _status_ok(L)
    _unchanged([(q, qh), (kc, dd["k_cache"]), (vc, dd["v_cache"]), (sl, dd["seqlen"])])
    ro, rl = oracle.decode_attn(qh, dd["k_cache"], dd["v_cache"], dd["seqlen"], n, mode, W, scale,
                                final_only=final)
    check(host64(out), ro, O_MAX, O_MEAN, "decode O")
    check(host64(lse), rl, LSE_MAX, LSE_MAX, "decode LSE")


@pytest.mark.parametrize("which", ["libhd", "libhd_checked"])
@pytest.mark.parametrize("fin", [0, 1], ids=["all", "final"])
def test_rope_guarded(libs, which, fin):
    L = libs[which]
    B, Lt, n, Hq, Hkv, D = 2, 37, 3, 5, 3, 64
    Sq = Lt if fin else n * Lt
    qh, kh = syn.normal_bf16((B, Sq, Hq, D), 41), syn.normal_bf16((B, n * Lt, Hkv, D), 42)
    off_h = torch.tensor([0, 9], dtype=torch.int32)
    g = Guarded()
    q, k, off = g.like(qh.cuda()), g.like(kh.cuda()), g.like(off_h.cuda())
    _run(L, "hd_rope_expanded", q, k, off, B, Lt, n, Hq, Hkv, D, fin, 10000.0)
    g.check_bands()
    _status_ok(L)
    _unchanged([(off, off_h)])
    wq, wk = oracle.rope_expanded(qh, kh, n, bool(fin), 10000.0, token_offset=off_h.numpy())
    tol = 2.0 ** -8
    for got, want in ((q, wq), (k, wk)):
        err = np.abs(host64(got) - want)
        assert (err <= tol * np.abs(want) + 1e-5).all(), float(err.max())


@pytest.mark.parametrize("which", ["libhd", "libhd_checked"])
def test_lm_head_guarded(libs, which):
    L = libs[which]
    B, Lt, n, d, V = 2, 37, 3, 128, 300
    li = syn.lm_head_inputs(B, Lt, n, d, V, seed=51, ignore_every=7)
    g = Guarded()
    x, w, lab = g.like(li["x"].cuda()), g.like(li["w"].cuda()), g.like(li["labels"].cuda())
    loss = g.empty((B, Lt), torch.float32)
    lse = g.empty((B, Lt), torch.float32)
    ws_n = L.hd_lm_head_ce_workspace_bytes(B, Lt, V)
    ws = g.empty((ws_n,), torch.uint8)
    _run(L, "hd_lm_head_ce", x, w, lab, loss, lse, B, Lt, n, d, V, ws, ws_n)
    dh = g.empty((B, Lt, d), torch.bfloat16)
    dw = g.empty((V, d), torch.float32)
    wsb_n = L.hd_lm_head_ce_bwd_workspace_bytes(B, Lt, V)
    wsb = g.empty((wsb_n,), torch.uint8)
    import ctypes

    _run(L, "hd_lm_head_ce_bwd", x, w, lab, lse, ctypes.c_float(1.0), dh, dw, B, Lt, n, d, V, wsb, wsb_n)
    g.check_bands()
    _status_ok(L)
    _unchanged([(x, li["x"]), (w, li["w"]), (lab, li["labels"])])
    wl, wsl = oracle.lm_head_ce(li["x"], li["w"], li["labels"], n)
    check(host64(loss), wl, 2e-3, 2e-3, "loss")
    check(host64(lse), wsl, 2e-3, 2e-3, "lse")
    _, dh_ref, dw_ref = oracle.lm_head_ce_grad(li["x"], li["w"], li["labels"], n)
    for got, want, what in ((dh, dh_ref, "dh"), (dw, dw_ref, "dW")):
        sc = float(np.abs(want).max())
        err = np.abs(host64(got) - want)
        assert err.max() <= 2e-2 * sc and err.mean() <= 2e-3 * sc, (what, err.max(), sc)
