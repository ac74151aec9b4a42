"""The bounds-checked build at the benchmark's full sizes.

libhd_checked.so is the same library compiled with HD_CHECK_BOUNDS: every
computed index of a plain (non-TMA) load or store is tested against its
buffer's size, and one out of range records HD_ERR_DEVICE_INDEX instead of
being performed. Each workload configuration runs here at the size the bench
times, through both builds on the same inputs. The checked build's status word
must stay HD_OK, so no index left its buffer at any of these sizes, and its
outputs must equal the normal build's bit for bit: the checks add branches,
not arithmetic. The one exception is dQ, which many CTAs add into an fp32
accumulator in an order that differs from run to run (even for one build);
after the bf16 rounding two runs differ there by at most one bf16 step.
"""
import ctypes
import math

import pytest
import torch

import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import _lib
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    need_gpu()
    from structured_causal_attention_b200.build import build

    build(checked=True)
    return _lib.lib(), _lib.lib_checked()


def _stream():
    return int(torch.cuda.current_stream().cuda_stream)


def _gen(shape, seed, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn(shape, device="cuda", generator=g).to(dtype)


def _both(libs, fn, summed=()):
    """fn(L) -> tuple of output tensors; run through both builds and compare.

    Outputs whose index is in ``summed`` are sums in a run-dependent order:
    they must agree within one bf16 step (2^-7 of the value, plus 1e-6 for
    values that cancel to near zero); all others bit for bit.
    """
    outs = []
    for L in libs:
        outs.append(fn(L))
        torch.cuda.synchronize()
        st = L.hd_device_status(_stream(), 1)
        assert st == hd.HD_OK, hd.status_string(st)
    for i, (a, b) in enumerate(zip(*outs)):
        if i in summed:
            a32, b32 = a.float(), b.float()
            tol = 2.0 ** -7 * torch.maximum(a32.abs(), b32.abs()) + 1e-6
            assert ((a32 - b32).abs() <= tol).all(), \
                "the checked build changed a summed output by more than one bf16 step"
        else:
            assert torch.equal(a, b), "the checked build changed an output"


ATTN = [  # name, B, L, n, Hq, Hkv, D, mode, W, final_only, backward
    ("intra_train", 4, 2048, 4, 16, 4, 128, hd.INTRA, 0, 0, True),
    ("cross_window", 2, 8192, 4, 32, 8, 128, hd.CROSS_WINDOW, 1024, 0, True),
    ("long_cross_full", 1, 32768, 4, 32, 8, 128, hd.CROSS_FULL, 0, 0, False),
    ("long_cross_final_only", 1, 32768, 4, 32, 8, 128, hd.CROSS_FULL, 0, 1, True),
]


@pytest.mark.parametrize("cfg", ATTN, ids=[c[0] for c in ATTN])
def test_attention_checked_build_full_size(libs, cfg):
    _, B, L, n, Hq, Hkv, D, mode, W, fin, bwd = cfg
    S = n * L
    Sq = L if fin else S
    q, k, v = _gen((B, Sq, Hq, D), 1), _gen((B, S, Hkv, D), 2), _gen((B, S, Hkv, D), 3)
    do = _gen((B, Sq, Hq, D), 4) if bwd else None
    sc = 1.0 / math.sqrt(D)

    def run(Lb):
        out = torch.empty_like(q)
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
        assert Lb.hd_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, L, n,
                              Hq, Hkv, D, mode, W, fin, ctypes.c_float(sc), _stream()) == hd.HD_OK
        if not bwd:
            return out, lse
        wsn = Lb.hd_attn_bwd_workspace_bytes(B, L, n, Hq, Hkv, D, fin)
        ws = torch.empty(wsn, dtype=torch.uint8, device="cuda")
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        assert Lb.hd_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                              do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, L, n, Hq, Hkv, D,
                              mode, W, fin, ctypes.c_float(sc), ws.data_ptr(), wsn, _stream()) == hd.HD_OK
        return out, lse, dq, dk, dv

    _both(libs, run, summed=(2,))


@pytest.mark.parametrize("B", [8, 64])
@pytest.mark.parametrize("mode", [hd.CROSS_FULL, hd.INTRA], ids=["CROSS_FULL", "INTRA"])
def test_decode_checked_build_full_size(libs, B, mode):
    n, T, Hq, Hkv, D = 4, 16384, 32, 8, 128
    Tcap = T + 1
    q = _gen((B, n, Hq, D), 5)
    kc, vc = _gen((B, Tcap * n, Hkv, D), 6), _gen((B, Tcap * n, Hkv, D), 7)
    seqlen = torch.full((B,), Tcap, dtype=torch.int32, device="cuda")
    sc = 1.0 / math.sqrt(D)

    def run(Lb):
        out = torch.empty_like(q)
        lse = torch.empty((B, Hq, n), dtype=torch.float32, device="cuda")
        wsn = Lb.hd_decode_workspace_bytes(B, n, Tcap, Hq, Hkv, D)
        ws = torch.empty(wsn, dtype=torch.uint8, device="cuda")
        assert Lb.hd_decode_attn(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), seqlen.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), B, n, Tcap, Hq, Hkv, D, mode, 1024, ctypes.c_float(sc),
                                 ws.data_ptr(), wsn, _stream()) == hd.HD_OK
        return out, lse

    _both(libs, run)


def test_expand_checked_build_full_size(libs):
    B, L, n, V, d = 4, 8192, 4, 32000, 4096
    g = torch.Generator(device="cuda")
    g.manual_seed(8)
    ids = torch.randint(0, V, (B, L), device="cuda", generator=g, dtype=torch.int64).to(torch.int32)
    tables = torch.empty((n, V, d), device="cuda").normal_(0, 0.02, generator=g)

    def run(Lb):
        out = torch.empty((B, L * n, d), device="cuda")
        assert Lb.hd_expand_embed(ids.data_ptr(), tables.data_ptr(), out.data_ptr(), B, L, n, V, d, 4,
                                  _stream()) == hd.HD_OK
        return (out,)

    _both(libs, run)
