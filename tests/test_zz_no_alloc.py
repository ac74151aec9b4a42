"""hd_decode_attn_noalloc: the decode step without a caller-supplied workspace.

Some callers cannot allocate device memory while they decode (their framework
owns every byte of the GPU through its own pool, or their loop must never enter
cudaMalloc). This entry point keeps its split-K scratch in a fixed array inside
the library. The test calls it through the C ABI twice in a row, on different
inputs, and checks each result against the float64 oracle and against
hd_decode_attn with a caller-allocated workspace. It lives in its own file,
collected last, and passes both alone in a fresh process and after the other
tests.
"""
import ctypes
import math

import pytest
import torch

import oracle
import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import synthetic as syn
from tests.gpu_util import LSE_MAX, O_MAX, O_MEAN, check, host64, need_gpu

pytestmark = pytest.mark.gpu


def _noalloc(inp, out, lse, B, n, Tcap, Hq, Hkv, D, mode, W, scale):
    L = hd.lib()
    return L.hd_decode_attn_noalloc(
        ctypes.c_void_p(inp["q"].data_ptr()), ctypes.c_void_p(inp["k_cache"].data_ptr()),
        ctypes.c_void_p(inp["v_cache"].data_ptr()), ctypes.c_void_p(inp["seqlen"].data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), B, n, Tcap, Hq, Hkv, D,
        mode, W, ctypes.c_float(scale), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("mode", [hd.CROSS_FULL, hd.INTRA, hd.CROSS_WINDOW],
                         ids=["CROSS_FULL", "INTRA", "CROSS_WINDOW"])
def test_noalloc_decode_matches_workspace_decode_twice(mode):
    need_gpu()
    cases = [(4, 4, 700, 760, 16, 4, 128, 33, 1), (3, 3, 150, 160, 6, 2, 64, 7, 2)]
    for (B, n, T, Tcap, Hq, Hkv, D, W, seed) in cases:  # two calls in a row
        host = syn.decode_inputs(B, n, T, Tcap, Hq, Hkv, D, seed=seed, ragged=True)
        inp = {k: v.cuda() for k, v in host.items()}
        scale = 1.0 / math.sqrt(D)
        out = torch.empty_like(inp["q"])
        lse = torch.empty((B, Hq, n), dtype=torch.float32, device="cuda")
        assert _noalloc(inp, out, lse, B, n, Tcap, Hq, Hkv, D, mode, W, scale) == hd.HD_OK
        ref_o, ref_l = hd.decode_attn(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlen"], mode, W,
                                      scale)
        torch.cuda.synchronize()
        assert hd.hd_device_status() == hd.HD_OK
        want_o, want_l = oracle.decode_attn(host["q"], host["k_cache"], host["v_cache"], host["seqlen"], n,
                                            mode, W, scale)
        check(host64(out), want_o, O_MAX, O_MEAN, "O vs oracle")
        check(host64(lse), want_l, LSE_MAX, LSE_MAX, "LSE vs oracle")
        check(host64(out), host64(ref_o), O_MAX, O_MEAN, "O vs hd_decode_attn")
        check(host64(lse), host64(ref_l), LSE_MAX, LSE_MAX, "LSE vs hd_decode_attn")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    need_gpu()
    B, n, Tcap, Hq, Hkv, D = 64, 4, 1000, 64, 64, 128
    assert hd.hd_decode_workspace_bytes(B, n, Tcap, Hq, Hkv, D) > (16 << 20)
    L = hd.lib()
    st = L.hd_decode_attn_noalloc(*([ctypes.c_void_p(0x10000)] * 6), B, n, Tcap, Hq, Hkv, D,
                                  hd.CROSS_FULL, 1, ctypes.c_float(0.1), None)
    assert st == hd.HD_ERR_UNSUPPORTED
