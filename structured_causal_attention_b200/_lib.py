"""ctypes binding to libhd.so: the C ABI of include/hd.h, argument marshalling only.

The functions here carry the C names and take device pointers as Python ints
(or torch tensors, whose ``data_ptr()`` is passed). Every computation happens in
the CUDA kernels behind the C ABI; there is no fallback of any kind: if the
library is missing or does not load, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhd.so")
# the same library built with HD_CHECK_BOUNDS (bounds-checked kernels), for tests
LIB_CHECKED_PATH = os.path.join(HERE, "libhd_checked.so")

HD_OK = 0
HD_ERR_INVALID_ARG = 1
HD_ERR_UNSUPPORTED = 2
HD_ERR_CUDA = 3
HD_ERR_TIMEOUT = 4
HD_ERR_DEVICE_INDEX = 5

# every symbol include/hd.h declares, with (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t
_D = ctypes.c_double
SIGNATURES = {
    "hd_status_string": (ctypes.c_char_p, [_I]),
    "hd_version": (_I, []),
    "hd_build_flags": (_I, []),
    "hd_expand_embed": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "hd_rope_expanded": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _D, _P]),
    "hd_final_readout": (_I, [_P, _P, _I, _I, _I, _I, _I, _P]),
    "hd_lm_head_ce_workspace_bytes": (_Z, [_I, _I, _I]),
    "hd_lm_head_ce": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "hd_lm_head_ce_bwd_workspace_bytes": (_Z, [_I, _I, _I]),
    "hd_lm_head_ce_bwd": (_I, [_P, _P, _P, _P, _F, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "hd_attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "hd_attn_bwd_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "hd_attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                         _F, _P, _Z, _P]),
    "hd_decode_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _I]),
    "hd_decode_attn": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _Z,
                            _P]),
    "hd_decode_final_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _I]),
    "hd_decode_attn_final": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                                  _Z, _P]),
    "hd_decode_attn_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                                    _P]),
    "hd_selftest_wait_timeout": (_I, [ctypes.c_longlong, _P]),
    "hd_device_status": (_I, [_P, _I]),
}

_lib = None
_lib_checked = None


class HDError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def _load(path):
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m structured_causal_attention_b200.build`")
    handle = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    return handle


def lib():
    """Load libhd.so once; raise if it is absent (no fallback exists)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


def lib_checked():
    """Load the checked build, libhd_checked.so (same ABI, bounds-checked kernels)."""
    global _lib_checked
    if _lib_checked is None:
        _lib_checked = _load(LIB_CHECKED_PATH)
    return _lib_checked


def status_string(status: int) -> str:
    return lib().hd_status_string(int(status)).decode()


def ptr(x) -> int:
    """Device pointer of a tensor (or an int passed through); None -> 0."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def stream_handle(stream) -> int:
    if stream is None:
        import torch

        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check(st: int, what: str) -> int:
    if st != HD_OK:
        raise HDError(st, what)
    return st


def hd_expand_embed(ids, tables, out, B, L, n, V, d, elem_bytes, stream=None):
    return _check(lib().hd_expand_embed(ptr(ids), ptr(tables), ptr(out), B, L, n, V, d, elem_bytes,
                                        stream_handle(stream)), "hd_expand_embed")


def hd_rope_expanded(q, k, token_offset, B, L, n, Hq, Hkv, D, final_only, base, stream=None):
    return _check(lib().hd_rope_expanded(ptr(q), ptr(k), ptr(token_offset), B, L, n, Hq, Hkv, D,
                                         int(final_only), float(base), stream_handle(stream)),
                  "hd_rope_expanded")


def hd_final_readout(x, out, B, L, n, d, elem_bytes, stream=None):
    return _check(lib().hd_final_readout(ptr(x), ptr(out), B, L, n, d, elem_bytes,
                                         stream_handle(stream)), "hd_final_readout")


def hd_lm_head_ce_workspace_bytes(B, L, V):
    return int(lib().hd_lm_head_ce_workspace_bytes(B, L, V))


def hd_lm_head_ce(x, w, labels, loss, lse, B, L, n, d, V, workspace, workspace_bytes, stream=None):
    return _check(lib().hd_lm_head_ce(ptr(x), ptr(w), ptr(labels), ptr(loss), ptr(lse), B, L, n, d,
                                      V, ptr(workspace), workspace_bytes, stream_handle(stream)),
                  "hd_lm_head_ce")


def hd_lm_head_ce_bwd_workspace_bytes(B, L, V):
    return int(lib().hd_lm_head_ce_bwd_workspace_bytes(B, L, V))


def hd_lm_head_ce_bwd(x, w, labels, lse, grad_scale, dh, dw, B, L, n, d, V, workspace, workspace_bytes,
                      stream=None):
    return _check(lib().hd_lm_head_ce_bwd(ptr(x), ptr(w), ptr(labels), ptr(lse), float(grad_scale), ptr(dh),
                                          ptr(dw), B, L, n, d, V, ptr(workspace), workspace_bytes,
                                          stream_handle(stream)), "hd_lm_head_ce_bwd")


def hd_attn_fwd(q, k, v, out, lse, B, L, n, Hq, Hkv, D, mode, W_tokens, final_only, scale,
                stream=None):
    return _check(lib().hd_attn_fwd(ptr(q), ptr(k), ptr(v), ptr(out), ptr(lse), B, L, n, Hq, Hkv, D,
                                    mode, W_tokens, int(final_only), float(scale),
                                    stream_handle(stream)), "hd_attn_fwd")


def hd_attn_bwd_workspace_bytes(B, L, n, Hq, Hkv, D, final_only):
    return int(lib().hd_attn_bwd_workspace_bytes(B, L, n, Hq, Hkv, D, int(final_only)))


def hd_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, L, n, Hq, Hkv, D, mode, W_tokens,
                final_only, scale, workspace, workspace_bytes, stream=None):
    return _check(lib().hd_attn_bwd(ptr(q), ptr(k), ptr(v), ptr(out), ptr(lse), ptr(dout), ptr(dq),
                                    ptr(dk), ptr(dv), B, L, n, Hq, Hkv, D, mode, W_tokens,
                                    int(final_only), float(scale), ptr(workspace),
                                    int(workspace_bytes), stream_handle(stream)), "hd_attn_bwd")


def hd_decode_workspace_bytes(B, n, Tcap, Hq, Hkv, D):
    return int(lib().hd_decode_workspace_bytes(B, n, Tcap, Hq, Hkv, D))


def hd_decode_attn(q, k_cache, v_cache, seqlen, out, lse, B, n, Tcap, Hq, Hkv, D, mode, W_tokens,
                   scale, workspace, workspace_bytes, stream=None):
    return _check(lib().hd_decode_attn(ptr(q), ptr(k_cache), ptr(v_cache), ptr(seqlen), ptr(out),
                                       ptr(lse), B, n, Tcap, Hq, Hkv, D, mode, W_tokens, float(scale),
                                       ptr(workspace), int(workspace_bytes), stream_handle(stream)),
                  "hd_decode_attn")


def hd_decode_final_workspace_bytes(B, n, Tcap, Hq, Hkv, D):
    return int(lib().hd_decode_final_workspace_bytes(B, n, Tcap, Hq, Hkv, D))


def hd_decode_attn_final(q, k_cache, v_cache, seqlen, out, lse, B, n, Tcap, Hq, Hkv, D, mode,
                         W_tokens, scale, workspace, workspace_bytes, stream=None):
    return _check(lib().hd_decode_attn_final(ptr(q), ptr(k_cache), ptr(v_cache), ptr(seqlen),
                                             ptr(out), ptr(lse), B, n, Tcap, Hq, Hkv, D, mode,
                                             W_tokens, scale, ptr(workspace), workspace_bytes,
                                             stream_handle(stream)),
                  "hd_decode_attn_final")


def hd_decode_attn_noalloc(q, k_cache, v_cache, seqlen, out, lse, B, n, Tcap, Hq, Hkv, D, mode,
                           W_tokens, scale, stream=None):
    """hd_decode_attn with the library's fixed scratch array (no workspace argument)."""
    return _check(lib().hd_decode_attn_noalloc(ptr(q), ptr(k_cache), ptr(v_cache), ptr(seqlen),
                                               ptr(out), ptr(lse), B, n, Tcap, Hq, Hkv, D, mode,
                                               W_tokens, float(scale), stream_handle(stream)),
                  "hd_decode_attn_noalloc")


def hd_selftest_wait_timeout(limit_cycles, stream=None):
    return _check(lib().hd_selftest_wait_timeout(int(limit_cycles), stream_handle(stream)),
                  "hd_selftest_wait_timeout")


def hd_device_status(stream=None, clear=True):
    return int(lib().hd_device_status(stream_handle(stream), int(clear)))
