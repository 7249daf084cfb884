"""ctypes binding of libdl.so (C ABI declared in include/dl.h).

Argument marshalling only: each function passes device pointers, sizes and the
CUDA stream handle straight to the C entry point of the same name and returns
its ``dl_status`` code.  There is no fallback: if ``libdl.so`` is missing the
first call raises.

Tensor arguments may be torch tensors (their ``data_ptr()`` is passed), plain
integers (raw addresses) or ``None`` (a null pointer).  ``stream`` defaults to
torch's current CUDA stream.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdl.so")

DL_OK = 0
DL_ERR_INVALID_ARG = 1
DL_ERR_UNSUPPORTED = 2
DL_ERR_ALIGNMENT = 3
DL_ERR_WORKSPACE = 4
DL_ERR_CUDA = 5
DL_ERR_TIMEOUT = 6
DL_ERR_DEVICE_ARG = 7

DL_FLAG_PDL = 1
DL_FLAG_DEBUG_TIMEOUT = 2
DL_FLAG_XQ_READY = 4
DL_FLAG_COPY_NO_WAIT = 16
DL_FLAG_SPLIT_SHIFT = 8
DL_PACK_PLAIN = 0
DL_PACK_SWIGLU = 1

_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_U = ctypes.c_uint
_LL = ctypes.c_longlong
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "dl_pack_fp8_weight": (_I, [_P, _P, _I, _I, _I, _P]),
    "dl_workspace_bytes": (_SZ, [_I, _I]),
    "dl_fc13_swiglu": (_I, [_P, _I, _I, _P, _P, _I, _P, _P, _SZ, _P, _U]),
    "dl_fc13_swiglu_static_ws": (_I, [_P, _I, _I, _P, _P, _I, _P, _P, _P, _U]),
    "dl_fc_qkv_scale": (_I, [_P, _I, _I, _P, _P, _I, _I, _I, _F, _P, _P, _SZ, _P, _U]),
    "dl_moe_fc13_swiglu_grouped": (_I, [_P, _I, _I, _P, _I, _P, _P, _I, _P, _P, _SZ, _P, _U]),
    "dl_gemm_e4m3": (_I, [_P, _I, _I, _P, _P, _I, _P, _P, _SZ, _P, _U]),
    "dl_moe_gemm_grouped": (_I, [_P, _I, _I, _P, _I, _P, _P, _I, _P, _P, _SZ, _P, _U]),
    "dl_add_rmsnorm_quant": (_I, [_P, _P, _P, _P, _I, _I, _F, _P, _SZ, _P, _U]),
    "dl_rmsnorm_fc_qkv_scale": (_I, [_P, _P, _P, _P, _F, _I, _I, _P, _P, _I, _I, _I, _F, _P, _P, _SZ, _P, _U]),
    "dl_rmsnorm_fc13_swiglu": (_I, [_P, _P, _P, _P, _F, _I, _I, _P, _P, _I, _P, _P, _SZ, _P, _U]),
    "dl_spec_verify_greedy": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _U]),
    "dl_decode_attn": (_I, [_P, _LL, _I, _I, _I, _I, _I, _P, _P, _I, _P, _F, _I, _P, _P, _SZ, _P, _U]),
    "dl_decode_attn_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "dl_decode_attn_fp8kv": (_I, [_P, _LL, _I, _I, _I, _I, _I, _P, _P, _P, _I, _P, _F, _I, _P, _P, _SZ, _P, _U]),
    "dl_decode_attn_fp8kv_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "dl_copy": (_I, [_P, _P, _SZ, _P, _U]),
    "dl_read_status": (_I, [_P, _P]),
    "dl_status_string": (ctypes.c_char_p, [_I]),
}


class DLError(RuntimeError):
    pass


def lib():
    """Load libdl.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m latency_decode_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(ws, ws_bytes):
    if ws_bytes is not None:
        return int(ws_bytes)
    return ws.numel() * ws.element_size() if ws is not None and not isinstance(ws, int) else 0


def dl_status_string(status: int) -> str:
    return lib().dl_status_string(int(status)).decode()


def check(status: int) -> None:
    if status != DL_OK:
        raise DLError(dl_status_string(status))


def dl_workspace_bytes(M: int, K: int) -> int:
    return int(lib().dl_workspace_bytes(M, K))


def dl_pack_fp8_weight(w_nk, w_packed, N, K, kind, stream=None) -> int:
    return lib().dl_pack_fp8_weight(_ptr(w_nk), _ptr(w_packed), N, K, kind, _stream(stream))


def dl_fc13_swiglu(x, M, K, w_packed, w_scale, N2, out, ws, ws_bytes=None, stream=None,
                   flags=DL_FLAG_PDL) -> int:
    return lib().dl_fc13_swiglu(_ptr(x), M, K, _ptr(w_packed), _ptr(w_scale), N2, _ptr(out), _ptr(ws),
                                _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_fc13_swiglu_static_ws(x, M, K, w_packed, w_scale, N2, out, status=None, stream=None,
                             flags=DL_FLAG_PDL) -> int:
    return lib().dl_fc13_swiglu_static_ws(_ptr(x), M, K, _ptr(w_packed), _ptr(w_scale), N2, _ptr(out),
                                          _ptr(status), _stream(stream), flags)


def dl_fc_qkv_scale(x, M, K, w_packed, w_scale, Hq, Hkv, d, q_scale, qkv, ws, ws_bytes=None,
                    stream=None, flags=DL_FLAG_PDL) -> int:
    return lib().dl_fc_qkv_scale(_ptr(x), M, K, _ptr(w_packed), _ptr(w_scale), Hq, Hkv, d, float(q_scale),
                                 _ptr(qkv), _ptr(ws), _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_moe_fc13_swiglu_grouped(x, T, K, expert_ids, E, w_packed, w_scales, N2, out, ws, ws_bytes=None,
                               stream=None, flags=DL_FLAG_PDL) -> int:
    return lib().dl_moe_fc13_swiglu_grouped(_ptr(x), T, K, _ptr(expert_ids), E, _ptr(w_packed),
                                            _ptr(w_scales), N2, _ptr(out), _ptr(ws), _nbytes(ws, ws_bytes),
                                            _stream(stream), flags)


def dl_gemm_e4m3(x, M, K, w_packed, w_scale, N, out, ws, ws_bytes=None, stream=None, flags=DL_FLAG_PDL) -> int:
    return lib().dl_gemm_e4m3(_ptr(x), M, K, _ptr(w_packed), _ptr(w_scale), N, _ptr(out), _ptr(ws),
                              _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_moe_gemm_grouped(x, T, K, expert_ids, E, w_packed, w_scales, N, out, ws, ws_bytes=None, stream=None,
                        flags=DL_FLAG_PDL) -> int:
    return lib().dl_moe_gemm_grouped(_ptr(x), T, K, _ptr(expert_ids), E, _ptr(w_packed), _ptr(w_scales), N,
                                     _ptr(out), _ptr(ws), _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_add_rmsnorm_quant(x, residual, h_out, gamma, M, K, eps, ws, ws_bytes=None, stream=None,
                         flags=DL_FLAG_PDL) -> int:
    return lib().dl_add_rmsnorm_quant(_ptr(x), _ptr(residual), _ptr(h_out), _ptr(gamma), M, K, float(eps),
                                      _ptr(ws), _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_spec_verify_greedy(logits, B, T, V, draft_ids, target_ids, n_accepted, emitted, seq_lens=None, stream=None,
                          flags=DL_FLAG_PDL) -> int:
    return lib().dl_spec_verify_greedy(_ptr(logits), B, T, V, _ptr(draft_ids), _ptr(target_ids), _ptr(n_accepted),
                                       _ptr(emitted), _ptr(seq_lens), _stream(stream), flags)


def dl_rmsnorm_fc_qkv_scale(x, residual, h_out, gamma, eps, M, K, w_packed, w_scale, Hq, Hkv, d, q_scale, qkv, ws,
                            ws_bytes=None, stream=None, flags=DL_FLAG_PDL) -> int:
    return lib().dl_rmsnorm_fc_qkv_scale(_ptr(x), _ptr(residual), _ptr(h_out), _ptr(gamma), float(eps), M, K,
                                         _ptr(w_packed), _ptr(w_scale), Hq, Hkv, d, float(q_scale), _ptr(qkv),
                                         _ptr(ws), _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_rmsnorm_fc13_swiglu(x, residual, h_out, gamma, eps, M, K, w_packed, w_scale, N2, out, ws, ws_bytes=None,
                           stream=None, flags=DL_FLAG_PDL) -> int:
    return lib().dl_rmsnorm_fc13_swiglu(_ptr(x), _ptr(residual), _ptr(h_out), _ptr(gamma), float(eps), M, K,
                                        _ptr(w_packed), _ptr(w_scale), N2, _ptr(out), _ptr(ws),
                                        _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_decode_attn(q, q_token_stride, B, T, Hq, Hkv, d, k_cache, v_cache, Lcap, seq_lens, softmax_scale,
                   cluster_size, out, ws, ws_bytes=None, stream=None, flags=DL_FLAG_PDL) -> int:
    return lib().dl_decode_attn(_ptr(q), int(q_token_stride), B, T, Hq, Hkv, d, _ptr(k_cache), _ptr(v_cache),
                                Lcap, _ptr(seq_lens), float(softmax_scale), cluster_size, _ptr(out), _ptr(ws),
                                _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_decode_attn_fp8kv(q, q_token_stride, B, T, Hq, Hkv, d, k_cache, vt_cache, kv_scale, Lcap, seq_lens,
                         softmax_scale, cluster_size, out, ws, ws_bytes=None, stream=None, flags=DL_FLAG_PDL) -> int:
    return lib().dl_decode_attn_fp8kv(_ptr(q), int(q_token_stride), B, T, Hq, Hkv, d, _ptr(k_cache), _ptr(vt_cache),
                                      _ptr(kv_scale), Lcap, _ptr(seq_lens), float(softmax_scale), cluster_size,
                                      _ptr(out), _ptr(ws), _nbytes(ws, ws_bytes), _stream(stream), flags)


def dl_decode_attn_fp8kv_workspace_bytes(B, T, Hq, Hkv, d, Lcap, cluster_size) -> int:
    return int(lib().dl_decode_attn_fp8kv_workspace_bytes(B, T, Hq, Hkv, d, Lcap, cluster_size))


def dl_decode_attn_workspace_bytes(B, T, Hq, Hkv, d, Lcap, cluster_size) -> int:
    return int(lib().dl_decode_attn_workspace_bytes(B, T, Hq, Hkv, d, Lcap, cluster_size))


def dl_copy(src, dst, nbytes, stream=None, flags=DL_FLAG_PDL) -> int:
    return lib().dl_copy(_ptr(src), _ptr(dst), int(nbytes), _stream(stream), flags)


def dl_read_status(ws, stream=None) -> int:
    return lib().dl_read_status(_ptr(ws), _stream(stream))
