"""Python binding of the CPU oracle (``oracle/oracle.cpp``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``latency_decode_b200``) never imports it and never falls back to it.

Every function takes numpy arrays holding the raw input bytes (bf16 as
``uint16``, e4m3 as ``uint8``, weights in nn.Linear ``[N, K]`` order) and returns
float64 results.  The arithmetic lives in the C++ file; this module only
marshals arguments.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "oracle.cpp")
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_LL = ctypes.c_longlong


def build(force: bool = False) -> str:
    """Compile ``oracle.cpp`` into ``liboracle.so`` next to it (plain g++)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h"))
    ):
        cmd = [
            "g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
            "-Wall", "-Wextra", "-o", _SO, _SRC,
        ]
        subprocess.run(cmd, check=True)
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        sig = {
            "oracle_bf16_to_f64": (ctypes.c_double, [ctypes.c_uint16]),
            "oracle_f64_to_bf16": (ctypes.c_uint16, [ctypes.c_double]),
            "oracle_e4m3_to_f64": (ctypes.c_double, [ctypes.c_uint8]),
            "oracle_f32_to_e4m3": (ctypes.c_uint8, [ctypes.c_float]),
            "oracle_act_quant": (None, [_P, _I, _I, _P, _P]),
            "oracle_gemm_q": (None, [_P, _F, _P, _F, _I, _I, _I, _P]),
            "oracle_fc13_swiglu_q": (None, [_P, _F, _P, _F, _I, _I, _I, _P]),
            "oracle_fc13_swiglu": (None, [_P, _I, _I, _P, _F, _I, _P]),
            "oracle_fc_qkv_scale_q": (None, [_P, _F, _P, _F, _I, _I, _I, _I, _I, _F, _P]),
            "oracle_fc_qkv_scale": (None, [_P, _I, _I, _P, _F, _I, _I, _I, _F, _P]),
            "oracle_moe_fc13_swiglu": (None, [_P, _I, _I, _P, _I, _P, _P, _I, _P]),
            "oracle_linear": (None, [_P, _I, _I, _P, _F, _I, _P]),
            "oracle_moe_linear": (None, [_P, _I, _I, _P, _I, _P, _P, _I, _P]),
            "oracle_add_rmsnorm": (None, [_P, _P, _P, _I, _I, _F, _P, _P]),
            "oracle_quant_f32": (None, [_P, _LL, _P, _P]),
            "oracle_spec_verify_greedy": (None, [_P, _I, _I, _I, _P, _P, _P, _P]),
            "oracle_decode_attn_fp8kv": (None, [_P, _LL, _I, _I, _I, _I, _I, _P, _P, _I, _P, _F, _F, _F, _P]),
            "oracle_decode_attn": (None, [_P, _LL, _I, _I, _I, _I, _I, _P, _P, _I, _P, _F, _P]),
            "oracle_attn_partial": (None, [_P, _LL, _I, _I, _I, _I, _P, _P, _I, _I, _I, _I, _I,
                                           _F, _I, _I, _P, _P, _P]),
            "oracle_lse_combine": (None, [_I, _P, _P, _P, _I, _P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- number formats --------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    lib = _load()
    b = _c(bits, np.uint16).ravel()
    return np.array([lib.oracle_bf16_to_f64(int(v)) for v in b]).reshape(np.shape(bits))


def bf16_array_to_f64(bits: np.ndarray) -> np.ndarray:
    """Vectorised bf16 decode (the top half of a float32; format definition)."""
    b = _c(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(v) -> np.ndarray:
    lib = _load()
    arr = np.asarray(v, dtype=np.float64)
    out = np.array([lib.oracle_f64_to_bf16(float(x)) for x in arr.ravel()], dtype=np.uint16)
    return out.reshape(arr.shape)


def e4m3_to_f64(codes) -> np.ndarray:
    lib = _load()
    arr = np.asarray(codes, dtype=np.uint8)
    out = np.array([lib.oracle_e4m3_to_f64(int(c)) for c in arr.ravel()], dtype=np.float64)
    return out.reshape(arr.shape)


def f32_to_e4m3(v) -> np.ndarray:
    lib = _load()
    arr = np.asarray(v, dtype=np.float32)
    out = np.array([lib.oracle_f32_to_e4m3(float(x)) for x in arr.ravel()], dtype=np.uint8)
    return out.reshape(arr.shape)


# ---- the path ----------------------------------------------------------------

def act_quant(x_bf16: np.ndarray):
    """Returns (xq uint8 [M, K], s_x float32)."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    xq = np.zeros((M, K), dtype=np.uint8)
    sx = np.zeros(1, dtype=np.float32)
    lib.oracle_act_quant(_ptr(x), M, K, _ptr(xq), _ptr(sx))
    return xq, np.float32(sx[0])


def gemm_q(xq, s_x, w, s_w) -> np.ndarray:
    lib = _load()
    xq = _c(xq, np.uint8)
    w = _c(w, np.uint8)
    M, K = xq.shape
    N = w.shape[0]
    assert w.shape[1] == K
    y = np.zeros((M, N), dtype=np.float64)
    lib.oracle_gemm_q(_ptr(xq), float(s_x), _ptr(w), float(s_w), M, N, K, _ptr(y))
    return y


def fc13_swiglu_q(xq, s_x, w, s_w) -> np.ndarray:
    lib = _load()
    xq = _c(xq, np.uint8)
    w = _c(w, np.uint8)
    M, K = xq.shape
    N2 = w.shape[0]
    out = np.zeros((M, N2 // 2), dtype=np.float64)
    lib.oracle_fc13_swiglu_q(_ptr(xq), float(s_x), _ptr(w), float(s_w), M, K, N2, _ptr(out))
    return out


def fc13_swiglu(x_bf16, w, s_w) -> np.ndarray:
    lib = _load()
    x = _c(x_bf16, np.uint16)
    w = _c(w, np.uint8)
    M, K = x.shape
    N2 = w.shape[0]
    out = np.zeros((M, N2 // 2), dtype=np.float64)
    lib.oracle_fc13_swiglu(_ptr(x), M, K, _ptr(w), float(s_w), N2, _ptr(out))
    return out


def fc_qkv_scale_q(xq, s_x, w, s_w, Hq, Hkv, d, q_scale) -> np.ndarray:
    lib = _load()
    xq = _c(xq, np.uint8)
    w = _c(w, np.uint8)
    M, K = xq.shape
    N = (Hq + 2 * Hkv) * d
    assert w.shape == (N, K)
    out = np.zeros((M, N), dtype=np.float64)
    lib.oracle_fc_qkv_scale_q(_ptr(xq), float(s_x), _ptr(w), float(s_w), M, K, Hq, Hkv, d,
                              float(q_scale), _ptr(out))
    return out


def fc_qkv_scale(x_bf16, w, s_w, Hq, Hkv, d, q_scale) -> np.ndarray:
    lib = _load()
    x = _c(x_bf16, np.uint16)
    w = _c(w, np.uint8)
    M, K = x.shape
    N = (Hq + 2 * Hkv) * d
    assert w.shape == (N, K)
    out = np.zeros((M, N), dtype=np.float64)
    lib.oracle_fc_qkv_scale(_ptr(x), M, K, _ptr(w), float(s_w), Hq, Hkv, d, float(q_scale),
                            _ptr(out))
    return out


def moe_fc13_swiglu(x_bf16, ids, w, s_w) -> np.ndarray:
    """w is [E, N2, K] uint8, s_w is [E] float32."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    ids = _c(ids, np.int32)
    w = _c(w, np.uint8)
    s_w = _c(s_w, np.float32)
    T, K = x.shape
    E, N2, K2 = w.shape
    assert K2 == K and s_w.shape == (E,)
    out = np.zeros((T, N2 // 2), dtype=np.float64)
    lib.oracle_moe_fc13_swiglu(_ptr(x), T, K, _ptr(ids), E, _ptr(w), _ptr(s_w), N2, _ptr(out))
    return out


def linear(x_bf16, w, s_w) -> np.ndarray:
    """Plain-epilogue FP8 projection: act_quant(x), then y = s_x*s_w*x_q.W^T.  [M, N]."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    w = _c(w, np.uint8)
    M, K = x.shape
    N = w.shape[0]
    assert w.shape[1] == K
    out = np.zeros((M, N), dtype=np.float64)
    lib.oracle_linear(_ptr(x), M, K, _ptr(w), float(s_w), N, _ptr(out))
    return out


def moe_linear(x_bf16, ids, w, s_w) -> np.ndarray:
    """Grouped plain projection; w is [E, N, K] uint8, s_w [E] float32.  [T, N]."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    ids = _c(ids, np.int32)
    w = _c(w, np.uint8)
    s_w = _c(s_w, np.float32)
    T, K = x.shape
    E, N, K2 = w.shape
    assert K2 == K and s_w.shape == (E,)
    out = np.zeros((T, N), dtype=np.float64)
    lib.oracle_moe_linear(_ptr(x), T, K, _ptr(ids), E, _ptr(w), _ptr(s_w), N, _ptr(out))
    return out


def add_rmsnorm(x_bf16, r_bf16, gamma_bf16, eps):
    """Returns (h bf16 bits [M, K], y float64 [M, K]); r_bf16 may be None."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    g = _c(gamma_bf16, np.uint16)
    assert g.shape == (K,)
    r = None if r_bf16 is None else _c(r_bf16, np.uint16)
    if r is not None:
        assert r.shape == x.shape
    h = np.zeros((M, K), dtype=np.uint16)
    y = np.zeros((M, K), dtype=np.float64)
    lib.oracle_add_rmsnorm(_ptr(x), None if r is None else _ptr(r), _ptr(g), M, K, float(eps), _ptr(h), _ptr(y))
    return h, y


def quant_f32(y) -> tuple:
    """Returns (xq uint8, s_x float32) of float32 values (shape kept)."""
    lib = _load()
    yf = _c(y, np.float32)
    xq = np.zeros(yf.shape, dtype=np.uint8)
    sx = np.zeros(1, dtype=np.float32)
    lib.oracle_quant_f32(_ptr(yf), int(yf.size), _ptr(xq), _ptr(sx))
    return xq, np.float32(sx[0])


def add_rmsnorm_quant(x_bf16, r_bf16, gamma_bf16, eps):
    """Residual add + RMSNorm + Quantize: (h bits, y float64, xq, s_x), the
    quantisation taken on float32(y)."""
    h, y = add_rmsnorm(x_bf16, r_bf16, gamma_bf16, eps)
    xq, sx = quant_f32(y.astype(np.float32))
    return h, y, xq, sx


def spec_verify_greedy(logits_bf16, draft):
    """logits [B, T, V] bf16 bits, draft [B, T-1] int32 ->
    (target_ids [B, T], n_accepted [B], emitted [B, T]) int32."""
    lib = _load()
    lg = _c(logits_bf16, np.uint16)
    B, T, V = lg.shape
    dr = _c(draft, np.int32).reshape(B, T - 1)
    tid = np.zeros((B, T), dtype=np.int32)
    nacc = np.zeros(B, dtype=np.int32)
    em = np.zeros((B, T), dtype=np.int32)
    lib.oracle_spec_verify_greedy(_ptr(lg), B, T, V, _ptr(dr), _ptr(tid), _ptr(nacc), _ptr(em))
    return tid, nacc, em


def decode_attn(q, q_stride, B, T, Hq, Hkv, d, k_cache, v_cache, seq_lens, scale) -> np.ndarray:
    """q is a flat uint16 buffer addressed as q[(b*T+t)*q_stride + h*d + i];
    k_cache / v_cache are [B, Hkv, Lcap, d] uint16.  Returns [B, T, Hq, d]."""
    lib = _load()
    q = _c(q, np.uint16)
    k = _c(k_cache, np.uint16)
    v = _c(v_cache, np.uint16)
    sl = _c(seq_lens, np.int32)
    Lcap = k.shape[2]
    assert k.shape == (B, Hkv, Lcap, d) and v.shape == k.shape and sl.shape == (B,)
    out = np.zeros((B, T, Hq, d), dtype=np.float64)
    lib.oracle_decode_attn(_ptr(q), int(q_stride), B, T, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap,
                           _ptr(sl), float(scale), _ptr(out))
    return out


def decode_attn_fp8kv(q, q_stride, B, T, Hq, Hkv, d, k_codes, vt_codes, seq_lens, scale, s_k, s_v) -> np.ndarray:
    """As decode_attn, with e4m3 caches and per-tensor scales: k_codes uint8
    [B, Hkv, Lcap, d], vt_codes uint8 [B, Hkv, d, Lcap] (V stored transposed)."""
    lib = _load()
    q = _c(q, np.uint16)
    k = _c(k_codes, np.uint8)
    v = _c(vt_codes, np.uint8)
    sl = _c(seq_lens, np.int32)
    Lcap = k.shape[2]
    assert k.shape == (B, Hkv, Lcap, d) and v.shape == (B, Hkv, d, Lcap) and sl.shape == (B,)
    out = np.zeros((B, T, Hq, d), dtype=np.float64)
    lib.oracle_decode_attn_fp8kv(_ptr(q), int(q_stride), B, T, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(sl),
                                 float(scale), float(s_k), float(s_v), _ptr(out))
    return out


def attn_partial(q, q_stride, T, Hq, Hkv, d, k_cache, v_cache, b, t, h, L, scale, key_lo, key_hi):
    """Returns (m, l, o[d]) of one query row over keys [key_lo, key_hi)."""
    lib = _load()
    q = _c(q, np.uint16)
    k = _c(k_cache, np.uint16)
    v = _c(v_cache, np.uint16)
    Lcap = k.shape[2]
    m = np.zeros(1)
    l = np.zeros(1)
    o = np.zeros(d)
    lib.oracle_attn_partial(_ptr(q), int(q_stride), T, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap,
                            b, t, h, L, float(scale), key_lo, key_hi, _ptr(m), _ptr(l), _ptr(o))
    return float(m[0]), float(l[0]), o


def lse_combine(m, l, o_parts) -> np.ndarray:
    lib = _load()
    m = _c(m, np.float64)
    l = _c(l, np.float64)
    o = _c(o_parts, np.float64)
    S, d = o.shape
    out = np.zeros(d)
    lib.oracle_lse_combine(S, _ptr(m), _ptr(l), _ptr(o), d, _ptr(out))
    return out
