"""Shared test helpers: the packed-weight layout restated from include/dl.h,
tolerance checks, and device/host tensor plumbing.  No method arithmetic."""
from __future__ import annotations

import numpy as np

try:
    import torch
except ImportError:  # pragma: no cover
    torch = None

GEMM_REL_L2 = 1e-2
GEMM_MAX_ABS = 3e-2
ATTN_REL_L2 = 5e-3


def pack_reference(w: np.ndarray, kind: int) -> np.ndarray:
    """The packed layout of dl_pack_fp8_weight, written from its definition in
    include/dl.h: 16384-byte blocks, byte c of row r of a block at
    (r/8)*1024 + (r%8)*128 + ((c/16) ^ (r%8))*16 + c%16; PLAIN orders blocks
    (tile, kb); SWIGLU orders them (tile, kb, gate|up)."""
    N, K = w.shape
    KB = K // 128
    r = np.arange(128)[:, None]
    c = np.arange(128)[None, :]
    intra = ((r // 8) * 1024 + (r % 8) * 128 + ((c // 16) ^ (r % 8)) * 16 + c % 16).ravel()

    def blocks_of(mat):
        n = mat.shape[0]
        return mat.reshape(n // 128, 128, KB, 128).transpose(0, 2, 1, 3)  # (t, kb, r, c)

    if kind == 0:
        blk = blocks_of(w).reshape(-1, 128 * 128)
    else:
        F = N // 2
        g, u = blocks_of(w[:F]), blocks_of(w[F:])
        blk = np.stack([g, u], axis=2).reshape(-1, 128 * 128)
    out = np.empty((blk.shape[0], 128 * 128), dtype=np.uint8)
    out[:, intra] = blk
    return out.ravel()


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_round_f64(ref: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even) via torch."""
    t = torch.from_numpy(np.ascontiguousarray(ref, dtype=np.float64)).to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((got - ref).ravel()) / (den if den > 0 else 1.0))


def check_gemm(got_bits: np.ndarray, ref: np.ndarray, what: str = "", slack=None) -> dict:
    """bf16 GEMM outputs vs the float64 oracle: relative L2 <= 1e-2 over the
    call, and max-abs <= 3e-2 against the bf16-rounded reference, where an
    element whose bf16 spacing exceeds 3e-2 may sit one spacing away (a
    rounding-boundary flip of a correct fp32 result).  `slack`, when given, is
    a per-element allowance added to both rules (a derived bound for inputs
    whose e4m3 codes may legitimately differ at rounding ties)."""
    got = bf16_to_f64(got_bits)
    rl2 = rel_l2(got, ref)
    rb = bf16_round_f64(ref)
    diff = np.abs(got - rb)
    ulp = bf16_ulp(rb)
    if slack is not None:
        diff = np.maximum(diff - slack, 0.0)
    bad = (diff > GEMM_MAX_ABS) & ~((ulp > GEMM_MAX_ABS) & (diff <= ulp * 1.0000001))
    stats = {"rel_l2": rl2, "max_abs_vs_bf16ref": float(diff.max(initial=0.0)),
             "raw_max_abs": float(np.abs(got - ref).max(initial=0.0)), "n_bad": int(bad.sum())}
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert rl2 <= GEMM_REL_L2, f"{what}: rel L2 {rl2:.3e} > {GEMM_REL_L2} ({stats})"
    assert not bad.any(), f"{what}: {bad.sum()} elements beyond max-abs rule ({stats})"
    return stats


def check_attn(got_bits: np.ndarray, ref: np.ndarray, what: str = "") -> float:
    got = bf16_to_f64(got_bits)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    rl2 = rel_l2(got, ref)
    assert rl2 <= ATTN_REL_L2, f"{what}: rel L2 {rl2:.3e} > {ATTN_REL_L2}"
    return rl2


def dev_u8(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_u16(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda()


def dev_i32(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def dev_f32(a):
    return torch.tensor(np.atleast_1d(np.asarray(a, dtype=np.float32)), device="cuda")


def host_u16(t) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint16)


def new_ws(M: int, K: int):
    from latency_decode_b200 import dl
    n = dl.dl_workspace_bytes(M, K)
    return torch.zeros(n, dtype=torch.uint8, device="cuda"), n


def gpu_available() -> bool:
    return torch is not None and torch.cuda.is_available()
