"""Seeded synthetic inputs for the decode path, shared by the tests, the smoke
check and the benchmark.

This module holds no arithmetic of the method (no activation quantisation, no
GEMM, no softmax).  It draws random numbers, rounds them to the storage formats
the path consumes (bf16 activations and KV cache, e4m3 weights with one
per-tensor scale) using torch's own casts, and packages them with the workload
shapes.  The e4m3 weight scale follows the per-tensor max-abs rule the
workloads name: ``s_w = max|W| / 448`` in float32, ``W_q = e4m3(W / s_w)``.

Workloads (named by what they are):
  tiny      1 token, FC13 512 -> 2x1024, attention 8/2 heads d=64, KV length 256
  layer_b1  1 token, FC_QKV 5120 -> 7168, FC13 5120 -> 2x8192, attention 40/8 heads
            d=128, KV length 4096
  verify4   4 query tokens (1 + draft 3), causal, KV length 32768, weights as layer_b1
  batch16x4 16 sequences x 4 tokens (GEMM M=64), KV lengths uniform in [1024, 16384]
  moe64     64 tokens, 128 experts top-1 uniform, each expert FC13 5120 -> 2x8192
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

E4M3_MAX = 448.0
# Vocabulary of the verification workloads: the size of Llama 4 Maverick's
# tokenizer (the pages do not state it; public model configuration).
VOCAB = 202048


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    K: int              # hidden size (GEMM reduction length)
    M: int              # GEMM rows = tokens in the step
    N2: int             # FC13 output rows (gate + up)
    Hq: int
    Hkv: int
    d: int
    B: int              # sequences
    T: int              # query tokens per sequence
    L: int              # KV length (fixed) or 0 when drawn per sequence
    Lcap: int           # KV cache capacity per sequence
    experts: int = 0    # MoE experts (0 = dense)
    cluster: int = 8    # attention split-KV cluster size (the measured best for the shape)

    @property
    def n_qkv(self) -> int:
        return (self.Hq + 2 * self.Hkv) * self.d

    @property
    def k_o(self) -> int:
        """Attention output projection: reduction length Hq*d, output rows K."""
        return self.Hq * self.d

    @property
    def k_fc2(self) -> int:
        """FC2 down projection: reduction length F = N2/2, output rows K."""
        return self.N2 // 2


WORKLOADS = {
    "tiny": Workload("tiny", 0, K=512, M=1, N2=2048, Hq=8, Hkv=2, d=64, B=1, T=1, L=256,
                     Lcap=256, cluster=8),
    "layer_b1": Workload("layer_b1", 1, K=5120, M=1, N2=16384, Hq=40, Hkv=8, d=128, B=1, T=1,
                         L=4096, Lcap=4096, cluster=8),
    "verify4": Workload("verify4", 2, K=5120, M=4, N2=16384, Hq=40, Hkv=8, d=128, B=1, T=4,
                        L=32768, Lcap=32768, cluster=4),
    "batch16x4": Workload("batch16x4", 3, K=5120, M=64, N2=16384, Hq=40, Hkv=8, d=128, B=16,
                          T=4, L=0, Lcap=16384, cluster=4),
    "moe64": Workload("moe64", 4, K=5120, M=64, N2=16384, Hq=40, Hkv=8, d=128, B=0, T=0, L=0,
                      Lcap=0, experts=128),
}


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (torch's round-to-nearest-even cast)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_normal(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return bf16_bits(g.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def e4m3_codes_from_f32(w: np.ndarray):
    """Per-tensor max-abs e4m3 quantisation of a weight tensor (input preparation).
    Returns (codes uint8 same shape, s_w float32)."""
    t = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32))
    amax = float(t.abs().max()) if t.numel() else 0.0
    s_w = np.float32(amax) / np.float32(E4M3_MAX) if amax > 0 else np.float32(1.0)
    q = (t / torch.tensor(float(s_w), dtype=torch.float32)).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, np.float32(s_w)


def e4m3_weight(g: np.random.Generator, N: int, K: int, std: float = 0.02):
    w = g.standard_normal(size=(N, K), dtype=np.float32) * np.float32(std)
    return e4m3_codes_from_f32(w)


def e4m3_weight_torch(gen: torch.Generator, N: int, K: int, device, std: float = 0.02):
    """Same rule, drawn with a seeded torch generator on ``device`` (used for the
    10.7 GB expert bank, too large to draw on the host).  Returns (codes uint8
    tensor [N, K] on device, s_w float32 python float)."""
    w = torch.randn((N, K), generator=gen, device=device, dtype=torch.float32) * std
    amax = float(w.abs().max())
    s_w = float(np.float32(amax) / np.float32(E4M3_MAX))
    q = (w / torch.tensor(s_w, dtype=torch.float32, device=device)).clamp_(-E4M3_MAX, E4M3_MAX)
    return q.to(torch.float8_e4m3fn).view(torch.uint8), s_w


def seq_lens_for(wl: Workload, g: np.random.Generator) -> np.ndarray:
    if wl.L > 0:
        return np.full(wl.B, wl.L, dtype=np.int32)
    return g.integers(1024, 16384, endpoint=True, size=wl.B).astype(np.int32)


def expert_ids_for(wl: Workload, g: np.random.Generator) -> np.ndarray:
    return g.integers(0, wl.experts, size=wl.M).astype(np.int32)


def rmsnorm_gain(g: np.random.Generator, K: int) -> np.ndarray:
    """A synthetic RMSNorm gain: bf16 of 1 + 0.1 N(0, 1)."""
    return bf16_bits(np.float32(1.0) + g.standard_normal(size=K, dtype=np.float32) * np.float32(0.1))


def dense_layer_inputs(wl: Workload, with_weights: bool = True, with_kv: bool = True):
    """Host arrays for one dense decode layer of workload ``wl``.

    Keys: x1 [M,K] bf16 (QKV input), x2 [M,K] bf16 (FC13 input, drawn fresh and
    independent of the attention output), w_qkv/s_qkv, w13/s13, k_cache, v_cache
    [B,Hkv,Lcap,d] bf16, seq_lens [B] int32, q_scale = 1/sqrt(d)."""
    g = rng(wl.seed)
    out = {}
    out["x1"] = bf16_normal(g, (wl.M, wl.K))
    out["x2"] = bf16_normal(g, (wl.M, wl.K))
    out["q_scale"] = np.float32(1.0 / math.sqrt(wl.d))
    if with_weights:
        if wl.Hq > 0 and wl.n_qkv % 128 == 0:
            out["w_qkv"], out["s_qkv"] = e4m3_weight(g, wl.n_qkv, wl.K)
        out["w13"], out["s13"] = e4m3_weight(g, wl.N2, wl.K)
    if with_kv and wl.B > 0:
        out["seq_lens"] = seq_lens_for(wl, g)
        out["k_cache"] = bf16_normal(g, (wl.B, wl.Hkv, wl.Lcap, wl.d))
        out["v_cache"] = bf16_normal(g, (wl.B, wl.Hkv, wl.Lcap, wl.d))
    return out


def full_layer_inputs(wl: Workload):
    """Host arrays for the whole pre-norm layer of workload ``wl``: x (the
    previous layer's output) and h (the residual stream) [M, K] bf16; weights
    w_qkv, w_o [K, Hq*d], w13, w2 [K, F] e4m3 with their scales; RMSNorm gains
    g1, g2 [K] bf16; the KV caches, seq_lens and q_scale."""
    g = rng(1000 + wl.seed)
    out = {"x": bf16_normal(g, (wl.M, wl.K)), "h": bf16_normal(g, (wl.M, wl.K)),
           "q_scale": np.float32(1.0 / math.sqrt(wl.d))}
    out["w_qkv"], out["s_qkv"] = e4m3_weight(g, wl.n_qkv, wl.K)
    out["w_o"], out["s_o"] = e4m3_weight(g, wl.K, wl.k_o)
    out["w13"], out["s13"] = e4m3_weight(g, wl.N2, wl.K)
    out["w2"], out["s2"] = e4m3_weight(g, wl.K, wl.k_fc2)
    out["g1"] = rmsnorm_gain(g, wl.K)
    out["g2"] = rmsnorm_gain(g, wl.K)
    out["seq_lens"] = seq_lens_for(wl, g)
    out["k_cache"] = bf16_normal(g, (wl.B, wl.Hkv, wl.Lcap, wl.d))
    out["v_cache"] = bf16_normal(g, (wl.B, wl.Hkv, wl.Lcap, wl.d))
    return out
