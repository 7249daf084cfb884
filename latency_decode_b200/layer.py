"""One decode layer's hot path on one GPU, as a sequence of C-ABI calls.

``DecodeLayer`` owns the packed FP8 weights, the weight scales, one workspace
per call and the output buffers, and issues

    act-quant(x1) -> FC_QKV + attention scaling -> split-KV attention (q read in
    place from the QKV output, softmax scale 1 since Q is pre-scaled)
    act-quant(x2) -> FC13 + SwiGLU

on one stream, each kernel chained to the previous one with Programmatic
Dependent Launch ([XZY] "程序化依赖启动（PDL）").  Every step runs in libdl.so;
this module only allocates buffers and passes pointers.

The FC13 input ``x2`` is a separate activation: the layer pieces between the
attention output and FC13 (output projection, residual, norm) are not part of
this path.
"""
from __future__ import annotations

import torch

from . import dl


def _scale_tensor(v, device):
    return torch.tensor([float(v)], dtype=torch.float32, device=device)


class DecodeLayer:
    def __init__(self, w_qkv: torch.Tensor, s_qkv: float, w13: torch.Tensor, s13: float, *, Hq: int, Hkv: int,
                 d: int, q_scale: float, M: int, B: int, T: int, cluster: int = 8,
                 device: torch.device | str = "cuda"):
        """w_qkv [(Hq+2Hkv)*d, K] and w13 [N2, K]: canonical e4m3 bytes (uint8, on device)."""
        assert M == B * T, "the GEMM rows are the B*T query tokens"
        self.device = torch.device(device)
        self.Hq, self.Hkv, self.d, self.M, self.B, self.T = Hq, Hkv, d, M, B, T
        self.cluster = cluster
        self.q_scale = float(q_scale)
        self.N_qkv, self.K = w_qkv.shape
        self.N2 = w13.shape[0]
        self.wp_qkv = torch.empty_like(w_qkv)
        self.wp_13 = torch.empty_like(w13)
        dl.check(dl.dl_pack_fp8_weight(w_qkv, self.wp_qkv, self.N_qkv, self.K, dl.DL_PACK_PLAIN))
        dl.check(dl.dl_pack_fp8_weight(w13, self.wp_13, self.N2, self.K, dl.DL_PACK_SWIGLU))
        self.s_qkv = _scale_tensor(s_qkv, self.device)
        self.s_13 = _scale_tensor(s13, self.device)
        nq = dl.dl_workspace_bytes(M, self.K)
        self.ws_qkv = torch.zeros(nq, dtype=torch.uint8, device=self.device)
        self.ws_13 = torch.zeros(nq, dtype=torch.uint8, device=self.device)
        self.Lcap_hint = None
        self.ws_attn = None
        self.qkv = torch.empty((M, self.N_qkv), dtype=torch.int16, device=self.device)
        self.attn_out = torch.empty((B, T, Hq, d), dtype=torch.int16, device=self.device)
        self.ffn_out = torch.empty((M, self.N2 // 2), dtype=torch.int16, device=self.device)

    @property
    def weight_bytes(self) -> int:
        return self.N_qkv * self.K + self.N2 * self.K

    def step(self, x1: torch.Tensor, x2: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
             seq_lens: torch.Tensor, stream=None, flags: int = dl.DL_FLAG_PDL) -> None:
        """x1, x2: bf16 bits [M, K] (int16); k_cache, v_cache: bf16 bits [B, Hkv, Lcap, d];
        seq_lens: int32 [B].  Results land in self.attn_out and self.ffn_out."""
        Lcap = k_cache.shape[2]
        if self.ws_attn is None or self.Lcap_hint != Lcap:
            n = dl.dl_decode_attn_workspace_bytes(self.B, self.T, self.Hq, self.Hkv, self.d, Lcap, self.cluster)
            self.ws_attn = torch.zeros(n, dtype=torch.uint8, device=self.device)
            self.Lcap_hint = Lcap
        dl.check(dl.dl_fc_qkv_scale(x1, self.M, self.K, self.wp_qkv, self.s_qkv, self.Hq, self.Hkv, self.d,
                                    self.q_scale, self.qkv, self.ws_qkv, stream=stream, flags=flags))
        dl.check(dl.dl_decode_attn(self.qkv, self.N_qkv, self.B, self.T, self.Hq, self.Hkv, self.d, k_cache,
                                   v_cache, Lcap, seq_lens, 1.0, self.cluster, self.attn_out, self.ws_attn,
                                   stream=stream, flags=flags))
        dl.check(dl.dl_fc13_swiglu(x2, self.M, self.K, self.wp_13, self.s_13, self.N2, self.ffn_out, self.ws_13,
                                   stream=stream, flags=flags))

    def read_status(self, stream=None) -> None:
        for ws in (self.ws_qkv, self.ws_attn, self.ws_13):
            if ws is not None:
                dl.check(dl.dl_read_status(ws, stream))
