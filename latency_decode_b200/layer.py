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
        # both results in one buffer, so a caller can fetch them with one copy
        n_attn = B * T * Hq * d
        self.out_buf = torch.empty(n_attn + M * (self.N2 // 2), dtype=torch.int16, device=self.device)
        self.attn_out = self.out_buf[:n_attn].view(B, T, Hq, d)
        self.ffn_out = self.out_buf[n_attn:].view(M, self.N2 // 2)

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

    def step_host(self, x_host: torch.Tensor, out_host: torch.Tensor, k_cache, v_cache, seq_lens, stream=None,
                  flags: int = dl.DL_FLAG_PDL, overlap_upload: bool = False) -> None:
        """One step whose activations come from, and whose results go to, pinned
        host memory: x_host is [2, M, K] bf16 bits (x1, x2) from cudaHostAlloc
        (torch's pin_memory), out_host has the layout of self.out_buf.  The two
        transfers are kernels of the same PDL chain (dl_copy), so the QKV GEMM
        streams its weights while the activations arrive.

        overlap_upload: the kernel just before this call in the stream is the
        result download of a previous step_host (of this or another
        DecodeLayer), which reads only that layer's out_buf and writes its host
        buffer; the upload then starts beside it (DL_FLAG_COPY_NO_WAIT), using
        the other direction of the host link.  That download waited for its
        step's kernels before it let this one start, so x_dev is free."""
        if not hasattr(self, "x_dev"):
            self.x_dev = torch.empty((2, self.M, self.K), dtype=torch.int16, device=self.device)
        up_flags = flags | (dl.DL_FLAG_COPY_NO_WAIT if overlap_upload else 0)
        dl.check(dl.dl_copy(x_host, self.x_dev, self.x_dev.numel() * 2, stream=stream, flags=up_flags))
        self.step(self.x_dev[0], self.x_dev[1], k_cache, v_cache, seq_lens, stream=stream, flags=flags)
        dl.check(dl.dl_copy(self.out_buf, out_host, self.out_buf.numel() * 2, stream=stream, flags=flags))

    def read_status(self, stream=None) -> None:
        for ws in (self.ws_qkv, self.ws_attn, self.ws_13):
            if ws is not None:
                dl.check(dl.dl_read_status(ws, stream))


class FullDecodeLayer:
    """The whole pre-norm decode layer of a dense model on one GPU:

        h1 = x + h;  qkv = FC_QKV(RMSNorm(h1) * g1)         (dl_rmsnorm_fc_qkv_scale)
        o  = attention(q, K cache, V cache)                 (dl_decode_attn, q read in place)
        a  = O_proj(o)                                      (dl_gemm_e4m3)
        h  <- a + h1;  f = SwiGLU(FC13(RMSNorm(h) * g2))    (dl_rmsnorm_fc13_swiglu)
        y  = FC2(f)                                         (dl_gemm_e4m3)

    ``y`` is the layer's output and ``h`` its residual stream (updated in place);
    the next layer's first step adds them.  Each RMSNorm call is the producer
    kernel followed by its GEMM: seven kernels at batch 1 (more when an input
    is too large for a GEMM to quantise itself), all chained with PDL on one
    stream.  Everything runs in libdl.so; this class only holds buffers."""

    def __init__(self, w_qkv, s_qkv, w_o, s_o, w13, s13, w2, s2, g1, g2, *, Hq, Hkv, d, q_scale, M, B, T,
                 eps: float = 1e-5, cluster: int = 8, device="cuda"):
        """Weights: canonical e4m3 bytes (uint8, on device) in nn.Linear [N, K] order:
        w_qkv [(Hq+2Hkv)d, D], w_o [D, Hq d], w13 [2F, D], w2 [D, F].  g1, g2:
        bf16 bits [D] (int16, on device)."""
        assert M == B * T
        self.device = torch.device(device)
        self.Hq, self.Hkv, self.d, self.M, self.B, self.T = Hq, Hkv, d, M, B, T
        self.cluster, self.eps, self.q_scale = cluster, float(eps), float(q_scale)
        self.N_qkv, self.D = w_qkv.shape
        self.N2 = w13.shape[0]
        self.F = self.N2 // 2
        assert w_o.shape == (self.D, Hq * d) and w2.shape == (self.D, self.F)
        self.wp = {}
        for name, w, kind in (("qkv", w_qkv, dl.DL_PACK_PLAIN), ("o", w_o, dl.DL_PACK_PLAIN),
                              ("13", w13, dl.DL_PACK_SWIGLU), ("2", w2, dl.DL_PACK_PLAIN)):
            p = torch.empty_like(w)
            dl.check(dl.dl_pack_fp8_weight(w, p, w.shape[0], w.shape[1], kind))
            self.wp[name] = p
        self.s = {k: _scale_tensor(v, self.device) for k, v in (("qkv", s_qkv), ("o", s_o), ("13", s13),
                                                                 ("2", s2))}
        self.g1, self.g2 = g1, g2

        def ws(K):
            return torch.zeros(dl.dl_workspace_bytes(M, K), dtype=torch.uint8, device=self.device)

        self.ws_qkv, self.ws_o, self.ws_13, self.ws_2 = ws(self.D), ws(Hq * d), ws(self.D), ws(self.F)
        self.ws_attn = None
        self.Lcap_hint = None
        self.h_mid = torch.empty((M, self.D), dtype=torch.int16, device=self.device)  # h1
        self.qkv = torch.empty((M, self.N_qkv), dtype=torch.int16, device=self.device)
        self.attn_out = torch.empty((M, Hq * d), dtype=torch.int16, device=self.device)
        self.a = torch.empty((M, self.D), dtype=torch.int16, device=self.device)
        self.f = torch.empty((M, self.F), dtype=torch.int16, device=self.device)
        self.y = torch.empty((M, self.D), dtype=torch.int16, device=self.device)

    @property
    def weight_bytes(self) -> int:
        return sum(int(p.numel()) for p in self.wp.values())

    def step(self, x, h, k_cache, v_cache, seq_lens, stream=None, flags: int = dl.DL_FLAG_PDL) -> None:
        """x: the previous layer's output, h: the residual stream (updated in
        place), both bf16 bits [M, D]; caches [B, Hkv, Lcap, d]; seq_lens int32
        [B].  The output lands in self.y."""
        M, D = self.M, self.D
        Lcap = k_cache.shape[2]
        if self.ws_attn is None or self.Lcap_hint != Lcap:
            n = dl.dl_decode_attn_workspace_bytes(self.B, self.T, self.Hq, self.Hkv, self.d, Lcap, self.cluster)
            self.ws_attn = torch.zeros(n, dtype=torch.uint8, device=self.device)
            self.Lcap_hint = Lcap
        dl.check(dl.dl_rmsnorm_fc_qkv_scale(x, h, self.h_mid, self.g1, self.eps, M, D, self.wp["qkv"],
                                            self.s["qkv"], self.Hq, self.Hkv, self.d, self.q_scale, self.qkv,
                                            self.ws_qkv, stream=stream, flags=flags))
        dl.check(dl.dl_decode_attn(self.qkv, self.N_qkv, self.B, self.T, self.Hq, self.Hkv, self.d, k_cache,
                                   v_cache, Lcap, seq_lens, 1.0, self.cluster, self.attn_out, self.ws_attn,
                                   stream=stream, flags=flags))
        dl.check(dl.dl_gemm_e4m3(self.attn_out, M, self.Hq * self.d, self.wp["o"], self.s["o"], D, self.a,
                                 self.ws_o, stream=stream, flags=flags))
        dl.check(dl.dl_rmsnorm_fc13_swiglu(self.a, self.h_mid, h, self.g2, self.eps, M, D, self.wp["13"],
                                           self.s["13"], self.N2, self.f, self.ws_13, stream=stream, flags=flags))
        dl.check(dl.dl_gemm_e4m3(self.f, M, self.F, self.wp["2"], self.s["2"], D, self.y, self.ws_2,
                                 stream=stream, flags=flags))

    def read_status(self, stream=None) -> None:
        for ws in (self.ws_qkv, self.ws_attn, self.ws_o, self.ws_13, self.ws_2):
            if ws is not None:
                dl.check(dl.dl_read_status(ws, stream))
