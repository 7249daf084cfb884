"""Failure detection on the GPU without a GPU fault.

DL_FLAG_DEBUG_TIMEOUT makes the producer of each kernel withhold its last
pipeline load (the load is simply never issued) and shortens every bounded
wait to ~2 ms.  The consumer's wait then runs out: the kernel records the
timeout in the workspace status word, lets its other loads land, frees its
Tensor Memory and returns.  The host reads DL_ERR_TIMEOUT, and the next normal
call on the same context must succeed and match the oracle."""
import math

import numpy as np
import pytest
import torch

import helpers
import oracle
from helpers import dev_f32, dev_i32, dev_u8, dev_u16, host_u16, new_ws
from latency_decode_b200 import build as dl_build
from latency_decode_b200 import datagen as dg
from latency_decode_b200 import dl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not helpers.gpu_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def lib():
    dl_build.build()
    return dl.lib()


def _fc13_case(seed=1, M=2, K=512, N2=256):
    g = np.random.default_rng(seed)
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N2, K)
    wd = dev_u8(w)
    wp = torch.empty_like(wd)
    dl.check(dl.dl_pack_fp8_weight(wd, wp, N2, K, dl.DL_PACK_SWIGLU))
    return x, w, s_w, wp


@pytest.mark.parametrize("M,K", [(2, 512), (64, 1024)])
def test_gemm_timeout_is_reported_and_context_stays_usable(M, K):
    # (64, 1024): x_q is streamed into the GEMM by tensor loads beside the weights
    x, w, s_w, wp = _fc13_case(M=M, K=K)
    M, K = x.shape
    N2 = w.shape[0]
    out = torch.empty((M, N2 // 2), dtype=torch.int16, device="cuda")
    ws, n = new_ws(M, K)
    assert dl.dl_fc13_swiglu(dev_u16(x), M, K, wp, dev_f32(s_w), N2, out, ws, n,
                             flags=dl.DL_FLAG_PDL | dl.DL_FLAG_DEBUG_TIMEOUT) == dl.DL_OK
    assert dl.dl_read_status(ws) == dl.DL_ERR_TIMEOUT
    assert dl.dl_read_status(ws) == dl.DL_OK  # cleared by the read
    dl.check(dl.dl_fc13_swiglu(dev_u16(x), M, K, wp, dev_f32(s_w), N2, out, ws, n))
    assert dl.dl_read_status(ws) == dl.DL_OK
    helpers.check_gemm(host_u16(out), oracle.fc13_swiglu(x, w, s_w), "after timeout")


@pytest.mark.parametrize("M", [1, 64])
def test_qkv_timeout_with_a_single_stage_per_cta(M):
    # N = 256, one k-block per CTA: no weight block is loaded at all (at M = 64,
    # K = 1024, M*K is past the fused quantiser and the k-block's activations
    # still arrive by their tensor load)
    g = np.random.default_rng(3)
    K, Hq, Hkv, d = (512 if M == 1 else 1024), 2, 1, 64
    split = K // 128 if M > 1 else 4
    N = (Hq + 2 * Hkv) * d
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N, K)
    wd = dev_u8(w)
    wp = torch.empty_like(wd)
    dl.check(dl.dl_pack_fp8_weight(wd, wp, N, K, dl.DL_PACK_PLAIN))
    out = torch.empty((M, N), dtype=torch.int16, device="cuda")
    ws, n = new_ws(M, K)
    flags = dl.DL_FLAG_DEBUG_TIMEOUT | (split << dl.DL_FLAG_SPLIT_SHIFT)
    assert dl.dl_fc_qkv_scale(dev_u16(x), M, K, wp, dev_f32(s_w), Hq, Hkv, d, 0.125, out, ws, n,
                              flags=flags) == dl.DL_OK
    assert dl.dl_read_status(ws) == dl.DL_ERR_TIMEOUT


def test_attention_timeout_is_reported_and_context_stays_usable():
    g = np.random.default_rng(4)
    B, T, Hq, Hkv, d, L = 1, 1, 8, 2, 128, 300
    q = dg.bf16_normal(g, (B, T, Hq, d))
    k = dg.bf16_normal(g, (B, Hkv, L, d))
    v = dg.bf16_normal(g, (B, Hkv, L, d))
    sl = np.int32([L])
    out = torch.empty((B, T, Hq, d), dtype=torch.int16, device="cuda")
    ws, n = new_ws(0, 0)
    args = (dev_u16(q), Hq * d, B, T, Hq, Hkv, d, dev_u16(k), dev_u16(v), L, dev_i32(sl), 1 / math.sqrt(d), 8, out,
            ws, n)
    assert dl.dl_decode_attn(*args, flags=dl.DL_FLAG_PDL | dl.DL_FLAG_DEBUG_TIMEOUT) == dl.DL_OK
    assert dl.dl_read_status(ws) == dl.DL_ERR_TIMEOUT
    dl.check(dl.dl_decode_attn(*args))
    assert dl.dl_read_status(ws) == dl.DL_OK
    ref = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, 1 / math.sqrt(d))
    helpers.check_attn(host_u16(out), ref, "after timeout")


def test_fp8kv_attention_timeouts_are_reported_and_context_stays_usable():
    """FP8-cache attention under the test hook: the producer withholds its last
    tile, and each owner CTA expects 16 bytes more than its peers push, so both
    the tile wait and the merge's receive wait run out.  Every CTA still waits
    at the cluster barrier for its peers' pushes before it exits; the status is
    reported and the next normal call matches the oracle."""
    g = np.random.default_rng(5)
    B, T, Hq, Hkv, d, L = 1, 4, 8, 2, 128, 320
    q = dg.bf16_normal(g, (B, T, Hq, d))
    kc = g.integers(0, 0x7E, size=(B, Hkv, L, d)).astype(np.uint8)
    vt = g.integers(0, 0x7E, size=(B, Hkv, d, L)).astype(np.uint8)
    sl = np.int32([L])
    s_k, s_v = np.float32(0.01), np.float32(0.02)
    out = torch.empty((B, T, Hq, d), dtype=torch.int16, device="cuda")
    n = dl.dl_decode_attn_fp8kv_workspace_bytes(B, T, Hq, Hkv, d, L, 4)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    args = (dev_u16(q), Hq * d, B, T, Hq, Hkv, d, dev_u8(kc), dev_u8(vt), dev_f32([s_k, s_v]), L, dev_i32(sl),
            1 / math.sqrt(d), 4, out, ws, n)
    assert dl.dl_decode_attn_fp8kv(*args, flags=dl.DL_FLAG_PDL | dl.DL_FLAG_DEBUG_TIMEOUT) == dl.DL_OK
    assert dl.dl_read_status(ws) == dl.DL_ERR_TIMEOUT
    dl.check(dl.dl_decode_attn_fp8kv(*args))
    assert dl.dl_read_status(ws) == dl.DL_OK
    ref = oracle.decode_attn_fp8kv(q.ravel(), Hq * d, B, T, Hq, Hkv, d, kc, vt, sl, 1 / math.sqrt(d), s_k, s_v)
    helpers.check_attn(host_u16(out), ref, "after timeout")


def test_moe_timeout_is_reported():
    g = np.random.default_rng(6)
    T, E, K, N2 = 4, 3, 512, 256
    x = dg.bf16_normal(g, (T, K))
    bank = np.stack([dg.e4m3_weight(g, N2, K)[0] for _ in range(E)])
    wd = dev_u8(bank)
    wp = torch.empty_like(wd)
    for e in range(E):
        dl.check(dl.dl_pack_fp8_weight(wd[e], wp[e], N2, K, dl.DL_PACK_SWIGLU))
    out = torch.empty((T, N2 // 2), dtype=torch.int16, device="cuda")
    ws, n = new_ws(T, K)
    assert dl.dl_moe_fc13_swiglu_grouped(dev_u16(x), T, K, dev_i32(np.int32([0, 2, 2, 1])), E, wp,
                                         dev_f32(np.ones(E)), N2, out, ws, n,
                                         flags=dl.DL_FLAG_DEBUG_TIMEOUT) == dl.DL_OK
    assert dl.dl_read_status(ws) == dl.DL_ERR_TIMEOUT
