"""GPU parity of the FP8 GEMM family through the C ABI against the CPU oracle:
the offline pack (bit-exact against its stated layout), the activation
quantisation (bit-exact codes and scale), FC13+SwiGLU and FC_QKV+scaling over
many M / K / N / split-K shapes including ragged M, and the full-size layer
shapes.  Tolerances: relative L2 <= 1e-2 and max-abs <= 3e-2 (helpers.check_gemm)."""
import numpy as np
import pytest
import torch

import helpers
import oracle
from helpers import dev_f32, dev_u8, dev_u16, host_u16, new_ws
from latency_decode_b200 import build as dl_build
from latency_decode_b200 import datagen as dg
from latency_decode_b200 import dl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not helpers.gpu_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def lib():
    dl_build.build()
    return dl.lib()


def pack(w: np.ndarray, kind: int):
    N, K = w.shape
    wd = dev_u8(w)
    wp = torch.empty_like(wd)
    dl.check(dl.dl_pack_fp8_weight(wd, wp, N, K, kind))
    return wp


def run_fc13(x, w, s_w, flags=dl.DL_FLAG_PDL, split=0, wp=None):
    M, K = x.shape
    N2 = w.shape[0]
    wp = pack(w, dl.DL_PACK_SWIGLU) if wp is None else wp
    out = torch.full((M, N2 // 2), -1, dtype=torch.int16, device="cuda")
    ws, n = new_ws(M, K)
    dl.check(dl.dl_fc13_swiglu(dev_u16(x), M, K, wp, dev_f32(s_w), N2, out, ws, n,
                               flags=flags | (split << dl.DL_FLAG_SPLIT_SHIFT)))
    dl.check(dl.dl_read_status(ws))
    return host_u16(out), ws.cpu().numpy()


def run_qkv(x, w, s_w, Hq, Hkv, d, q_scale, flags=dl.DL_FLAG_PDL, split=0):
    M, K = x.shape
    N = w.shape[0]
    wp = pack(w, dl.DL_PACK_PLAIN)
    out = torch.full((M, N), -1, dtype=torch.int16, device="cuda")
    ws, n = new_ws(M, K)
    dl.check(dl.dl_fc_qkv_scale(dev_u16(x), M, K, wp, dev_f32(s_w), Hq, Hkv, d, q_scale, out, ws, n,
                                flags=flags | (split << dl.DL_FLAG_SPLIT_SHIFT)))
    dl.check(dl.dl_read_status(ws))
    return host_u16(out), ws.cpu().numpy()


@pytest.mark.parametrize("N,K,kind", [(512, 384, 0), (512, 384, 1), (256, 128, 1), (7168, 5120, 0),
                                      (16384, 5120, 1)])
def test_pack_matches_stated_layout(N, K, kind):
    g = np.random.default_rng(N + K + kind)
    w = g.integers(0, 256, size=(N, K)).astype(np.uint8)
    got = pack(w, kind).cpu().numpy().ravel()
    assert np.array_equal(got, helpers.pack_reference(w, kind))


@pytest.mark.parametrize("M,K", [(1, 512), (3, 256), (4, 5120), (64, 5120), (17, 1280)])
def test_act_quant_codes_and_scale_bit_exact(M, K):
    g = np.random.default_rng(100 + M)
    x = dg.bf16_normal(g, (M, K))
    x[0, :3] = dg.bf16_bits(np.float32([0.0, -0.0, 1e-30]))  # zeros and an underflowing value
    w, s_w = dg.e4m3_weight(g, 256, K)
    _, ws = run_fc13(x, w, s_w)
    xq_ref, sx_ref = oracle.act_quant(x)
    xq = ws[256:256 + M * K].reshape(M, K)
    sx = ws[8:12].view(np.float32)[0]
    assert sx == sx_ref
    mism = np.argwhere(xq != xq_ref)
    assert mism.size == 0, f"{len(mism)} codes differ, first {mism[:5].tolist()}"


@pytest.mark.parametrize("M,split", [(2, 2), (2, 3), (3, 4), (4, 4), (5, 5), (4, 8), (6, 8), (1, 4)])
def test_cooperative_quantiser_codes_bit_exact(M, split):
    """The fused quantiser at M*K > 8192 with a split-K cluster: each CTA loads
    only its K slice and the cluster exchanges the slice maxima (uneven slices
    at 3 and 5 CTAs; M = 1 takes the whole-x path).  The published codes and
    s_x are bit-exact against the oracle's, and the GEMM output holds the GEMM
    rule."""
    K, N2 = 5120, 512
    g = np.random.default_rng(400 + 10 * M + split)
    x = dg.bf16_normal(g, (M, K))
    x[M - 1, K - 5:] = dg.bf16_bits(np.float32([0.0, -0.0, 1e-30, 30.0, -2.0]))  # the maximum in the last slice
    w, s_w = dg.e4m3_weight(g, N2, K)
    out, ws = run_fc13(x, w, s_w, split=split)
    xq_ref, sx_ref = oracle.act_quant(x)
    assert ws[8:12].view(np.float32)[0] == sx_ref
    xq = ws[256:256 + M * K].reshape(M, K)
    mism = np.argwhere(xq != xq_ref)
    assert mism.size == 0, f"{len(mism)} codes differ, first {mism[:5].tolist()}"
    helpers.check_gemm(out, oracle.fc13_swiglu(x, w, s_w), f"cooperative quantiser M={M} split={split}")


def test_act_quant_all_zero_input():
    x = np.zeros((2, 256), dtype=np.uint16)
    g = np.random.default_rng(5)
    w, s_w = dg.e4m3_weight(g, 256, 256)
    out, ws = run_fc13(x, w, s_w)
    assert ws[8:12].view(np.float32)[0] == 1.0
    assert not ws[256:256 + 512].any()
    assert not helpers.bf16_to_f64(out).any()


def test_fc13_tiny_workload():
    wl = dg.WORKLOADS["tiny"]
    inp = dg.dense_layer_inputs(wl, with_kv=False)
    out, _ = run_fc13(inp["x2"], inp["w13"], inp["s13"])
    ref = oracle.fc13_swiglu(inp["x2"], inp["w13"], inp["s13"])
    helpers.check_gemm(out, ref, "fc13 tiny")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 7, 8, 9, 16, 33, 64])
def test_fc13_ragged_m(M):
    g = np.random.default_rng(200 + M)
    K, N2 = 1280, 768
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N2, K)
    out, _ = run_fc13(x, w, s_w)
    helpers.check_gemm(out, oracle.fc13_swiglu(x, w, s_w), f"fc13 M={M}")


@pytest.mark.parametrize("split", [1, 2, 3, 4, 5, 7, 8])
def test_fc13_split_k_cluster_sizes(split):
    g = np.random.default_rng(300 + split)
    M, K, N2 = 5, 1024, 512
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N2, K)
    out, _ = run_fc13(x, w, s_w, split=split)
    helpers.check_gemm(out, oracle.fc13_swiglu(x, w, s_w), f"fc13 split={split}")


@pytest.mark.parametrize("M,split", [(7, 0), (13, 3), (40, 5), (64, 1), (64, 8)])
def test_fc13_streamed_activations_by_tensor_loads(M, split):
    # M*K > 32768: x is quantised by its own kernel and each k-block of x_q
    # reaches the GEMM by one tensor load (padding rows M..npad-1 zero-filled
    # by the copy), over uneven split-K slices and a B ring that wraps 10 times
    # at split 1
    g = np.random.default_rng(600 + M + split)
    K, N2 = 5120, 512
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N2, K)
    out, _ = run_fc13(x, w, s_w, split=split)
    helpers.check_gemm(out, oracle.fc13_swiglu(x, w, s_w), f"fc13 streamed B M={M} split={split}")


def test_fc13_pdl_flag_does_not_change_bits():
    g = np.random.default_rng(7)
    x = dg.bf16_normal(g, (4, 512))
    w, s_w = dg.e4m3_weight(g, 512, 512)
    a, _ = run_fc13(x, w, s_w, flags=dl.DL_FLAG_PDL)
    b, _ = run_fc13(x, w, s_w, flags=0)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("wl_name", ["layer_b1", "verify4"])
def test_fc13_full_size(wl_name):
    wl = dg.WORKLOADS[wl_name]
    inp = dg.dense_layer_inputs(wl, with_kv=False)
    out, _ = run_fc13(inp["x2"], inp["w13"], inp["s13"])
    ref = oracle.fc13_swiglu(inp["x2"], inp["w13"], inp["s13"])
    helpers.check_gemm(out, ref, f"fc13 {wl_name}")


def test_fc13_batch16x4_sampled_columns():
    """M=64 at full weight size; the oracle computes a sample of 512 output
    columns (their gate and up rows), with the same shared activation scale."""
    wl = dg.WORKLOADS["batch16x4"]
    inp = dg.dense_layer_inputs(wl, with_kv=False)
    x, w, s_w = inp["x2"], inp["w13"], inp["s13"]
    out, _ = run_fc13(x, w, s_w)
    F = w.shape[0] // 2
    cols = np.sort(np.random.default_rng(1).choice(F, size=512, replace=False))
    xq, sx = oracle.act_quant(x)
    sub = np.concatenate([w[cols], w[F + cols]])
    ref = oracle.fc13_swiglu_q(xq, sx, sub, s_w)
    helpers.check_gemm(out[:, cols], ref, "fc13 M=64 sampled")


@pytest.mark.parametrize("M,Hq,Hkv,d,K", [(1, 8, 2, 64, 512), (3, 4, 2, 128, 384), (16, 2, 1, 64, 256)])
def test_qkv_small(M, Hq, Hkv, d, K):
    g = np.random.default_rng(400 + M)
    N = (Hq + 2 * Hkv) * d
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N, K)
    qs = np.float32(1.0 / np.sqrt(d))
    out, _ = run_qkv(x, w, s_w, Hq, Hkv, d, qs)
    ref = oracle.fc_qkv_scale(x, w, s_w, Hq, Hkv, d, qs)
    helpers.check_gemm(out, ref, f"qkv M={M}")
    # the scaling touches the Q columns only: unscaled run differs exactly there
    out1, _ = run_qkv(x, w, s_w, Hq, Hkv, d, 1.0)
    assert np.array_equal(out1[:, Hq * d:], out[:, Hq * d:])


@pytest.mark.parametrize("wl_name", ["layer_b1", "verify4", "batch16x4"])
def test_qkv_full_size(wl_name):
    wl = dg.WORKLOADS[wl_name]
    inp = dg.dense_layer_inputs(wl, with_kv=False)
    out, _ = run_qkv(inp["x1"], inp["w_qkv"], inp["s_qkv"], wl.Hq, wl.Hkv, wl.d, inp["q_scale"])
    ref = oracle.fc_qkv_scale(inp["x1"], inp["w_qkv"], inp["s_qkv"], wl.Hq, wl.Hkv, wl.d, inp["q_scale"])
    helpers.check_gemm(out, ref, f"qkv {wl_name}")
