"""GPU tests of the copy kernel (dl_copy) that keeps a step's host transfers
inside its PDL chain: device->device, pinned host->device and device->pinned
host, bit-exact, several sizes; chained under PDL ahead of a GEMM that reads
what it copied; and a whole decode step from pinned host memory to pinned host
memory (DecodeLayer.step_host) equal to the same step on device buffers."""
import math

import numpy as np
import pytest
import torch

import helpers
from helpers import dev_f32, dev_u8, new_ws
from latency_decode_b200 import build as dl_build
from latency_decode_b200 import datagen as dg
from latency_decode_b200 import dl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not helpers.gpu_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def lib():
    dl_build.build()
    return dl.lib()


@pytest.mark.parametrize("nbytes", [16, 4096 + 16, 20480, 1 << 20, 3 * (1 << 20) + 48])
@pytest.mark.parametrize("route", ["d2d", "h2d", "d2h"])
def test_copy_is_exact(nbytes, route):
    g = np.random.default_rng(nbytes % 1000)
    src_np = g.integers(0, 256, size=nbytes, dtype=np.uint8)
    src = torch.from_numpy(src_np)
    src = src.pin_memory() if route == "h2d" else src.cuda()
    dst = torch.zeros(nbytes, dtype=torch.uint8)
    dst = dst.pin_memory() if route == "d2h" else dst.cuda()
    dl.check(dl.dl_copy(src, dst, nbytes))
    torch.cuda.synchronize()
    assert np.array_equal(dst.cpu().numpy(), src_np)


def test_zero_bytes_launch_nothing():
    a = torch.zeros(16, dtype=torch.uint8, device="cuda")
    b = torch.ones(16, dtype=torch.uint8, device="cuda")
    dl.check(dl.dl_copy(a, b, 0))
    torch.cuda.synchronize()
    assert (b.cpu().numpy() == 1).all()


def test_pdl_chain_copy_then_gemm_reads_the_copied_input():
    """host -> device copy kernel, then FC13 under PDL reading what was copied;
    equals the same GEMM on a device-resident input."""
    import oracle
    g = np.random.default_rng(3)
    M, K, N2 = 1, 1024, 512
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N2, K)
    wp = torch.empty((N2, K), dtype=torch.uint8, device="cuda")
    dl.check(dl.dl_pack_fp8_weight(dev_u8(w), wp, N2, K, dl.DL_PACK_SWIGLU))
    hx = torch.from_numpy(x.view(np.int16)).pin_memory()
    dx = torch.full((M, K), 7, dtype=torch.int16, device="cuda")
    out = torch.empty((M, N2 // 2), dtype=torch.int16, device="cuda")
    ws, n = new_ws(M, K)
    for _ in range(3):  # repeated chains on one stream
        dl.check(dl.dl_copy(hx, dx, M * K * 2))
        dl.check(dl.dl_fc13_swiglu(dx, M, K, wp, dev_f32(s_w), N2, out, ws, n))
    assert dl.dl_read_status(ws) == dl.DL_OK
    helpers.check_gemm(helpers.host_u16(out), oracle.fc13_swiglu(x, w, s_w), "copy -> fc13")


def test_step_host_equals_device_step():
    from latency_decode_b200.layer import DecodeLayer
    wl = dg.WORKLOADS["tiny"]
    inp = dg.dense_layer_inputs(wl)
    lay = DecodeLayer(dev_u8(inp["w_qkv"]), inp["s_qkv"], dev_u8(inp["w13"]), inp["s13"], Hq=wl.Hq, Hkv=wl.Hkv,
                      d=wl.d, q_scale=inp["q_scale"], M=wl.M, B=wl.B, T=wl.T, cluster=wl.cluster)
    kc = helpers.dev_u16(inp["k_cache"])
    vc = helpers.dev_u16(inp["v_cache"])
    sl = helpers.dev_i32(inp["seq_lens"])
    x1, x2 = helpers.dev_u16(inp["x1"]), helpers.dev_u16(inp["x2"])
    lay.step(x1, x2, kc, vc, sl)
    ref = lay.out_buf.clone()
    hx = torch.stack([x1, x2]).cpu().pin_memory()
    hout = torch.zeros_like(lay.out_buf, device="cpu").pin_memory()
    lay.out_buf.zero_()
    lay.step_host(hx, hout, kc, vc, sl)
    torch.cuda.synchronize()
    lay.read_status()
    assert torch.equal(hout, ref.cpu())
