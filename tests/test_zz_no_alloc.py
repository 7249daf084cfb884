"""dl_fc13_swiglu_static_ws: FC13 + SwiGLU for callers that cannot allocate
device memory (a plugin given only its inputs and outputs, an engine whose
memory pool is fixed at start-up, a loop where cudaMalloc would synchronise
the device).  Its activation scratch is a fixed array inside libdl.so instead
of a caller workspace.

Each case runs two calls in a row with different inputs (and activation
scales), so the second call must fully replace what the first left in the
shared array.  Each output is checked against the CPU oracle on the same e4m3
weight bytes and scale, with the GEMM tolerances of every other GEMM test, and
against dl_fc13_swiglu (the caller-workspace entry point) as well.  The shapes
cover the quantiser fused into the GEMM (M*K <= 32768), the separate cluster
quantiser, an odd M that pads the token dimension, and M = 64, K = 8192, which
fills the array exactly.  Kept in a file that pytest collects last."""
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


@pytest.mark.parametrize("M,K,N2", [(1, 5120, 2048), (3, 4096, 1024), (4, 5120, 2048), (16, 4096, 768),
                                    (64, 8192, 512)])
def test_static_scratch_variant_matches_the_oracle_twice_in_a_row(M, K, N2):
    g = np.random.default_rng(2024 + M)
    w, s_w = dg.e4m3_weight(g, N2, K)
    wd = dev_u8(w)
    wp = torch.empty_like(wd)
    dl.check(dl.dl_pack_fp8_weight(wd, wp, N2, K, dl.DL_PACK_SWIGLU))
    sw = dev_f32(s_w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        x = dg.bf16_normal(g, (M, K), std=1.0 + call)  # a different input (and scale) each call
        xd = dev_u16(x)
        out = torch.full((M, N2 // 2), -1, dtype=torch.int16, device="cuda")
        dl.check(dl.dl_fc13_swiglu_static_ws(xd, M, K, wp, sw, N2, out, status))
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = host_u16(out)
        helpers.check_gemm(got, oracle.fc13_swiglu(x, w, s_w), f"static scratch M={M} K={K}, call {call}")
        ws_out = torch.empty((M, N2 // 2), dtype=torch.int16, device="cuda")
        ws, n = new_ws(M, K)
        dl.check(dl.dl_fc13_swiglu(xd, M, K, wp, sw, N2, ws_out, ws, n))
        dl.check(dl.dl_read_status(ws))
        helpers.check_gemm(got, helpers.bf16_to_f64(host_u16(ws_out)), f"vs workspace variant, call {call}")


def test_static_scratch_rejects_sizes_beyond_its_array():
    # M*K above 64*8192 bytes, or M above 64: refused before any launch
    assert dl.dl_fc13_swiglu_static_ws(1 << 20, 64, 8320, 1 << 20, 1 << 20, 256, 1 << 20) == dl.DL_ERR_WORKSPACE
    assert dl.dl_fc13_swiglu_static_ws(1 << 20, 65, 128, 1 << 20, 1 << 20, 256, 1 << 20) == dl.DL_ERR_WORKSPACE
