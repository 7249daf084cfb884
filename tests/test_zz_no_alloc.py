"""dl_fc13_swiglu_static_ws: FC13 + SwiGLU for callers that cannot allocate
device memory (a plugin given only its inputs and outputs, an engine whose
memory pool is fixed at start-up, a loop where cudaMalloc would synchronise
the device).  Its activation scratch is a fixed array inside libdl.so instead
of a caller workspace.

Checked through the C ABI against dl_fc13_swiglu (which uses a caller
workspace) on two calls in a row with different inputs, so the second call
must fully replace what the first left in the shared array.  The tolerance is
the one the GEMM parity tests use.  Kept in a file that pytest collects last."""
import numpy as np
import pytest
import torch

import helpers
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


def test_static_scratch_variant_matches_workspace_variant_twice_in_a_row():
    g = np.random.default_rng(2024)
    M, K, N2 = 4, 5120, 2048
    w, s_w = dg.e4m3_weight(g, N2, K)
    wd = dev_u8(w)
    wp = torch.empty_like(wd)
    dl.check(dl.dl_pack_fp8_weight(wd, wp, N2, K, dl.DL_PACK_SWIGLU))
    sw = dev_f32(s_w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        x = dg.bf16_normal(g, (M, K), std=1.0 + call)  # a different input (and scale) each call
        xd = dev_u16(x)
        ref_out = torch.empty((M, N2 // 2), dtype=torch.int16, device="cuda")
        ws, n = new_ws(M, K)
        dl.check(dl.dl_fc13_swiglu(xd, M, K, wp, sw, N2, ref_out, ws, n))
        dl.check(dl.dl_read_status(ws))
        out = torch.full((M, N2 // 2), -1, dtype=torch.int16, device="cuda")
        dl.check(dl.dl_fc13_swiglu_static_ws(xd, M, K, wp, sw, N2, out, status))
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = helpers.bf16_to_f64(host_u16(ref_out))
        helpers.check_gemm(host_u16(out), ref, f"static scratch, call {call}")


def test_static_scratch_rejects_sizes_beyond_its_array():
    # M*K above 64*8192 bytes, or M above 64: refused before any launch
    assert dl.dl_fc13_swiglu_static_ws(1 << 20, 64, 8320, 1 << 20, 1 << 20, 256, 1 << 20) == dl.DL_ERR_WORKSPACE
    assert dl.dl_fc13_swiglu_static_ws(1 << 20, 65, 128, 1 << 20, 1 << 20, 256, 1 << 20) == dl.DL_ERR_WORKSPACE
