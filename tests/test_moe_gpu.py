"""GPU parity of the grouped MoE expert FC13+SwiGLU (top-1, routing on the
device) through the C ABI against the CPU oracle: small banks with full
checks (one expert, every token on one expert, every token on its own expert,
random routes), the full 64-token x 128-expert bank with sampled columns, and a
bad expert id reported on the device."""
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


def pack_bank(w_bank: torch.Tensor, N2: int, K: int) -> torch.Tensor:
    E = w_bank.shape[0]
    out = torch.empty_like(w_bank)
    for e in range(E):
        dl.check(dl.dl_pack_fp8_weight(w_bank[e], out[e], N2, K, dl.DL_PACK_SWIGLU))
    return out


def run_moe(x, ids, wp_bank, s_w, N2, flags=dl.DL_FLAG_PDL, split=0, expect=dl.DL_OK):
    T, K = x.shape
    E = wp_bank.shape[0]
    out = torch.full((T, N2 // 2), -1, dtype=torch.int16, device="cuda")
    ws, n = new_ws(T, K)
    dl.check(dl.dl_moe_fc13_swiglu_grouped(dev_u16(x), T, K, dev_i32(ids), E, wp_bank, dev_f32(s_w), N2, out, ws,
                                           n, flags=flags | (split << dl.DL_FLAG_SPLIT_SHIFT)))
    assert dl.dl_read_status(ws) == expect
    return host_u16(out)


def small_bank(seed, E, N2, K):
    g = np.random.default_rng(seed)
    ws, scales = zip(*(dg.e4m3_weight(g, N2, K) for _ in range(E)))
    return np.stack(ws), np.array(scales, dtype=np.float32), g


@pytest.mark.parametrize("T,E,route", [(1, 1, "random"), (5, 3, "random"), (64, 16, "random"),
                                       (64, 4, "same"), (16, 16, "distinct"), (9, 40, "random"),
                                       (33, 1024, "random")])
def test_moe_small_banks(T, E, route):
    K, N2 = 512, 512
    w, s_w, g = small_bank(T * 1000 + E, E, N2, K)
    x = dg.bf16_normal(g, (T, K))
    if route == "same":
        ids = np.full(T, E - 1, dtype=np.int32)
    elif route == "distinct":
        ids = g.permutation(E)[:T].astype(np.int32)
    else:
        ids = g.integers(0, E, size=T).astype(np.int32)
    wp = pack_bank(dev_u8(w), N2, K)
    got = run_moe(x, ids, wp, s_w, N2)
    ref = oracle.moe_fc13_swiglu(x, ids, w, s_w)
    helpers.check_gemm(got, ref, f"moe T={T} E={E} {route}")


@pytest.mark.parametrize("split", [1, 2, 4, 8])
def test_moe_split_sizes(split):
    T, E, K, N2 = 12, 5, 1024, 768
    w, s_w, g = small_bank(77 + split, E, N2, K)
    x = dg.bf16_normal(g, (T, K))
    ids = g.integers(0, E, size=T).astype(np.int32)
    got = run_moe(x, ids, pack_bank(dev_u8(w), N2, K), s_w, N2, split=split)
    helpers.check_gemm(got, oracle.moe_fc13_swiglu(x, ids, w, s_w), f"moe split={split}")


def test_moe64_full_bank_sampled_columns():
    """64 tokens, 128 experts of [16384, 5120] e4m3 (10.7 GB, drawn on the device
    with a seeded torch generator), top-1 uniform routes.  The oracle checks 96
    output columns of every token against that token's expert rows."""
    wl = dg.WORKLOADS["moe64"]
    g = dg.rng(wl.seed)
    x = dg.bf16_normal(g, (wl.M, wl.K))
    ids = dg.expert_ids_for(wl, g)
    gen = torch.Generator(device="cuda").manual_seed(wl.seed)
    bank = torch.empty((wl.experts, wl.N2, wl.K), dtype=torch.uint8, device="cuda")
    s_w = np.zeros(wl.experts, dtype=np.float32)
    for e in range(wl.experts):
        codes, s = dg.e4m3_weight_torch(gen, wl.N2, wl.K, "cuda")
        bank[e].copy_(codes)
        s_w[e] = s
    wp = pack_bank(bank, wl.N2, wl.K)
    got = run_moe(x, ids, wp, s_w, wl.N2)
    del wp
    F = wl.N2 // 2
    cols = np.sort(np.random.default_rng(2).choice(F, size=96, replace=False))
    xq, sx = oracle.act_quant(x)
    rows = torch.from_numpy(np.concatenate([cols, F + cols])).cuda()
    for t in range(wl.M):
        e = int(ids[t])
        sub = bank[e].index_select(0, rows).cpu().numpy()
        ref = oracle.fc13_swiglu_q(xq[t:t + 1], sx, sub, s_w[e])
        helpers.check_gemm(got[t:t + 1, cols], ref, f"moe64 token {t} expert {e}")
    assert len(np.unique(ids)) > 30  # a real spread of touched experts


def test_moe_bad_expert_id_is_reported():
    T, E, K, N2 = 4, 3, 256, 256
    w, s_w, g = small_bank(5, E, N2, K)
    x = dg.bf16_normal(g, (T, K))
    ids = np.int32([0, 1, 7, 2])
    run_moe(x, ids, pack_bank(dev_u8(w), N2, K), s_w, N2, expect=dl.DL_ERR_DEVICE_ARG)
