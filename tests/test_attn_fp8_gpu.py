"""GPU parity of split-KV decode attention over an FP8 (e4m3) KV cache through
the C ABI against the CPU oracle (oracle.decode_attn_fp8kv): the named
workloads at full size, every cluster size (both the one-CTA-per-SM and the
two-CTAs-per-SM variants), 1..4 query-row tiles, ragged and minimal lengths,
clusters per head merged through the workspace, q read in place from a QKV
row.  The cache holds K as [key][d] and V transposed as [d][key]; Lcap is a
multiple of 16.  Tolerance: relative L2 <= 5e-3 (as for the bf16 cache; the
device rounds q and the probabilities to f16, the oracle stays in double)."""
import math

import numpy as np
import pytest
import torch

import helpers
import oracle
from helpers import dev_f32, dev_i32, dev_u8, dev_u16, host_u16
from latency_decode_b200 import build as dl_build
from latency_decode_b200 import datagen as dg
from latency_decode_b200 import dl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not helpers.gpu_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def lib():
    dl_build.build()
    return dl.lib()


def fp8_cache(g, shape, transpose=False):
    """e4m3 codes of N(0,1) values with a per-tensor scale; transpose=True stores
    [B, Hkv, Lcap, d] as [B, Hkv, d, Lcap] (the V^T layout)."""
    codes, s = dg.e4m3_codes_from_f32(g.standard_normal(size=shape, dtype=np.float32))
    if transpose:
        codes = np.ascontiguousarray(codes.transpose(0, 1, 3, 2))
    return codes, np.float32(s)


def run(q_flat, q_stride, B, T, Hq, Hkv, d, kc, vc, s_k, s_v, seq_lens, scale, cluster, splits=0,
        expect=dl.DL_OK):
    Lcap = kc.shape[2]
    out = torch.full((B, T, Hq, d), -1, dtype=torch.int16, device="cuda")
    n = dl.dl_decode_attn_fp8kv_workspace_bytes(B, T, Hq, Hkv, d, Lcap, cluster)
    flags = dl.DL_FLAG_PDL
    if splits:
        n = max(n, 256 + 4096 + 2 * 65536 + B * Hkv * splits * (Hq // Hkv) * T * d * 4 + 65536)
        flags |= splits << dl.DL_FLAG_SPLIT_SHIFT
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    dl.check(dl.dl_decode_attn_fp8kv(dev_u16(q_flat), q_stride, B, T, Hq, Hkv, d, dev_u8(kc), dev_u8(vc),
                                     dev_f32([s_k, s_v]), Lcap, dev_i32(seq_lens), scale, cluster, out, ws, n,
                                     flags=flags))
    assert dl.dl_read_status(ws) == expect
    return host_u16(out)


def check(seed, B, T, Hq, Hkv, Lcap, seq_lens, cluster, splits=0, scale=None):
    d = 128
    g = np.random.default_rng(seed)
    q = dg.bf16_normal(g, (B, T, Hq, d))
    kc, s_k = fp8_cache(g, (B, Hkv, Lcap, d))
    vc, s_v = fp8_cache(g, (B, Hkv, Lcap, d), transpose=True)
    sl = np.asarray(seq_lens, dtype=np.int32)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    got = run(q.ravel(), Hq * d, B, T, Hq, Hkv, d, kc, vc, s_k, s_v, sl, scale, cluster, splits)
    ref = oracle.decode_attn_fp8kv(q.ravel(), Hq * d, B, T, Hq, Hkv, d, kc, vc, sl, scale, s_k, s_v)
    return helpers.check_attn(got, ref, f"fp8kv B={B} T={T} Hq={Hq} Hkv={Hkv} L={seq_lens} S={cluster} P={splits}")


@pytest.mark.parametrize("name", ["layer_b1", "verify4"])
def test_workloads_full_size(name):
    wl = dg.WORKLOADS[name]
    check(900 + wl.seed, wl.B, wl.T, wl.Hq, wl.Hkv, wl.Lcap, [wl.L], wl.cluster)


def test_batch16x4_full_size_sampled_sequences():
    wl = dg.WORKLOADS["batch16x4"]
    g = np.random.default_rng(903)
    sl = dg.seq_lens_for(wl, g)
    d = wl.d
    q = dg.bf16_normal(g, (wl.B, wl.T, wl.Hq, d))
    kc, s_k = fp8_cache(g, (wl.B, wl.Hkv, wl.Lcap, d))
    vc, s_v = fp8_cache(g, (wl.B, wl.Hkv, wl.Lcap, d), transpose=True)
    got = run(q.ravel(), wl.Hq * d, wl.B, wl.T, wl.Hq, wl.Hkv, d, kc, vc, s_k, s_v, sl, 1 / math.sqrt(d),
              wl.cluster).reshape(wl.B, wl.T, wl.Hq, d)
    for b in (0, 7, 15):
        ref = oracle.decode_attn_fp8kv(q[b:b + 1].ravel(), wl.Hq * d, 1, wl.T, wl.Hq, wl.Hkv, d, kc[b:b + 1],
                                       vc[b:b + 1], sl[b:b + 1], 1 / math.sqrt(d), s_k, s_v)
        helpers.check_attn(got[b:b + 1], ref, f"fp8kv batch16x4 seq {b}")


@pytest.mark.parametrize("cluster", [1, 2, 4, 8, 16])
def test_cluster_sizes_ragged(cluster):
    check(910 + cluster, 2, 2, 10, 2, 704, [700, 333], cluster)


@pytest.mark.parametrize("G,T", [(1, 1), (5, 1), (8, 1), (3, 3), (5, 4), (8, 4)])
def test_query_row_tiles(G, T):
    check(920 + G * T, 1, T, G * 2, 2, 304, [300], 8)


@pytest.mark.parametrize("L", [1, 15, 17, 64, 129, 1000])
def test_lengths(L):
    check(930 + L, 1, 1, 4, 1, 1024, [L], 16)


@pytest.mark.parametrize("splits", [2, 3, 5])
def test_clusters_per_head(splits):
    check(940 + splits, 2, 4, 10, 2, 2000, [2000, 731], 8, splits=splits)


def test_q_in_place_from_qkv_row_and_scales_matter():
    g = np.random.default_rng(950)
    B, T, Hq, Hkv, d, L = 2, 2, 8, 2, 128, 208
    W = (Hq + 2 * Hkv) * d
    wide = dg.bf16_normal(g, (B * T, W), std=0.1)
    kc, s_k = fp8_cache(g, (B, Hkv, L, d))
    vc, s_v = fp8_cache(g, (B, Hkv, L, d), transpose=True)
    sl = np.int32([200, 150])
    got = run(wide.ravel(), W, B, T, Hq, Hkv, d, kc, vc, s_k, s_v, sl, 1.0, 8)
    ref = oracle.decode_attn_fp8kv(wide.ravel(), W, B, T, Hq, Hkv, d, kc, vc, sl, 1.0, s_k, s_v)
    helpers.check_attn(got, ref, "fp8kv q in qkv row")
    got2 = run(wide.ravel(), W, B, T, Hq, Hkv, d, kc, vc, s_k, 2 * s_v, sl, 1.0, 8)  # s_v is linear
    assert helpers.rel_l2(helpers.bf16_to_f64(got2), 2 * helpers.bf16_to_f64(got)) < 1e-2


def test_bad_seq_len_is_reported_on_device():
    g = np.random.default_rng(951)
    q = dg.bf16_normal(g, (2, 2, 4, 128))
    kc, s_k = fp8_cache(g, (2, 1, 128, 128))
    out = run(q.ravel(), 4 * 128, 2, 2, 4, 1, 128, kc, np.ascontiguousarray(kc.transpose(0, 1, 3, 2)), s_k, s_k,
              np.int32([1, 200]), 0.1, 8, expect=dl.DL_ERR_DEVICE_ARG)
    assert not helpers.bf16_to_f64(out).any()


def test_many_heads_use_the_two_ctas_per_sm_variant():
    """B*Hkv*S = 12*8*4 = 384 CTAs > SMs: the W = 4, two-CTAs-per-SM variant
    (64-byte V^T rows, 64-byte swizzle)."""
    g = np.random.default_rng(960)
    sl = g.integers(64, 2048, size=12).astype(np.int32)
    check(961, 12, 2, 16, 8, 2048, sl.tolist(), 4)
