"""GPU parity of split-KV decode attention (cluster DSMEM merge) through the C
ABI against the CPU oracle: the named workloads at full size, every cluster
size, both head dims, 1..4 query-row tiles, ragged and minimal lengths, empty
chunks, q read in place from a fused QKV row.  Tolerance: relative L2 <= 5e-3."""
import math

import numpy as np
import pytest
import torch

import helpers
import oracle
from helpers import dev_i32, dev_u16, host_u16, new_ws
from latency_decode_b200 import build as dl_build
from latency_decode_b200 import datagen as dg
from latency_decode_b200 import dl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not helpers.gpu_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def lib():
    dl_build.build()
    return dl.lib()


def run_attn(q_flat, q_stride, B, T, Hq, Hkv, d, k, v, seq_lens, scale, cluster, flags=dl.DL_FLAG_PDL,
             expect=dl.DL_OK, splits=0):
    Lcap = k.shape[2]
    out = torch.full((B, T, Hq, d), -1, dtype=torch.int16, device="cuda")
    n = dl.dl_decode_attn_workspace_bytes(B, T, Hq, Hkv, d, Lcap, cluster)
    if splits:
        n = max(n, 256 + 4096 + 2 * 65536 + B * Hkv * splits * (Hq // Hkv) * T * d * 4 + 65536)
        flags |= splits << dl.DL_FLAG_SPLIT_SHIFT
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    dl.check(dl.dl_decode_attn(dev_u16(q_flat), q_stride, B, T, Hq, Hkv, d, dev_u16(k), dev_u16(v), Lcap,
                               dev_i32(seq_lens), scale, cluster, out, ws, n, flags=flags))
    assert dl.dl_read_status(ws) == expect
    return host_u16(out)


def case(seed, B, T, Hq, Hkv, d, Lcap, seq_lens):
    g = np.random.default_rng(seed)
    q = dg.bf16_normal(g, (B, T, Hq, d))
    k = dg.bf16_normal(g, (B, Hkv, Lcap, d))
    v = dg.bf16_normal(g, (B, Hkv, Lcap, d))
    return q, k, v, np.asarray(seq_lens, dtype=np.int32)


def check(seed, B, T, Hq, Hkv, d, Lcap, seq_lens, cluster, scale=None, splits=0):
    q, k, v, sl = case(seed, B, T, Hq, Hkv, d, Lcap, seq_lens)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    got = run_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, scale, cluster, splits=splits)
    ref = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, scale)
    return helpers.check_attn(got, ref, f"B={B} T={T} Hq={Hq} Hkv={Hkv} d={d} L={seq_lens} S={cluster}")


def test_tiny_workload():
    wl = dg.WORKLOADS["tiny"]
    check(wl.seed, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, wl.Lcap, [wl.L], wl.cluster)


@pytest.mark.parametrize("cluster", [8, 16])
def test_layer_b1_full(cluster):
    wl = dg.WORKLOADS["layer_b1"]
    check(wl.seed, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, wl.Lcap, [wl.L], cluster)


@pytest.mark.parametrize("cluster", [8, 16])
def test_verify4_full(cluster):
    wl = dg.WORKLOADS["verify4"]
    check(wl.seed, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, wl.Lcap, [wl.L], cluster)


def test_batch16x4_full_size_sampled_sequences():
    """16 sequences with lengths drawn in [1024, 16384]; the GPU computes all of
    them, the oracle checks the longest and the shortest drawn sequence, the
    first and the last, and two more."""
    wl = dg.WORKLOADS["batch16x4"]
    g = dg.rng(wl.seed)
    sl = dg.seq_lens_for(wl, g)
    q, k, v, _ = case(wl.seed, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, wl.Lcap, sl)
    scale = 1.0 / math.sqrt(wl.d)
    got = run_attn(q.ravel(), wl.Hq * wl.d, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, k, v, sl, scale, wl.cluster)
    got = got.reshape(wl.B, wl.T, wl.Hq, wl.d)
    picks = [int(np.argmax(sl)), int(np.argmin(sl)), 0, wl.B - 1, 5, 10]
    picks = sorted(set(picks))
    assert int(np.argmax(sl)) in picks and len(picks) >= 4
    for b in picks:
        ref = oracle.decode_attn(q[b:b + 1].ravel(), wl.Hq * wl.d, 1, wl.T, wl.Hq, wl.Hkv, wl.d, k[b:b + 1],
                                 v[b:b + 1], sl[b:b + 1], scale)
        helpers.check_attn(got[b:b + 1], ref, f"batch16x4 seq {b} L={sl[b]}")


@pytest.mark.parametrize("cluster", [1, 2, 4, 8, 16])
def test_cluster_sizes_ragged(cluster):
    check(10 + cluster, 2, 2, 10, 2, 128, 700, [700, 333], cluster)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G,T", [(1, 1), (5, 1), (8, 1), (3, 3), (4, 4), (5, 4), (6, 4), (8, 4)])
def test_query_row_tiles(d, G, T):
    # R = G*T query rows per kv head: 1, 5, 8, 9, 16, 20, 24, 32 -> 1..4 row tiles
    check(20 + G * T + d, 1, T, G * 2, 2, d, 300, [300], 8)


@pytest.mark.parametrize("L", [1, 2, 15, 16, 17, 63, 64, 65, 129, 1000])
def test_lengths_ragged_and_minimal(L):
    T = 1
    check(30 + L, 1, T, 4, 1, 64, 1024, [L], 16)


def test_minimal_length_equals_tokens_causal():
    check(41, 1, 4, 8, 2, 128, 64, [4], 8)  # L == T: query t sees keys 0..t
    check(42, 3, 4, 8, 2, 128, 64, [4, 37, 64], 4)


def test_empty_chunks_in_large_cluster():
    # L=20 with 16 CTAs: chunks of 16 keys, CTAs 2..15 see nothing
    check(43, 1, 1, 8, 1, 128, 64, [20], 16)


def test_q_read_in_place_from_qkv_row_with_unit_scale():
    g = np.random.default_rng(44)
    B, T, Hq, Hkv, d, L = 2, 2, 8, 2, 128, 200
    W = (Hq + 2 * Hkv) * d
    wide = dg.bf16_normal(g, (B * T, W), std=0.1)
    k = dg.bf16_normal(g, (B, Hkv, L, d))
    v = dg.bf16_normal(g, (B, Hkv, L, d))
    sl = np.int32([L, 150])
    got = run_attn(wide.ravel(), W, B, T, Hq, Hkv, d, k, v, sl, 1.0, 8)
    ref = oracle.decode_attn(wide.ravel(), W, B, T, Hq, Hkv, d, k, v, sl, 1.0)
    helpers.check_attn(got, ref, "q in qkv row")


def test_identical_keys_give_mean_of_values():
    g = np.random.default_rng(45)
    B, T, Hq, Hkv, d, L = 1, 1, 8, 2, 128, 513
    q, k, v, sl = case(45, B, T, Hq, Hkv, d, L, [L])
    k[:] = k[:, :, :1, :]
    got = helpers.bf16_to_f64(run_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, 0.2, 8))
    vf = helpers.bf16_to_f64(v)
    for h in range(Hq):
        mean = vf[0, h // 4].mean(axis=0)
        assert helpers.rel_l2(got[0, 0, h], mean) < 5e-3


@pytest.mark.parametrize("splits", [1, 2, 3, 4, 5])
def test_clusters_per_head_merge_through_workspace(splits):
    # P clusters per (b, kv head): DSMEM merge inside each, workspace merge across them
    check(60 + splits, 2, 4, 10, 2, 128, 2000, [2000, 731], 8, splits=splits)


@pytest.mark.parametrize("splits", [2, 7])
def test_clusters_per_head_with_empty_clusters_and_small_d(splits):
    check(70 + splits, 1, 1, 8, 2, 64, 512, [100], 4, splits=splits)


def test_workspace_counters_return_to_zero_and_repeat_calls_agree():
    B, T, Hq, Hkv, d, L = 1, 4, 40, 8, 128, 8192
    q, k, v, sl = case(80, B, T, Hq, Hkv, d, L, [L])
    n = dl.dl_decode_attn_workspace_bytes(B, T, Hq, Hkv, d, L, 4)
    assert n > 256  # long sequences split each head over several clusters
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    args = (dev_u16(q.ravel()), Hq * d, B, T, Hq, Hkv, d, dev_u16(k), dev_u16(v), L, dev_i32(sl), 0.088, 4)
    outs = []
    for _ in range(3):
        out = torch.empty((B, T, Hq, d), dtype=torch.int16, device="cuda")
        dl.check(dl.dl_decode_attn(*args, out, ws))
        assert dl.dl_read_status(ws) == dl.DL_OK
        outs.append(host_u16(out))
    assert not ws[256:256 + 4 * B * Hkv * 4].any()  # every per-(head, owner) counter is back to zero
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])
    ref = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, 0.088)
    helpers.check_attn(outs[0], ref, "repeat calls")


def test_bad_seq_len_is_reported_on_device():
    q, k, v, _ = case(46, 2, 2, 4, 1, 64, 128, [1, 1])
    out = run_attn(q.ravel(), 4 * 64, 2, 2, 4, 1, 64, k, v, np.int32([1, 200]), 0.125, 8,
                   expect=dl.DL_ERR_DEVICE_ARG)
    assert not helpers.bf16_to_f64(out).any()  # both sequences invalid -> zeros
