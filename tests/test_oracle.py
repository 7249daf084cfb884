"""Pins of the CPU oracle against things other than itself: format definitions
checked against torch's casts, hand-derived worked examples (tests/golden/),
closed forms, invariants, library routines (torch float64 matmul and
scaled_dot_product_attention) and brute force on tiny inputs.

A plausible mistake anywhere in the oracle (a dropped term, a wrong sign or
index, a transposed operand, gate/up swapped, the wrong kv head) fails at
least one of these tests.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from latency_decode_b200 import datagen as dg


def _bits_of(vals):
    return dg.bf16_bits(np.asarray(vals, dtype=np.float32))


def _dequant_torch(codes):
    """Library decode of e4m3 bytes (torch), independent of the oracle's table."""
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def _bf16_torch(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------- formats --

def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = _dequant_torch(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decode_definition_points():
    # format definition: bias 7, subnormal step 2^-9, max S.1111.110 = 448
    assert oracle.e4m3_to_f64(0x38) == 1.0
    assert oracle.e4m3_to_f64(0xB8) == -1.0
    assert oracle.e4m3_to_f64(0x7E) == 448.0
    assert oracle.e4m3_to_f64(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_f64(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_f64(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_to_f64(0x44) == 3.0


def test_e4m3_encode_roundtrips_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_to_f64(codes).astype(np.float32)
    back = oracle.f32_to_e4m3(vals)
    assert np.array_equal(back, codes)  # includes 0x80 for -0.0


def test_e4m3_encode_matches_torch_on_random_and_midpoints():
    g = np.random.default_rng(123)
    mags = np.exp2(g.uniform(-12, math.log2(440), size=4000)).astype(np.float32)
    vals = mags * np.where(g.random(4000) < 0.5, -1, 1).astype(np.float32)
    # exact midpoints between neighbouring finite codes (ties go to even)
    pos = np.sort(oracle.e4m3_to_f64(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids])
    ours = oracle.f32_to_e4m3(vals)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    # ties to even: every midpoint lands on an even mantissa
    assert np.all(oracle.f32_to_e4m3(mids[1:]) % 2 == 0)


def test_e4m3_encode_saturates():
    assert oracle.f32_to_e4m3(np.float32(448.0)) == 0x7E
    assert oracle.f32_to_e4m3(np.float32(460.0)) == 0x7E
    assert oracle.f32_to_e4m3(np.float32(1e6)) == 0x7E
    assert oracle.f32_to_e4m3(np.float32(-1e30)) == 0xFE
    assert oracle.f32_to_e4m3(np.float32(np.inf)) == 0x7E
    assert oracle.f32_to_e4m3(np.float32(-0.0)) == 0x80
    assert oracle.f32_to_e4m3(np.float32(2.0 ** -11)) == 0x00  # below half the smallest subnormal


def test_bf16_decode_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    sample = bits[::97]  # every 97th pattern keeps the ctypes loop short
    ours = oracle.bf16_to_f64(sample)
    ref = _bf16_torch(sample)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_round_matches_torch():
    g = np.random.default_rng(7)
    vals = (g.standard_normal(3000) * np.exp2(g.uniform(-30, 30, 3000))).astype(np.float32)
    # exact ties between neighbouring bf16 values
    base = _bits_of(g.standard_normal(500).astype(np.float32)).astype(np.uint32)
    ties = ((base << 16) | 0x8000).astype(np.uint32).view(np.float32)
    vals = np.concatenate([vals, ties, np.float32([0.0, -0.0, 3e38, -3e38])])
    ours = oracle.f64_to_bf16(vals.astype(np.float64))
    ref = _bits_of(vals)
    assert np.array_equal(ours, ref)


# ------------------------------------------------------ activation quant --

def test_act_quant_hand_example(golden_dir):
    gold = json.load(open(os.path.join(golden_dir, "act_quant_hand.json")))
    x = _bits_of(gold["x"]).reshape(1, -1)
    xq, sx = oracle.act_quant(x)
    assert xq.ravel().tolist() == gold["xq"]
    assert sx == np.float32(1.0) / np.float32(112.0)


def test_act_quant_properties():
    g = np.random.default_rng(11)
    x = dg.bf16_normal(g, (4, 256))
    xq, sx = oracle.act_quant(x)
    xf = _bf16_torch(x)
    amax = np.abs(xf).max()
    assert sx == np.float32(amax) / np.float32(448.0)
    i = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    assert xq[i] in (0x7E, 0xFE)
    # every code is within half a code step of x*inv (relative 1/16 for normals)
    deq = _dequant_torch(xq) * float(sx)
    assert np.allclose(deq, xf, rtol=1 / 16 + 1e-6, atol=float(sx) * 2.0 ** -9)


def test_act_quant_zero_input():
    x = np.zeros((2, 128), dtype=np.uint16)
    xq, sx = oracle.act_quant(x)
    assert sx == 1.0 and not xq.any()


# ------------------------------------------------------------------- GEMM --

def test_gemm_swiglu_hand_example(golden_dir):
    gold = json.load(open(os.path.join(golden_dir, "gemm_swiglu_hand.json")))
    xq = np.array([gold["xq"]], dtype=np.uint8)
    w = np.array(gold["w"], dtype=np.uint8)
    y = oracle.gemm_q(xq, gold["s_x"], w, gold["s_w"])
    assert y.ravel().tolist() == gold["y"]
    out = oracle.fc13_swiglu_q(xq, gold["s_x"], w, gold["s_w"])
    assert out.ravel()[0] == pytest.approx(gold["swiglu"][0], rel=1e-15)


def test_gemm_one_hot_selects_column():
    g = np.random.default_rng(3)
    K, N = 256, 64
    w, s_w = dg.e4m3_weight(g, N, K)
    for k in (0, 17, 255):
        x = np.zeros((1, K), dtype=np.float32)
        x[0, k] = 1.0
        xb = dg.bf16_bits(x)
        xq, sx = oracle.act_quant(xb)
        assert xq[0, k] == 0x7E and np.count_nonzero(xq) == 1
        y = oracle.gemm_q(xq, sx, w, s_w)
        expect = float(sx) * float(s_w) * 448.0 * _dequant_torch(w[:, k])
        assert np.array_equal(y[0], expect)


def test_gemm_matches_torch_matmul_of_dequantised_bytes():
    g = np.random.default_rng(5)
    M, N, K = 3, 96, 384  # non-square: a transposed operand cannot match
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N, K)
    xq, sx = oracle.act_quant(x)
    y = oracle.gemm_q(xq, sx, w, s_w)
    ref = (torch.from_numpy(_dequant_torch(xq)) @ torch.from_numpy(_dequant_torch(w)).T).numpy()
    ref = ref * float(sx) * float(s_w)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_gemm_brute_force_tiny():
    g = np.random.default_rng(9)
    for _ in range(20):
        M, N, K = g.integers(1, 4, endpoint=True, size=3)
        xq = g.integers(0, 256, size=(M, K)).astype(np.uint8)
        w = g.integers(0, 256, size=(N, K)).astype(np.uint8)
        xq[(xq & 0x7F) == 0x7F] = 0x38  # no NaN codes
        w[(w & 0x7F) == 0x7F] = 0x30
        sx, sw = np.float32(g.uniform(0.1, 2)), np.float32(g.uniform(0.1, 2))
        y = oracle.gemm_q(xq, sx, w, sw)
        xd, wd = _dequant_torch(xq), _dequant_torch(w)
        for m in range(M):
            for n in range(N):
                acc = math.fsum(xd[m, k] * wd[n, k] for k in range(K))
                assert y[m, n] == pytest.approx(acc * float(sx) * float(sw), rel=1e-12, abs=1e-300)


def test_gemm_linear_in_weight_scale():
    g = np.random.default_rng(13)
    x = dg.bf16_normal(g, (2, 128))
    w, s_w = dg.e4m3_weight(g, 32, 128)
    xq, sx = oracle.act_quant(x)
    y1 = oracle.gemm_q(xq, sx, w, s_w)
    y2 = oracle.gemm_q(xq, sx, w, np.float32(2.0) * s_w)
    assert np.allclose(y2, 2 * y1, rtol=1e-15, atol=0)


# ---------------------------------------------------------------- SwiGLU --

def test_swiglu_closed_form_and_order():
    g = np.random.default_rng(17)
    M, K, F = 2, 128, 48
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, 2 * F, K)
    xq, sx = oracle.act_quant(x)
    y = oracle.gemm_q(xq, sx, w, s_w)
    gate, up = y[:, :F], y[:, F:]
    out = oracle.fc13_swiglu_q(xq, sx, w, s_w)
    sig = 1.0 / (1.0 + np.exp(-gate))
    assert np.allclose(out, gate * sig * up, rtol=1e-13, atol=1e-300)
    swapped = up / (1.0 + np.exp(-up)) * gate
    assert not np.allclose(out, swapped, rtol=1e-3)
    # the unquantised entry point equals act_quant followed by the quantised one
    assert np.array_equal(oracle.fc13_swiglu(x, w, s_w), out)


def test_silu_limits():
    # silu(0) = 0, silu(g) -> g for large g, -> 0 for very negative g
    K = 128
    xq = np.zeros((1, K), dtype=np.uint8)
    xq[0, 0] = 0x38  # 1.0
    w = np.zeros((2, K), dtype=np.uint8)
    w[1, 0] = 0x38  # up = 1 * s
    for gate_code, expect in ((0x00, 0.0), (0x7E, 448.0), (0xFE, 0.0)):
        w[0, 0] = gate_code
        out = oracle.fc13_swiglu_q(xq, 1.0, w, 1.0)[0, 0]
        assert out == pytest.approx(expect, abs=1e-12)


# ------------------------------------------------------------- QKV scale --

def test_qkv_scale_only_touches_q_columns():
    g = np.random.default_rng(19)
    Hq, Hkv, d, K = 4, 2, 16, 128
    N = (Hq + 2 * Hkv) * d
    x = dg.bf16_normal(g, (3, K))
    w, s_w = dg.e4m3_weight(g, N, K)
    qs = np.float32(1 / math.sqrt(d))
    out = oracle.fc_qkv_scale(x, w, s_w, Hq, Hkv, d, qs)
    plain = oracle.fc_qkv_scale(x, w, s_w, Hq, Hkv, d, 1.0)
    xq, sx = oracle.act_quant(x)
    assert np.array_equal(plain, oracle.gemm_q(xq, sx, w, s_w))
    assert np.array_equal(out[:, : Hq * d], plain[:, : Hq * d] * float(qs))
    assert np.array_equal(out[:, Hq * d:], plain[:, Hq * d:])


# ------------------------------------------------------------- attention --

def _attn_case(g, B, T, Hq, Hkv, d, Lcap, seq_lens):
    q = dg.bf16_normal(g, (B, T, Hq, d))
    k = dg.bf16_normal(g, (B, Hkv, Lcap, d))
    v = dg.bf16_normal(g, (B, Hkv, Lcap, d))
    return q, k, v, np.asarray(seq_lens, dtype=np.int32)


def _sdpa_ref(q, k, v, seq_lens, scale, T, Hq, Hkv):
    """torch scaled_dot_product_attention in float64, GQA expanded, explicit
    bottom-right causal mask."""
    B = q.shape[0]
    g = Hq // Hkv
    outs = []
    for b in range(B):
        L = int(seq_lens[b])
        qt = torch.from_numpy(_bf16_torch(q[b])).permute(1, 0, 2)  # [Hq, T, d]
        kt = torch.from_numpy(_bf16_torch(k[b, :, :L])).repeat_interleave(g, 0)
        vt = torch.from_numpy(_bf16_torch(v[b, :, :L])).repeat_interleave(g, 0)
        mask = torch.arange(L)[None, :] <= (L - T + torch.arange(T))[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(
            qt[None], kt[None], vt[None], attn_mask=mask[None, None], scale=float(scale))
        outs.append(o[0].permute(1, 0, 2).numpy())
    return np.stack(outs)


def test_attn_hand_example(golden_dir):
    gold = json.load(open(os.path.join(golden_dir, "attn_hand.json")))
    q = _bits_of(gold["q"]).reshape(1, 1, 2, 2)
    k = _bits_of(gold["k"]).reshape(1, 1, 2, 2)
    v = _bits_of(gold["v"]).reshape(1, 1, 2, 2)
    out = oracle.decode_attn(q.ravel(), 4, 1, 1, 2, 1, 2, k, v, np.int32([2]), 1.0)
    assert np.allclose(out.reshape(2, 2), np.array(gold["out"]), rtol=1e-15, atol=0)


def test_attn_matches_torch_sdpa_gqa_causal():
    g = np.random.default_rng(23)
    B, T, Hq, Hkv, d, Lcap = 2, 4, 10, 2, 32, 96
    seq = [96, 37]
    q, k, v, sl = _attn_case(g, B, T, Hq, Hkv, d, Lcap, seq)
    scale = 1 / math.sqrt(d)
    out = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, scale)
    ref = _sdpa_ref(q, k, v, sl, np.float32(scale), T, Hq, Hkv)
    assert np.allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_attn_identical_keys_give_mean_of_values():
    g = np.random.default_rng(29)
    B, T, Hq, Hkv, d, L = 1, 1, 4, 2, 16, 50
    q, k, v, sl = _attn_case(g, B, T, Hq, Hkv, d, L, [L])
    k[:] = k[:, :, :1, :]  # every key equal to key 0
    out = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, 0.3)
    vf = _bf16_torch(v)
    for h in range(Hq):
        assert np.allclose(out[0, 0, h], vf[0, h // 2].mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attn_scale_zero_is_mean_over_visible_keys():
    g = np.random.default_rng(31)
    B, T, Hq, Hkv, d, Lcap = 1, 4, 2, 1, 8, 20
    q, k, v, sl = _attn_case(g, B, T, Hq, Hkv, d, Lcap, [20])
    out = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, 0.0)
    vf = _bf16_torch(v)
    for t in range(T):
        vis = 20 - T + t + 1
        assert np.allclose(out[0, t, 0], vf[0, 0, :vis].mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attn_dominant_logit_selects_value_row_and_stays_in_hull():
    g = np.random.default_rng(37)
    B, T, Hq, Hkv, d, L = 1, 1, 1, 1, 8, 12
    q, k, v, sl = _attn_case(g, B, T, Hq, Hkv, d, L, [L])
    qv = np.zeros(d, dtype=np.float32)
    qv[0] = 1.0
    q[:] = dg.bf16_bits(qv)
    kk = np.zeros((L, d), dtype=np.float32)
    kk[7, 0] = 64.0  # logit 64*scale on key 7, zero elsewhere
    k[0, 0] = dg.bf16_bits(kk)
    out = oracle.decode_attn(q.ravel(), d, B, T, Hq, Hkv, d, k, v, sl, 1.0)
    vf = _bf16_torch(v)[0, 0]
    assert np.allclose(out[0, 0, 0], vf[7], rtol=0, atol=1e-20)
    # random logits: output inside [min V, max V] coordinate-wise
    q2, k2, v2, _ = _attn_case(g, B, T, Hq, Hkv, d, L, [L])
    o2 = oracle.decode_attn(q2.ravel(), d, B, T, Hq, Hkv, d, k2, v2, sl, 0.5)[0, 0, 0]
    v2f = _bf16_torch(v2)[0, 0]
    assert np.all(o2 >= v2f.min(axis=0) - 1e-12) and np.all(o2 <= v2f.max(axis=0) + 1e-12)


def test_lse_merge_of_any_split_equals_unsplit():
    g = np.random.default_rng(41)
    B, T, Hq, Hkv, d, L = 1, 4, 5, 1, 16, 200
    q, k, v, sl = _attn_case(g, B, T, Hq, Hkv, d, L, [L])
    full = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, 0.25)
    for trial in range(6):
        S = int(g.integers(1, 17))
        cuts = np.sort(g.integers(0, L + 1, size=S - 1))
        bounds = [0, *cuts.tolist(), L + 8]  # some chunks empty, one past L
        for t in range(T):
            for h in range(Hq):
                parts = [oracle.attn_partial(q.ravel(), Hq * d, T, Hq, Hkv, d, k, v, 0, t, h, L,
                                             0.25, bounds[i], bounds[i + 1]) for i in range(S)]
                m = np.array([p[0] for p in parts])
                l = np.array([p[1] for p in parts])
                o = np.stack([p[2] for p in parts])
                merged = oracle.lse_combine(m, l, o)
                assert np.allclose(merged, full[0, t, h], rtol=1e-12, atol=1e-14)


def test_causal_rows_equal_single_token_decode_at_shorter_length():
    g = np.random.default_rng(43)
    B, T, Hq, Hkv, d, L = 1, 4, 5, 1, 32, 64
    q, k, v, sl = _attn_case(g, B, T, Hq, Hkv, d, L, [L])
    out = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, 0.2)
    for t in range(T):
        one = oracle.decode_attn(q[:, t:t + 1].ravel(), Hq * d, B, 1, Hq, Hkv, d, k, v,
                                 np.int32([L - T + 1 + t]), 0.2)
        assert np.allclose(out[0, t], one[0, 0], rtol=1e-13, atol=1e-15)


def test_q_stride_reads_q_inside_a_wider_row():
    # q taken from a fused QKV row of width (Hq+2Hkv)*d must equal q packed alone
    g = np.random.default_rng(47)
    B, T, Hq, Hkv, d, L = 1, 2, 4, 2, 8, 16
    q, k, v, sl = _attn_case(g, B, T, Hq, Hkv, d, L, [L])
    W = (Hq + 2 * Hkv) * d
    wide = dg.bf16_normal(g, (B * T, W))
    wide[:, : Hq * d] = q.reshape(B * T, Hq * d)
    a = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, k, v, sl, 0.3)
    b = oracle.decode_attn(wide.ravel(), W, B, T, Hq, Hkv, d, k, v, sl, 0.3)
    assert np.array_equal(a, b)


# ------------------------------------------------------------------- MoE --

def test_moe_equals_per_token_dense_with_shared_scale():
    g = np.random.default_rng(53)
    T, K, F, E = 9, 128, 32, 5
    x = dg.bf16_normal(g, (T, K))
    ws, scales = zip(*(dg.e4m3_weight(g, 2 * F, K) for _ in range(E)))
    w = np.stack(ws)
    s_w = np.array(scales, dtype=np.float32)
    ids = g.integers(0, E, size=T).astype(np.int32)
    out = oracle.moe_fc13_swiglu(x, ids, w, s_w)
    xq, sx = oracle.act_quant(x)  # one scale over all tokens
    for t in range(T):
        ref = oracle.fc13_swiglu_q(xq[t:t + 1], sx, w[ids[t]], s_w[ids[t]])
        assert np.array_equal(out[t], ref[0])
    # a token routed elsewhere gives a different row (the expert id matters)
    other = (ids[0] + 1) % E
    assert not np.allclose(out[0], oracle.fc13_swiglu_q(xq[:1], sx, w[other], s_w[other])[0])


# ------------------------------------------- plain projections (o_proj, FC2) --

def test_linear_equals_unit_scaled_qkv_and_one_hot_column():
    g = np.random.default_rng(61)
    M, K, N = 3, 256, 160
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N, K)
    # the QKV entry with q_scale = 1 is the plain projection (N = (Hq + 2Hkv) d)
    assert np.array_equal(oracle.linear(x, w, s_w), oracle.fc_qkv_scale(x, w, s_w, 6, 2, 16, 1.0))
    # one-hot input selects column k of W, times the known scales
    xo = np.zeros((1, K), dtype=np.float32)
    xo[0, 77] = -2.0
    y = oracle.linear(dg.bf16_bits(xo), w, s_w)
    expect = float(np.float32(2.0) / np.float32(448.0)) * float(s_w) * -448.0 * _dequant_torch(w[:, 77])
    assert np.array_equal(y[0], expect)


def test_moe_linear_equals_per_token_projection_with_shared_scale():
    g = np.random.default_rng(62)
    T, K, N, E = 7, 128, 64, 4
    x = dg.bf16_normal(g, (T, K))
    ws, scales = zip(*(dg.e4m3_weight(g, N, K) for _ in range(E)))
    w = np.stack(ws)
    s_w = np.array(scales, dtype=np.float32)
    ids = np.array([3, 0, 3, 1, 2, 0, 3], dtype=np.int32)
    out = oracle.moe_linear(x, ids, w, s_w)
    xq, sx = oracle.act_quant(x)
    xd, = (_dequant_torch(xq),)
    for t in range(T):
        ref = xd[t] @ _dequant_torch(w[ids[t]]).T * float(sx) * float(s_w[ids[t]])
        assert np.allclose(out[t], ref, rtol=1e-12, atol=1e-14)
    bad = oracle.moe_linear(x, np.array([0, 9, 0, 0, 0, 0, 0], dtype=np.int32), w, s_w)
    assert np.isnan(bad[1]).all() and not np.isnan(bad[0]).any()


# ------------------------------------------ residual add + RMSNorm + quant --

def test_add_rmsnorm_quant_hand_example(golden_dir):
    gold = json.load(open(os.path.join(golden_dir, "add_rmsnorm_quant_hand.json")))
    x = _bits_of(gold["x"])
    r = _bits_of(gold["r"])
    gam = _bits_of(gold["gamma"])
    h, y, xq, sx = oracle.add_rmsnorm_quant(x, r, gam, gold["eps"])
    assert np.array_equal(h, _bits_of(gold["h"]))
    assert y[0].tolist() == gold["y_row0"]
    assert xq[0].tolist() == gold["xq_row0"]
    assert sx == np.float32(1.0) / np.float32(112.0)


def test_rmsnorm_matches_torch_rms_norm():
    g = np.random.default_rng(63)
    M, K = 5, 640
    x = dg.bf16_normal(g, (M, K))
    gam = dg.bf16_normal(g, (K,), std=0.5)
    for eps in (1e-5, 0.25):
        h, y = oracle.add_rmsnorm(x, None, gam, eps)
        assert np.array_equal(h, x)  # no residual: h is x
        ref = torch.nn.functional.rms_norm(torch.from_numpy(_bf16_torch(x)), (K,),
                                           weight=torch.from_numpy(_bf16_torch(gam)), eps=float(np.float32(eps)))
        assert np.allclose(y, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_residual_add_matches_torch_bf16_add_and_norm_uses_the_rounded_sum():
    g = np.random.default_rng(64)
    M, K = 3, 512
    x = dg.bf16_normal(g, (M, K))
    r = dg.bf16_normal(g, (M, K), std=3.0)
    gam = dg.bf16_bits(np.ones(K, dtype=np.float32))
    h, y = oracle.add_rmsnorm(x, r, gam, 1e-6)
    tx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    tr = torch.from_numpy(r.view(np.int16)).view(torch.bfloat16)
    assert np.array_equal(h, (tx + tr).view(torch.int16).numpy().view(np.uint16))
    # the norm is taken of h (the rounded sum): normalising h itself gives y
    h2, y2 = oracle.add_rmsnorm(h, None, gam, 1e-6)
    assert np.array_equal(h2, h) and np.array_equal(y2, y)


def test_rmsnorm_invariants():
    g = np.random.default_rng(65)
    M, K = 4, 256
    x = dg.bf16_normal(g, (M, K))
    one = dg.bf16_bits(np.ones(K, dtype=np.float32))
    _, y = oracle.add_rmsnorm(x, None, one, 0.0)
    assert np.allclose((y ** 2).mean(axis=1), 1.0, rtol=1e-13)  # unit gain, eps = 0: unit mean square
    xs = dg.bf16_bits(_bf16_torch(x).astype(np.float32) * np.float32(8.0))  # exact power-of-two scaling
    _, ys = oracle.add_rmsnorm(xs, None, one, 0.0)
    assert np.allclose(ys, y, rtol=1e-14, atol=0)
    _, yp = oracle.add_rmsnorm(x[::-1].copy(), None, one, 0.0)  # rows are independent
    assert np.array_equal(yp, y[::-1])
    # a constant row c gives sign(c) * gamma; gamma enters per column
    gam = dg.bf16_normal(g, (K,))
    c = dg.bf16_bits(np.full((1, K), -3.0, dtype=np.float32))
    _, yc = oracle.add_rmsnorm(c, None, gam, 0.0)
    assert np.array_equal(yc[0], -_bf16_torch(gam))
    # a zero row with eps > 0 normalises to zero, not NaN
    _, yz = oracle.add_rmsnorm(np.zeros((1, K), dtype=np.uint16), None, gam, 1e-6)
    assert not yz.any()


def test_quant_f32_reduces_to_act_quant_on_bf16_values():
    g = np.random.default_rng(66)
    x = dg.bf16_normal(g, (3, 384))
    xq, sx = oracle.act_quant(x)
    xq2, sx2 = oracle.quant_f32(_bf16_torch(x).astype(np.float32))
    assert sx2 == sx and np.array_equal(xq2, xq)
    z, sz = oracle.quant_f32(np.zeros(10, dtype=np.float32))
    assert sz == 1.0 and not z.any()


def test_quant_f32_codes_are_nearest_by_brute_force():
    g = np.random.default_rng(67)
    y = (g.standard_normal(300) * np.exp(g.uniform(-6, 3, 300))).astype(np.float32)
    xq, sx = oracle.quant_f32(y)
    inv = np.float32(448.0) / np.float32(np.abs(y).max())
    assert sx == np.float32(np.abs(y).max()) / np.float32(448.0)
    codes = np.arange(256, dtype=np.uint8)
    vals = _dequant_torch(codes)
    finite = ~np.isnan(vals)
    for i in range(y.size):
        p = float(np.float32(y[i] * inv))
        best = np.min(np.abs(vals[finite] - p))
        assert abs(vals[xq[i]] - p) == best, (i, p, vals[xq[i]])


# ------------------------------------------------ speculative verification --

def test_spec_verify_hand_example(golden_dir):
    gold = json.load(open(os.path.join(golden_dir, "spec_verify_hand.json")))
    T, V = len(gold["hot"]), gold["V"]
    lg = np.zeros((1, T, V), dtype=np.float32)
    for t, v in enumerate(gold["hot"]):
        lg[0, t, v] = 1.0
    tid, nacc, em = oracle.spec_verify_greedy(dg.bf16_bits(lg), np.array([gold["draft"]], dtype=np.int32))
    assert tid[0].tolist() == gold["target_ids"]
    assert int(nacc[0]) == gold["n_accepted"]
    assert em[0].tolist() == gold["emitted"]


def _signed_zero_logits(gold):
    """Logits of the signed-zero fixture as bf16 bits: -1.0 everywhere, then
    the listed -0 (0x8000) and +0 (0x0000) entries."""
    T, V = len(gold["target_ids"]), gold["V"]
    lg = np.full((1, T, V), dg.bf16_bits(np.float32([-1.0]))[0], dtype=np.uint16)
    for t, v in gold["neg_zero"]:
        lg[0, t, v] = 0x8000
    for t, v in gold["pos_zero"]:
        lg[0, t, v] = 0x0000
    return lg


def test_spec_verify_signed_zero_tie(golden_dir):
    """-0 and +0 are one value: the lower index wins, whatever its sign (numpy's
    argmax on the decoded values agrees)."""
    gold = json.load(open(os.path.join(golden_dir, "spec_verify_signed_zero.json")))
    lg = _signed_zero_logits(gold)
    tid, nacc, em = oracle.spec_verify_greedy(lg, np.array([gold["draft"]], dtype=np.int32))
    assert tid[0].tolist() == gold["target_ids"]
    assert tid[0].tolist() == np.argmax(_bf16_torch(lg)[0], axis=1).tolist()
    assert int(nacc[0]) == gold["n_accepted"] and em[0].tolist() == gold["emitted"]


def test_spec_verify_matches_numpy_argmax_and_brute_force_acceptance():
    g = np.random.default_rng(71)
    B, T, V = 6, 4, 1000
    lg = dg.bf16_normal(g, (B, T, V))
    lg[0, 1, 7] = lg[0, 1, 9] = dg.bf16_bits(np.float32([50.0]))[0]  # a tie: the lower index wins
    ref = np.argmax(_bf16_torch(lg), axis=2)  # numpy returns the first maximal index
    assert ref[0, 1] == 7
    draft = g.integers(0, V, size=(B, T - 1)).astype(np.int32)
    # plant accept runs of every length 0..T-1
    for b, n in enumerate([0, 1, 2, 3, 3, 1]):
        draft[b, :n] = ref[b, :n]
        if n < T - 1 and draft[b, n] == ref[b, n]:
            draft[b, n] = (ref[b, n] + 1) % V
    tid, nacc, em = oracle.spec_verify_greedy(lg, draft)
    assert np.array_equal(tid, ref)
    for b in range(B):
        n = 0
        for i in range(T - 1):  # brute force: longest matching prefix
            if all(draft[b, j] == ref[b, j] for j in range(i + 1)):
                n = i + 1
        assert nacc[b] == n
        assert em[b, :n + 1].tolist() == ref[b, :n + 1].tolist() and (em[b, n + 1:] == -1).all()
    assert nacc.tolist() == [0, 1, 2, 3, 3, 1]


def test_spec_verify_single_position_emits_one_token():
    g = np.random.default_rng(72)
    lg = dg.bf16_normal(g, (3, 1, 50))
    tid, nacc, em = oracle.spec_verify_greedy(lg, np.zeros((3, 0), dtype=np.int32))
    assert (nacc == 0).all() and np.array_equal(em[:, 0], tid[:, 0])
    assert np.array_equal(tid[:, 0], np.argmax(_bf16_torch(lg)[:, 0], axis=1))


# ------------------------------------------------------ FP8 KV attention --

def test_fp8kv_attention_equals_bf16_attention_on_exactly_representable_caches():
    """With power-of-two scales every s * e4m3 value is exact in bf16, so the
    FP8-cache attention must equal the (pinned) bf16 attention on those values."""
    g = np.random.default_rng(81)
    B, T, Hq, Hkv, d, Lcap = 2, 4, 8, 2, 64, 96
    q = dg.bf16_normal(g, (B, T, Hq, d))
    kc = g.integers(0, 256, size=(B, Hkv, Lcap, d)).astype(np.uint8)
    vc = g.integers(0, 256, size=(B, Hkv, Lcap, d)).astype(np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x30  # no NaN codes
    vc[(vc & 0x7F) == 0x7F] = 0x38
    s_k, s_v = np.float32(2.0 ** -7), np.float32(2.0 ** -5)
    sl = np.int32([96, 37])
    vt = np.ascontiguousarray(vc.transpose(0, 1, 3, 2))  # the FP8 cache stores V as [d][key]
    got = oracle.decode_attn_fp8kv(q.ravel(), Hq * d, B, T, Hq, Hkv, d, kc, vt, sl, 0.125, s_k, s_v)
    kb = dg.bf16_bits((_dequant_torch(kc) * float(s_k)).astype(np.float32))
    vb = dg.bf16_bits((_dequant_torch(vc) * float(s_v)).astype(np.float32))
    assert np.array_equal(_bf16_torch(kb), _dequant_torch(kc) * float(s_k))  # exact in bf16
    ref = oracle.decode_attn(q.ravel(), Hq * d, B, T, Hq, Hkv, d, kb, vb, sl, 0.125)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_fp8kv_scales_enter_as_stated():
    """s_v scales the output linearly; s_k acts as a softmax temperature
    (s_k * scale is all that matters)."""
    g = np.random.default_rng(82)
    B, T, Hq, Hkv, d, Lcap = 1, 1, 4, 1, 64, 50
    q = dg.bf16_normal(g, (B, T, Hq, d))
    kc = g.integers(0, 0x7E, size=(B, Hkv, Lcap, d)).astype(np.uint8)
    vc = g.integers(0, 0x7E, size=(B, Hkv, Lcap, d)).astype(np.uint8)
    sl = np.int32([50])
    vt = np.ascontiguousarray(vc.transpose(0, 1, 3, 2))
    a = oracle.decode_attn_fp8kv(q.ravel(), Hq * d, B, T, Hq, Hkv, d, kc, vt, sl, 0.5, 0.01, 1.0)
    b = oracle.decode_attn_fp8kv(q.ravel(), Hq * d, B, T, Hq, Hkv, d, kc, vt, sl, 0.25, 0.02, 3.0)
    assert np.allclose(b, 3.0 * a, rtol=1e-12)
