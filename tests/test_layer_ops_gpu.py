"""GPU parity of the layer's remaining operations through the C ABI against the
CPU oracle: the plain-epilogue projection (attention output projection, FC2
down projection) dense and grouped per expert, and the residual add + RMSNorm +
Quantize producer handing x_q to a GEMM through the workspace
(DL_FLAG_XQ_READY).

Tolerances: GEMM outputs as for every GEMM here (relative L2 <= 1e-2, the
max-abs rule of helpers.check_gemm).  The producer's h is bit-exact (a single
bf16 rounding of an exact sum); its e4m3 codes are decided on fp32 y on both
sides, whose last bits depend on the order of the row sum of squares, so a
code may sit one step away only where y*inv lies at a rounding midpoint (to
1e-5 relative; at most 1e-3 of the codes), and s_x agrees to 1e-6."""
import numpy as np
import pytest
import torch

import helpers
import oracle
from helpers import dev_f32, dev_i32, dev_u8, dev_u16, host_u16, new_ws
from latency_decode_b200 import build as dl_build
from latency_decode_b200 import datagen as dg
from latency_decode_b200 import dl
from layer_chain_ref import chain_tolerance, oracle_full_layer

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not helpers.gpu_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def lib():
    dl_build.build()
    return dl.lib()


def pack(w_dev, N, K):
    out = torch.empty_like(w_dev)
    dl.check(dl.dl_pack_fp8_weight(w_dev, out, N, K, dl.DL_PACK_PLAIN))
    return out


def run_linear(x, w, s_w, split=0, flags=dl.DL_FLAG_PDL):
    M, K = x.shape
    N = w.shape[0]
    out = torch.full((M, N), -1, dtype=torch.int16, device="cuda")
    ws, n = new_ws(M, K)
    dl.check(dl.dl_gemm_e4m3(dev_u16(x), M, K, pack(dev_u8(w), N, K), dev_f32(s_w), N, out, ws, n,
                             flags=flags | (split << dl.DL_FLAG_SPLIT_SHIFT)))
    assert dl.dl_read_status(ws) == dl.DL_OK
    return host_u16(out)


# ------------------------------------------------------------ plain GEMM --

@pytest.mark.parametrize("M,K,N", [(1, 512, 256), (3, 1024, 384), (8, 640, 128), (17, 2048, 640),
                                   (64, 1280, 256), (64, 8192, 128)])
def test_linear_small(M, K, N):
    g = np.random.default_rng(M * 7 + K + N)
    x = dg.bf16_normal(g, (M, K))
    w, s_w = dg.e4m3_weight(g, N, K)
    helpers.check_gemm(run_linear(x, w, s_w), oracle.linear(x, w, s_w), f"linear M={M} K={K} N={N}")


@pytest.mark.parametrize("split", [1, 2, 3, 5, 8])
def test_linear_forced_splits(split):
    g = np.random.default_rng(90 + split)
    x = dg.bf16_normal(g, (4, 2048))
    w, s_w = dg.e4m3_weight(g, 256, 2048)
    helpers.check_gemm(run_linear(x, w, s_w, split=split), oracle.linear(x, w, s_w), f"linear split={split}")


@pytest.mark.parametrize("name", ["layer_b1", "verify4", "batch16x4"])
def test_output_and_down_projections_full_size(name):
    """o_proj [K x Hq*d] and FC2 [K x F] at the workload's M; the oracle checks
    128 sampled output columns of every token (the scale is over all of x)."""
    wl = dg.WORKLOADS[name]
    g = dg.rng(100 + wl.seed)
    cols = np.sort(np.random.default_rng(5).choice(wl.K, size=128, replace=False))
    for Kin in (wl.k_o, wl.k_fc2):
        x = dg.bf16_normal(g, (wl.M, Kin))
        w, s_w = dg.e4m3_weight(g, wl.K, Kin)
        got = run_linear(x, w, s_w)
        xq, sx = oracle.act_quant(x)
        ref = oracle.gemm_q(xq, sx, np.ascontiguousarray(w[cols]), s_w)
        helpers.check_gemm(got[:, cols], ref, f"{name} projection K={Kin}")


def test_linear_zero_input_gives_zero():
    x = np.zeros((2, 512), dtype=np.uint16)
    w, s_w = dg.e4m3_weight(np.random.default_rng(1), 256, 512)
    assert not helpers.bf16_to_f64(run_linear(x, w, s_w)).any()


# ----------------------------------------------------------- grouped MoE --

def run_moe_linear(x, ids, w_bank, s_w, split=0):
    T, K = x.shape
    E, N, _ = w_bank.shape
    bank = dev_u8(w_bank) if isinstance(w_bank, np.ndarray) else w_bank
    wp = torch.empty_like(bank)
    for e in range(E):
        dl.check(dl.dl_pack_fp8_weight(bank[e], wp[e], N, K, dl.DL_PACK_PLAIN))
    out = torch.full((T, N), -1, dtype=torch.int16, device="cuda")
    ws, n = new_ws(T, K)
    dl.check(dl.dl_moe_gemm_grouped(dev_u16(x), T, K, dev_i32(ids), E, wp, dev_f32(s_w), N, out, ws, n,
                                    flags=dl.DL_FLAG_PDL | (split << dl.DL_FLAG_SPLIT_SHIFT)))
    assert dl.dl_read_status(ws) == dl.DL_OK
    return host_u16(out)


@pytest.mark.parametrize("T,E,split", [(1, 1, 0), (7, 3, 0), (64, 16, 0), (33, 200, 0), (12, 5, 3), (64, 8, 8)])
def test_moe_linear_small_banks(T, E, split):
    K, N = 1024, 384
    g = np.random.default_rng(T * 31 + E)
    ws_, scales = zip(*(dg.e4m3_weight(g, N, K) for _ in range(E)))
    w, s_w = np.stack(ws_), np.array(scales, dtype=np.float32)
    x = dg.bf16_normal(g, (T, K))
    ids = g.integers(0, E, size=T).astype(np.int32)
    got = run_moe_linear(x, ids, w, s_w, split)
    helpers.check_gemm(got, oracle.moe_linear(x, ids, w, s_w), f"moe linear T={T} E={E} split={split}")


def test_moe_fc2_full_bank_sampled_columns():
    """64 tokens, 128 experts of FC2 [5120, 8192] e4m3 (5.4 GB, drawn on the
    device), top-1 uniform routes; 96 sampled output columns per token."""
    wl = dg.WORKLOADS["moe64"]
    g = dg.rng(200 + wl.seed)
    F = wl.k_fc2
    x = dg.bf16_normal(g, (wl.M, F))
    ids = dg.expert_ids_for(wl, g)
    gen = torch.Generator(device="cuda").manual_seed(200 + wl.seed)
    bank = torch.empty((wl.experts, wl.K, F), dtype=torch.uint8, device="cuda")
    s_w = np.zeros(wl.experts, dtype=np.float32)
    for e in range(wl.experts):
        codes, s = dg.e4m3_weight_torch(gen, wl.K, F, "cuda")
        bank[e].copy_(codes)
        s_w[e] = s
    got = run_moe_linear(x, ids, bank, s_w)
    cols = np.sort(np.random.default_rng(3).choice(wl.K, size=96, replace=False))
    xq, sx = oracle.act_quant(x)
    rows = torch.from_numpy(cols).cuda()
    for t in range(wl.M):
        e = int(ids[t])
        sub = bank[e].index_select(0, rows).cpu().numpy()
        helpers.check_gemm(got[t:t + 1, cols], oracle.gemm_q(xq[t:t + 1], sx, sub, s_w[e]), f"fc2 token {t}")
    del bank
    torch.cuda.empty_cache()


# ------------------------------------------ residual add + RMSNorm + quant --

def run_norm(x, r, gamma, eps, h_mode="separate"):
    """h_mode: 'separate' (own h_out), 'none' (h_out NULL), 'into_r' / 'into_x' (in place)."""
    M, K = x.shape
    xd = dev_u16(x)
    rd = dev_u16(r) if r is not None else None
    if h_mode == "separate":
        hd = torch.full((M, K), -1, dtype=torch.int16, device="cuda")
    elif h_mode == "into_r":
        hd = rd
    elif h_mode == "into_x":
        hd = xd
    else:
        hd = None
    ws, n = new_ws(M, K)
    dl.check(dl.dl_add_rmsnorm_quant(xd, rd, hd, dev_u16(gamma), M, K, eps, ws, n))
    assert dl.dl_read_status(ws) == dl.DL_OK
    xq = ws[256:256 + M * K].cpu().numpy().reshape(M, K)
    sx = np.float32(ws[8:12].view(torch.float32).item())
    return (host_u16(hd) if hd is not None else None), xq, sx, ws, n


def e4m3_values(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def codes_close(got, ref, y_ref, what):
    """Codes may differ only where the oracle's fp32 product y*inv sits at the
    rounding midpoint of the two neighbouring e4m3 values (to 1e-5 relative):
    there the last bits of fp32 y, which depend on the order of the row's sum
    of squares, decide the rounding."""
    diff = got != ref
    assert diff.mean() <= 1e-3, f"{what}: {diff.sum()} of {diff.size} codes differ"
    if not diff.any():
        return
    gm, rm = got[diff].astype(int), ref[diff].astype(int)
    assert np.all((gm & 0x80) == (rm & 0x80)) and np.all(np.abs((gm & 0x7F) - (rm & 0x7F)) == 1), what
    yf = y_ref.astype(np.float32)
    inv = np.float32(448.0) / np.float32(np.abs(yf).max())
    p = (yf[diff] * inv).astype(np.float64)
    mid = (e4m3_values(got[diff]) + e4m3_values(ref[diff])) / 2
    assert np.all(np.abs(p - mid) <= 1e-5 * np.abs(mid)), f"{what}: a code differs away from a rounding midpoint"


@pytest.mark.parametrize("M", [1, 2, 4, 5, 16, 33, 64])
@pytest.mark.parametrize("residual", [True, False])
def test_add_rmsnorm_quant_rows(M, residual):
    K = 5120
    g = np.random.default_rng(300 + M + 1000 * residual)
    x = dg.bf16_normal(g, (M, K))
    r = dg.bf16_normal(g, (M, K), std=2.0) if residual else None
    gam = dg.rmsnorm_gain(g, K)
    h, xq, sx, _, _ = run_norm(x, r, gam, 1e-5)
    h_ref, y_ref, xq_ref, sx_ref = oracle.add_rmsnorm_quant(x, r, gam, 1e-5)
    assert np.array_equal(h, h_ref)
    assert abs(float(sx) / float(sx_ref) - 1.0) <= 1e-6
    codes_close(xq, xq_ref, y_ref, f"norm M={M} residual={residual}")


@pytest.mark.parametrize("h_mode", ["none", "into_r", "into_x"])
def test_add_rmsnorm_quant_outputs_in_place_and_rows_beyond_registers(h_mode):
    M, K = 64, 8192  # 16 vectors per thread: the part beyond the register set is re-read
    g = np.random.default_rng(400)
    x = dg.bf16_normal(g, (M, K))
    r = dg.bf16_normal(g, (M, K))
    gam = dg.rmsnorm_gain(g, K)
    h, xq, sx, _, _ = run_norm(x, r, gam, 1e-6, h_mode)
    h_ref, y_ref, xq_ref, sx_ref = oracle.add_rmsnorm_quant(x, r, gam, 1e-6)
    if h is not None:
        assert np.array_equal(h, h_ref)
    assert abs(float(sx) / float(sx_ref) - 1.0) <= 1e-6
    codes_close(xq, xq_ref, y_ref, f"norm in-place {h_mode}")


def test_add_rmsnorm_quant_zero_rows_and_large_eps():
    M, K = 3, 1024
    g = np.random.default_rng(401)
    x = dg.bf16_normal(g, (M, K))
    x[1] = 0  # a zero row normalises to zero
    gam = dg.rmsnorm_gain(g, K)
    h, xq, sx, _, _ = run_norm(x, None, gam, 4.0)
    h_ref, y_ref, xq_ref, sx_ref = oracle.add_rmsnorm_quant(x, None, gam, 4.0)
    assert not xq[1].any() and not y_ref[1].any()
    assert abs(float(sx) / float(sx_ref) - 1.0) <= 1e-6
    codes_close(xq, xq_ref, y_ref, "zero row")
    _, xq0, sx0, _, _ = run_norm(np.zeros((2, 256), np.uint16), None, gam[:256], 1e-5)
    assert sx0 == 1.0 and not xq0.any()  # all-zero input: s_x = 1, codes 0


def tie_flip_bound(y_ref, xq_ref, sx, w, s_w, swiglu):
    """Largest change of each output that the producer's admissible code flips
    can cause, from the oracle's own quantities only.

    The producer's codes may differ from the oracle's only where the oracle's
    fp32 product y*inv sits at a rounding midpoint of two e4m3 values (to 1e-5
    relative, as codes_close checks).  A flip there moves the code by one e4m3
    spacing, delta = 2|p - dec(c)|.  For one token row m and output column n
    the pre-activation then moves by at most
        D[m, n] = s_x * s_w * sum over tie positions k of delta[m, k] * |dec(W[n, k])|.
    A plain output moves by D.  For SwiGLU, out = silu(g) u with |silu'| <= 1.1,
    so over the box g +- Dg, u +- Du it moves by at most
        1.1 Dg (|u| + Du) + (|silu(g)| + 1.1 Dg) Du.
    Returns that bound, shaped like the output ([M, N] or [M, F])."""
    yf = y_ref.astype(np.float32)
    amax = np.float32(np.abs(yf).max())
    inv = np.float32(448.0) / amax
    p = (yf * inv).astype(np.float64)
    table = e4m3_values(np.arange(256, dtype=np.uint8))
    finite = np.isfinite(table)
    grid = np.unique(table[finite])
    v = e4m3_values(xq_ref)
    # the neighbouring e4m3 value on the side of p, and the midpoint towards it
    idx = np.searchsorted(grid, v)
    up = grid[np.minimum(idx + 1, grid.size - 1)]
    dn = grid[np.maximum(idx - 1, 0)]
    nb = np.where(p >= v, up, dn)
    mid = (v + nb) / 2
    tie = np.abs(p - mid) <= 1e-5 * np.maximum(np.abs(mid), 1e-30)
    delta = np.where(tie, np.abs(nb - v), 0.0)
    wv = np.abs(e4m3_values(w))
    D = float(sx) * float(s_w) * (delta @ wv.T)
    if not swiglu:
        return D
    F = w.shape[0] // 2
    y = float(sx) * float(s_w) * (e4m3_values(xq_ref) @ e4m3_values(w).T)
    g, u = y[:, :F], y[:, F:]
    Dg, Du = D[:, :F], D[:, F:]
    silu = g / (1.0 + np.exp(-g))
    return 1.1 * Dg * (np.abs(u) + Du) + (np.abs(silu) + 1.1 * Dg) * Du


EPS_EXACT = 2.0 ** -40  # below half an fp32 ulp of mean(h^2) >= 1/4: rsqrt sees mean(h^2) alone


def exact_rows(g, M, K):
    """Rows of constant power-of-two magnitude with random signs: mean(h^2) is a
    power of two summed exactly in any order, so with eps = EPS_EXACT RMSNorm
    gives y = +-gamma on both sides bit for bit and the codes cannot differ."""
    mag = np.float32(2.0) ** (np.arange(M) % 4 - 1).astype(np.float32)
    sign = np.where(g.random((M, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    return dg.bf16_bits(sign * mag[:, None])


@pytest.mark.parametrize("name", ["layer_b1", "verify4", "batch16x4"])
@pytest.mark.parametrize("inputs", ["exact", "random"])
def test_norm_then_gemm_through_the_workspace(name, inputs):
    """h = x + r, RMSNorm, Quantize into the GEMM's workspace, then FC13 + SwiGLU
    with DL_FLAG_XQ_READY (x = NULL), chained under PDL on one stream; the
    oracle checks 128 sampled output columns of every token.  'exact' inputs
    make the two sides' codes identical, so the GEMM output is held to the
    element-wise GEMM rule.  With 'random' inputs a code at a rounding tie may
    differ (codes_close checks that every difference is such a tie); the GEMM
    rule then holds with each output's allowance widened by tie_flip_bound,
    the most that the admissible flips can move it."""
    wl = dg.WORKLOADS[name]
    g = dg.rng(500 + wl.seed)
    if inputs == "exact":
        x = exact_rows(g, wl.M, wl.K)
        r = x.copy()  # h = 2x, exact
    else:
        x = dg.bf16_normal(g, (wl.M, wl.K))
        r = dg.bf16_normal(g, (wl.M, wl.K))
    gam = dg.rmsnorm_gain(g, wl.K)
    eps = EPS_EXACT if inputs == "exact" else 1e-5
    w13, s13 = dg.e4m3_weight(g, wl.N2, wl.K)
    F = wl.N2 // 2
    wp = torch.empty((wl.N2, wl.K), dtype=torch.uint8, device="cuda")
    dl.check(dl.dl_pack_fp8_weight(dev_u8(w13), wp, wl.N2, wl.K, dl.DL_PACK_SWIGLU))
    ws, n = new_ws(wl.M, wl.K)
    hd = torch.empty((wl.M, wl.K), dtype=torch.int16, device="cuda")
    out = torch.empty((wl.M, F), dtype=torch.int16, device="cuda")
    dl.check(dl.dl_add_rmsnorm_quant(dev_u16(x), dev_u16(r), hd, dev_u16(gam), wl.M, wl.K, eps, ws, n))
    dl.check(dl.dl_fc13_swiglu(None, wl.M, wl.K, wp, dev_f32(s13), wl.N2, out, ws, n,
                               flags=dl.DL_FLAG_PDL | dl.DL_FLAG_XQ_READY))
    assert dl.dl_read_status(ws) == dl.DL_OK
    h_ref, _, xq_ref, sx_ref = oracle.add_rmsnorm_quant(x, r, gam, eps)
    assert np.array_equal(host_u16(hd), h_ref)
    cols = np.sort(np.random.default_rng(6).choice(F, size=128, replace=False))
    sub = np.ascontiguousarray(np.concatenate([w13[cols], w13[F + cols]]))
    ref = oracle.fc13_swiglu_q(xq_ref, sx_ref, sub, s13)
    got = host_u16(out)[:, cols]
    xq_gpu = ws[256:256 + wl.M * wl.K].cpu().numpy().reshape(wl.M, wl.K)
    if inputs == "exact":
        assert np.array_equal(xq_gpu, xq_ref)
        helpers.check_gemm(got, ref, f"{name} norm -> fc13 (exact rows)")
    else:
        _, y_ref, _, _ = oracle.add_rmsnorm_quant(x, r, gam, eps)
        codes_close(xq_gpu, xq_ref, y_ref, f"{name} norm codes")
        slack = tie_flip_bound(y_ref, xq_ref, sx_ref, sub, s13, swiglu=True)
        helpers.check_gemm(got, ref, f"{name} norm -> fc13 (random rows)", slack=slack)


def test_xq_ready_plain_and_qkv_entries_read_the_producer_output():
    M, K = 4, 1024
    g = np.random.default_rng(600)
    x = exact_rows(g, M, K)
    gam = dg.rmsnorm_gain(g, K)
    w, s_w = dg.e4m3_weight(g, 384, K)
    wp = pack(dev_u8(w), 384, K)
    ws, n = new_ws(M, K)
    dl.check(dl.dl_add_rmsnorm_quant(dev_u16(x), None, None, dev_u16(gam), M, K, EPS_EXACT, ws, n))
    o1 = torch.empty((M, 384), dtype=torch.int16, device="cuda")
    o2 = torch.empty((M, 384), dtype=torch.int16, device="cuda")
    f = dl.DL_FLAG_PDL | dl.DL_FLAG_XQ_READY
    dl.check(dl.dl_gemm_e4m3(None, M, K, wp, dev_f32(s_w), 384, o1, ws, n, flags=f))
    dl.check(dl.dl_fc_qkv_scale(None, M, K, wp, dev_f32(s_w), 2, 1, 96, 0.5, o2, ws, n, flags=f))
    assert dl.dl_read_status(ws) == dl.DL_OK
    _, _, xq_ref, sx_ref = oracle.add_rmsnorm_quant(x, None, gam, EPS_EXACT)
    helpers.check_gemm(host_u16(o1), oracle.gemm_q(xq_ref, sx_ref, w, s_w), "xq-ready plain")
    helpers.check_gemm(host_u16(o2), oracle.fc_qkv_scale_q(xq_ref, sx_ref, w, s_w, 2, 1, 96, 0.5), "xq-ready qkv")


# ------------------------------------------------------------ whole layer --

def run_full_layer(wl, inp):
    from latency_decode_b200.layer import FullDecodeLayer
    lay = FullDecodeLayer(dev_u8(inp["w_qkv"]), inp["s_qkv"], dev_u8(inp["w_o"]), inp["s_o"], dev_u8(inp["w13"]),
                          inp["s13"], dev_u8(inp["w2"]), inp["s2"], dev_u16(inp["g1"]), dev_u16(inp["g2"]),
                          Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, q_scale=inp["q_scale"], M=wl.M, B=wl.B, T=wl.T,
                          cluster=wl.cluster)
    h = dev_u16(inp["h"])
    lay.step(dev_u16(inp["x"]), h, dev_u16(inp["k_cache"]), dev_u16(inp["v_cache"]), dev_i32(inp["seq_lens"]))
    lay.read_status()
    return helpers.bf16_to_f64(host_u16(lay.y)), host_u16(h)


@pytest.mark.parametrize("name", ["tiny", "layer_b1"])
def test_full_layer_chain(name):
    """The seven-kernel layer under PDL against the oracle chain.  Each later
    stage re-quantises to e4m3, so an attention output that is right within its
    tolerance still moves downstream codes; the bound is the oracle chain's own
    spread under attention noise at the attention tolerance
    (layer_chain_ref.chain_tolerance)."""
    wl = dg.WORKLOADS[name]
    inp = dg.full_layer_inputs(wl)
    y, h = run_full_layer(wl, inp)
    y_ref, h_ref = oracle_full_layer(inp, wl, 1e-5)
    tol_y, tol_h = chain_tolerance(inp, wl, 1e-5, y_ref, h_ref)
    assert np.isfinite(y).all()
    assert helpers.rel_l2(y, y_ref) <= tol_y, (helpers.rel_l2(y, y_ref), tol_y)
    assert helpers.rel_l2(helpers.bf16_to_f64(h), helpers.bf16_to_f64(h_ref)) <= tol_h


@pytest.mark.parametrize("name", ["tiny", "layer_b1"])
def test_full_layer_chain_identical_keys_at_the_gemm_bound(name):
    """With every cached key equal, the attention output is the mean of the
    visible values, which both sides compute to within a bf16 rounding; the
    seven-kernel chain then holds the GEMM bound (relative L2 <= 1e-2) at its
    output and on the residual stream."""
    wl = dg.WORKLOADS[name]
    inp = dg.full_layer_inputs(wl)
    inp["k_cache"] = np.ascontiguousarray(np.broadcast_to(inp["k_cache"][:, :, :1, :], inp["k_cache"].shape))
    y, h = run_full_layer(wl, inp)
    y_ref, h_ref = oracle_full_layer(inp, wl, 1e-5)
    assert np.isfinite(y).all()
    assert helpers.rel_l2(y, y_ref) <= helpers.GEMM_REL_L2, helpers.rel_l2(y, y_ref)
    assert helpers.rel_l2(helpers.bf16_to_f64(h), helpers.bf16_to_f64(h_ref)) <= helpers.GEMM_REL_L2


# ------------------------------------- RMSNorm producer + GEMM in one call --

@pytest.mark.parametrize("M", [1, 3, 8, 9, 24])
@pytest.mark.parametrize("inputs", ["exact", "random"])
def test_rmsnorm_fused_into_fc13(M, inputs):
    """dl_rmsnorm_fc13_swiglu (producer kernel + GEMM in one call).  Exact rows:
    codes identical to the oracle's, element-wise GEMM rule; random rows: codes
    may differ only at rounding ties, and the GEMM rule holds with the
    allowance widened by tie_flip_bound."""
    K, N2 = 2048, 512
    g = np.random.default_rng(700 + M + (inputs == "exact") * 50)
    if inputs == "exact":
        x = exact_rows(g, M, K)
        r = x.copy()
        eps = EPS_EXACT
    else:
        x = dg.bf16_normal(g, (M, K))
        r = dg.bf16_normal(g, (M, K), std=2.0)
        eps = 1e-5
    gam = dg.rmsnorm_gain(g, K)
    w, s_w = dg.e4m3_weight(g, N2, K)
    wp = torch.empty((N2, K), dtype=torch.uint8, device="cuda")
    dl.check(dl.dl_pack_fp8_weight(dev_u8(w), wp, N2, K, dl.DL_PACK_SWIGLU))
    ws, n = new_ws(M, K)
    hd = torch.full((M, K), -1, dtype=torch.int16, device="cuda")
    out = torch.empty((M, N2 // 2), dtype=torch.int16, device="cuda")
    for _ in range(2):  # twice on one stream: the second call must not see the first's h
        dl.check(dl.dl_rmsnorm_fc13_swiglu(dev_u16(x), dev_u16(r), hd, dev_u16(gam), eps, M, K, wp, dev_f32(s_w), N2,
                                           out, ws, n))
    assert dl.dl_read_status(ws) == dl.DL_OK
    h_ref, _, xq_ref, sx_ref = oracle.add_rmsnorm_quant(x, r, gam, eps)
    assert np.array_equal(host_u16(hd), h_ref)
    ref = oracle.fc13_swiglu_q(xq_ref, sx_ref, w, s_w)
    xq_gpu = ws[256:256 + M * K].cpu().numpy().reshape(M, K)
    if inputs == "exact":
        assert np.array_equal(xq_gpu, xq_ref)
        helpers.check_gemm(host_u16(out), ref, f"fused norm fc13 M={M}")
    else:
        _, y_ref, _, _ = oracle.add_rmsnorm_quant(x, r, gam, eps)
        codes_close(xq_gpu, xq_ref, y_ref, f"fused norm codes M={M}")
        slack = tie_flip_bound(y_ref, xq_ref, sx_ref, w, s_w, swiglu=True)
        helpers.check_gemm(host_u16(out), ref, f"fused norm fc13 M={M} (random rows)", slack=slack)


@pytest.mark.parametrize("M", [1, 5])
def test_rmsnorm_fused_into_qkv_without_residual_or_h(M):
    K, Hq, Hkv, d = 1024, 4, 2, 64
    N = (Hq + 2 * Hkv) * d
    g = np.random.default_rng(760 + M)
    x = exact_rows(g, M, K)
    gam = dg.rmsnorm_gain(g, K)
    w, s_w = dg.e4m3_weight(g, N, K)
    ws, n = new_ws(M, K)
    out = torch.empty((M, N), dtype=torch.int16, device="cuda")
    dl.check(dl.dl_rmsnorm_fc_qkv_scale(dev_u16(x), None, None, dev_u16(gam), EPS_EXACT, M, K, pack(dev_u8(w), N, K),
                                        dev_f32(s_w), Hq, Hkv, d, 0.125, out, ws, n))
    assert dl.dl_read_status(ws) == dl.DL_OK
    _, _, xq_ref, sx_ref = oracle.add_rmsnorm_quant(x, None, gam, EPS_EXACT)
    helpers.check_gemm(host_u16(out), oracle.fc_qkv_scale_q(xq_ref, sx_ref, w, s_w, Hq, Hkv, d, 0.125),
                       f"fused norm qkv M={M}")
