"""CUDA-graph replay of the PDL-chained decode step against the CPU oracle.

Xinzhiyuan report, section "通过 CUDA Graph 和重叠调度器减少主机端开销": the
step's kernels run from a CUDA graph, so the host launches one graph per step.
These tests capture the step exactly as the benchmark does (one graph holding
the PDL-chained steps of two layer replicas), replay it over rotating inputs
written into the buffers the graph reads, and check every replay's outputs
against the oracle on the same inputs (100 replays of the decode step at the
tiny and batch-1 shapes):

  - DecodeLayer.step (FC_QKV + scaling -> split-KV attention -> FC13 +
    SwiGLU) at tiny, layer_b1 and verify4; verify4 splits each kv head over
    several clusters, whose per-(head, owner) counters in the attention
    workspace must be back at zero after every replay;
  - DecodeLayer.step_host (copy kernels from and to pinned host memory around
    the chain) at tiny and layer_b1;
  - FullDecodeLayer.step (seven kernels, residual stream updated in place) at
    tiny and layer_b1.

Tolerances are those of the eager tests: GEMM rule for the projections,
relative L2 <= 5e-3 for attention, and the whole layer's derived bound; each
whole-layer replay must also reproduce an eager step's bits exactly."""
import dataclasses

import numpy as np
import pytest
import torch

import helpers
import oracle
from helpers import dev_i32, dev_u8, dev_u16, host_u16
from latency_decode_b200 import build as dl_build
from latency_decode_b200 import datagen as dg
from latency_decode_b200 import dl
from latency_decode_b200.layer import DecodeLayer, FullDecodeLayer
from layer_chain_ref import chain_tolerance, oracle_full_layer

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not helpers.gpu_available(), reason="needs a CUDA GPU")]

REPLICAS = 2
INPUT_SETS = [0, 1, 0]  # the input set written before each checked replay
# DecodeLayer.step: checked replays per workload, cycling through three input sets
# (the oracle runs once per set and replica)
STEP_REPLAYS = {"tiny": 100, "layer_b1": 100, "verify4": 12}


@pytest.fixture(scope="module", autouse=True)
def lib():
    dl_build.build()
    return dl.lib()


def replica_inputs(wl, r):
    """Weights and KV cache of replica r (its own seed)."""
    return dg.dense_layer_inputs(dataclasses.replace(wl, seed=9000 + 100 * wl.seed + r))


def activation_set(wl, r, j):
    g = dg.rng(9500 + 100 * wl.seed + 10 * r + j)
    return dg.bf16_normal(g, (wl.M, wl.K)), dg.bf16_normal(g, (wl.M, wl.K))


def oracle_step(wl, inp, x1, x2):
    """The chain on the oracle: its attention reads the oracle's own q (its
    QKV output in bf16)."""
    qkv = oracle.fc_qkv_scale(x1, inp["w_qkv"], inp["s_qkv"], wl.Hq, wl.Hkv, wl.d, inp["q_scale"])
    attn = oracle.decode_attn(oracle.f64_to_bf16(qkv).ravel(), wl.n_qkv, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d,
                              inp["k_cache"], inp["v_cache"], inp["seq_lens"], 1.0)
    ffn = oracle.fc13_swiglu(x2, inp["w13"], inp["s13"])
    return qkv, attn, ffn


def build_layers(wl):
    reps = []
    for r in range(REPLICAS):
        inp = replica_inputs(wl, r)
        lay = DecodeLayer(dev_u8(inp["w_qkv"]), inp["s_qkv"], dev_u8(inp["w13"]), inp["s13"], Hq=wl.Hq, Hkv=wl.Hkv,
                          d=wl.d, q_scale=inp["q_scale"], M=wl.M, B=wl.B, T=wl.T, cluster=wl.cluster)
        reps.append({"inp": inp, "lay": lay, "k": dev_u16(inp["k_cache"]), "v": dev_u16(inp["v_cache"]),
                     "sl": dev_i32(inp["seq_lens"])})
    return reps


def capture(fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        fn()
    return g


def counters_zero(lay, wl):
    n = 4 * wl.B * wl.Hkv * wl.cluster
    ws = lay.ws_attn
    return ws.numel() <= 256 or not ws[256:256 + n].any()


def check_step(wl, rep, j, x1, x2, attn_bits, ffn_bits, qkv_bits, what):
    if j not in rep.setdefault("refs", {}):  # the oracle's results for input set j, computed once
        rep["refs"][j] = oracle_step(wl, rep["inp"], x1, x2)
    qkv, attn, ffn = rep["refs"][j]
    if qkv_bits is not None:
        helpers.check_gemm(qkv_bits, qkv, f"{what} qkv")
    helpers.check_attn(attn_bits.reshape(attn.shape), attn, f"{what} attention")
    helpers.check_gemm(ffn_bits, ffn, f"{what} fc13")


@pytest.mark.parametrize("name", ["tiny", "layer_b1", "verify4"])
def test_decode_step_graph_replay_matches_the_oracle(name):
    wl = dg.WORKLOADS[name]
    reps = build_layers(wl)
    xin = [(torch.empty((wl.M, wl.K), dtype=torch.int16, device="cuda"),
            torch.empty((wl.M, wl.K), dtype=torch.int16, device="cuda")) for _ in range(REPLICAS)]

    def steps():
        for r, rep in enumerate(reps):
            rep["lay"].step(xin[r][0], xin[r][1], rep["k"], rep["v"], rep["sl"],
                            stream=torch.cuda.current_stream().cuda_stream)

    for r in range(REPLICAS):  # an eager step first: workspaces and kernel attributes are set up outside capture
        x1, x2 = activation_set(wl, r, 0)
        xin[r][0].copy_(dev_u16(x1))
        xin[r][1].copy_(dev_u16(x2))
    steps()
    torch.cuda.synchronize()
    graph = capture(steps)
    sets = {j: [activation_set(wl, r, j) for r in range(REPLICAS)] for j in range(3)}
    dev_sets = {j: [(dev_u16(a[0]), dev_u16(a[1])) for a in sets[j]] for j in sets}
    for k in range(STEP_REPLAYS[name]):
        j = (0, 1, 0, 2)[k % 4]
        acts = sets[j]
        for r in range(REPLICAS):
            xin[r][0].copy_(dev_sets[j][r][0])
            xin[r][1].copy_(dev_sets[j][r][1])
            reps[r]["lay"].attn_out.fill_(-1)
            reps[r]["lay"].ffn_out.fill_(-1)
        graph.replay()
        torch.cuda.synchronize()
        for r, rep in enumerate(reps):
            rep["lay"].read_status()
            assert counters_zero(rep["lay"], wl), f"replay {k}: attention counters not reset"
            check_step(wl, rep, j, acts[r][0], acts[r][1], host_u16(rep["lay"].attn_out),
                       host_u16(rep["lay"].ffn_out), host_u16(rep["lay"].qkv), f"{name} replay {k} replica {r}")
    # a burst of back-to-back replays with no host synchronisation in between
    j_last = (0, 1, 0, 2)[(STEP_REPLAYS[name] - 1) % 4]
    for _ in range(8):
        graph.replay()
    torch.cuda.synchronize()
    for r, rep in enumerate(reps):
        rep["lay"].read_status()
        assert counters_zero(rep["lay"], wl)
        check_step(wl, rep, j_last, sets[j_last][r][0], sets[j_last][r][1], host_u16(rep["lay"].attn_out),
                   host_u16(rep["lay"].ffn_out), None, f"{name} burst replica {r}")
    del graph


@pytest.mark.parametrize("name,overlap", [("tiny", False), ("layer_b1", False), ("tiny", True), ("layer_b1", True)])
def test_step_host_graph_replay_matches_the_oracle(name, overlap):
    """Activations from pinned host memory, results to pinned host memory, the
    transfers being copy kernels of the same PDL chain inside the graph (with
    overlap, each replica's upload runs beside the previous replica's
    download, DL_FLAG_COPY_NO_WAIT)."""
    wl = dg.WORKLOADS[name]
    reps = build_layers(wl)
    hx = [torch.empty((2, wl.M, wl.K), dtype=torch.int16).pin_memory() for _ in range(REPLICAS)]
    hout = [torch.empty_like(rep["lay"].out_buf, device="cpu").pin_memory() for rep in reps]

    def steps():
        for r, rep in enumerate(reps):
            rep["lay"].step_host(hx[r], hout[r], rep["k"], rep["v"], rep["sl"],
                                 stream=torch.cuda.current_stream().cuda_stream, overlap_upload=overlap)

    def write_inputs(j):
        acts = [activation_set(wl, r, j) for r in range(REPLICAS)]
        for r in range(REPLICAS):
            hx[r][0].copy_(torch.from_numpy(acts[r][0].view(np.int16)))
            hx[r][1].copy_(torch.from_numpy(acts[r][1].view(np.int16)))
            hout[r].fill_(-1)
        return acts

    write_inputs(0)
    steps()
    torch.cuda.synchronize()
    graph = capture(steps)
    n_attn = wl.B * wl.T * wl.Hq * wl.d
    for k, j in enumerate(INPUT_SETS):
        acts = write_inputs(j)
        graph.replay()
        torch.cuda.synchronize()
        for r, rep in enumerate(reps):
            rep["lay"].read_status()
            out = hout[r].numpy().view(np.uint16)
            check_step(wl, rep, j, acts[r][0], acts[r][1], out[:n_attn], out[n_attn:].reshape(wl.M, wl.N2 // 2),
                       None, f"{name} host replay {k} replica {r}")
    del graph


@pytest.mark.parametrize("name", ["tiny", "layer_b1"])
def test_full_layer_graph_replay_matches_the_oracle(name):
    """The seven-kernel layer captured once and replayed; before each replay the
    layer input x and the residual stream h (which the layer updates in place)
    are rewritten from an input set.  Each replay must give exactly the bits of
    an eager step on the same inputs (every kernel is deterministic), and match
    the oracle chain within the chain's derived bound
    (layer_chain_ref.chain_tolerance)."""
    wl = dg.WORKLOADS[name]
    base = dg.full_layer_inputs(wl)
    lay = FullDecodeLayer(dev_u8(base["w_qkv"]), base["s_qkv"], dev_u8(base["w_o"]), base["s_o"],
                          dev_u8(base["w13"]), base["s13"], dev_u8(base["w2"]), base["s2"], dev_u16(base["g1"]),
                          dev_u16(base["g2"]), Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, q_scale=base["q_scale"], M=wl.M,
                          B=wl.B, T=wl.T, cluster=wl.cluster)
    kc, vc, sl = dev_u16(base["k_cache"]), dev_u16(base["v_cache"]), dev_i32(base["seq_lens"])
    x = torch.empty((wl.M, wl.K), dtype=torch.int16, device="cuda")
    h = torch.empty((wl.M, wl.K), dtype=torch.int16, device="cuda")

    def sets(j):
        g = dg.rng(9700 + 100 * wl.seed + j)
        return dg.bf16_normal(g, (wl.M, wl.K)), dg.bf16_normal(g, (wl.M, wl.K))

    def step():
        lay.step(x, h, kc, vc, sl, stream=torch.cuda.current_stream().cuda_stream)

    def load(j):
        xj, hj = sets(j)
        x.copy_(dev_u16(xj))
        h.copy_(dev_u16(hj))
        lay.y.fill_(-1)
        return xj, hj

    eager = {}
    for j in sorted(set(INPUT_SETS)):  # eager steps first (also sets up the workspaces outside capture)
        load(j)
        step()
        torch.cuda.synchronize()
        lay.read_status()
        eager[j] = (host_u16(lay.y).copy(), host_u16(h).copy())
    graph = capture(step)
    refs = {}
    for k, j in enumerate(INPUT_SETS):
        xj, hj = load(j)
        graph.replay()
        torch.cuda.synchronize()
        lay.read_status()
        y_bits, h_bits = host_u16(lay.y), host_u16(h)
        assert np.array_equal(y_bits, eager[j][0]) and np.array_equal(h_bits, eager[j][1]), f"replay {k}"
        if j not in refs:
            inp = dict(base, x=xj, h=hj)
            y_ref, h_ref = oracle_full_layer(inp, wl, 1e-5)
            refs[j] = (y_ref, h_ref) + chain_tolerance(inp, wl, 1e-5, y_ref, h_ref)
        y_ref, h_ref, tol_y, tol_h = refs[j]
        y = helpers.bf16_to_f64(y_bits)
        assert np.isfinite(y).all()
        assert helpers.rel_l2(y, y_ref) <= tol_y, (k, helpers.rel_l2(y, y_ref), tol_y)
        assert helpers.rel_l2(helpers.bf16_to_f64(h_bits), helpers.bf16_to_f64(h_ref)) <= tol_h
    del graph
