#!/usr/bin/env python
"""Benchmark of one decode layer's hot path on B200: act-quant -> FC_QKV +
attention scaling -> split-KV attention with cluster DSMEM merge -> act-quant ->
FC13 + SwiGLU, PDL-chained, all in libdl.so.

Default workload: the batch-1 decode layer (1 token, FC_QKV 5120->7168,
FC13 5120->2x8192, attention 40/8 heads d=128 over 4096 cached keys).  Inputs
are synthetic and seeded.  Every timed step runs on a different copy of the
layer (weights and KV cache), and one rotation over the copies moves more than
three times the 126 MB L2, so each step streams its weights and KV from HBM.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on the
same workload instead (the deliberately slow reference arm).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs per decode layer; achieved HBM TB/s vs B200 peak (FP8 GEMM, split-KV attn)"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="layer_b1")
    p.add_argument("--cluster", type=int, default=0, help="attention cluster size (0 = workload default)")
    p.add_argument("--replicas", type=int, default=0, help="layer copies to rotate through (0 = auto)")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle CPU-baseline sample length")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-full-layer", action="store_true", help="skip the whole-layer (7-kernel) figure")
    p.add_argument("--configs", default="verify4,batch16x4,moe64",
                   help="other workloads measured after the headline (comma list, or 'none')")
    p.add_argument("--profile-steps", type=int, default=0,
                   help="only run this many direct-launch layer steps (for a profiler), print no JSON line")
    p.add_argument("--profile-moe", type=int, default=0,
                   help="only run this many grouped MoE FC13 + SwiGLU calls of the moe64 workload (for a "
                        "profiler), print no JSON line")
    p.add_argument("--profile-next", type=int, default=0,
                   help="only run this many direct-launch whole-layer steps, FP8-cache attention calls and "
                        "verification calls (for a profiler), print no JSON line")
    return p.parse_args()


def env_int(name, default):
    v = os.environ.get(name)
    return int(v) if v is not None else default


def max_over_ranks(value: float) -> float:
    """The largest of `value` over all ranks (one process per GPU); the value
    itself when torch.distributed is not initialised.  Every rank must call it
    at the same point."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config(wl, cluster):
    # L = 0 in the table means per-sequence lengths drawn uniformly from [1024, 16384] (seeded)
    kv = wl.L if wl.L > 0 else "U[1024,16384]"
    return {"workload": f"{wl.name}: M={wl.M} K={wl.K} FC_QKV N={wl.n_qkv} FC13 N2={wl.N2} "
                        f"attn B={wl.B} T={wl.T} Hq={wl.Hq} Hkv={wl.Hkv} d={wl.d} L={kv} cluster={cluster}",
            "tokens": wl.M, "hidden": wl.K, "kv_len": kv, "heads_q": wl.Hq, "heads_kv": wl.Hkv,
            "head_dim": wl.d, "cluster": cluster,
            "l2": "inputs larger than L2: each step uses another layer copy; one rotation > 3x L2"}


# ---------------------------------------------------------------- oracle arm --

def oracle_layer_inputs(wl):
    from latency_decode_b200 import datagen as dg
    return dg.dense_layer_inputs(wl)


def oracle_layer(wl, inp):
    """One layer through the CPU oracle (same steps as the GPU path).  Returns
    (qkv, attention output, FC13 output), float64."""
    import numpy as np
    import oracle
    from latency_decode_b200 import datagen as dg
    qkv = oracle.fc_qkv_scale(inp["x1"], inp["w_qkv"], inp["s_qkv"], wl.Hq, wl.Hkv, wl.d, inp["q_scale"])
    qb = dg.bf16_bits(qkv.astype(np.float32))
    attn = oracle.decode_attn(qb.ravel(), wl.n_qkv, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, inp["k_cache"],
                              inp["v_cache"], inp["seq_lens"], 1.0)
    ffn = oracle.fc13_swiglu(inp["x2"], inp["w13"], inp["s13"])
    return qkv, attn, ffn


def time_oracle(wl, inp, seconds, min_reps=1, max_reps=10**6):
    reps, t0 = 0, time.perf_counter()
    while reps < min_reps or (time.perf_counter() - t0 < seconds and reps < max_reps):
        oracle_layer(wl, inp)
        reps += 1
    dt = time.perf_counter() - t0
    return dt / reps * 1e6, reps, dt


def host_cores(cap=16):
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, cap))


def sliced_oracle_inputs(wl, inp, fc13_cols=256):
    """The slices of one layer's inputs that oracle_layer_sliced hands to its
    threads: the QKV weight rows of each head, the FC13 gate and up rows of each
    range of `fc13_cols` output columns (gate rows then the matching up rows),
    and the K and V caches of each kv head.  Built once, outside any timing."""
    import numpy as np
    d, F = wl.d, wl.N2 // 2
    heads = [(c0, c0 + d) for c0 in range(0, wl.n_qkv, d)]
    w_heads = [np.ascontiguousarray(inp["w_qkv"][c0:c1]) for c0, c1 in heads]
    cols = [(j0, min(F, j0 + fc13_cols)) for j0 in range(0, F, fc13_cols)]
    w13 = [np.ascontiguousarray(np.concatenate([inp["w13"][j0:j1], inp["w13"][F + j0:F + j1]])) for j0, j1 in cols]
    kv = [(np.ascontiguousarray(inp["k_cache"][:, hk:hk + 1]), np.ascontiguousarray(inp["v_cache"][:, hk:hk + 1]))
          for hk in range(wl.Hkv)]
    return {"heads": heads, "w_heads": w_heads, "cols": cols, "w13": w13, "kv": kv}


def oracle_layer_sliced(wl, inp, sl, pool):
    """One layer through the CPU oracle with its independent outputs spread over
    the threads of `pool`: FC_QKV one head of output columns per task, the
    attention one query head per task, FC13 one range of output columns per
    task (FC13 runs beside QKV and attention: its input does not depend on
    them).  Every task is a call of the oracle's own function on a slice of the
    weights, or on one head, and the tasks fill disjoint parts of the outputs,
    so the result equals oracle_layer's bit for bit.  ctypes releases the GIL
    for the duration of each call, so the tasks run on as many host cores as
    the pool has threads.  Returns (qkv, attention output, FC13 output)."""
    import numpy as np
    import oracle
    from latency_decode_b200 import datagen as dg
    d, Hq, Hkv = wl.d, wl.Hq, wl.Hkv
    G = Hq // Hkv
    qkv = np.zeros((wl.M, wl.n_qkv))
    ffn = np.zeros((wl.M, wl.N2 // 2))
    attn = np.zeros((wl.B, wl.T, Hq, d))

    def qkv_task(i):
        c0, c1 = sl["heads"][i]
        if c0 < Hq * d:  # one query head: scaled columns
            qkv[:, c0:c1] = oracle.fc_qkv_scale(inp["x1"], sl["w_heads"][i], inp["s_qkv"], 1, 0, d, inp["q_scale"])
        else:            # one K or V head: plain columns
            qkv[:, c0:c1] = oracle.linear(inp["x1"], sl["w_heads"][i], inp["s_qkv"])

    def fc13_task(i):
        j0, j1 = sl["cols"][i]
        ffn[:, j0:j1] = oracle.fc13_swiglu(inp["x2"], sl["w13"][i], inp["s13"])

    def attn_task(h, qb):
        kc, vc = sl["kv"][h // G]
        attn[:, :, h:h + 1] = oracle.decode_attn(qb[h * d:], wl.n_qkv, wl.B, wl.T, 1, 1, d, kc, vc,
                                                 inp["seq_lens"], 1.0)

    f13 = [pool.submit(fc13_task, i) for i in range(len(sl["cols"]))]
    for f in [pool.submit(qkv_task, i) for i in range(len(sl["heads"]))]:
        f.result()
    qb = dg.bf16_bits(qkv.astype(np.float32)).ravel()
    for f in [pool.submit(attn_task, h, qb) for h in range(Hq)] + f13:
        f.result()
    return qkv, attn, ffn


def time_oracle_threads(wl, inp, seconds, cores, min_reps=1):
    """Per-layer latency of the oracle with each layer's outputs spread over
    `cores` host threads (oracle_layer_sliced).  Returns (us per layer, layers
    timed, seconds)."""
    from concurrent.futures import ThreadPoolExecutor
    sl = sliced_oracle_inputs(wl, inp)
    with ThreadPoolExecutor(max_workers=cores) as pool:
        oracle_layer_sliced(wl, inp, sl, pool)  # warm-up
        reps, t0 = 0, time.perf_counter()
        while reps < min_reps or time.perf_counter() - t0 < seconds:
            oracle_layer_sliced(wl, inp, sl, pool)
            reps += 1
        dt = time.perf_counter() - t0
    return dt / reps * 1e6, reps, dt


def run_reference(args):
    rank = env_int("RANK", 0)
    if rank != 0:
        return 0
    from latency_decode_b200 import datagen as dg
    wl = dg.WORKLOADS[args.workload]
    cluster = args.cluster or wl.cluster
    inp = oracle_layer_inputs(wl)
    for _ in range(args.warmup):
        oracle_layer(wl, inp)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_layer(wl, inp)
        times.append(time.perf_counter() - t0)
    us = sum(times) / len(times) * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": "us", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, cluster),
        "cpu_baseline": {"value": us, "unit": "us", "cores": 1, "kind": "oracle",
                         "sample": f"{args.steps} full {wl.name} layers (QKV GEMM, attention, FC13) "
                                   "through the single-threaded FP64 C++ oracle"},
        "e2e": {"value": us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- clocks --------

class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of one GPU
    through NVML from a background thread (~1 kHz), so that even a
    sub-second timed region gets samples.  Read-only: changes no setting."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, torch_device_index):
        self.idx = torch_device_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._nvml = None
        self._handle = None

    def start(self):
        import threading
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(self.idx)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self._handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM))
            self._nvml = pynvml
        except Exception:  # NVML unavailable: report "unsampled"
            self._nvml = None
            return
        self._stop = threading.Event()

        def loop():
            nv, h = self._nvml, self._handle
            bits = {k: getattr(nv, v) for k, v in self.REASONS.items()}
            while not self._stop.is_set():
                try:
                    self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for k, b in bits.items():
                        if r & b:
                            self.reasons.add(k)
                except Exception:
                    pass
                time.sleep(0.001)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        self._stop.set()
        self._thread.join(timeout=5)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------- GPU arm --------

def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) that
    a committed ncu summary under profiles/ records for this kernel and
    workload, or None when there is no record or when the kernel source has
    changed since the capture (the record carries the source's sha256)."""
    import glob
    import hashlib
    import re
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        for line in open(path):
            if not line.startswith("traffic-record:"):
                continue
            f = dict(kv.split("=", 1) for kv in line.split()[1:] if "=" in kv)
            if f.get("kernel") != kernel or f.get("workload") != workload:
                continue
            src = os.path.join(ROOT, f.get("source", ""))
            if not os.path.isfile(src):
                return None
            digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
            return int(f["bytes_per_launch"]) if digest == f.get("sha256_16") else None
    return None


def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def make_layers(wl, R, seed_base, device, cluster):
    import torch
    from latency_decode_b200 import datagen as dg
    from latency_decode_b200.layer import DecodeLayer
    import numpy as np
    layers, kvs, xs = [], [], []
    g = dg.rng(wl.seed)
    sl = dg.seq_lens_for(wl, g)
    seq_lens = torch.from_numpy(sl).to(device)
    for r in range(R):
        gen = torch.Generator(device=device).manual_seed(seed_base + r)
        wq, sq = dg.e4m3_weight_torch(gen, wl.n_qkv, wl.K, device)
        w13, s13 = dg.e4m3_weight_torch(gen, wl.N2, wl.K, device)
        layer = DecodeLayer(wq, sq, w13, s13, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, q_scale=1.0 / math.sqrt(wl.d),
                            M=wl.M, B=wl.B, T=wl.T, cluster=cluster, device=device)
        del wq, w13
        kc = torch.randn((wl.B, wl.Hkv, wl.Lcap, wl.d), generator=gen, device=device).to(torch.bfloat16)
        vc = torch.randn((wl.B, wl.Hkv, wl.Lcap, wl.d), generator=gen, device=device).to(torch.bfloat16)
        x1 = torch.randn((wl.M, wl.K), generator=gen, device=device).to(torch.bfloat16)
        x2 = torch.randn((wl.M, wl.K), generator=gen, device=device).to(torch.bfloat16)
        layers.append(layer)
        kvs.append((kc.view(torch.int16), vc.view(torch.int16)))
        xs.append((x1.view(torch.int16), x2.view(torch.int16)))
    torch.cuda.synchronize()
    return layers, kvs, xs, seq_lens, sl


def make_full_layers(wl, R, seed_base, device, cluster):
    """R independent whole pre-norm layers (QKV, attention, O_proj, FC13, FC2,
    two RMSNorms), random weights of the workload's shapes drawn on the device."""
    import torch
    from latency_decode_b200 import datagen as dg
    from latency_decode_b200.layer import FullDecodeLayer
    out = []
    for r in range(R):
        gen = torch.Generator(device=device).manual_seed(seed_base + r)
        wq, sq = dg.e4m3_weight_torch(gen, wl.n_qkv, wl.K, device)
        wo, so = dg.e4m3_weight_torch(gen, wl.K, wl.k_o, device)
        w13, s13 = dg.e4m3_weight_torch(gen, wl.N2, wl.K, device)
        w2, s2 = dg.e4m3_weight_torch(gen, wl.K, wl.k_fc2, device)
        gains = [(1.0 + 0.1 * torch.randn(wl.K, generator=gen, device=device)).to(torch.bfloat16).view(torch.int16)
                 for _ in range(2)]
        lay = FullDecodeLayer(wq, sq, wo, so, w13, s13, w2, s2, gains[0], gains[1], Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d,
                              q_scale=1.0 / math.sqrt(wl.d), M=wl.M, B=wl.B, T=wl.T, cluster=cluster,
                              device=device)
        del wq, wo, w13, w2
        kc = torch.randn((wl.B, wl.Hkv, wl.Lcap, wl.d), generator=gen, device=device).to(torch.bfloat16)
        vc = torch.randn((wl.B, wl.Hkv, wl.Lcap, wl.d), generator=gen, device=device).to(torch.bfloat16)
        x = torch.randn((wl.M, wl.K), generator=gen, device=device).to(torch.bfloat16)
        hres = torch.randn((wl.M, wl.K), generator=gen, device=device).to(torch.bfloat16)
        out.append((lay, kc.view(torch.int16), vc.view(torch.int16), x.view(torch.int16), hres.view(torch.int16)))
    torch.cuda.synchronize()
    return out


def measure_next_rows(wl, fl, seq_lens, device, cluster, steps, per_call_us, peak):
    """Per-call device time of the rows beyond the headline chain, each timed the
    way the headline kernels are (graphs of back-to-back calls over more than
    3x L2 of distinct inputs, exactly `steps` calls), with its algorithmic bytes
    and roofline fraction."""
    import torch
    from latency_decode_b200 import dl

    out = {}
    RF = len(fl)

    def entry(res, nbytes, extra=None):
        us, mode, lengths = res
        gbs = nbytes / (us * 1e-6) / 1e9
        e = {"us_per_call": us, "alg_bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / peak, "mode": mode,
             "graph_steps": lengths}
        e.update(extra or {})
        return e

    h = lambda: torch.cuda.current_stream().cuda_stream
    G = RF * max(1, 24 // RF)
    # NEXT-1: plain projections and the RMSNorm producer
    def o_proj(i):
        lay = fl[i % RF][0]
        dl.check(dl.dl_gemm_e4m3(lay.attn_out, wl.M, wl.k_o, lay.wp["o"], lay.s["o"], wl.K, lay.a, lay.ws_o,
                                 stream=h()))
    def fc2(i):
        lay = fl[i % RF][0]
        dl.check(dl.dl_gemm_e4m3(lay.f, wl.M, wl.k_fc2, lay.wp["2"], lay.s["2"], wl.K, lay.y, lay.ws_2, stream=h()))
    def norm(i):
        lay, kc, vc, x, hres = fl[i % RF]
        dl.check(dl.dl_add_rmsnorm_quant(x, hres, hres, lay.g1, wl.M, wl.K, 1e-5, lay.ws_qkv, stream=h()))
    out["o_proj"] = entry(per_call_us(o_proj, G, steps), wl.K * wl.k_o)
    out["fc2"] = entry(per_call_us(fc2, G, steps), wl.K * wl.k_fc2)
    out["add_rmsnorm_quant"] = entry(per_call_us(norm, G, steps), 3 * wl.M * wl.K * 2 + wl.M * wl.K,
                                     {"note": "latency-bound at this size"})
    out.update(measure_fp8_attn_and_verify(wl, [f[0] for f in fl], seq_lens, device, cluster, steps,
                                           per_call_us, peak))
    torch.cuda.empty_cache()
    return out


def measure_fp8_attn_and_verify(wl, q_layers, seq_lens, device, cluster, steps, per_call_us, peak):
    """Per-call device time of NEXT-3 (attention over an e4m3 cache, half the
    bytes of the bf16 cache; q from the layers' QKV outputs) and NEXT-4 (greedy
    verification over the full vocabulary at the workload's B and T), timed as
    the headline kernels are: graphs of back-to-back calls over more than 3x L2
    of distinct inputs, exactly `steps` calls."""
    import torch
    from latency_decode_b200 import datagen as dg
    from latency_decode_b200 import dl

    out = {}
    RL = len(q_layers)
    h = lambda: torch.cuda.current_stream().cuda_stream

    def entry(res, nbytes, extra=None):
        us, mode, lengths = res
        gbs = nbytes / (us * 1e-6) / 1e9
        e = {"us_per_call": us, "alg_bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / peak, "mode": mode,
             "graph_steps": lengths}
        e.update(extra or {})
        return e

    if wl.d == 128:
        sl_host = seq_lens.cpu().numpy()
        kv8 = int(sum(2 * wl.Hkv * int(L) * wl.d for L in sl_host))
        R8 = max(2, -(-3 * 126 * 10**6 // (2 * wl.B * wl.Hkv * wl.Lcap * wl.d)))
        gen = torch.Generator(device=device).manual_seed(77)
        caches = [tuple(torch.randint(0, 0x7E, shape, generator=gen, device=device, dtype=torch.uint8)
                        for shape in ((wl.B, wl.Hkv, wl.Lcap, wl.d), (wl.B, wl.Hkv, wl.d, wl.Lcap)))  # K, V^T
                  for _ in range(R8)]
        scales = torch.tensor([0.01, 0.02], dtype=torch.float32, device=device)
        n = dl.dl_decode_attn_fp8kv_workspace_bytes(wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, wl.Lcap, cluster)
        wss = [torch.zeros(n, dtype=torch.uint8, device=device) for _ in range(R8)]

        def attn8(i):
            r = i % R8
            lay = q_layers[i % RL]
            dl.check(dl.dl_decode_attn_fp8kv(lay.qkv, lay.N_qkv, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, caches[r][0],
                                             caches[r][1], scales, wl.Lcap, seq_lens, 1.0, cluster, lay.attn_out,
                                             wss[r], stream=h()))

        for i in range(3):
            attn8(i)
        out["decode_attn_fp8kv"] = entry(per_call_us(attn8, R8 * max(1, 24 // R8), steps), kv8)
        for w in wss:
            dl.check(dl.dl_read_status(w))
        del caches, wss
    V = dg.VOCAB
    per = wl.B * wl.T * V * 2
    RV = max(2, min(2048, -(-3 * 126 * 10**6 // per)))
    lg = torch.randn((RV, wl.B, wl.T, V), device=device).to(torch.bfloat16).view(torch.int16)
    dr = torch.randint(0, V, (wl.B, max(1, wl.T - 1)), device=device, dtype=torch.int32)
    tid = torch.empty((wl.B, wl.T), dtype=torch.int32, device=device)
    nacc = torch.empty((wl.B,), dtype=torch.int32, device=device)
    em = torch.empty((wl.B, wl.T), dtype=torch.int32, device=device)

    def verify(i):
        dl.check(dl.dl_spec_verify_greedy(lg[i % RV], wl.B, wl.T, V, dr, tid, nacc, em, None, stream=h()))

    out["spec_verify_greedy"] = entry(per_call_us(verify, RV * max(1, 24 // RV) if RV < 24 else RV, steps), per,
                                      {"vocab": V})
    del lg
    torch.cuda.empty_cache()
    return out


def profile_moe(n, device, experts=16):
    """n grouped FC13 + SwiGLU calls at the moe64 shapes (64 tokens, experts of
    [16384, 5120] e4m3 drawn on the device, top-1 uniform routes) over a bank of
    `experts` experts: 16 (1.3 GB) keeps a multi-pass profiler capture small."""
    import torch
    from latency_decode_b200 import datagen as dg
    from latency_decode_b200 import dl

    wl = dg.WORKLOADS["moe64"]
    g = dg.rng(wl.seed)
    x = torch.from_numpy(dg.bf16_normal(g, (wl.M, wl.K)).view("int16")).to(device)
    ids = torch.from_numpy(g.integers(0, experts, size=wl.M).astype("int32")).to(device)
    gen = torch.Generator(device=device).manual_seed(wl.seed)
    bank = torch.empty((experts, wl.N2, wl.K), dtype=torch.uint8, device=device)
    scales = torch.empty(experts, dtype=torch.float32, device=device)
    for e in range(experts):
        codes, s = dg.e4m3_weight_torch(gen, wl.N2, wl.K, device)
        dl.check(dl.dl_pack_fp8_weight(codes, bank[e], wl.N2, wl.K, dl.DL_PACK_SWIGLU))
        scales[e] = s
    out = torch.empty((wl.M, wl.N2 // 2), dtype=torch.int16, device=device)
    ws = torch.zeros(dl.dl_workspace_bytes(wl.M, wl.K), dtype=torch.uint8, device=device)
    for _ in range(n):
        dl.check(dl.dl_moe_fc13_swiglu_grouped(x, wl.M, wl.K, ids, experts, bank, scales, wl.N2, out, ws))
    dl.check(dl.dl_read_status(ws))


def profile_next_rows(wl, n, seq_lens, device, cluster):
    """n direct-launch steps of the whole layer, n FP8-cache attention calls and
    n verification calls over the full vocabulary, on two replicas (the input of
    an ncu capture of those kernels)."""
    import torch
    from latency_decode_b200 import datagen as dg
    from latency_decode_b200 import dl

    fl = make_full_layers(wl, 2, 7000, device, cluster)
    gen = torch.Generator(device=device).manual_seed(78)
    c8 = [torch.randint(0, 0x7E, shape, generator=gen, device=device, dtype=torch.uint8)
          for shape in ((wl.B, wl.Hkv, wl.Lcap, wl.d), (wl.B, wl.Hkv, wl.d, wl.Lcap))]  # K, V^T
    scales = torch.tensor([0.01, 0.02], dtype=torch.float32, device=device)
    ws8 = torch.zeros(dl.dl_decode_attn_fp8kv_workspace_bytes(wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, wl.Lcap, cluster),
                      dtype=torch.uint8, device=device)
    V = dg.VOCAB
    lg = torch.randn((wl.B, wl.T, V), generator=gen, device=device).to(torch.bfloat16).view(torch.int16)
    dr = torch.randint(0, V, (wl.B, max(1, wl.T - 1)), generator=gen, device=device, dtype=torch.int32)
    tid = torch.empty((wl.B, wl.T), dtype=torch.int32, device=device)
    nacc = torch.empty((wl.B,), dtype=torch.int32, device=device)
    em = torch.empty((wl.B, wl.T), dtype=torch.int32, device=device)
    h = torch.cuda.current_stream().cuda_stream
    for i in range(n):
        lay, kc, vc, x, hres = fl[i % 2]
        lay.step(x, hres, kc, vc, seq_lens, stream=h)
        dl.check(dl.dl_decode_attn_fp8kv(lay.qkv, lay.N_qkv, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, c8[0], c8[1], scales,
                                         wl.Lcap, seq_lens, 1.0, cluster, lay.attn_out, ws8, stream=h))
        dl.check(dl.dl_spec_verify_greedy(lg, wl.B, wl.T, V, dr, tid, nacc, em, None, stream=h))
    for entry in fl:
        entry[0].read_status(h)
    dl.check(dl.dl_read_status(ws8, h))


def gemm_launches(M, K):
    """Kernels one GEMM entry point launches: the GEMM quantises inputs of up to
    32768 elements itself, larger ones get a quantise kernel first."""
    return 1 if M * K <= 32768 else 2


def replay_plan(n: int, period: int) -> list:
    """Lengths of the CUDA graphs replayed, in order, to run exactly n steps:
    graphs of `period` PDL-chained steps, then one graph of the remaining
    n mod period steps.  Every replayed graph chains several steps (a run of
    fewer than `period` steps is one graph of n steps), so the timed region
    has the same shape whatever n is; `period` is a multiple of the replica
    count, so each graph starts again at replica 0."""
    if n <= 0:
        return []
    q, rem = divmod(n, period)
    return [period] * q + ([rem] if rem else [])


class GraphReplayer:
    """CUDA graphs of fn(0), fn(1), ... fn(L-1) for each length L that
    replay_plan asks for, captured once; run(n) replays exactly n steps."""

    def __init__(self, fn, period, capture):
        self.fn, self.period, self.capture = fn, period, capture
        self.graphs = {}

    def prepare(self, n):
        for length in sorted(set(replay_plan(n, self.period))):
            if length not in self.graphs:
                self.graphs[length] = self.capture(self.fn, range(length))
        return self

    def run(self, n):
        self.prepare(n)
        for length in replay_plan(n, self.period):
            self.graphs[length].replay()

    def warm(self, n):
        """One untimed replay of the plan's first graph (the graphs must be
        prepared): queued right before the timed replays, so that the first
        timed graph is launched while another graph runs, as every graph after
        the first is, instead of after an idle stream."""
        plan = replay_plan(n, self.period)
        if plan:
            self.graphs[plan[0]].replay()

    def lengths(self, n):
        return sorted(set(replay_plan(n, self.period)), reverse=True)

    def release(self):
        self.graphs.clear()


def timed(fn, steps, stream):
    import torch
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        fn(i)
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end)  # ms


def peak_bf16_tflops():
    """Dense bf16 tensor peak (TFLOP/s): the measured burst figure when the
    generated file exists, else the recorded fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback"


def measure_dense_config(name, steps, device, rank, per_call_us, peak, peak_bf16):
    """Chain and per-call figures of one more dense workload (verify4,
    batch16x4): its own layer copies (> 3x L2 per rotation), the chain
    FC_QKV -> attention -> FC13 replayed from CUDA graphs, and each kernel
    family per call, with algorithmic bytes, the fraction of the HBM peak and
    the tensor-core rate (FP8 GEMMs against twice the bf16 peak, the nominal
    ratio; bf16 attention against the bf16 peak)."""
    import torch
    from latency_decode_b200 import datagen as dg
    from latency_decode_b200 import dl

    wl = dg.WORKLOADS[name]
    cluster = wl.cluster
    per_layer = wl.n_qkv * wl.K + wl.N2 * wl.K + 2 * wl.B * wl.Hkv * wl.Lcap * wl.d * 2
    R = max(2, math.ceil(3 * L2_BYTES / per_layer))
    layers, kvs, xs, seq_lens, sl = make_layers(wl, R, 3000 * (rank + 1) + 100 * wl.seed, device, cluster)
    h = lambda: torch.cuda.current_stream().cuda_stream

    def step(i):
        r = i % R
        layers[r].step(xs[r][0], xs[r][1], kvs[r][0], kvs[r][1], seq_lens, stream=h())

    def call_qkv(i):
        r = i % R
        L_ = layers[r]
        dl.check(dl.dl_fc_qkv_scale(xs[r][0], wl.M, wl.K, L_.wp_qkv, L_.s_qkv, wl.Hq, wl.Hkv, wl.d, L_.q_scale,
                                    L_.qkv, L_.ws_qkv, stream=h()))

    def call_attn(i):
        r = i % R
        L_ = layers[r]
        dl.check(dl.dl_decode_attn(L_.qkv, L_.N_qkv, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, kvs[r][0], kvs[r][1],
                                   wl.Lcap, seq_lens, 1.0, cluster, L_.attn_out, L_.ws_attn, stream=h()))

    def call_fc13(i):
        r = i % R
        L_ = layers[r]
        dl.check(dl.dl_fc13_swiglu(xs[r][1], wl.M, wl.K, L_.wp_13, L_.s_13, wl.N2, L_.ffn_out, L_.ws_13,
                                   stream=h()))

    G = R * max(1, 24 // R)
    for i in range(3):
        step(i)
    chain_us, chain_mode, lengths = per_call_us(step, G, steps)
    kv_bytes = int(sum(2 * wl.Hkv * int(L) * wl.d * 2 for L in sl))
    attn_flops = float(sum(4 * wl.Hq * wl.T * int(L) * wl.d for L in sl))  # QK^T and PV, every key of every row
    fam = {"fc_qkv_scale": (call_qkv, wl.n_qkv * wl.K, 2.0 * wl.M * wl.n_qkv * wl.K, 2 * peak_bf16),
           "decode_attn": (call_attn, kv_bytes, attn_flops, peak_bf16),
           "fc13_swiglu": (call_fc13, wl.N2 * wl.K, 2.0 * wl.M * wl.N2 * wl.K, 2 * peak_bf16)}
    kernels = {}
    for kname, (fn, nbytes, flops, tpeak) in fam.items():
        for i in range(3):
            fn(i)
        us, mode, _ = per_call_us(fn, G, steps)
        gbs = nbytes / (us * 1e-6) / 1e9
        kernels[kname] = {"us_per_call": us, "alg_bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / peak,
                          "tensor_tflops": flops / (us * 1e-6) / 1e12,
                          "tensor_frac": flops / (us * 1e-6) / 1e12 / tpeak, "mode": mode}
    for lay in layers:
        lay.read_status(h())
    for kname, e in measure_fp8_attn_and_verify(wl, layers, seq_lens, device, cluster, steps, per_call_us,
                                                peak).items():
        kernels[kname] = e
    layer_bytes = wl.n_qkv * wl.K + wl.N2 * wl.K + kv_bytes
    out = {"workload": f"{wl.name}: M={wl.M} B={wl.B} T={wl.T} L={'U[1024,16384]' if wl.L == 0 else wl.L} "
                       f"cluster={cluster}",
           "chain_us": chain_us, "alg_bytes": layer_bytes, "achieved_gbs": layer_bytes / (chain_us * 1e-6) / 1e9,
           "frac": layer_bytes / (chain_us * 1e-6) / 1e9 / peak, "mode": chain_mode, "graph_steps": lengths,
           "replicas": R, "kernels": kernels}
    del layers, kvs, xs
    torch.cuda.empty_cache()
    return out


def measure_moe_config(steps, device, per_call_us, peak, peak_bf16):
    """Grouped MoE FC13 + SwiGLU at the moe64 shapes: 64 tokens routed top-1
    uniformly (seeded) over 128 experts of [16384, 5120] e4m3 drawn on the
    device (10.7 GB); each call reads only the touched experts (> 4 GB, far
    beyond L2)."""
    import numpy as np
    import torch
    from latency_decode_b200 import datagen as dg
    from latency_decode_b200 import dl

    wl = dg.WORKLOADS["moe64"]
    g = dg.rng(wl.seed)
    x = torch.from_numpy(dg.bf16_normal(g, (wl.M, wl.K)).view("int16")).to(device)
    ids_h = dg.expert_ids_for(wl, g)
    ids = torch.from_numpy(ids_h).to(device)
    gen = torch.Generator(device=device).manual_seed(wl.seed)
    bank = torch.empty((wl.experts, wl.N2, wl.K), dtype=torch.uint8, device=device)
    scales = torch.empty(wl.experts, dtype=torch.float32, device=device)
    for e in range(wl.experts):
        codes, s = dg.e4m3_weight_torch(gen, wl.N2, wl.K, device)
        dl.check(dl.dl_pack_fp8_weight(codes, bank[e], wl.N2, wl.K, dl.DL_PACK_SWIGLU))
        scales[e] = s
        del codes
    out = torch.empty((wl.M, wl.N2 // 2), dtype=torch.int16, device=device)
    ws = torch.zeros(dl.dl_workspace_bytes(wl.M, wl.K), dtype=torch.uint8, device=device)

    def call(i):
        dl.check(dl.dl_moe_fc13_swiglu_grouped(x, wl.M, wl.K, ids, wl.experts, bank, scales, wl.N2, out, ws,
                                               stream=torch.cuda.current_stream().cuda_stream))

    for i in range(3):
        call(i)
    us, mode, lengths = per_call_us(call, 8, steps)
    dl.check(dl.dl_read_status(ws))
    touched = int(np.unique(ids_h).size)
    nbytes = touched * wl.N2 * wl.K
    flops = 2.0 * wl.M * wl.N2 * wl.K
    gbs = nbytes / (us * 1e-6) / 1e9
    res = {"workload": f"moe64: T={wl.M} E={wl.experts} top-1, FC13 {wl.K}->{wl.N2} per expert",
           "us_per_call": us, "touched_experts": touched, "alg_bytes": nbytes, "achieved_gbs": gbs,
           "frac": gbs / peak, "tensor_tflops": flops / (us * 1e-6) / 1e12,
           "tensor_frac": flops / (us * 1e-6) / 1e12 / (2 * peak_bf16), "mode": mode, "graph_steps": lengths}
    del bank, x, out, ws
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist
    from latency_decode_b200 import build as dl_build
    from latency_decode_b200 import datagen as dg
    from latency_decode_b200 import dl

    rank, world, local = env_int("RANK", 0), env_int("WORLD_SIZE", 1), env_int("LOCAL_RANK", 0)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU for --impl ours")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    dl_build.build()
    dl.lib()

    if args.profile_moe > 0:  # the grouped expert GEMM alone, for a profiler
        profile_moe(args.profile_moe, device)
        if world > 1:
            dist.destroy_process_group()
        return 0

    wl = dg.WORKLOADS[args.workload]
    cluster = args.cluster or wl.cluster
    per_layer = wl.n_qkv * wl.K + wl.N2 * wl.K + 2 * wl.B * wl.Hkv * wl.Lcap * wl.d * 2
    R = args.replicas or max(2, math.ceil(3 * L2_BYTES / per_layer))
    layers, kvs, xs, seq_lens, sl = make_layers(wl, R, 1000 * (rank + 1), device, cluster)
    stream = torch.cuda.current_stream()
    h = stream.cuda_stream

    def step(i, flags=dl.DL_FLAG_PDL):
        # launch on torch's current stream: the eager stream, or the capturing one inside a graph capture
        r = i % R
        layers[r].step(xs[r][0], xs[r][1], kvs[r][0], kvs[r][1], seq_lens,
                       stream=torch.cuda.current_stream().cuda_stream, flags=flags)

    if args.profile_next > 0:  # a short, graph-free run of the rows beyond the headline chain
        profile_next_rows(wl, args.profile_next, seq_lens, device, cluster)
        if world > 1:
            dist.destroy_process_group()
        return 0
    if args.profile_steps > 0:  # a short, graph-free run of the chain for a profiler
        for i in range(args.profile_steps):
            step(i)
        for lay in layers:
            lay.read_status(h)
        if world > 1:
            dist.destroy_process_group()
        return 0

    for i in range(max(args.warmup, 3)):
        step(i)
    for lay in layers:
        lay.read_status(h)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize()

    # ---- CUDA graphs of the PDL-chained steps (the launch mode the pages pair with PDL) ----
    cap_stream = torch.cuda.Stream(device)

    def capture(fn, idxs):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            for i in idxs:
                fn(i)
        return g

    def timed_replay(rp, n):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        # The start event follows one untimed replay of the first graph: a graph
        # launched onto an idle stream starts ~30 us late (measured: 36.2 us
        # per layer_b1 step over one 20-step graph, 35.3 with this replay before
        # it, 35.0 over 2000 steps), while in a run of replays each graph is
        # launched as the previous one executes.  The timed region still holds
        # exactly the n steps, in stream order after the untimed replay.
        rp.warm(n)
        start.record()
        rp.run(n)
        end.record()
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    def per_call_us(fn, period, n):
        """Device time per call of exactly n calls fn(0..n-1), replayed from CUDA
        graphs of `period` chained calls (the same plan as the headline), or
        launched directly when capture fails.  Returns (us, mode, graph lengths)."""
        try:
            rp = GraphReplayer(fn, period, capture).prepare(n)
            rp.run(n)  # untimed: the same graphs once through
            us = timed_replay(rp, n) * 1e3 / n
            lengths = rp.lengths(n)
            rp.release()
            return us, "graph", lengths
        except Exception:
            return timed(fn, n, torch.cuda.current_stream()) * 1e3 / n, "direct", []

    G = R * max(1, 24 // R)
    main_rp, graph_error = None, None
    try:
        main_rp = GraphReplayer(step, G, capture).prepare(args.steps)
        for _ in range(2):
            main_rp.run(args.steps)  # untimed warm-up replays of the timed graphs
    except Exception as exc:  # capture refused: fall back to direct launches, and say so
        main_rp = None
        graph_error = repr(exc)[:200]
    torch.cuda.synchronize()

    # ---- timed region: exactly K whole-layer steps ----
    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    if main_rp is not None:
        ms = timed_replay(main_rp, args.steps)
        graph_lengths = main_rp.lengths(args.steps)
        launch_mode = (f"CUDA graphs of {' and '.join(map(str, graph_lengths))} PDL-chained layer steps, replayed "
                       f"({len(replay_plan(args.steps, G))} replays for {args.steps} steps)")
    else:
        ms = timed(step, args.steps, stream)
        graph_lengths = []
        launch_mode = "direct launches (graph capture failed: " + graph_error + ")"
    barrier()
    clk = clocks.stop()
    for lay in layers:
        lay.read_status(h)
    if main_rp is not None:
        main_rp.release()
    us_layer = max_over_ranks(ms * 1e3 / args.steps)
    layer_bytes = wl.n_qkv * wl.K + wl.N2 * wl.K + int(sum(2 * wl.Hkv * int(L) * wl.d * 2 for L in sl))
    if layer_bytes / (us_layer * 1e-6) / 1e9 > 1.2 * peak_hbm()[0]:
        raise SystemExit(f"timed region did not do the work: {us_layer:.3f} us per layer is faster than HBM allows")

    # ---- context: direct launches through the public API (PDL on / off), host time per step ----
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ms_direct = timed(step, args.steps, stream)
    host_us = (time.perf_counter() - t0) * 1e6 / args.steps
    us_layer_direct = ms_direct * 1e3 / args.steps
    us_layer_nopdl = timed(lambda i: step(i, 0), args.steps, stream) * 1e3 / args.steps

    # ---- per-call loops, for the roofline of each kernel family ----
    K = wl.K
    def call_qkv(i):
        r = i % R
        L_ = layers[r]
        dl.check(dl.dl_fc_qkv_scale(xs[r][0], wl.M, K, L_.wp_qkv, L_.s_qkv, wl.Hq, wl.Hkv, wl.d, L_.q_scale, L_.qkv,
                                    L_.ws_qkv, stream=torch.cuda.current_stream().cuda_stream))

    def call_attn(i):
        r = i % R
        L_ = layers[r]
        dl.check(dl.dl_decode_attn(L_.qkv, L_.N_qkv, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, kvs[r][0], kvs[r][1],
                                   wl.Lcap, seq_lens, 1.0, cluster, L_.attn_out, L_.ws_attn,
                                   stream=torch.cuda.current_stream().cuda_stream))

    def call_fc13(i):
        r = i % R
        L_ = layers[r]
        dl.check(dl.dl_fc13_swiglu(xs[r][1], wl.M, K, L_.wp_13, L_.s_13, wl.N2, L_.ffn_out, L_.ws_13,
                                   stream=torch.cuda.current_stream().cuda_stream))

    kv_bytes = int(sum(2 * wl.Hkv * int(L) * wl.d * 2 for L in sl))
    gl = gemm_launches(wl.M, K)
    fam = {
        "fc13_swiglu": (call_fc13, wl.N2 * wl.K, gl),
        "fc_qkv_scale": (call_qkv, wl.n_qkv * wl.K, gl),
        "decode_attn": (call_attn, kv_bytes, 1),
    }
    peak, peak_kind = peak_hbm()
    peak_bf16, peak_bf16_kind = peak_bf16_tflops()
    kernels = {}
    for name, (fn, nbytes, launches) in fam.items():
        for i in range(3):
            fn(i)
        us, mode, lengths = per_call_us(fn, G, args.steps)
        gbs = nbytes / (us * 1e-6) / 1e9
        kernels[name] = {"us_per_call": us, "alg_bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / peak,
                         "launches_per_call": launches, "mode": mode, "graph_steps": lengths}
    for lay in layers:
        lay.read_status(h)

    # ---- the whole pre-norm layer (adds O_proj, FC2 and both RMSNorm producers) ----
    full = None
    next_rows = None
    if not args.no_full_layer:
        fbytes = wl.n_qkv * K + wl.K * wl.k_o + wl.N2 * K + wl.K * wl.k_fc2
        RF = max(2, math.ceil(3 * L2_BYTES / (fbytes + 2 * wl.B * wl.Hkv * wl.Lcap * wl.d * 2)))
        fl = make_full_layers(wl, RF, 5000 * (rank + 1), device, cluster)

        def full_step(i):
            lay, kc, vc, x, hres = fl[i % RF]
            lay.step(x, hres, kc, vc, seq_lens, stream=torch.cuda.current_stream().cuda_stream)

        for i in range(3):
            full_step(i)
        us_full, fmode, flengths = per_call_us(full_step, RF * max(1, 24 // RF), args.steps)
        for entry in fl:
            entry[0].read_status(h)
        us_full = max_over_ranks(us_full)
        # norm1, QKV (x_q from the norm), attention, O_proj, norm2, FC13 (x_q from the norm), FC2
        f_launches = 1 + 1 + 1 + gemm_launches(wl.M, wl.k_o) + 1 + 1 + gemm_launches(wl.M, wl.k_fc2)
        full = {"us": us_full, "alg_bytes": fbytes + kv_bytes,
                "achieved_gbs": (fbytes + kv_bytes) / (us_full * 1e-6) / 1e9,
                "frac": (fbytes + kv_bytes) / (us_full * 1e-6) / 1e9 / peak,
                "launches_per_step": f_launches, "mode": fmode, "graph_steps": flengths, "replicas": RF,
                "steps": "add+RMSNorm+quant -> FC_QKV -> attention -> O_proj -> add+RMSNorm+quant -> FC13+SwiGLU "
                         "-> FC2"}
        next_rows = measure_next_rows(wl, fl, seq_lens, device, cluster, args.steps, per_call_us, peak)
        del fl
        torch.cuda.empty_cache()

    # ---- end to end through the public API with host buffers ----
    # The step's two activations travel in one pinned buffer and its two
    # results come back in one (DecodeLayer keeps them contiguous).
    hx = torch.stack([xs[0][0], xs[0][1]]).cpu().pin_memory()
    hout = torch.empty_like(layers[0].out_buf, device="cpu").pin_memory()
    dx = [torch.empty_like(hx, device=device) for _ in range(R)]

    def e2e_step(i):  # copy engine transfers, direct launches
        r = i % R
        dx[r].copy_(hx, non_blocking=True)
        layers[r].step(dx[r][0], dx[r][1], kvs[r][0], kvs[r][1], seq_lens, stream=h)
        hout.copy_(layers[r].out_buf, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    us_e2e_direct = max_over_ranks(timed(e2e_step, args.steps, stream) * 1e3 / args.steps)

    # The way the pages run decode steps: every step's transfers and kernels in
    # CUDA graphs, one PDL chain.  DecodeLayer.step_host moves the activations
    # in from pinned host memory and the results out with copy kernels, so the
    # chain is not broken by copy nodes.  Each step's upload runs beside the
    # previous step's download (the two touch disjoint buffers, and the download
    # has waited for its own step's kernels), one in each direction of the link.
    def e2e_graph_step(i):
        r = i % R
        layers[r].step_host(hx, hout, kvs[r][0], kvs[r][1], seq_lens,
                            stream=torch.cuda.current_stream().cuda_stream, overlap_upload=True)

    for i in range(3):
        e2e_graph_step(i)
    us_e2e, e2e_kind, e2e_lengths = per_call_us(e2e_graph_step, G, args.steps)
    us_e2e = max_over_ranks(us_e2e)

    # The same with every upload waiting for the previous step's download, as a
    # decode loop whose next input depends on the last result has to run
    def e2e_graph_step_seq(i):
        r = i % R
        layers[r].step_host(hx, hout, kvs[r][0], kvs[r][1], seq_lens,
                            stream=torch.cuda.current_stream().cuda_stream)

    for i in range(3):
        e2e_graph_step_seq(i)
    us_e2e_seq = max_over_ranks(per_call_us(e2e_graph_step_seq, G, args.steps)[0])
    if e2e_kind == "graph":
        e2e_mode = (f"CUDA graphs of {' and '.join(map(str, e2e_lengths))} steps, each: copy kernel host->device "
                    "(beside the previous step's download), the chain, copy kernel device->host")
    else:
        e2e_mode = "direct (graph capture failed)"
    h2d = hx.numel() * 2
    d2h = hout.numel() * 2
    for lay in layers:
        lay.read_status(h)
    del layers, kvs, xs, dx
    torch.cuda.empty_cache()

    # ---- the other workloads: per-config chain and kernel figures ----
    configs = {}
    names = [] if args.configs == "none" else [c for c in args.configs.split(",") if c and c != wl.name]
    for name in names:
        if name == "moe64":
            configs[name] = measure_moe_config(args.steps, device, per_call_us, peak, peak_bf16)
        else:
            configs[name] = measure_dense_config(name, args.steps, device, rank, per_call_us, peak, peak_bf16)

    cpu = cpu_all = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:  # the CPU baseline is an N = 1 figure
        inp = oracle_layer_inputs(wl)
        us_cpu, reps, secs = time_oracle(wl, inp, args.cpu_seconds, min_reps=1)
        cpu = {"value": us_cpu, "unit": "us", "cores": 1, "kind": "oracle",
               "sample": f"{reps} full {wl.name} layers ({secs:.1f} s) through the single-threaded FP64 C++ "
                         "oracle on the host"}
        cores = host_cores()
        if cores > 1:
            us_all, reps_all, secs_all = time_oracle_threads(wl, inp, args.cpu_seconds, cores)
            cpu_all = {"value": us_all, "unit": "us", "cores": cores, "kind": "oracle",
                       "sample": f"{reps_all} full {wl.name} layers ({secs_all:.1f} s), one at a time, each "
                                 f"layer's output columns and query heads spread over {cores} host threads "
                                 "(per-layer latency; the oracle's own functions on slices)"}

    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank != 0:
        return 0
    dom = kernels["fc13_swiglu"]
    line = {
        "metric": METRIC, "value": us_layer, "unit": "us", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us_layer / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8e4m3xfp8e4m3->f32 GEMM, bf16 attention (f32 softmax)",
        "data": "synthetic", "config": workload_config(wl, cluster),
        "roofline": {"bound": "hbm",
                     "kernel": "gemm_e4m3_kernel<1> (FC13 + SwiGLU, " +
                               ("fused e4m3 quantiser)" if gemm_launches(wl.M, wl.K) == 1 else
                                "x_q from the quantise kernel by tensor loads)"),
                     "achieved": dom["achieved_gbs"], "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": dom["achieved_gbs"] / peak,
                     "traffic": recorded_traffic("gemm_e4m3_kernel<1>", wl.name),
                     "alg_bytes_per_launch": wl.N2 * wl.K},
        "kernels": kernels,
        "graph_steps": graph_lengths,
        "layer_us_direct_launch": us_layer_direct,
        "layer_us_direct_no_pdl": us_layer_nopdl,
        "host_us_per_step_direct": host_us,
        "launch": launch_mode,
        "layer_alg_bytes": wl.n_qkv * wl.K + wl.N2 * wl.K + kv_bytes,
        "layer_achieved_gbs": (wl.n_qkv * wl.K + wl.N2 * wl.K + kv_bytes) / (us_layer * 1e-6) / 1e9,
        "e2e": {"value": us_e2e, "unit": "us", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": e2e_mode, "direct_launch_us": us_e2e_direct,
                "sequential_us": us_e2e_seq,
                "sequential_mode": "as value, but each upload waits for the previous step's download"},
        "cpu_baseline": cpu,
        "cpu_baseline_all_cores": cpu_all,
        "gpu_launches": (2 * gl + 1) * args.steps,
        "full_layer": full,
        "next_rows": next_rows,
        "configs": configs,
        "peak_bf16_tflops": {"value": peak_bf16, "kind": peak_bf16_kind},
        "clocks": clk,
        "replicas": R,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
