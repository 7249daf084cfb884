"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
entry point include/dl.h declares, links none of the oracle, and rejects bad
arguments before launching anything.  Only argument combinations that fail
validation are passed, so no call here reaches the GPU; the fake device
addresses are never dereferenced."""
import os
import re
import subprocess

import numpy as np
import pytest

from latency_decode_b200 import build as dl_build
from latency_decode_b200 import dl
import helpers

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x7F0000000000  # 256-byte aligned, never dereferenced


@pytest.fixture(scope="module", autouse=True)
def built_lib():
    dl_build.build()
    return dl.lib()


def declared_entry_points():
    text = open(os.path.join(ROOT, "include", "dl.h")).read()
    return sorted(set(re.findall(r"^\s*(?:dl_status|size_t|const char\*)\s+(dl_\w+)\s*\(", text, re.M)))


def test_binding_constants_match_the_header():
    """Every DL_* integer macro of include/dl.h (flags, pack kinds, status codes)
    has the same value in the Python binding."""
    text = open(os.path.join(ROOT, "include", "dl.h")).read()
    macros = dict((name, int(val)) for name, val in re.findall(r"^#define\s+(DL_\w+)\s+(\d+)u?\b", text, re.M))
    macros.update((name, int(val)) for name, val in re.findall(r"^\s*(DL_(?:OK|ERR_\w+))\s*=\s*(\d+)", text, re.M))
    assert "DL_FLAG_PDL" in macros and "DL_FLAG_COPY_NO_WAIT" in macros and "DL_ERR_DEVICE_ARG" in macros
    for name, val in macros.items():
        assert getattr(dl, name) == val, name


def test_exports_every_declared_entry_point():
    names = declared_entry_points()
    assert len(names) >= 8
    out = subprocess.run(["nm", "-D", "--defined-only", dl.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, f"not exported: {missing}"
    for n in names:
        getattr(dl.lib(), n)


def test_library_has_no_oracle_code():
    out = subprocess.run(["nm", "-D", dl.LIB_PATH], capture_output=True, text=True, check=True).stdout
    assert "oracle" not in out


def test_only_sm100a_code():
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", dl.LIB_PATH], capture_output=True,
                         text=True).stdout
    arches = set(re.findall(r"sm_(\d+a?)", out))
    assert arches == {"100a"}, arches


def test_status_strings():
    for code, name in [(0, "DL_OK"), (1, "DL_ERR_INVALID_ARG"), (4, "DL_ERR_WORKSPACE"),
                       (6, "DL_ERR_TIMEOUT"), (7, "DL_ERR_DEVICE_ARG")]:
        assert dl.dl_status_string(code) == name
    assert dl.dl_status_string(99) == "DL_ERR_UNKNOWN"


def test_workspace_bytes():
    assert dl.dl_workspace_bytes(0, 0) == 256
    assert dl.dl_workspace_bytes(1, 5120) == 256 + 5120
    assert dl.dl_workspace_bytes(64, 5120) == 256 + 64 * 5120
    assert dl.dl_workspace_bytes(1, 100) == 512


def test_attention_workspace_bytes():
    assert dl.dl_decode_attn_workspace_bytes(1, 4, 40, 8, 128, 32768, 8) > 256  # long: splits over clusters
    assert dl.dl_decode_attn_workspace_bytes(1, 1, 40, 8, 128, 4096, 8) == 256  # batch-1 layer: one cluster
    assert dl.dl_decode_attn_workspace_bytes(16, 4, 40, 8, 128, 16384, 8) == 256  # enough CTAs already
    assert dl.dl_decode_attn_workspace_bytes(1, 1, 8, 2, 64, 256, 8) == 256  # too short to split
    assert dl.dl_decode_attn_workspace_bytes(1, 1, 6, 4, 64, 256, 8) == 0  # Hq % Hkv != 0


def _fc13(**kw):
    a = dict(x=FAKE, M=1, K=512, w_packed=FAKE, w_scale=FAKE, N2=2048, out=FAKE, ws=FAKE,
             ws_bytes=1 << 20, stream=0, flags=0)
    a.update(kw)
    return dl.dl_fc13_swiglu(**a)


def test_fc13_argument_errors():
    assert _fc13(x=None) == dl.DL_ERR_INVALID_ARG
    assert _fc13(w_scale=None) == dl.DL_ERR_INVALID_ARG
    assert _fc13(M=0) == dl.DL_ERR_INVALID_ARG
    assert _fc13(M=65) == dl.DL_ERR_UNSUPPORTED
    assert _fc13(K=520) == dl.DL_ERR_UNSUPPORTED
    assert _fc13(N2=2048 + 128) == dl.DL_ERR_UNSUPPORTED
    assert _fc13(N2=128) == dl.DL_ERR_INVALID_ARG
    assert _fc13(x=FAKE + 8) == dl.DL_ERR_ALIGNMENT
    assert _fc13(out=FAKE + 2) == dl.DL_ERR_ALIGNMENT
    assert _fc13(w_packed=FAKE + 4) == dl.DL_ERR_ALIGNMENT
    assert _fc13(ws=None) == dl.DL_ERR_WORKSPACE
    assert _fc13(ws=FAKE + 16) == dl.DL_ERR_WORKSPACE
    assert _fc13(ws_bytes=256 + 511) == dl.DL_ERR_WORKSPACE
    assert _fc13(flags=dl.DL_FLAG_PDL | (9 << dl.DL_FLAG_SPLIT_SHIFT)) == dl.DL_ERR_INVALID_ARG


def test_qkv_argument_errors():
    base = dict(x=FAKE, M=1, K=512, w_packed=FAKE, w_scale=FAKE, Hq=8, Hkv=2, d=64, q_scale=0.125, qkv=FAKE,
                ws=FAKE, ws_bytes=1 << 20, stream=0, flags=0)
    assert dl.dl_fc_qkv_scale(**{**base, "Hq": 0}) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_fc_qkv_scale(**{**base, "d": 40}) == dl.DL_ERR_UNSUPPORTED  # (8+4)*40 % 128 != 0
    assert dl.dl_fc_qkv_scale(**{**base, "qkv": None}) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_fc_qkv_scale(**{**base, "ws_bytes": 100}) == dl.DL_ERR_WORKSPACE


def test_moe_argument_errors():
    base = dict(x=FAKE, T=4, K=512, expert_ids=FAKE, E=8, w_packed=FAKE, w_scales=FAKE, N2=512, out=FAKE,
                ws=FAKE, ws_bytes=1 << 20, stream=0, flags=0)
    assert dl.dl_moe_fc13_swiglu_grouped(**{**base, "expert_ids": None}) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_moe_fc13_swiglu_grouped(**{**base, "E": 0}) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_moe_fc13_swiglu_grouped(**{**base, "E": 2000}) == dl.DL_ERR_UNSUPPORTED
    assert dl.dl_moe_fc13_swiglu_grouped(**{**base, "T": 65}) == dl.DL_ERR_UNSUPPORTED
    assert dl.dl_moe_fc13_swiglu_grouped(**{**base, "expert_ids": FAKE + 2}) == dl.DL_ERR_ALIGNMENT


def _attn(**kw):
    a = dict(q=FAKE, q_token_stride=1024, B=1, T=1, Hq=8, Hkv=2, d=64, k_cache=FAKE, v_cache=FAKE, Lcap=256,
             seq_lens=FAKE, softmax_scale=0.125, cluster_size=8, out=FAKE, ws=FAKE, ws_bytes=256, stream=0,
             flags=0)
    a.update(kw)
    return dl.dl_decode_attn(**a)


def test_attn_argument_errors():
    assert _attn(q=None) == dl.DL_ERR_INVALID_ARG
    assert _attn(seq_lens=None) == dl.DL_ERR_INVALID_ARG
    assert _attn(Hq=6, Hkv=4) == dl.DL_ERR_INVALID_ARG
    assert _attn(d=96) == dl.DL_ERR_UNSUPPORTED
    assert _attn(Hq=40, Hkv=1, T=1) == dl.DL_ERR_UNSUPPORTED  # 40 query rows per kv head > 32
    assert _attn(T=0) == dl.DL_ERR_INVALID_ARG
    assert _attn(cluster_size=3) == dl.DL_ERR_INVALID_ARG
    assert _attn(cluster_size=32) == dl.DL_ERR_INVALID_ARG
    assert _attn(q_token_stride=500) == dl.DL_ERR_ALIGNMENT  # < Hq*d
    assert _attn(q_token_stride=516) == dl.DL_ERR_ALIGNMENT  # not a multiple of 8
    assert _attn(k_cache=FAKE + 8) == dl.DL_ERR_ALIGNMENT
    assert _attn(ws_bytes=255) == dl.DL_ERR_WORKSPACE


def test_pack_argument_errors():
    assert dl.dl_pack_fp8_weight(None, FAKE, 128, 128, 0, 0) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_pack_fp8_weight(FAKE, FAKE + 4096, 128, 128, 0, 0) == dl.DL_ERR_INVALID_ARG  # overlap
    assert dl.dl_pack_fp8_weight(FAKE, FAKE + (1 << 20), 128, 100, 0, 0) == dl.DL_ERR_UNSUPPORTED
    assert dl.dl_pack_fp8_weight(FAKE, FAKE + (1 << 20), 128, 128, 1, 0) == dl.DL_ERR_UNSUPPORTED  # SwiGLU N%256
    assert dl.dl_pack_fp8_weight(FAKE, FAKE + (1 << 20), 128, 128, 7, 0) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_read_status(None, 0) == dl.DL_ERR_WORKSPACE


def test_pack_reference_is_a_permutation_with_the_stated_layout():
    g = np.random.default_rng(0)
    N, K = 512, 384
    w = g.integers(0, 256, size=(N, K)).astype(np.uint8)
    for kind in (0, 1):
        p = helpers.pack_reference(w, kind)
        assert p.size == w.size
        assert np.array_equal(np.sort(p), np.sort(w.ravel()))
    # spot-check the stated formula on a few bytes (PLAIN)
    p = helpers.pack_reference(w, 0)
    KB = K // 128
    for (n, k) in [(0, 0), (5, 17), (130, 300), (511, 383)]:
        t, r, kb, c = n // 128, n % 128, k // 128, k % 128
        off = (t * KB + kb) * 16384 + (r // 8) * 1024 + (r % 8) * 128 + ((c // 16) ^ (r % 8)) * 16 + c % 16
        assert p[off] == w[n, k]
    # SWIGLU: gate row j and up row F+j of the same K bytes sit in neighbouring blocks
    p = helpers.pack_reference(w, 1)
    F = N // 2
    for (j, k) in [(0, 0), (3, 129), (255, 383)]:
        t, r, kb, c = j // 128, j % 128, k // 128, k % 128
        intra = (r // 8) * 1024 + (r % 8) * 128 + ((c // 16) ^ (r % 8)) * 16 + c % 16
        blk = 2 * (t * KB + kb)
        assert p[blk * 16384 + intra] == w[j, k]
        assert p[(blk + 1) * 16384 + intra] == w[F + j, k]


def test_plain_and_grouped_projection_argument_errors():
    base = dict(x=FAKE, M=1, K=512, w_packed=FAKE, w_scale=FAKE, N=256, out=FAKE, ws=FAKE, ws_bytes=1 << 20,
                stream=0, flags=0)
    assert dl.dl_gemm_e4m3(**{**base, "x": None}) == dl.DL_ERR_INVALID_ARG  # x needed without XQ_READY
    assert dl.dl_gemm_e4m3(**{**base, "N": 64}) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_gemm_e4m3(**{**base, "N": 320}) == dl.DL_ERR_UNSUPPORTED
    assert dl.dl_gemm_e4m3(**{**base, "M": 64, "K": 8320}) == dl.DL_ERR_UNSUPPORTED  # M*K > 64*8192
    assert dl.dl_gemm_e4m3(**{**base, "out": FAKE + 2}) == dl.DL_ERR_ALIGNMENT
    assert dl.dl_gemm_e4m3(**{**base, "ws_bytes": 256 + 511}) == dl.DL_ERR_WORKSPACE
    assert dl.dl_gemm_e4m3(**{**base, "flags": 9 << dl.DL_FLAG_SPLIT_SHIFT}) == dl.DL_ERR_INVALID_ARG
    m = dict(x=FAKE, T=4, K=512, expert_ids=FAKE, E=8, w_packed=FAKE, w_scales=FAKE, N=128, out=FAKE, ws=FAKE,
             ws_bytes=1 << 20, stream=0, flags=0)
    assert dl.dl_moe_gemm_grouped(**{**m, "N": 192}) == dl.DL_ERR_UNSUPPORTED
    assert dl.dl_moe_gemm_grouped(**{**m, "expert_ids": None}) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_moe_gemm_grouped(**{**m, "E": 1025}) == dl.DL_ERR_UNSUPPORTED
    assert dl.dl_moe_gemm_grouped(**{**m, "T": 0}) == dl.DL_ERR_INVALID_ARG
    # the plain grouped entry accepts N % 128 where the SwiGLU one needs N % 256
    assert dl.dl_moe_fc13_swiglu_grouped(**{**{k: v for k, v in m.items() if k != "N"}, "N2": 128}) \
        == dl.DL_ERR_INVALID_ARG


def _norm(**kw):
    a = dict(x=FAKE, residual=FAKE + (1 << 24), h_out=FAKE + (2 << 24), gamma=FAKE + (3 << 24), M=4, K=5120,
             eps=1e-5, ws=FAKE + (4 << 24), ws_bytes=1 << 20, stream=0, flags=0)
    a.update(kw)
    return dl.dl_add_rmsnorm_quant(**a)


def test_rmsnorm_quant_argument_errors():
    assert _norm(x=None) == dl.DL_ERR_INVALID_ARG
    assert _norm(gamma=None) == dl.DL_ERR_INVALID_ARG
    assert _norm(eps=0.0) == dl.DL_ERR_INVALID_ARG
    assert _norm(eps=-1.0) == dl.DL_ERR_INVALID_ARG
    assert _norm(eps=float("nan")) == dl.DL_ERR_INVALID_ARG
    assert _norm(eps=float("inf")) == dl.DL_ERR_INVALID_ARG
    assert _norm(M=0) == dl.DL_ERR_INVALID_ARG
    assert _norm(K=5000) == dl.DL_ERR_UNSUPPORTED
    assert _norm(M=65) == dl.DL_ERR_UNSUPPORTED
    assert _norm(M=64, K=8320) == dl.DL_ERR_UNSUPPORTED
    assert _norm(gamma=FAKE + (3 << 24) + 2) == dl.DL_ERR_ALIGNMENT
    assert _norm(residual=FAKE + (1 << 24) + 8) == dl.DL_ERR_ALIGNMENT
    assert _norm(h_out=FAKE + 4096) == dl.DL_ERR_INVALID_ARG  # partial overlap with x
    assert _norm(h_out=FAKE + (1 << 24) - 4096) == dl.DL_ERR_INVALID_ARG  # partial overlap with residual
    assert _norm(ws_bytes=256 + 4 * 5120 - 1) == dl.DL_ERR_WORKSPACE
    assert _norm(ws=None) == dl.DL_ERR_WORKSPACE


def test_spec_verify_argument_errors():
    base = dict(logits=FAKE, B=2, T=4, V=1024, draft_ids=FAKE, target_ids=FAKE, n_accepted=FAKE, emitted=FAKE,
                seq_lens=None, stream=0, flags=0)
    f = dl.dl_spec_verify_greedy
    assert f(**{**base, "logits": None}) == dl.DL_ERR_INVALID_ARG
    assert f(**{**base, "draft_ids": None}) == dl.DL_ERR_INVALID_ARG  # T > 1 needs drafts
    assert f(**{**base, "T": 0}) == dl.DL_ERR_INVALID_ARG
    assert f(**{**base, "V": 4}) == dl.DL_ERR_INVALID_ARG
    assert f(**{**base, "T": 33}) == dl.DL_ERR_UNSUPPORTED
    assert f(**{**base, "V": 1001}) == dl.DL_ERR_UNSUPPORTED
    assert f(**{**base, "B": 70000}) == dl.DL_ERR_UNSUPPORTED
    assert f(**{**base, "logits": FAKE + 8}) == dl.DL_ERR_ALIGNMENT
    assert f(**{**base, "seq_lens": FAKE + 2}) == dl.DL_ERR_ALIGNMENT
    assert f(**{**base, "emitted": None}) == dl.DL_ERR_INVALID_ARG


def test_fp8kv_attention_argument_errors():
    a = dict(q=FAKE, q_token_stride=1024, B=1, T=1, Hq=8, Hkv=2, d=128, k_cache=FAKE, vt_cache=FAKE, kv_scale=FAKE,
             Lcap=256, seq_lens=FAKE, softmax_scale=0.125, cluster_size=8, out=FAKE, ws=FAKE, ws_bytes=256,
             stream=0, flags=0)
    f = dl.dl_decode_attn_fp8kv
    assert f(**{**a, "kv_scale": None}) == dl.DL_ERR_INVALID_ARG
    assert f(**{**a, "d": 64, "q_token_stride": 512}) == dl.DL_ERR_UNSUPPORTED  # the e4m3 path is d = 128 only
    assert f(**{**a, "k_cache": FAKE + 8}) == dl.DL_ERR_ALIGNMENT
    assert f(**{**a, "kv_scale": FAKE + 2}) == dl.DL_ERR_ALIGNMENT
    assert f(**{**a, "cluster_size": 3}) == dl.DL_ERR_INVALID_ARG
    assert f(**{**a, "ws_bytes": 255}) == dl.DL_ERR_WORKSPACE
    assert dl.dl_decode_attn_fp8kv_workspace_bytes(1, 1, 8, 2, 64, 256, 8) == 0


def test_copy_argument_errors():
    assert dl.dl_copy(None, FAKE, 16, 0, 0) == dl.DL_ERR_INVALID_ARG
    assert dl.dl_copy(FAKE, FAKE + 4096, 17, 0, 0) == dl.DL_ERR_ALIGNMENT
    assert dl.dl_copy(FAKE + 8, FAKE + 4096, 16, 0, 0) == dl.DL_ERR_ALIGNMENT
    assert dl.dl_copy(FAKE, FAKE + 16, 64, 0, 0) == dl.DL_ERR_INVALID_ARG  # overlap


def test_fp8kv_cache_capacity_must_be_a_multiple_of_16():
    a = dict(q=FAKE, q_token_stride=1024, B=1, T=1, Hq=8, Hkv=2, d=128, k_cache=FAKE, vt_cache=FAKE, kv_scale=FAKE,
             Lcap=200 + 4, seq_lens=FAKE, softmax_scale=0.125, cluster_size=8, out=FAKE, ws=FAKE, ws_bytes=256,
             stream=0, flags=0)
    assert dl.dl_decode_attn_fp8kv(**a) == dl.DL_ERR_ALIGNMENT


def test_fused_rmsnorm_gemm_argument_errors():
    base = dict(x=FAKE, residual=FAKE + (1 << 24), h_out=FAKE + (2 << 24), gamma=FAKE + (3 << 24), eps=1e-5, M=1,
                K=512, w_packed=FAKE + (4 << 24), w_scale=FAKE + (5 << 24), N2=512, out=FAKE + (6 << 24),
                ws=FAKE + (7 << 24), ws_bytes=1 << 20, stream=0, flags=0)
    f = dl.dl_rmsnorm_fc13_swiglu
    assert f(**{**base, "h_out": FAKE + (1 << 24) + 512}) == dl.DL_ERR_INVALID_ARG  # partial overlap with residual
    assert f(**{**base, "h_out": FAKE + 512}) == dl.DL_ERR_INVALID_ARG  # partial overlap with x
    assert f(**{**base, "gamma": None}) == dl.DL_ERR_INVALID_ARG
    assert f(**{**base, "eps": 0.0}) == dl.DL_ERR_INVALID_ARG
    assert f(**{**base, "gamma": FAKE + (3 << 24) + 2}) == dl.DL_ERR_ALIGNMENT
    assert f(**{**base, "N2": 384}) == dl.DL_ERR_UNSUPPORTED
    q = dict(x=FAKE, residual=None, h_out=None, gamma=FAKE + (3 << 24), eps=1e-5, M=1, K=512, w_packed=FAKE,
             w_scale=FAKE, Hq=8, Hkv=2, d=64, q_scale=0.125, qkv=FAKE + (6 << 24), ws=FAKE + (7 << 24),
             ws_bytes=100, stream=0, flags=0)
    assert dl.dl_rmsnorm_fc_qkv_scale(**q) == dl.DL_ERR_WORKSPACE
