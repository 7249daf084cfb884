"""The whole pre-norm layer restated with oracle steps only, and the tolerance
a GPU run of that chain can be held to.

Every hand-over between steps is rounded to bf16 (the storage format between
kernels).  The chain re-quantises its data to e4m3 three more times after
attention (the O_proj input, the FC13 input after the second RMSNorm, the FC2
input), so an attention output that is correct within the attention tolerance
still moves codes across rounding midpoints downstream, and each such code
moves a later output by a whole e4m3 step.  The bound therefore comes from the
chain itself: chain_tolerance runs the oracle chain again with relative noise
on the attention output at the attention tolerance and takes the largest
deviation of the layer output, with a safety factor."""
from __future__ import annotations

import numpy as np

import helpers
import oracle


def oracle_full_layer(inp, wl, eps, att_noise: float = 0.0, rng=None):
    """(y, h2): the layer output (float64) and the updated residual stream (bf16
    bits).  att_noise > 0 multiplies the attention output by (1 + att_noise * z),
    z ~ N(0, 1) drawn from `rng`, before it is rounded and handed on."""
    rnd = lambda a: oracle.f64_to_bf16(a)
    h1, _, xq1, sx1 = oracle.add_rmsnorm_quant(inp["x"], inp["h"], inp["g1"], eps)
    qkv = rnd(oracle.fc_qkv_scale_q(xq1, sx1, inp["w_qkv"], inp["s_qkv"], wl.Hq, wl.Hkv, wl.d, inp["q_scale"]))
    att = oracle.decode_attn(qkv.ravel(), wl.n_qkv, wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, inp["k_cache"],
                             inp["v_cache"], inp["seq_lens"], 1.0)
    if att_noise > 0.0:
        att = att * (1.0 + att_noise * rng.standard_normal(att.shape))
    att = rnd(att).reshape(wl.M, wl.k_o)
    a = rnd(oracle.linear(att, inp["w_o"], inp["s_o"]))
    h2, _, xq2, sx2 = oracle.add_rmsnorm_quant(a, h1, inp["g2"], eps)
    f = rnd(oracle.fc13_swiglu_q(xq2, sx2, inp["w13"], inp["s13"]))
    return oracle.linear(f, inp["w2"], inp["s2"]), h2


def chain_tolerance(inp, wl, eps, y_ref, h_ref, trials: int = 6, seed: int = 0, floor: float = 1e-2):
    """Relative-L2 bounds (layer output, residual stream): 1.5 x the largest
    deviation of the oracle chain's own results over `trials` runs with
    relative noise of helpers.ATTN_REL_L2 on its attention output, and never
    below `floor` (the GEMM bound)."""
    rng = np.random.default_rng(seed)
    wy = wh = 0.0
    for _ in range(trials):
        y, h = oracle_full_layer(inp, wl, eps, helpers.ATTN_REL_L2, rng)
        wy = max(wy, helpers.rel_l2(y, y_ref))
        wh = max(wh, helpers.rel_l2(helpers.bf16_to_f64(h), helpers.bf16_to_f64(h_ref)))
    return max(floor, 1.5 * wy), max(floor, 1.5 * wh)
