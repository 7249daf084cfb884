"""GPU parity of the on-device greedy speculative verification through the C
ABI against the CPU oracle.  Integer work: target ids, accepted counts, emitted
tokens and the updated sequence lengths must match exactly.  Cases: the pages'
d2-d4 example, every accept length, ties inside one vector, across CTA slices
and across the whole row, all-negative and infinite logits, T = 1 and T = 32,
one to sixty-four sequences, and the full vocabulary (202,048) at the verify
and batch shapes."""
import json
import os

import numpy as np
import pytest
import torch

import helpers
import oracle
from helpers import dev_i32, dev_u16
from latency_decode_b200 import build as dl_build
from latency_decode_b200 import datagen as dg
from latency_decode_b200 import dl

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not helpers.gpu_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def lib():
    dl_build.build()
    return dl.lib()


def run_verify(lg, draft, seq_lens=None):
    B, T, V = lg.shape
    tid = torch.full((B, T), -7, dtype=torch.int32, device="cuda")
    nacc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    em = torch.full((B, T), -7, dtype=torch.int32, device="cuda")
    sl = dev_i32(seq_lens) if seq_lens is not None else None
    dr = dev_i32(draft.reshape(B, T - 1)) if T > 1 else None
    dl.check(dl.dl_spec_verify_greedy(dev_u16(lg), B, T, V, dr, tid, nacc, em, sl))
    torch.cuda.synchronize()
    return (tid.cpu().numpy(), nacc.cpu().numpy(), em.cpu().numpy(),
            sl.cpu().numpy() if sl is not None else None)


def check(lg, draft, seq_lens=None, what=""):
    B, T, V = lg.shape
    got = run_verify(lg, draft, seq_lens)
    tid, nacc, em = oracle.spec_verify_greedy(lg, draft.reshape(B, T - 1))
    assert np.array_equal(got[0], tid), f"{what}: target ids"
    assert np.array_equal(got[1], nacc), f"{what}: accepted"
    assert np.array_equal(got[2], em), f"{what}: emitted"
    if seq_lens is not None:
        assert np.array_equal(got[3], np.asarray(seq_lens) - (T - 1 - nacc)), f"{what}: seq_lens"
    return nacc


def planted(g, B, T, V, runs, std=1.0):
    lg = dg.bf16_normal(g, (B, T, V), std=std)
    ref = oracle.spec_verify_greedy(lg, np.zeros((B, T - 1), np.int32))[0]
    draft = g.integers(0, V, size=(B, T - 1)).astype(np.int32)
    for b in range(B):
        n = runs[b % len(runs)]
        draft[b, :n] = ref[b, :n]
        if n < T - 1 and draft[b, n] == ref[b, n]:
            draft[b, n] = (ref[b, n] + 1) % V
    return lg, draft


def test_pages_worked_example(golden_dir):
    gold = json.load(open(os.path.join(golden_dir, "spec_verify_hand.json")))
    T, V = len(gold["hot"]), gold["V"]
    lg = np.zeros((1, T, V), dtype=np.float32)
    for t, v in enumerate(gold["hot"]):
        lg[0, t, v] = 1.0
    tid, nacc, em, sl = run_verify(dg.bf16_bits(lg), np.array([gold["draft"]], np.int32), [1000])
    assert tid[0].tolist() == gold["target_ids"] and int(nacc[0]) == gold["n_accepted"]
    assert em[0].tolist() == gold["emitted"] and int(sl[0]) == 1000 - 1


def test_signed_zero_tie_lowest_index_wins(golden_dir):
    """The largest logit is 0, present as -0 before +0 (and +0 before -0): the
    lower index wins, as in the oracle; also with the zeros in different CTA
    slices of the full vocabulary."""
    gold = json.load(open(os.path.join(golden_dir, "spec_verify_signed_zero.json")))
    T, V = len(gold["target_ids"]), gold["V"]
    lg = np.full((1, T, V), dg.bf16_bits(np.float32([-1.0]))[0], dtype=np.uint16)
    for t, v in gold["neg_zero"]:
        lg[0, t, v] = 0x8000
    for t, v in gold["pos_zero"]:
        lg[0, t, v] = 0x0000
    tid, nacc, em, _ = run_verify(lg, np.array([gold["draft"]], np.int32))
    assert tid[0].tolist() == gold["target_ids"] and int(nacc[0]) == gold["n_accepted"]
    assert em[0].tolist() == gold["emitted"]
    big = np.full((2, 3, dg.VOCAB), dg.bf16_bits(np.float32([-2.0]))[0], dtype=np.uint16)
    big[0, 0, 7], big[0, 0, 150001] = 0x8000, 0x0000        # -0 first, far apart
    big[0, 1, 100], big[0, 1, 190000] = 0x0000, 0x8000      # +0 first
    big[0, 2, 24], big[0, 2, 25] = 0x8000, 0x0000           # inside one 16-byte vector
    big[1, :, 202047] = 0x0000
    big[1, :, 202046] = 0x8000
    check(big, np.array([[7, 100], [202046, 5]], np.int32), None, "signed zeros")


@pytest.mark.parametrize("B,T,V", [(1, 4, 1000), (3, 4, 4096), (16, 4, 32000), (64, 2, 2048), (5, 8, 800),
                                   (2, 32, 128), (1, 1, 64), (3, 3, 5000), (2, 5, 70000), (1, 17, 3000)])
def test_every_accept_length(B, T, V):
    g = np.random.default_rng(B * 100 + T * 7 + V)
    lg, draft = planted(g, B, T, V, list(range(T)))
    nacc = check(lg, draft, g.integers(T, 5000, size=B).astype(np.int32), f"B={B} T={T} V={V}")
    assert set(nacc.tolist()) == set(range(min(T, B)))


def test_ties_lowest_index_wins_across_cta_slices():
    g = np.random.default_rng(7)
    B, T, V = 2, 4, 202048
    lg = dg.bf16_normal(g, (B, T, V))
    big = dg.bf16_bits(np.float32([100.0]))[0]
    lg[0, 0, [5, 150000]] = big            # far apart: different CTAs of the cluster
    lg[0, 1, [202047, 101024]] = big       # the higher index comes first in the list; the lower one wins
    lg[0, 2, [16, 17]] = big               # inside one 16-byte vector
    lg[1, :, :] = dg.bf16_bits(np.float32([-3.0]))[0]  # a whole row of equal, negative logits -> index 0
    lg[1, 3, 99] = dg.bf16_bits(np.float32([np.inf]))[0]
    draft = np.array([[5, 101024, 9], [0, 0, 0]], dtype=np.int32)
    nacc = check(lg, draft, None, "ties")
    assert nacc.tolist() == [2, 3]


@pytest.mark.parametrize("T", [1, 4])
def test_ties_between_threads_and_warps_of_one_row_slice(T):
    # equal maxima in vectors that different threads and different warps of
    # one CTA's row group scan (8 logits per vector; the group has 512 / T
    # threads), and equal maxima at +0 / -0: the lowest index wins in each row
    g = np.random.default_rng(11 + T)
    B, V = 1, 202048
    lg = dg.bf16_normal(g, (B, T, V))
    big = dg.bf16_bits(np.float32([50.0]))[0]
    expect = []
    for t in range(T):
        idx = [8 * (7 + 40 * t) + 3, 8 * (1 + 40 * t) + 6, 8 * (300 + 40 * t) + 1]  # vectors 1, 7, 300 (+40 t)
        lg[0, t, idx] = big
        expect.append(min(idx))
    draft = np.array([expect[:T - 1]], dtype=np.int32)
    nacc = check(lg, draft, None, f"ties across threads T={T}")
    assert nacc.tolist() == [T - 1]


@pytest.mark.parametrize("name", ["verify4", "batch16x4"])
def test_full_vocabulary_at_the_verify_shapes(name):
    """The workload's sequences and T, vocabulary 202,048, logits N(0, 2) with
    every accept length planted."""
    wl = dg.WORKLOADS[name]
    g = dg.rng(800 + wl.seed)
    lg, draft = planted(g, wl.B, wl.T, dg.VOCAB, list(range(wl.T)), std=2.0)
    check(lg, draft, dg.seq_lens_for(wl, g), name)


def test_repeat_calls_are_deterministic():
    g = np.random.default_rng(9)
    lg, draft = planted(g, 4, 4, 50000, [0, 1, 2, 3])
    a = run_verify(lg, draft)
    b = run_verify(lg, draft)
    for x, y in zip(a[:3], b[:3]):
        assert np.array_equal(x, y)
