"""Pins for the oracle's block_merge and bf16 rounding (CPU only).

block_merge follows the CSDN DeepSeek-V4 CSA/HCA code page, section 1
(block_merge: per-channel softmax of the block weights over the m positions,
then a weighted sum of the m tokens) and section 2 (block_compress: all-ones
weights, i.e. the mean).  Each test below fixes a value that a plausible slip
(softmax over the wrong axis, a dropped token, a shifted block) would change.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits(torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16))


def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        # exact halfway cases between two bf16 neighbours (ties)
        (1.0 + (2 * rng.integers(0, 128, 2000) + 1) * 2.0 ** -8) * 2.0 ** rng.integers(-20, 20, 2000),
        [0.0, -0.0, 1.0, -1.0, 65504.0, 3.0e38, -3.0e38, 1e-39, 1e-42],
    ]).astype(np.float32)
    want = oracle.bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    got = oracle.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_round_bf16_hand_ties():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    got = oracle.round_bf16(np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -30]))
    assert list(got) == [0x3F80, 0x3F82, 0x3F81]


def test_zero_weights_give_the_block_mean():
    # block_compress with all-equal weights: the softmax over m is uniform, so each
    # compressed entry is the plain mean of its m tokens (numpy's mean is the check).
    rng = np.random.default_rng(1)
    B, L, H, d, m = 2, 37, 3, 8, 4
    x = _bits(rng.standard_normal((B, L, H, d)))
    out, _ = oracle.block_merge(x, np.zeros((m, d), np.float32), m)
    xf = oracle.bf16_to_f64(x)
    Nc = L // m
    want = xf[:, :Nc * m].reshape(B, Nc, m, H, d).mean(axis=2)
    np.testing.assert_allclose(out, want, rtol=1e-15, atol=1e-15)


def test_large_one_hot_weight_selects_one_token():
    rng = np.random.default_rng(2)
    B, L, H, d, m = 1, 64, 2, 16, 8
    x = _bits(rng.standard_normal((B, L, H, d)))
    for i_star in (0, 5, m - 1):
        w = np.zeros((m, d), np.float32)
        w[i_star] = 60.0
        _, ob = oracle.block_merge(x, w, m)
        assert np.array_equal(ob, x[:, i_star::m][:, : L // m])


def test_softmax_runs_over_positions_per_channel():
    # channel c puts all weight on position c % m; a softmax over channels (the
    # wrong axis) or a weight shared by all channels would not reproduce this.
    rng = np.random.default_rng(3)
    B, L, H, d, m = 1, 32, 1, 12, 4
    x = _bits(rng.standard_normal((B, L, H, d)))
    w = np.zeros((m, d), np.float32)
    for c in range(d):
        w[c % m, c] = 60.0
    _, ob = oracle.block_merge(x, w, m)
    for j in range(L // m):
        for c in range(d):
            assert ob[0, j, 0, c] == x[0, j * m + c % m, 0, c]


def test_known_weight_ratios():
    # weights log(a_i) give the convex combination sum a_i x_i / sum a_i
    m, d = 4, 2
    a = np.array([1.0, 2.0, 4.0, 1.0])
    w = np.tile(np.log(a).astype(np.float32)[:, None], (1, d))
    x = np.zeros((1, 4, 1, d), np.float32)
    x[0, :, 0, 0] = [8.0, 0.0, 0.0, 0.0]
    x[0, :, 0, 1] = [0.0, 0.0, 1.0, 0.0]
    out, _ = oracle.block_merge(_bits(x), w, m)
    pw = np.exp(w[:, 0].astype(np.float64))
    pw /= pw.sum()
    # 8 * 1/8 = 1 (up to the fp32 rounding of log(a)); 1 * 4/8 = 0.5
    np.testing.assert_allclose(out[0, 0, 0], [8 * pw[0], pw[2]], rtol=1e-15)
    np.testing.assert_allclose(out[0, 0, 0], [1.0, 0.5], rtol=1e-6)


def test_m1_is_identity_and_trailing_tokens_are_dropped():
    rng = np.random.default_rng(4)
    x = _bits(rng.standard_normal((2, 9, 2, 8)))
    _, ob = oracle.block_merge(x, rng.standard_normal((1, 8)).astype(np.float32), 1)
    assert np.array_equal(ob, x)
    w = rng.standard_normal((4, 8)).astype(np.float32)
    _, o1 = oracle.block_merge(x, w, 4)
    x2 = x.copy()
    x2[:, 8:] = 0  # the partial block (token 8) is never compressed
    _, o2 = oracle.block_merge(x2, w, 4)
    assert o1.shape == (2, 2, 2, 8) and np.array_equal(o1, o2)


def test_compressed_entry_counts_match_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "counts.json")))
    for item in g["compressed_entries"]:
        L, m = item["context"], item["m"]
        x = np.zeros((1, L, 1, 1), np.uint16)
        out, _ = oracle.block_merge(x, np.zeros((m, 1), np.float32), m)
        assert out.shape[1] == item["exact"]
        assert abs(out.shape[1] - item["page_figure"]) <= item["page_rel_tol"] * item["page_figure"]
