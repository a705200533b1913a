"""Pins for the oracle's lightning-indexer scores and exact top-K (CPU only)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a) -> np.ndarray:
    return oracle.bf16_bits(torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16))


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "indexer_hand.json")))
    qi = _bits(np.array(g["qi"])[None, None])            # [1, 1, Hi, di]
    wi = np.array(g["wi"], np.float32)[None, None]        # [1, 1, Hi]
    ki = _bits(np.array(g["ki"])[None])                   # [1, Nc, di]
    for case in g["cases"]:
        qpos = np.array([[case["t"]]], np.int32)
        sc, nv = oracle.index_scores(qi, wi, ki, g["m"], g["W"], q_pos=qpos)
        assert nv[0] == case["nvis"]
        assert np.array_equal(sc[0, :nv[0]], np.array(case["scores"]))
        assert np.all(np.isnan(sc[0, nv[0]:]))
        for k, want in case["topk"].items():
            assert oracle.topk(sc, nv, int(k))[0].tolist() == want


def test_visible_count_follows_the_block_rule():
    # entry j (raw positions j*m .. j*m+m-1) is visible to t iff its last
    # position precedes the window start t-W+1; enumerate j explicitly.
    for m, W, Nc in [(4, 128, 256), (128, 128, 64), (1, 0, 50), (4, 0, 40), (3, 5, 9)]:
        for t in range(0, Nc * m + W + 8):
            want = sum(1 for j in range(Nc) if j * m + (m - 1) <= t - W)
            assert oracle.visible_count(t, m, W, Nc) == want


def test_relu_and_linearity_invariants():
    rng = np.random.default_rng(5)
    B, L, Hi, di, Nc, m, W = 1, 40, 1, 16, 10, 4, 0
    qi = _bits(rng.standard_normal((B, L, Hi, di)))
    ki = _bits(rng.standard_normal((B, Nc, di)))
    wi = np.ones((B, L, Hi), np.float32)
    s_pos, nv = oracle.index_scores(qi, wi, ki, m, W)
    s_neg, _ = oracle.index_scores(qi ^ np.uint16(0x8000), wi, ki, m, W)
    # relu(x) - relu(-x) = x and relu(x) + relu(-x) = |x|
    dots = oracle.bf16_to_f64(qi)[0, :, 0] @ oracle.bf16_to_f64(ki)[0].T
    ok = ~np.isnan(s_pos)
    assert ok.sum() > 50
    np.testing.assert_allclose((s_pos - s_neg)[ok], dots[ok], rtol=1e-12, atol=1e-12)
    assert np.all(s_pos[ok] >= 0) and np.all(s_neg[ok] >= 0)
    assert np.all((s_pos[ok] == 0) | (s_neg[ok] == 0))
    # head weights enter linearly; a zero-weight head contributes nothing
    qi2 = _bits(rng.standard_normal((B, L, 3, di)))
    w3 = rng.random((B, L, 3)).astype(np.float32)
    s3, _ = oracle.index_scores(qi2, w3, ki, m, W)
    parts = []
    for h in range(3):
        wh = np.zeros_like(w3)
        wh[..., h] = w3[..., h]
        parts.append(oracle.index_scores(qi2, wh, ki, m, W)[0])
    np.testing.assert_allclose(s3[ok], sum(parts)[ok], rtol=1e-12)


def _lexsort_topk(scores, nv, K):
    out = np.full((len(nv), K), -1, np.int32)
    for r in range(len(nv)):
        n = nv[r]
        key = scores[r, :n].astype(np.float32)
        order = np.lexsort((np.arange(n), -key.astype(np.float64)))  # score desc, index asc
        sel = np.sort(order[:min(K, n)])
        out[r, :len(sel)] = sel
    return out


def test_topk_against_lexsort_with_ties():
    rng = np.random.default_rng(6)
    nrows, Nc = 50, 300
    sc = np.round(rng.random((nrows, Nc)) * 20) / 4  # many exact ties
    nv = rng.integers(0, Nc + 1, nrows).astype(np.int32)
    nv[:3] = [0, 1, Nc]
    for K in (1, 7, 64, 299, 300, 400):
        assert np.array_equal(oracle.topk(sc, nv, K), _lexsort_topk(sc, nv, K))


def test_topk_selects_all_visible_when_K_covers_them():
    sc = np.random.default_rng(7).random((4, 20))
    nv = np.array([0, 3, 19, 20], np.int32)
    got = oracle.topk(sc, nv, 25)
    for r in range(4):
        assert got[r, :nv[r]].tolist() == list(range(nv[r]))
        assert np.all(got[r, nv[r]:] == -1)


def test_selection_follows_a_permutation_of_the_entries():
    rng = np.random.default_rng(8)
    B, L, Hi, di, Nc, m, W = 1, 1, 4, 32, 64, 4, 8
    qi = _bits(rng.standard_normal((B, L, Hi, di)))
    wi = rng.random((B, L, Hi)).astype(np.float32)
    ki = _bits(rng.standard_normal((B, Nc, di)))
    qpos = np.array([[Nc * m + W]], np.int32)  # every entry visible
    sc, nv = oracle.index_scores(qi, wi, ki, m, W, q_pos=qpos)
    assert nv[0] == Nc
    perm = rng.permutation(Nc)
    sc_p, _ = oracle.index_scores(qi, wi, ki[:, perm], m, W, q_pos=qpos)
    K = 10
    a = set(oracle.topk(sc, nv, K)[0].tolist())
    b = set(perm[oracle.topk(sc_p, nv, K)[0]].tolist())
    assert a == b
