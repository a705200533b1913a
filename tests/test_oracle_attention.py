"""Pins for the oracle's hybrid attention (CPU only).

The attention is one softmax over the union of compressed keys (selected by
top-K for CSA, all visible ones for HCA) and the raw keys of a W-token window
("deepseek-v4" blog, section 1, SWA).  The oracle is checked against
  - an independent brute-force statement with an explicit mask (oracle/brute.py),
  - torch's scaled_dot_product_attention for m=1, W=0 (plain causal attention),
  - a hand-worked two-key case (one softmax across both parts),
  - label counting with q = 0 (uniform weights reveal the key sets),
  - the window-size entry count printed on the zwxr.cn post (section 4.2),
  - CSA with K >= n_vis equalling HCA dense, and softmax rows summing to 1,
  - the decode form (query position + raw ring buffer) equalling prefill.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a) -> np.ndarray:
    return oracle.bf16_bits(torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16))


def _f(bits):
    return oracle.bf16_to_f64(bits)


def _rand_case(rng, B, L, Hq, Hkv, d, m):
    q = _bits(rng.standard_normal((B, L, Hq, d)))
    k = _bits(rng.standard_normal((B, L, Hkv, d)))
    v = _bits(rng.standard_normal((B, L, Hkv, d)))
    Nc = L // m
    kc = _bits(rng.standard_normal((B, Nc, Hkv, d)))
    vc = _bits(rng.standard_normal((B, Nc, Hkv, d)))
    return q, k, v, kc, vc


def _random_idx(rng, L, Nc, m, W, K):
    idx = np.full((1, L, K), -1, np.int32)
    for t in range(L):
        nv = oracle.visible_count(t, m, W, Nc)
        if nv:
            sel = np.sort(rng.choice(nv, size=min(K, nv), replace=False))
            idx[0, t, :len(sel)] = sel
    return idx


@pytest.mark.parametrize("L,Hq,Hkv,d,m,W,K", [
    (96, 4, 1, 8, 4, 16, 5),
    (130, 4, 2, 16, 4, 8, 0),
    (200, 2, 2, 8, 8, 24, 0),
    (77, 6, 3, 8, 3, 10, 4),
])
def test_matches_brute_force_masked_attention(L, Hq, Hkv, d, m, W, K):
    rng = np.random.default_rng(L + 10 * K)
    q, k, v, kc, vc = _rand_case(rng, 1, L, Hq, Hkv, d, m)
    Nc = L // m
    idx = _random_idx(rng, L, Nc, m, W, K) if K else None
    res = oracle.hybrid_attention(q, kc, vc, idx, k, v, m, W, debug_maxkeys=Nc + W)
    o_b, lse_b, P_b = brute.attention(_f(q)[0], _f(kc)[0], _f(vc)[0], _f(k)[0], _f(v)[0], m, W,
                                      idx=None if idx is None else idx[0])
    np.testing.assert_allclose(res["o"], o_b, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse_b, rtol=1e-12)
    # the per-key weights agree too, mapped through the key labels
    for t in range(0, L, 7):
        keys = res["keys"][t]
        n = res["n_comp"][t] + res["n_win"][t]
        cols = [int(kk) if kk >= 0 else Nc + (-int(kk) - 1) for kk in keys[:n]]
        for h in range(Hq):
            np.testing.assert_allclose(res["p"][t, h, :n], P_b[h, t, cols], rtol=1e-10, atol=1e-14)
            assert abs(P_b[h, t].sum() - (1.0 if n else 0.0)) < 1e-12


def test_m1_without_window_is_causal_attention_sdpa():
    rng = np.random.default_rng(11)
    L, Hq, Hkv, d = 64, 4, 2, 16
    q = _bits(rng.standard_normal((1, L, Hq, d)))
    k = _bits(rng.standard_normal((1, L, Hkv, d)))
    v = _bits(rng.standard_normal((1, L, Hkv, d)))
    # m = 1: block_merge is the identity, every earlier-or-equal token is a visible entry
    _, kc = oracle.block_merge(k, np.zeros((1, d), np.float32), 1)
    _, vc = oracle.block_merge(v, np.zeros((1, d), np.float32), 1)
    res = oracle.hybrid_attention(q, kc, vc, None, k, v, m=1, W=0)
    qt = torch.from_numpy(_f(q)[0]).transpose(0, 1)
    kt = torch.from_numpy(_f(k)[0]).transpose(0, 1)
    vt = torch.from_numpy(_f(v)[0]).transpose(0, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                           enable_gqa=True)
    np.testing.assert_allclose(res["o"], ref.transpose(0, 1).numpy(), rtol=1e-10, atol=1e-12)


def test_two_key_hand_case_uses_one_softmax():
    # m=1, W=1, L=2: query 1 sees compressed entry 0 (= token 0) and raw token 1.
    # logits 0 and 1 (scale 1) -> weights 1/(1+e), e/(1+e).  Separate softmaxes per
    # part (then any gate) could not produce this split.
    q = np.zeros((1, 2, 1, 2)); q[0, 1, 0] = [1, 0]
    k = np.zeros((1, 2, 1, 2)); k[0, 1, 0] = [1, 0]
    v = np.zeros((1, 2, 1, 2)); v[0, 0, 0] = [1, 0]; v[0, 1, 0] = [0, 1]
    kb, vb = _bits(k), _bits(v)
    res = oracle.hybrid_attention(_bits(q), kb, vb, None, kb, vb, m=1, W=1, scale=1.0, rows=[1])
    e = math.e
    np.testing.assert_allclose(res["o"][0, 0], [1 / (1 + e), e / (1 + e)], rtol=1e-15)
    assert abs(res["lse"][0, 0] - math.log(1 + e)) < 1e-15
    assert res["n_comp"][0] == 1 and res["n_win"][0] == 1


def test_uniform_weights_count_the_key_sets():
    # q = 0 makes every key weigh the same, so o is the mean of the values.  Raw
    # values carry (1, position), compressed values (1000, entry index): the output
    # then tells how many keys of each kind were used and which.
    L, m, W, d, Nc = 256, 4, 32, 4, 64
    q = np.zeros((1, L, 1, d))
    v = np.zeros((1, L, 1, d)); v[0, :, 0, 0] = 1.0; v[0, :, 0, 1] = np.arange(L)
    vc = np.zeros((1, Nc, 1, d)); vc[0, :, 0, 2] = 1.0; vc[0, :, 0, 3] = np.arange(Nc)
    zb = _bits(np.zeros((1, L, 1, d)))
    res = oracle.hybrid_attention(_bits(q), _bits(np.zeros((1, Nc, 1, d))), _bits(vc), None, zb,
                                  _bits(v), m, W)
    for t in range(L):
        n_win = min(W, t + 1)
        n_cmp = sum(1 for j in range(Nc) if (j + 1) * m - 1 < t - W + 1)
        n = n_win + n_cmp
        o = res["o"][t, 0]
        assert abs(o[0] * n - n_win) < 1e-9 and abs(o[2] * n - n_cmp) < 1e-9
        lo = max(0, t - W + 1)
        assert abs(o[1] * n - sum(range(lo, t + 1))) < 1e-7
        assert abs(o[3] * n - sum(range(n_cmp))) < 1e-7
        # compressed history never reaches into the window, nor past t
        if n_cmp:
            assert (n_cmp - 1) * m + m - 1 < lo


def test_window_entry_count_of_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "counts.json")))["window_score_entries"]
    n, w = g[0]["n"], g[0]["w"]
    z = _bits(np.zeros((1, n, 1, 1)))
    zc = _bits(np.zeros((1, 1, 1, 1)))
    # m larger than n: no compressed entry is ever visible; only the window counts
    res = oracle.hybrid_attention(z, zc, zc, None, z, z, m=n + 1, W=w)
    assert int(res["n_comp"].sum()) == 0
    total = int(res["n_win"].sum())
    assert total == g[0]["with_causal_ramp"]
    # the page's figure ignores the causal ramp at the start: n * w
    assert n * int(res["n_win"].max()) == g[0]["product_n_times_w"]
    assert abs(g[0]["product_n_times_w"] - g[0]["page_figure"]) <= g[0]["page_rel_tol"] * g[0]["page_figure"]
    assert n * n // (n * w) == 8 and n * n // (n * g[1]["w"]) == g[1]["full_over_window"]


def test_topk_covering_all_visible_equals_dense():
    rng = np.random.default_rng(12)
    L, Hq, d, m, W = 160, 4, 8, 4, 16
    q, k, v, kc, vc = _rand_case(rng, 1, L, Hq, 1, d, m)
    Nc = L // m
    idx = np.full((1, L, Nc), -1, np.int32)
    for t in range(L):
        nv = oracle.visible_count(t, m, W, Nc)
        idx[0, t, :nv] = np.arange(nv)
    a = oracle.hybrid_attention(q, kc, vc, idx, k, v, m, W)
    b = oracle.hybrid_attention(q, kc, vc, None, k, v, m, W)
    np.testing.assert_array_equal(a["o"], b["o"])
    np.testing.assert_array_equal(a["lse"], b["lse"])


def test_decode_form_equals_prefill_row():
    # the last token of a sequence, computed from a W-row raw buffer and a query
    # position, must equal the prefill result for that row.
    rng = np.random.default_rng(13)
    B, L, Hq, d, m, W = 2, 300, 4, 8, 4, 32
    q, k, v, kc, vc = _rand_case(rng, B, L, Hq, 1, d, m)
    rows = [L - 1, 2 * L - 1]
    pre = oracle.hybrid_attention(q, kc, vc, None, k, v, m, W, rows=rows)
    qd = q[:, L - 1:L]
    kd, vd = k[:, L - W:], v[:, L - W:]
    qpos = np.full((B, 1), L - 1, np.int32)
    kv0 = np.full((B,), L - W, np.int32)
    dec = oracle.hybrid_attention(qd, kc, vc, None, kd, vd, m, W, q_pos=qpos, kv_pos0=kv0)
    np.testing.assert_array_equal(dec["o"], pre["o"])
    np.testing.assert_array_equal(dec["lse"], pre["lse"])


def test_empty_key_set_gives_zero_output():
    # W = 0 and t < m - 1: no window and no complete block yet
    z = _bits(np.ones((1, 8, 1, 4)))
    res = oracle.hybrid_attention(z, z[:, :2], z[:, :2], None, z, z, m=4, W=0, rows=[0, 1, 2, 3])
    assert np.all(res["o"][:3] == 0) and np.all(np.isneginf(res["lse"][:3]))
    assert res["n_comp"][3] == 1


def test_invalid_index_is_reported():
    z = _bits(np.ones((1, 8, 1, 4)))
    idx = np.full((1, 8, 2), -1, np.int32)
    idx[0, 7, 0] = 5  # Nc = 2
    with pytest.raises(ValueError):
        oracle.hybrid_attention(z, z[:, :2], z[:, :2], idx, z, z, m=4, W=0)
