"""Pins of the gated three-branch oracle against plain definitions."""
import numpy as np

import oracle
from oracle import brute


def _bits(rng, shape):
    return (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _case(seed=0, B=1, L=40, Hq=2, Hkv=1, d=8, m=4, W=6, K=3):
    rng = np.random.default_rng(seed)
    q = _bits(rng, (B, L, Hq, d))
    k = _bits(rng, (B, L, Hkv, d))
    v = _bits(rng, (B, L, Hkv, d))
    Nc = L // m
    kc = _bits(rng, (B, Nc, Hkv, d))
    vc = _bits(rng, (B, Nc, Hkv, d))
    idx = np.full((B, L, K), -1, np.int32)
    for b in range(B):
        for t in range(L):
            nv = min(Nc, (t + 1) // m)      # blocks ending at or before t
            if nv:
                idx[b, t, :min(K, nv)] = np.sort(rng.choice(nv, size=min(K, nv), replace=False))
    gate = rng.standard_normal((B, L, Hq, 3)).astype(np.float32)
    return q, kc, vc, idx, k, v, m, W, gate


def test_one_hot_gate_selects_a_branch():
    q, kc, vc, idx, k, v, m, W, gate = _case()
    for br in range(3):
        g = np.full(gate.shape, -1e30, np.float32)
        g[..., br] = 0.0
        res = oracle.gated_attention(q, kc, vc, idx, k, v, m, W, g)
        np.testing.assert_allclose(res["o"], res["branches"][br], atol=1e-12)


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_branches_against_brute_force_masks():
    # each branch equals dense attention under an explicit mask: blocks ending
    # at or before t (all, then the selected ones) with no raw key (W = 0), and
    # raw keys t-W+1..t with no compressed entry
    q, kc, vc, idx, k, v, m, W, gate = _case(seed=1)
    res = oracle.gated_attention(q, kc, vc, idx, k, v, m, W, gate)
    qf, kcf, vcf, kf, vf = (_f64(x[0]) for x in (q, kc, vc, k, v))
    none = np.zeros((0,) + kcf.shape[1:])
    refs = [brute.attention(qf, kcf, vcf, kf, vf, m, 0)[0],
            brute.attention(qf, kcf, vcf, kf, vf, m, 0, idx=idx[0])[0],
            brute.attention(qf, none, none, kf, vf, m, W)[0]]
    for br in range(3):
        np.testing.assert_allclose(res["branches"][br], refs[br], atol=1e-10)


def test_gate_is_a_convex_combination():
    q, kc, vc, idx, k, v, m, W, gate = _case(seed=2)
    res = oracle.gated_attention(q, kc, vc, idx, k, v, m, W, gate)
    g = np.exp(gate.astype(np.float64) - gate.max(-1, keepdims=True))
    g /= g.sum(-1, keepdims=True)
    want = (g.reshape(-1, 2, 3)[:, :, :, None] * np.moveaxis(res["branches"], 0, 2)).sum(2)
    np.testing.assert_allclose(res["o"], want, atol=1e-12)
