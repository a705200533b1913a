"""Pins for the backward oracle (oracle/backward.py): central finite
differences of the scalar losses sum(dO * o) and sum(dc * c) in fp64, and
the fp64 block_merge against the C oracle's."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bwd


def _fd(f, x, picks, eps=1e-6):
    out = []
    for i in picks:
        old = x.flat[i]
        x.flat[i] = old + eps
        hi = f()
        x.flat[i] = old - eps
        lo = f()
        x.flat[i] = old
        out.append((hi - lo) / (2 * eps))
    return np.array(out)


@pytest.mark.parametrize("K", [0, 3])
def test_attention_gradients_match_finite_differences(K):
    rng = np.random.default_rng(7 + K)
    L, Hq, Hkv, d, m, W = 21, 4, 2, 8, 2, 4
    Nc = L // m
    q, k, v = (rng.standard_normal((L, Hq if i == 0 else Hkv, d)) for i in range(3))
    kc, vc = rng.standard_normal((Nc, Hkv, d)), rng.standard_normal((Nc, Hkv, d))
    dout = rng.standard_normal((L, Hq, d))
    idx = None
    if K:
        idx = np.full((L, K), -1, np.int64)
        for t in range(L):
            nv = oracle.visible_count(t, m, W, Nc)
            if nv:
                s = np.sort(rng.choice(nv, size=min(K, nv), replace=False))
                idx[t, :len(s)] = s
    g = bwd.attention_bwd(q, kc, vc, k, v, m, W, dout, idx=idx)
    loss = lambda: float((dout * bwd.attention_f64(q, kc, vc, k, v, m, W, idx=idx)).sum())
    for name, x, gx in (("q", q, g["dq"]), ("kc", kc, g["dkc"]), ("vc", vc, g["dvc"]),
                        ("k", k, g["dk_raw"]), ("v", v, g["dv_raw"])):
        picks = rng.choice(x.size, size=min(60, x.size), replace=False)
        num = _fd(loss, x, picks)
        np.testing.assert_allclose(gx.flat[picks], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_unselected_and_invisible_keys_get_no_gradient():
    # a compressed entry no query selects, and raw rows after the last query's
    # window, have zero gradient
    rng = np.random.default_rng(3)
    L, Hq, Hkv, d, m, W, K = 16, 2, 1, 4, 2, 4, 2
    Nc = L // m
    q, k, v = (rng.standard_normal((L, Hq if i == 0 else Hkv, d)) for i in range(3))
    kc, vc = rng.standard_normal((Nc, Hkv, d)), rng.standard_normal((Nc, Hkv, d))
    idx = np.full((L, K), -1, np.int64)
    for t in range(L):
        nv = oracle.visible_count(t, m, W, Nc)
        sel = [j for j in range(nv) if j != 1][:K]
        idx[t, :len(sel)] = sel
    g = bwd.attention_bwd(q, kc, vc, k, v, m, W, rng.standard_normal((L, Hq, d)), idx=idx)
    assert not g["dkc"][1].any() and not g["dvc"][1].any()
    nv_last = oracle.visible_count(L - 1, m, W, Nc)
    assert not g["dkc"][nv_last:].any()


def test_block_merge_gradients_match_finite_differences():
    rng = np.random.default_rng(11)
    B, L, H, dx, m = 2, 9, 2, 4, 2          # L % m != 0: a trailing partial block
    x = rng.standard_normal((B, L, H, dx))
    w = rng.standard_normal((m, dx))
    dc = rng.standard_normal((B, L // m, H, dx))
    gx, gw = bwd.block_merge_bwd(x, w, m, dc)
    loss = lambda: float((dc * bwd.block_merge_f64(x, w, m)).sum())
    np.testing.assert_allclose(gx.ravel(), _fd(loss, x, range(x.size)), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(gw.ravel(), _fd(loss, w, range(w.size)), rtol=1e-6, atol=1e-8)
    assert not gx[:, (L // m) * m:].any()


def test_block_merge_f64_is_the_oracle_forward():
    g = torch.Generator().manual_seed(12)
    x = torch.randn((2, 24, 3, 16), generator=g).to(torch.bfloat16)
    w = torch.randn((4, 16), generator=g)
    ref, _ = oracle.block_merge(oracle.bf16_bits(x), w.numpy(), 4)
    got = bwd.block_merge_f64(x.double().numpy(), w.numpy().astype(np.float64), 4)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
