"""Brute-force masked attention (numpy fp64) for tiny prefill shapes.

TEST INFRASTRUCTURE ONLY.  A second, independent statement of the hybrid
attention, written as dense attention over the concatenation
[compressed entries ; raw tokens] with an explicit boolean mask, the way the
"DeepSeek-V4 architecture diagram" post (zwxr.cn, section 4, SWA) recommends
building and unit-testing a combined window + causal mask.  It pins the
oracle's per-row key lists: it never builds a key list itself.

Mask for query t (prefill, absolute position t), per the visibility rule of
the compressed history ("deepseek-v4" blog, section 1, SWA: recent raw KV plus
older compressed KV):
    M[t, j]      = (j + 1) * m - 1 < t - W + 1  and  (idx is None or j in idx[t])
    M[t, Nc + s] = t - W + 1 <= s <= t
"""
from __future__ import annotations

import numpy as np


def mask(L: int, Nc: int, m: int, W: int, idx=None) -> np.ndarray:
    t = np.arange(L)[:, None]
    j = np.arange(Nc)[None, :]
    comp = (j + 1) * m - 1 < t - W + 1
    if idx is not None:
        sel = np.zeros((L, Nc), dtype=bool)
        for tt in range(L):
            for jj in idx[tt]:
                if jj >= 0:
                    sel[tt, jj] = True
        comp = comp & sel
    s = np.arange(L)[None, :]
    raw = (s >= t - W + 1) & (s <= t)
    return np.concatenate([comp, raw], axis=1)


def attention(q, kc, vc, k_raw, v_raw, m: int, W: int, idx=None, scale=None):
    """q [L, Hq, d]; kc/vc [Nc, Hkv, d]; k_raw/v_raw [L, Hkv, d]; fp64 arrays.

    Returns (o [L, Hq, d], lse [L, Hq], P [Hq, L, Nc + L]).
    """
    L, Hq, d = q.shape
    Nc, Hkv = kc.shape[0], kc.shape[1]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    M = mask(L, Nc, m, W, idx)
    o = np.zeros((L, Hq, d))
    lse = np.full((L, Hq), -np.inf)
    P = np.zeros((Hq, L, Nc + L))
    for h in range(Hq):
        kh = np.concatenate([kc[:, h // g, :], k_raw[:, h // g, :]], axis=0)
        vh = np.concatenate([vc[:, h // g, :], v_raw[:, h // g, :]], axis=0)
        S = scale * (q[:, h, :] @ kh.T)
        S = np.where(M, S, -np.inf)
        mx = S.max(axis=1, keepdims=True)
        has = np.isfinite(mx[:, 0])
        mx = np.where(np.isfinite(mx), mx, 0.0)
        E = np.where(M, np.exp(S - mx), 0.0)
        den = E.sum(axis=1, keepdims=True)
        Pm = np.divide(E, den, out=np.zeros_like(E), where=den > 0)
        P[h] = Pm
        o[:, h, :] = Pm @ vh
        lse[has, h] = (mx[:, 0] + np.log(np.where(den[:, 0] > 0, den[:, 0], 1.0)))[has]
    return o, lse, P
