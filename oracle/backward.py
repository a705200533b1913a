"""Backward pass of the hybrid attention and of block_merge (numpy fp64).

TEST INFRASTRUCTURE ONLY: used by the tests and the benchmark's CPU legs,
never by the library.  The training follow-on of the Tiny-R2 README
("Training"): gradients of a loss through the attention step and through the
compression of K / V.  The pages define no gradient for the top-K selection;
it is taken as fixed (a straight selection): the indexer gets no gradient and
the selected set does not change with the inputs.

Attention, for one query row with key set S (compressed entries selected or
visible, raw window), softmax over S of s_j = scale * q . k_j:
    o = sum_j P_j v_j,  dP_j = dO . v_j,  dS_j = P_j (dP_j - sum_k P_k dP_k)
    dq = scale * sum_j dS_j k_j,  dk_j += scale * dS_j q,  dv_j += P_j dO
summed over the query heads sharing a KV head and over the queries that
select key j.  Written here on the dense masked form of oracle.brute (one
sequence, prefill positions), with numpy matrix products.

block_merge, c_j[c] = sum_i P[i, c] x_{jm+i}[c] with P = softmax over i of
w[:, c]:
    dx_{jm+i}[c] = P[i, c] dc_j[c]
    dw[i, c] = P[i, c] (G[i, c] - sum_k P[k, c] G[k, c]),
    G[i, c] = sum over blocks, batches, heads of dc_j[c] x_{jm+i}[c]
(rows of a trailing partial block get no gradient).

Pins: central finite differences of sum(dO * o) and sum(dc * c) in fp64
(tests/test_oracle_backward.py); block_merge_f64 against the C oracle's
block_merge on bf16 inputs.
"""
from __future__ import annotations

import numpy as np

from . import brute


def _softmax_rows(S, M):
    mx = np.where(M, S, -np.inf).max(axis=1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    E = np.where(M, np.exp(S - mx), 0.0)
    den = E.sum(axis=1, keepdims=True)
    return np.divide(E, den, out=np.zeros_like(E), where=den > 0)


def attention_f64(q, kc, vc, k_raw, v_raw, m: int, W: int, idx=None, scale=None):
    """Forward on fp64 inputs (one sequence): q [L, Hq, d], kc/vc [Nc, Hkv, d],
    k_raw/v_raw [L, Hkv, d].  Returns o [L, Hq, d]."""
    return brute.attention(q, kc, vc, k_raw, v_raw, m, W, idx=idx, scale=scale)[0]


def attention_bwd(q, kc, vc, k_raw, v_raw, m: int, W: int, dout, idx=None, scale=None):
    """Gradients of sum(dout * o) for one sequence (fp64 arrays, shapes as
    attention_f64).  Returns dict(dq, dkc, dvc, dk_raw, dv_raw)."""
    L, Hq, d = q.shape
    Nc, Hkv = kc.shape[0], kc.shape[1]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    M = brute.mask(L, Nc, m, W, idx)
    dq = np.zeros_like(q)
    dK = np.zeros((Hkv, Nc + L, d))
    dV = np.zeros((Hkv, Nc + L, d))
    for h in range(Hq):
        kv = h // g
        K = np.concatenate([kc[:, kv, :], k_raw[:, kv, :]], axis=0)
        V = np.concatenate([vc[:, kv, :], v_raw[:, kv, :]], axis=0)
        P = _softmax_rows(scale * (q[:, h, :] @ K.T), M)
        dP = dout[:, h, :] @ V.T
        dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
        dq[:, h, :] = scale * (dS @ K)
        dK[kv] += scale * (dS.T @ q[:, h, :])
        dV[kv] += P.T @ dout[:, h, :]
    return dict(dq=dq, dkc=dK[:, :Nc].transpose(1, 0, 2), dvc=dV[:, :Nc].transpose(1, 0, 2),
                dk_raw=dK[:, Nc:].transpose(1, 0, 2), dv_raw=dV[:, Nc:].transpose(1, 0, 2))


def block_merge_f64(x, w, m: int):
    """block_merge on fp64 x [B, L, H, dx] with weights w [m, dx]: [B, L//m, H, dx]."""
    B, L, H, dx = x.shape
    Nc = L // m
    P = np.exp(w - w.max(axis=0, keepdims=True))
    P = P / P.sum(axis=0, keepdims=True)
    xb = x[:, :Nc * m].reshape(B, Nc, m, H, dx)
    return np.einsum("bjihc,ic->bjhc", xb, P)


def block_merge_bwd(x, w, m: int, dc):
    """Gradients of sum(dc * block_merge_f64(x, w, m)).  Returns (dx, dw)."""
    B, L, H, dx_ = x.shape
    Nc = L // m
    P = np.exp(w - w.max(axis=0, keepdims=True))
    P = P / P.sum(axis=0, keepdims=True)
    xb = x[:, :Nc * m].reshape(B, Nc, m, H, dx_)
    dx = np.zeros_like(x)
    dx[:, :Nc * m] = (P[None, None, :, None, :] * dc[:, :, None, :, :]).reshape(B, Nc * m, H, dx_)
    G = np.einsum("bjhc,bjihc->ic", dc, xb)
    dw = P * (G - (P * G).sum(axis=0, keepdims=True))
    return dx, dw
