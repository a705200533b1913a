"""CPU oracle for hybrid compressed / sparse / sliding-window attention.

TEST INFRASTRUCTURE ONLY: this package is imported by the tests, by the smoke
check and by the CPU-baseline leg of the benchmark, never by the library.  It
shares no code with the CUDA path; its arithmetic lives in ``oracle.c`` (fp64,
OpenMP over query rows) and, for tiny shapes, in ``brute.py`` (numpy fp64 with
an explicit mask), which is an independent second statement used to pin it.

Inputs are numpy arrays.  bf16 tensors are passed as their raw bits
(``numpy.uint16``); fp32 tensors as ``numpy.float32``.  ``bf16_bits`` turns a
torch bf16 tensor into that form.

Parity status per function (what pins it, in tests/test_oracle_*.py):
  block_merge       closed forms (zero weights -> mean, one-hot weights ->
                    a single token, m=1 -> identity), softmax axis
  round_bf16        torch's fp32->bf16 conversion, hand-worked ties
  index_scores      hand-worked example (tests/golden), homogeneity and ReLU
                    invariants, head-weight linearity
  topk              numpy.lexsort brute force, K >= n_vis, permutation
  hybrid_attention  brute-force masked attention (brute.py), torch SDPA for
                    m=1/W=0, K >= n_vis equals dense, softmax rows sum to 1,
                    label-counting pins for the key sets, window-count pin
  decode_append     ring rows and emitted entries against block_merge of the
                    same positions, kv_pos0 closed form
  gated_attention   one-hot gates give one branch (brute-force masks per
                    branch), the output is the gate-weighted combination
  fp4_quantize /    exact levels, ties to even, constant rows, nibble order,
  fp4_dequantize    the half-step error bound, nearest level by brute force
  backward.*        (oracle/backward.py) attention and block_merge gradients:
                    central finite differences of the scalar losses in fp64
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I = ctypes.c_int
    I64 = ctypes.c_int64
    lib.oracle_round_bf16.argtypes = [P, P, I64]
    lib.oracle_round_bf16.restype = None
    lib.oracle_block_merge.argtypes = [P, I, I, I, I, I, P, P, P]
    lib.oracle_block_merge.restype = None
    lib.oracle_visible_count.argtypes = [I64, I, I, I]
    lib.oracle_visible_count.restype = I
    lib.oracle_index_scores.argtypes = [P, P, P, I, I, I, I, I, I, I, P, P, I, P, P]
    lib.oracle_index_scores.restype = None
    lib.oracle_topk.argtypes = [P, P, I, I, I, P]
    lib.oracle_topk.restype = None
    lib.oracle_hybrid_attention.argtypes = [P, P, P, P, I, P, P, I, I, I, I, I, I, I, I, I,
                                            ctypes.c_double, P, P, P, I, P, P, P, P, P, I, P]
    lib.oracle_hybrid_attention.restype = I
    _lib = lib
    return lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a: Optional[np.ndarray], dtype) -> Optional[np.ndarray]:
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def bf16_bits(t) -> np.ndarray:
    """Raw bits of a torch bf16 tensor (any device) as a numpy uint16 array."""
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits to float64 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); returns raw bits."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_round_bf16(_ptr(x), _ptr(out), x.size)
    return out


def visible_count(t: int, m: int, W: int, Nc: int) -> int:
    """Number of compressed entries visible to a query at absolute position t."""
    return int(_load().oracle_visible_count(t, m, W, Nc))


def block_merge(x_bits: np.ndarray, w: np.ndarray, m: int):
    """Compress x [B, L, H, dx] (bf16 bits) in blocks of m with weights w [m, dx].

    Returns (fp64 [B, L//m, H, dx], bf16 bits of the same shape).
    """
    x_bits = _c(x_bits, np.uint16)
    w = _c(w, np.float32)
    B, L, H, dx = x_bits.shape
    if w.shape != (m, dx):
        raise ValueError("block weights must be [m, dx]")
    Nc = L // m
    out = np.empty((B, Nc, H, dx), dtype=np.float64)
    out_b = np.empty((B, Nc, H, dx), dtype=np.uint16)
    _load().oracle_block_merge(_ptr(x_bits), B, L, H, dx, m, _ptr(w), _ptr(out), _ptr(out_b))
    return out, out_b


def decode_append(state: dict, t_new, k_new_bits, v_new_bits, wk, wv, m: int, W: int,
                  ki_new_bits=None, wib=None):
    """Decode cache maintenance, one new token per sequence ("deepseek-v4"
    blog, section 1: the window's raw KV and the compressed KV are separate
    caches with different lifetimes).

    state holds bf16 bits: k_ring / v_ring [B, 2W, Hkv, d], ki_ring [B, W, di]
    (CSA), kc / vc [B, Nc, Hkv, d], kic [B, Nc, di]; updated in place.
    The new row of position t goes to ring rows t mod W and t mod W + W (K, V)
    and t mod W (indexer key).  When (t + 1) is a multiple of m the block of
    positions j*m .. t, j = (t + 1) / m - 1, is compressed into entry j by
    block_merge.  Returns kv_pos0 [B] int32: lo - lo mod W, lo = max(0,
    t - W + 1), the position of ring row 0 for the contiguous window run.
    """
    t_new = np.asarray(t_new, dtype=np.int64).reshape(-1)
    B = len(t_new)
    kv_pos0 = np.zeros(B, dtype=np.int32)
    for b in range(B):
        t = int(t_new[b])
        s = t % W
        for name, new, two in (("k_ring", k_new_bits, True), ("v_ring", v_new_bits, True),
                               ("ki_ring", ki_new_bits, False)):
            if new is None:
                continue
            state[name][b, s] = new[b]
            if two:
                state[name][b, s + W] = new[b]
        lo = max(0, t - W + 1)
        kv_pos0[b] = lo - lo % W
        if (t + 1) % m == 0:
            j = (t + 1) // m - 1
            block = [(j * m + i) % W for i in range(m)]
            for ring, cache, w in (("k_ring", "kc", wk), ("v_ring", "vc", wv), ("ki_ring", "kic", wib)):
                if cache not in state or w is None or state.get(ring) is None:
                    continue
                rows = state[ring][b, block]               # [m, ...] bits
                x = rows.reshape(1, m, -1, rows.shape[-1]) if rows.ndim == 3 else rows.reshape(1, m, 1, -1)
                _, out_b = block_merge(x, w, m)
                state[cache][b, j] = out_b.reshape(state[cache][b, j].shape)
    return kv_pos0


def fp4_quantize(x_bits):
    """4-bit min/max affine quantization of every row (the last axis) of a bf16
    tensor, as the "FP4" cache storage of the DeepSeek-V4 CSDN article
    ("compress_to_fp4"): scale = (max - min) / 15, code = round((x - min) /
    scale) clamped to 0..15.

    Readings: min and max are taken per row (one compressed entry of one
    head), so that a cache can grow one entry at a time; round is to nearest,
    ties to even (torch.round); a row with max == min gets scale 0 and codes 0.
    The arithmetic that decides a code is fp32, one IEEE operation at a time.
    Codes are packed two per byte, element 2i in the low nibble of byte i.

    Returns (codes uint8 [..., dx / 2], qp float32 [..., 2] = (min, scale)).
    """
    bits = np.asarray(x_bits, dtype=np.uint16)
    if bits.shape[-1] % 2:
        raise ValueError("rows must have an even number of elements")
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    scale = np.float32(mx - mn) / np.float32(15.0)
    scale = np.asarray(scale, dtype=np.float32)
    q = np.zeros(x.shape, dtype=np.float32)
    pos = scale > 0
    if np.any(pos):
        diff = (x - mn[..., None]).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = (diff / np.where(pos, scale, np.float32(1.0))[..., None]).astype(np.float32)
        q = np.where(pos[..., None], np.rint(ratio), np.float32(0.0))
    q = np.clip(q, 0, 15).astype(np.uint8)
    codes = (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)
    qp = np.stack([mn, scale], axis=-1).astype(np.float32)
    return codes, qp


def fp4_dequantize(codes, qp):
    """Inverse of fp4_quantize ("decompress_from_fp4"): code * scale + min,
    the product and the sum each rounded to fp32, the result rounded to bf16
    (nearest, ties to even).  Returns bf16 bits [..., 2 * codes.shape[-1]]."""
    codes = np.asarray(codes, dtype=np.uint8)
    qp = np.asarray(qp, dtype=np.float32)
    q = np.empty(codes.shape[:-1] + (2 * codes.shape[-1],), dtype=np.float32)
    q[..., 0::2] = codes & 15
    q[..., 1::2] = codes >> 4
    prod = (q * qp[..., 1:2]).astype(np.float32)
    v = (prod + qp[..., 0:1]).astype(np.float32)
    return round_bf16(v.astype(np.float64))


def _rows(rows: Optional[Sequence[int]], total: int) -> np.ndarray:
    if rows is None:
        return np.arange(total, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def index_scores(qi_bits, wi, kic_bits, m: int, W: int, q_pos=None, rows=None):
    """Indexer scores for the selected query rows (row = b * Lq + t).

    qi [B, Lq, Hi, di] bf16 bits, wi [B, Lq, Hi] fp32, kic [B, Nc, di] bf16 bits.
    Returns (scores fp64 [nrows, Nc] with NaN past n_vis, n_vis int32 [nrows]).
    """
    qi_bits = _c(qi_bits, np.uint16)
    wi = _c(wi, np.float32)
    kic_bits = _c(kic_bits, np.uint16)
    B, Lq, Hi, di = qi_bits.shape
    Nc = kic_bits.shape[1]
    q_pos = _c(q_pos, np.int32)
    r = _rows(rows, B * Lq)
    scores = np.empty((len(r), Nc), dtype=np.float64)
    nvis = np.empty(len(r), dtype=np.int32)
    _load().oracle_index_scores(_ptr(qi_bits), _ptr(wi), _ptr(kic_bits), B, Lq, Hi, di, Nc, m, W,
                                _ptr(q_pos), _ptr(r), len(r), _ptr(scores), _ptr(nvis))
    return scores, nvis


def topk(scores: np.ndarray, nvis: np.ndarray, K: int) -> np.ndarray:
    """Exact top-K per row: ascending indices, -1 padded ([nrows, K] int32)."""
    scores = _c(scores, np.float64)
    nvis = _c(nvis, np.int32)
    nrows, Nc = scores.shape
    out = np.empty((nrows, K), dtype=np.int32)
    _load().oracle_topk(_ptr(scores), _ptr(nvis), nrows, Nc, K, _ptr(out))
    return out


def hybrid_attention(q_bits, kc_bits, vc_bits, idx, k_raw_bits, v_raw_bits, m: int, W: int,
                     scale: Optional[float] = None, q_pos=None, kv_pos0=None, rows=None,
                     debug_maxkeys: int = 0):
    """One softmax over (selected or all visible) compressed keys + raw window.

    q [B, Lq, Hq, d], kc/vc [B, Nc, Hkv, d], k_raw/v_raw [B, Lkv, Hkv, d] as bf16
    bits; idx [B, Lq, K] int32 or None (dense over visible entries).
    Returns dict with o [nrows, Hq, d] fp64, lse [nrows, Hq], n_comp, n_win and,
    when debug_maxkeys > 0, p [nrows, Hq, maxkeys] and keys [nrows, maxkeys].
    """
    q_bits = _c(q_bits, np.uint16)
    kc_bits = _c(kc_bits, np.uint16)
    vc_bits = _c(vc_bits, np.uint16)
    k_raw_bits = _c(k_raw_bits, np.uint16)
    v_raw_bits = _c(v_raw_bits, np.uint16)
    idx = _c(idx, np.int32)
    q_pos = _c(q_pos, np.int32)
    kv_pos0 = _c(kv_pos0, np.int32)
    B, Lq, Hq, d = q_bits.shape
    Nc, Hkv = kc_bits.shape[1], kc_bits.shape[2]
    Lkv = k_raw_bits.shape[1]
    topk_ = 0 if idx is None else idx.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = _rows(rows, B * Lq)
    n = len(r)
    o = np.empty((n, Hq, d), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    n_comp = np.empty(n, dtype=np.int32)
    n_win = np.empty(n, dtype=np.int32)
    p = keys = None
    if debug_maxkeys:
        p = np.zeros((n, Hq, debug_maxkeys), dtype=np.float64)
        keys = np.zeros((n, debug_maxkeys), dtype=np.int32)
    st = _load().oracle_hybrid_attention(
        _ptr(q_bits), _ptr(kc_bits), _ptr(vc_bits), _ptr(idx), topk_, _ptr(k_raw_bits),
        _ptr(v_raw_bits), B, Lq, Lkv, Hq, Hkv, d, m, W, Nc, float(scale), _ptr(q_pos),
        _ptr(kv_pos0), _ptr(r), n, _ptr(o), _ptr(lse), _ptr(n_comp), _ptr(n_win), _ptr(p),
        debug_maxkeys, _ptr(keys))
    if st != 0:
        raise ValueError(f"oracle_hybrid_attention: bad input (status {st})")
    res = dict(o=o, lse=lse, n_comp=n_comp, n_win=n_win)
    if debug_maxkeys:
        res["p"] = p
        res["keys"] = keys
    return res


def gated_attention(q_bits, kc_bits, vc_bits, idx, k_raw_bits, v_raw_bits, m: int, W: int,
                    gate_logits, scale: Optional[float] = None, q_pos=None, kv_pos0=None, rows=None):
    """The gated three-branch variant (Tiny-R2 README, "Attention Computation"
    and "branch_gate"): three attentions with separate softmaxes, then a
    softmax over the branches of per-(token, head) gate logits weights them.

      branch 1, compressed: every compressed block that ends at or before t
                (hybrid_attention with no selection and W = 0);
      branch 2, selected:   the listed blocks among those (idx, W = 0);
      branch 3, window:     the raw keys max(0, t-W+1) .. t (no compressed).
    A branch with no key contributes 0.  gate_logits [B, Lq, Hq, 3] (fp32).
    Returns dict(o [nrows, Hq, d], branches [3, nrows, Hq, d]).
    """
    kc_bits = _c(kc_bits, np.uint16)
    B, Nc, Hkv, d = kc_bits.shape
    none = np.zeros((B, 0, Hkv, d), dtype=np.uint16)
    o1 = hybrid_attention(q_bits, kc_bits, vc_bits, None, k_raw_bits, v_raw_bits, m, 0, scale=scale,
                          q_pos=q_pos, kv_pos0=kv_pos0, rows=rows)["o"]
    o2 = hybrid_attention(q_bits, kc_bits, vc_bits, idx, k_raw_bits, v_raw_bits, m, 0, scale=scale,
                          q_pos=q_pos, kv_pos0=kv_pos0, rows=rows)["o"]
    o3 = hybrid_attention(q_bits, none, none, None, k_raw_bits, v_raw_bits, m, W, scale=scale,
                          q_pos=q_pos, kv_pos0=kv_pos0, rows=rows)["o"]
    g = np.asarray(gate_logits, dtype=np.float64)
    Lq, Hq = g.shape[1], g.shape[2]
    g = g.reshape(-1, Hq, 3)[_rows(rows, B * Lq)]
    g = np.exp(g - g.max(axis=-1, keepdims=True))
    g /= g.sum(axis=-1, keepdims=True)
    br = np.stack([o1, o2, o3])
    o = np.einsum("nhk,knhd->nhd", g, br)
    return dict(o=o, branches=br)


def forward(inp: dict, m: int, W: int, topk_k: int, rows=None, scale=None):
    """The whole forward pass for prefill inputs (see workloads.make_inputs).

    block_merge of K, V (and indexer keys) -> indexer scores + top-K (CSA) ->
    hybrid attention, for the requested query rows.  Inputs are numpy bf16
    bits / fp32 arrays under the same names as the workload tensors.
    """
    _, kc = block_merge(inp["k"], inp["wk"], m)
    _, vc = block_merge(inp["v"], inp["wv"], m)
    res = dict(kc=kc, vc=vc)
    idx = None
    if topk_k:
        _, kic = block_merge(inp["ki"][:, :, None, :], inp["wib"], m)
        kic = kic[:, :, 0, :]
        scores, nvis = index_scores(inp["qi"], inp["wi"], kic, m, W, rows=rows)
        sel = topk(scores, nvis, topk_k)
        res.update(kic=kic, scores=scores, nvis=nvis, idx_rows=sel)
        B, L = inp["q"].shape[:2]
        idx = np.full((B * L, topk_k), -1, dtype=np.int32)
        r = _rows(rows, B * L)
        idx[r] = sel
        idx = idx.reshape(B, L, topk_k)
    att = hybrid_attention(inp["q"], kc, vc, idx, inp["k"], inp["v"], m, W, scale=scale,
                           rows=rows)
    res.update(att)
    return res
