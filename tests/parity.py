"""Comparison rules shared by the GPU parity tests.

Tolerances (bf16 inputs and outputs, fp32 accumulation on the GPU, fp64 in the
oracle):
  attention output   max |o_gpu - o_ref| <= 2e-2 and mean |o_gpu - o_ref| <= 2e-3
  lse                |lse_gpu - lse_ref| <= 2e-3 (natural log units)
  compressed caches  bit-exact bf16 except a fraction max(1e-4, 4 sqrt(m) 2^-16)
                     of elements (double rounding: fp32 sum then bf16 versus
                     fp64 sum then bf16), which stay within one bf16 ulp plus
                     the fp32 accumulation bound
  top-K indices      bit-exact per query row, except rows where the oracle's
                     K-th and (K+1)-th largest scores differ by less than 1e-4
                     relative (a near tie fp32 cannot resolve); for those rows
                     the GPU's set must still be a valid top-K within that
                     relative margin.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 2e-3
NEAR_TIE_REL = 1e-4


def bits(t: torch.Tensor) -> np.ndarray:
    return oracle.bf16_bits(t)


def from_bits(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def check_output(o_gpu: torch.Tensor, o_ref: np.ndarray, what: str = "o"):
    og = o_gpu.float().cpu().numpy().astype(np.float64).reshape(o_ref.shape)
    err = np.abs(og - o_ref)
    assert np.all(np.isfinite(og)), f"{what}: non-finite GPU output"
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    assert mx <= O_MAX_ABS and mean <= O_MEAN_ABS, f"{what}: max-abs {mx:.3e}, mean-abs {mean:.3e}"
    return mx, mean


def check_lse(lse_gpu: np.ndarray, lse_ref: np.ndarray):
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(lse_gpu)), "lse: -inf pattern differs"
    if fin.any():
        err = np.abs(lse_gpu[fin] - lse_ref[fin]).max()
        assert err <= LSE_ABS, f"lse: max-abs {err:.3e}"


def check_bf16_cache(gpu: torch.Tensor, ref_bits: np.ndarray, what: str = "cache",
                     abs_sum: np.ndarray = None, m: int = 1):
    """Compressed cache: bit-exact almost everywhere; elsewhere within one bf16
    ulp plus the fp32 accumulation bound (m + 8) * 2^-24 * sum_i P_i |x_i|
    (abs_sum, the oracle's block merge of |x|), which matters only where the
    weighted sum cancels to a value much smaller than its terms."""
    g = bits(gpu).reshape(ref_bits.shape)
    gf = oracle.bf16_to_f64(g)
    rf = oracle.bf16_to_f64(ref_bits)
    n = g.size
    exact = int((g == ref_bits).sum())
    ulp = np.maximum(np.abs(gf), np.abs(rf)) * 2.0 ** -7
    allowed = ulp + (0.0 if abs_sum is None else (m + 8) * 2.0 ** -24 * abs_sum)
    over = np.abs(gf - rf) > allowed
    assert not over.any(), f"{what}: {int(over.sum())} elements beyond tolerance"
    # Double rounding (fp32 sum, then bf16) differs from the oracle's rounding
    # when the exact sum lies within the fp32 accumulation error of a bf16
    # rounding midpoint: a typical error of sqrt(m) * 2^-24 relative against a
    # bf16 ulp of 2^-7 relative gives a rate near sqrt(m) * 2^-16.  Allowed:
    # four times that rate (and at least 1e-4).
    rate = max(1e-4, 4.0 * np.sqrt(m) * 2.0 ** -16)
    assert exact >= n - max(1, int(rate * n)), f"{what}: only {exact}/{n} bit-exact"
    return exact, n


def abs_merge(x_bits: np.ndarray, w: np.ndarray, m: int) -> np.ndarray:
    """sum_i P_i |x_i| per compressed element (oracle block merge of |x|)."""
    out, _ = oracle.block_merge(np.ascontiguousarray(x_bits) & np.uint16(0x7FFF), w, m)
    return out


def near_tie_rows(scores: np.ndarray, nvis: np.ndarray, K: int) -> np.ndarray:
    """Rows whose K-th and (K+1)-th largest oracle scores are a near tie."""
    out = np.zeros(len(nvis), dtype=bool)
    for r, n in enumerate(nvis):
        if n <= K:
            continue
        srt = np.sort(scores[r, :n])[::-1]
        a, b = srt[K - 1], srt[K]
        out[r] = a != b and abs(a - b) < NEAR_TIE_REL * max(abs(a), abs(b))
    return out


def check_topk(idx_gpu: np.ndarray, idx_ref: np.ndarray, scores: np.ndarray, nvis: np.ndarray,
               K: int):
    """Returns the boolean mask of rows compared bit-exactly."""
    tie = near_tie_rows(scores, nvis, K)
    exact = ~tie
    bad = np.where(exact & np.any(idx_gpu != idx_ref, axis=1))[0]
    assert len(bad) == 0, f"top-K differs on {len(bad)} rows, first {bad[:5]}"
    for r in np.where(tie)[0]:
        n = nvis[r]
        sel = idx_gpu[r][idx_gpu[r] >= 0]
        assert len(sel) == min(K, n) and len(set(sel.tolist())) == len(sel)
        assert np.all(np.diff(sel) > 0) and sel.max() < n
        kth = np.sort(scores[r, :n])[::-1][K - 1]
        tol = NEAR_TIE_REL * abs(kth) + 1e-30
        rest = np.setdiff1d(np.arange(n), sel)
        assert scores[r, sel].min() >= kth - tol
        if len(rest):
            assert scores[r, rest].max() <= kth + tol
    return exact
