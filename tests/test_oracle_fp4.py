"""Pins for the oracle's 4-bit cache quantization (DeepSeek-V4 CSDN article,
"compress_to_fp4" / "decompress_from_fp4": scale = (max - min) / 15, codes
round((x - min) / scale) clamped to 0..15, dequantized as code * scale + min)."""
import numpy as np
import pytest
import torch

import oracle



def _bits(vals):
    return oracle.bf16_bits(torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16))


def _unpack(codes):
    q = np.empty(codes.shape[:-1] + (2 * codes.shape[-1],), dtype=np.int64)
    q[..., 0::2] = codes & 15
    q[..., 1::2] = codes >> 4
    return q


def test_exact_levels_and_nibble_order():
    # min -8, max 7: scale exactly 1, every value sits on a level; element 2i
    # is the low nibble of byte i
    vals = [float(v) for v in range(-8, 8)]
    codes, qp = oracle.fp4_quantize(_bits(vals))
    assert qp.tolist() == [-8.0, 1.0]
    assert _unpack(codes).tolist() == list(range(16))
    assert codes[0] == 0x10 and codes[7] == 0xFE
    back = oracle.bf16_to_f64(oracle.fp4_dequantize(codes, qp))
    assert back.tolist() == vals


def test_ties_round_to_even():
    # scale 1 again (min 0, max 15); halfway values go to the even level,
    # as torch.round does
    vals = [0.0, 15.0, 0.5, 1.5, 2.5, 3.5, 4.5, 13.5]
    codes, qp = oracle.fp4_quantize(_bits(vals))
    assert qp.tolist() == [0.0, 1.0]
    assert _unpack(codes).tolist() == [0, 15, 0, 2, 2, 4, 4, 14]


def test_constant_row_reads_back_exactly():
    codes, qp = oracle.fp4_quantize(_bits([0.375] * 8))
    assert qp.tolist() == [0.375, 0.0]
    assert not codes.any()
    assert oracle.bf16_to_f64(oracle.fp4_dequantize(codes, qp)).tolist() == [0.375] * 8


def test_scale_from_row_extremes_only():
    # per-row min and max: one row's range does not affect another's
    rows = np.stack([_bits([1.0, 2.0, 4.0, 3.0]), _bits([-100.0, 100.0, 0.0, 50.0])])
    codes, qp = oracle.fp4_quantize(rows)
    assert qp[0].tolist() == [1.0, np.float32(3.0) / np.float32(15.0)]
    assert qp[1].tolist() == [-100.0, np.float32(200.0) / np.float32(15.0)]
    q = _unpack(codes)
    assert q[0, 0] == 0 and q[0, 2] == 15 and q[1, 0] == 0 and q[1, 1] == 15


def test_error_bound_and_nearest_level():
    # |dequant - x| <= scale / 2 (plus the final bf16 rounding), and each code
    # is the nearest of the 16 levels, checked by brute force in fp64
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(64, 128, generator=g) * torch.rand(64, 1, generator=g) * 4).to(torch.bfloat16)
    bits = oracle.bf16_bits(x)
    codes, qp = oracle.fp4_quantize(bits)
    xf = oracle.bf16_to_f64(bits)
    back = oracle.bf16_to_f64(oracle.fp4_dequantize(codes, qp))
    mn, sc = qp[:, 0:1].astype(np.float64), qp[:, 1:2].astype(np.float64)
    bound = sc / 2 * (1 + 1e-5) + np.abs(back) * 2.0 ** -8
    assert (np.abs(back - xf) <= bound).all()
    levels = mn[:, :, None] + sc[:, :, None] * np.arange(16)[None, None, :]
    dist = np.abs(levels - xf[:, :, None])
    best = dist.argmin(axis=-1)
    q = _unpack(codes)
    order = np.sort(dist, axis=-1)
    clear = (order[..., 1] - order[..., 0]) > 1e-4 * sc
    assert (q[clear] == best[clear]).all()
    assert clear.mean() > 0.99


def test_codes_cover_the_range():
    # the row minimum maps to code 0 and the maximum to code 15
    g = torch.Generator().manual_seed(6)
    x = torch.randn(32, 64, generator=g).to(torch.bfloat16)
    bits = oracle.bf16_bits(x)
    q = _unpack(oracle.fp4_quantize(bits)[0])
    xf = oracle.bf16_to_f64(bits)
    rows = np.arange(32)
    assert (q[rows, xf.argmin(axis=1)] == 0).all()
    assert (q[rows, xf.argmax(axis=1)] == 15).all()
