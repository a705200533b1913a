"""The C-ABI library loads and exports every entry point of include/hybattn.h,
and host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hybattn.h")


@pytest.fixture(scope="module")
def lib():
    from compressed_sparse_sliding_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hyb_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert {"hyb_hca_compress", "hyb_csa_index_topk", "hyb_attn_fwd", "hyb_fused_fwd",
            "hyb_workspace_size", "hyb_get_device_status", "hyb_error_string",
            "hyb_decode_append", "hyb_gated_fwd", "hyb_gated_workspace_size",
            "hyb_fp4_quantize", "hyb_fp4_dequantize", "hyb_fp4_workspace_size",
            "hyb_csa_index_topk_fp4", "hyb_attn_fwd_fp4", "hyb_decode_append_fp4",
            "hyb_attn_bwd", "hyb_hca_compress_bwd", "hyb_hca_compress_bwd_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_error_strings(lib):
    lib.hyb_error_string.restype = ctypes.c_char_p
    for code in range(-6, 1):
        assert lib.hyb_error_string(code)
    assert lib.hyb_error_string(0) == b"ok"


def test_host_side_argument_checks(lib):
    import compressed_sparse_sliding_b200 as hb
    # null inputs are rejected before any launch
    st = hb._lib.hyb_hca_compress(None, 1, 8, 1, 64, 4, None, None, None)
    assert st == hb.HYB_ERR_INVALID_ARG
    p = hb.problem(B=1, Lq=16, Lkv=16, Hq=4, Hkv=3, d=64, m=4, W=8)
    assert hb._lib.hyb_attn_fwd(ctypes.byref(p), None, None, None, None, None, None, None, None,
                                None) == hb.HYB_ERR_INVALID_ARG
    p = hb.problem(B=1, Lq=16, Lkv=16, Hq=4, Hkv=1, d=96, m=4, W=8)
    assert hb._lib.hyb_attn_fwd(ctypes.byref(p), None, None, None, None, None, None, None, None,
                                None) == hb.HYB_ERR_UNSUPPORTED
    # workspace: none when the selection runs in one kernel (64 or more query
    # rows per sequence, at most 4 indexer heads, Nc <= 65535) and the score
    # rows would take more than 256 MiB ...
    p = hb.problem(B=2, Lq=2048, Lkv=100, Hq=4, Hkv=1, d=64, m=4, W=8, topk=8, Hi=2, di=32, Nc=65535)
    assert hb.hyb_workspace_size(p) == 0
    p = hb.problem(B=1, Lq=32768, Lkv=32768, Hq=32, Hkv=1, d=128, m=4, W=128, topk=512, Hi=4, di=64,
                   Nc=8192)
    assert hb.hyb_workspace_size(p) == 0
    # ... otherwise the scores of every (query row, entry) pair, fp32, 256-byte rounded:
    # shapes the one kernel does not take, and smaller ones, which the two kernels finish first
    for lq, hi, nc in ((63, 2, 25), (100, 5, 25), (100, 2, 65536), (100, 2, 25), (16384, 4, 4096)):
        p = hb.problem(B=2 if lq < 16384 else 1, Lq=lq, Lkv=100, Hq=4, Hkv=1, d=64, m=4, W=8, topk=8, Hi=hi,
                       di=32, Nc=nc)
        assert hb.hyb_workspace_size(p) == (p.B * lq * nc * 4 + 255) // 256 * 256
    p.topk = 0
    assert hb.hyb_workspace_size(p) == 0
    # missing workspace is reported as such
    p = hb.problem(B=1, Lq=8, Lkv=8, Hq=4, Hkv=1, d=64, m=4, W=8, topk=4, Hi=2, di=32, Nc=2)
    buf = ctypes.c_void_p(256)
    st = hb._lib.hyb_csa_index_topk(ctypes.byref(p), buf, buf, buf, buf, None, None, 0, None)
    assert st == hb.HYB_ERR_WORKSPACE
    # the gather probes: null buffers, too few rows, stage counts outside 2..6
    for fn in (hb._lib.hyb_probe_l2_gather, hb._lib.hyb_probe_l2_gather_tma):
        assert fn(None, 1 << 20, 1024, 3, buf, None) == hb.HYB_ERR_INVALID_ARG
        assert fn(buf, 1 << 20, 1024, 3, None, None) == hb.HYB_ERR_INVALID_ARG
        assert fn(buf, 1 << 20, 64, 3, buf, None) == hb.HYB_ERR_INVALID_ARG
        assert fn(buf, 1 << 20, 1024, 7, buf, None) == hb.HYB_ERR_INVALID_ARG
        assert fn(buf, 1 << 20, 1024, 1, buf, None) == hb.HYB_ERR_INVALID_ARG


def test_decode_append_argument_checks(lib):
    import compressed_sparse_sliding_b200 as hb
    buf = ctypes.c_void_p(256)
    args = [buf] * 14 + [None]
    # the ring must hold 2W rows
    p = hb.problem(B=1, Lq=1, Lkv=8, Hq=4, Hkv=1, d=64, m=4, W=8, Nc=16)
    assert hb._lib.hyb_decode_append(ctypes.byref(p), *args) == hb.HYB_ERR_INVALID_ARG
    # a block longer than the window cannot be merged from the ring
    p = hb.problem(B=1, Lq=1, Lkv=16, Hq=4, Hkv=1, d=64, m=16, W=8, Nc=16)
    assert hb._lib.hyb_decode_append(ctypes.byref(p), *args) == hb.HYB_ERR_UNSUPPORTED
    # CSA needs the indexer-key ring and cache
    p = hb.problem(B=1, Lq=1, Lkv=16, Hq=4, Hkv=1, d=64, m=4, W=8, Nc=16, topk=4, Hi=2, di=32)
    a = [buf] * 3 + [None] + [buf] * 11 + [None]
    assert hb._lib.hyb_decode_append(ctypes.byref(p), *a) == hb.HYB_ERR_INVALID_ARG


def test_gated_argument_checks(lib):
    import compressed_sparse_sliding_b200 as hb
    buf = ctypes.c_void_p(256)
    p = hb.problem(B=1, Lq=16, Lkv=16, Hq=4, Hkv=1, d=64, m=4, W=8, topk=4, Nc=4)
    # the selection branch needs idx
    assert hb._lib.hyb_gated_fwd(ctypes.byref(p), buf, buf, buf, None, buf, buf, buf, buf, buf,
                                 1 << 20, None) == hb.HYB_ERR_INVALID_ARG
    # workspace: three bf16 branch outputs, each 256-byte rounded
    assert hb._lib.hyb_gated_workspace_size(ctypes.byref(p)) == 3 * ((16 * 4 * 64 * 2 + 255) // 256 * 256)
    assert hb._lib.hyb_gated_fwd(ctypes.byref(p), buf, buf, buf, buf, buf, buf, buf, buf, None, 0,
                                 None) == hb.HYB_ERR_WORKSPACE


def test_fp4_argument_checks(lib):
    import compressed_sparse_sliding_b200 as hb
    buf = ctypes.c_void_p(256)
    # row widths the quantizer handles: 64, 128, 256 channels
    assert hb._lib.hyb_fp4_quantize(buf, 4, 96, buf, buf, None) == hb.HYB_ERR_UNSUPPORTED
    assert hb._lib.hyb_fp4_quantize(None, 4, 64, buf, buf, None) == hb.HYB_ERR_INVALID_ARG
    assert hb._lib.hyb_fp4_dequantize(buf, buf, 4, 12, buf, None) == hb.HYB_ERR_INVALID_ARG
    # decode (Lq * topk < Nc): workspace = the selected K rows, then V rows, bf16
    p = hb.problem(B=2, Lq=1, Lkv=256, Hq=64, Hkv=1, d=128, m=4, W=128, topk=64, Hi=4, di=64, Nc=512)
    attn = 2 * ((2 * 64 * 128 * 2 + 255) // 256 * 256)
    index = (2 * 1 * 512 * 4 + 255) // 256 * 256          # scores; keys dequantized on chip
    assert hb.hyb_fp4_workspace_size(p) == max(attn, index)
    # prefill: the whole caches are dequantized
    p = hb.problem(B=1, Lq=64, Lkv=64, Hq=4, Hkv=1, d=64, m=4, W=8, topk=4, Hi=2, di=32, Nc=16)
    attn = 2 * ((16 * 64 * 2 + 255) // 256 * 256)
    # keys dequantized once, plus the score rows (small problems select from stored rows)
    index = (64 * 16 * 4 + 255) // 256 * 256 + (16 * 32 * 2 + 255) // 256 * 256
    assert hb.hyb_fp4_workspace_size(p) == max(attn, index)
    p.Hi = 5                                     # a shape only the two-kernel path takes: the same
    assert hb.hyb_fp4_workspace_size(p) == max(attn, index)
    p.Hi = 2
    assert hb._lib.hyb_attn_fwd_fp4(ctypes.byref(p), *([buf] * 10), None, 0, None) == hb.HYB_ERR_WORKSPACE
    assert hb._lib.hyb_csa_index_topk_fp4(ctypes.byref(p), *([buf] * 5), None, None, 0,
                                          None) == hb.HYB_ERR_WORKSPACE
    # the append shares the checks of hyb_decode_append
    p = hb.problem(B=1, Lq=1, Lkv=8, Hq=4, Hkv=1, d=64, m=4, W=8, Nc=16)
    assert hb._lib.hyb_decode_append_fp4(ctypes.byref(p), *([buf] * 17), None) == hb.HYB_ERR_INVALID_ARG


def test_backward_argument_checks(lib):
    import compressed_sparse_sliding_b200 as hb
    buf = ctypes.c_void_p(256)
    p = hb.problem(B=1, Lq=16, Lkv=16, Hq=4, Hkv=1, d=64, m=4, W=8, Nc=4)
    # lse is required (P is recomputed from it)
    args = [buf] * 7 + [None] + [buf] * 6 + [None]
    assert hb._lib.hyb_attn_bwd(ctypes.byref(p), *args) == hb.HYB_ERR_INVALID_ARG
    # block_merge backward: channels in multiples of 32, a G buffer of m * dx floats
    assert hb._lib.hyb_hca_compress_bwd_workspace_size(64, 4) == 1024
    assert hb._lib.hyb_hca_compress_bwd(buf, 1, 8, 1, 48, 4, buf, buf, buf, buf, buf, 1024,
                                        None) == hb.HYB_ERR_UNSUPPORTED
    assert hb._lib.hyb_hca_compress_bwd(buf, 1, 8, 1, 64, 4, buf, buf, buf, buf, buf, 512,
                                        None) == hb.HYB_ERR_WORKSPACE


def test_backward_rejects_misaligned_rows(lib):
    # the backward's kernels move 16-byte pieces of every row: a pointer off
    # that grid is refused on the host, before anything is launched
    import compressed_sparse_sliding_b200 as hb
    p = hb.problem(B=1, Lq=256, Lkv=256, Hq=2, Hkv=1, d=128, m=4, W=128, Nc=64)
    ok, bad = ctypes.c_void_p(256), ctypes.c_void_p(256 + 8)
    args = [ok] * 15   # q kc vc idx k v o lse dout dq dkc dvc dk dv stream
    args[3] = None     # dense: no selection
    args[14] = None    # default stream
    for i in (0, 1, 4, 6, 8, 9, 10, 12):
        a = list(args)
        a[i] = bad
        assert hb._lib.hyb_attn_bwd(ctypes.byref(p), *a) == hb.HYB_ERR_INVALID_ARG, i
