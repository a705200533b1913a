"""B200 (sm_100a) hybrid compressed / sparse / sliding-window attention.

Thin ctypes binding over ``libhybattn.so`` (C ABI in ``include/hybattn.h``).
Every step of the forward pass runs in the library's CUDA kernels; this module
only marshals arguments: it takes device tensors, passes their data pointers
and the current CUDA stream, and allocates outputs with torch.  There is no
CPU or PyTorch fallback: importing fails loudly when the library is missing.

Entry points (same names as the C ABI):
  hyb_hca_compress     block_merge of raw K / V / indexer keys
  hyb_csa_index_topk   lightning-indexer scores + exact per-query top-K
  hyb_attn_fwd         one softmax over compressed (selected / all visible)
                       keys and the raw sliding window
  hyb_fused_fwd        the three stages on one stream
  hyb_decode_append    decode cache maintenance: window ring + compressed entries
  hyb_gated_fwd        the gated three-branch variant (compressed, selected, window)
  hyb_fp4_*            4-bit compressed caches: quantize / dequantize, and the
                       indexer, attention and decode append over them
  hyb_attn_bwd,        gradients for training: through the attention (fixed
  hyb_hca_compress_bwd selection) and through block_merge
  hyb_workspace_size, hyb_get_device_status, hyb_error_string
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhybattn.so")

_BUILD_HINT = ("build it with `python compressed_sparse_sliding_b200/build.py` (nvcc, sm_100a). "
               "There is no fallback implementation.")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: {_BUILD_HINT}")

_lib = ctypes.CDLL(LIB_PATH)

HYB_OK = 0
HYB_ERR_INVALID_ARG = -1
HYB_ERR_UNSUPPORTED = -2
HYB_ERR_WORKSPACE = -3
HYB_ERR_CUDA = -4
HYB_ERR_DEVICE_TIMEOUT = -5
HYB_ERR_DEVICE_BOUNDS = -6


class HybProblem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("Lq", ctypes.c_int), ("Lkv", ctypes.c_int),
        ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
        ("m", ctypes.c_int), ("W", ctypes.c_int), ("topk", ctypes.c_int),
        ("Hi", ctypes.c_int), ("di", ctypes.c_int), ("Nc", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("q_pos", ctypes.c_void_p), ("kv_pos0", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int
_PP = ctypes.POINTER(HybProblem)
try:
    _lib.hyb_workspace_size.argtypes = [_PP]
    _lib.hyb_workspace_size.restype = ctypes.c_size_t
    _lib.hyb_hca_compress.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P, _P]
    _lib.hyb_hca_compress.restype = _I
    _lib.hyb_csa_index_topk.argtypes = [_PP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    _lib.hyb_csa_index_topk.restype = _I
    _lib.hyb_attn_fwd.argtypes = [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P]
    _lib.hyb_attn_fwd.restype = _I
    _lib.hyb_fused_fwd.argtypes = [_PP] + [_P] * 16 + [ctypes.c_size_t, _P]
    _lib.hyb_fused_fwd.restype = _I
    _lib.hyb_decode_append.argtypes = [_PP] + [_P] * 15
    _lib.hyb_decode_append.restype = _I
    _lib.hyb_gated_workspace_size.argtypes = [_PP]
    _lib.hyb_gated_workspace_size.restype = ctypes.c_size_t
    _lib.hyb_gated_fwd.argtypes = [_PP] + [_P] * 9 + [ctypes.c_size_t, _P]
    _lib.hyb_gated_fwd.restype = _I
    _lib.hyb_fp4_quantize.argtypes = [_P, ctypes.c_longlong, _I, _P, _P, _P]
    _lib.hyb_fp4_quantize.restype = _I
    _lib.hyb_fp4_dequantize.argtypes = [_P, _P, ctypes.c_longlong, _I, _P, _P]
    _lib.hyb_fp4_dequantize.restype = _I
    _lib.hyb_fp4_workspace_size.argtypes = [_PP]
    _lib.hyb_fp4_workspace_size.restype = ctypes.c_size_t
    _lib.hyb_csa_index_topk_fp4.argtypes = [_PP] + [_P] * 7 + [ctypes.c_size_t, _P]
    _lib.hyb_csa_index_topk_fp4.restype = _I
    _lib.hyb_attn_fwd_fp4.argtypes = [_PP] + [_P] * 11 + [ctypes.c_size_t, _P]
    _lib.hyb_attn_fwd_fp4.restype = _I
    _lib.hyb_decode_append_fp4.argtypes = [_PP] + [_P] * 18
    _lib.hyb_decode_append_fp4.restype = _I
    _lib.hyb_attn_bwd.argtypes = [_PP] + [_P] * 15
    _lib.hyb_attn_bwd.restype = _I
    _lib.hyb_hca_compress_bwd_workspace_size.argtypes = [_I, _I]
    _lib.hyb_hca_compress_bwd_workspace_size.restype = ctypes.c_size_t
    _lib.hyb_hca_compress_bwd.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    _lib.hyb_hca_compress_bwd.restype = _I
    _lib.hyb_get_device_status.argtypes = [_P]
    _lib.hyb_get_device_status.restype = _I
    _lib.hyb_error_string.argtypes = [_I]
    _lib.hyb_error_string.restype = ctypes.c_char_p
    _lib.hyb_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    _lib.hyb_set_wait_limit_ns.restype = _I
    _lib.hyb_trace_attach.argtypes = [_P, ctypes.c_size_t]
    _lib.hyb_trace_attach.restype = _I
    _lib.hyb_probe_l2_gather.argtypes = [_P, ctypes.c_longlong, ctypes.c_longlong, _I, _P, _P]
    _lib.hyb_probe_l2_gather.restype = _I
    _lib.hyb_probe_l2_gather_tma.argtypes = [_P, ctypes.c_longlong, ctypes.c_longlong, _I, _P, _P]
    _lib.hyb_probe_l2_gather_tma.restype = _I
except AttributeError as exc:   # a library built from older sources
    raise ImportError(f"{LIB_PATH} lacks an entry point ({exc}); rebuild: {_BUILD_HINT}") from exc


class HybError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {hyb_error_string(status)} ({status})")


def hyb_error_string(status: int) -> str:
    return _lib.hyb_error_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != HYB_OK:
        raise HybError(status, where)


def problem(B, Lq, Lkv, Hq, Hkv, d, m, W, topk=0, Hi=0, di=0, Nc=0, scale=0.0, q_pos=None,
            kv_pos0=None) -> HybProblem:
    """Builds the C problem struct; q_pos / kv_pos0 are int32 device tensors or None."""
    p = HybProblem(B, Lq, Lkv, Hq, Hkv, d, m, W, topk, Hi, di, Nc, float(scale), None, None)
    p.q_pos = None if q_pos is None else q_pos.data_ptr()
    p.kv_pos0 = None if kv_pos0 is None else kv_pos0.data_ptr()
    p._keep = (q_pos, kv_pos0)
    return p


def hyb_workspace_size(p: HybProblem) -> int:
    return int(_lib.hyb_workspace_size(ctypes.byref(p)))


def hyb_hca_compress(x: torch.Tensor, w: torch.Tensor, m: int, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """x [B, L, H, dx] (or [B, L, dx]) bf16, w [m, dx] fp32 -> [B, L//m, H, dx] bf16."""
    squeeze = x.dim() == 3
    xv = x.unsqueeze(2) if squeeze else x
    B, L, H, dx = xv.shape
    if out is None:
        out = torch.empty((B, L // m, H, dx), dtype=torch.bfloat16, device=x.device)
    st = _lib.hyb_hca_compress(_ptr(xv), B, L, H, dx, m, _ptr(w), _ptr(out), _stream(stream))
    _check(st, "hyb_hca_compress")
    return out.squeeze(2) if squeeze and out.dim() == 4 else out


def hyb_csa_index_topk(p: HybProblem, qi, wi, kic, idx=None, sel_scores=None, ws=None,
                       stream=None, ws_bytes: Optional[int] = None):
    """Top-K entry indices [B, Lq, topk] int32 (ascending, -1 padded).
    ws_bytes: the workspace bytes to declare (default: all of ws, which is
    allocated at hyb_workspace_size(p) when absent or short); 0 passes none,
    which runs the one-kernel path on the shapes it takes."""
    if idx is None:
        idx = torch.empty((p.B, p.Lq, p.topk), dtype=torch.int32, device=qi.device)
    if ws_bytes == 0:
        ws = None
    else:
        need = hyb_workspace_size(p)
        if ws is None or ws.numel() < need:
            ws = torch.empty(max(need, 256), dtype=torch.uint8, device=qi.device)
        ws_bytes = ws.numel() if ws_bytes is None else min(int(ws_bytes), ws.numel())
    st = _lib.hyb_csa_index_topk(ctypes.byref(p), _ptr(qi), _ptr(wi), _ptr(kic), _ptr(idx),
                                 _ptr(sel_scores), _ptr(ws), ws_bytes, _stream(stream))
    _check(st, "hyb_csa_index_topk")
    return idx


def hyb_attn_fwd(p: HybProblem, q, kc, vc, idx, k_raw, v_raw, o=None, lse=None, stream=None):
    """o [B, Lq, Hq, d] bf16 (and lse [B, Hq, Lq] fp32 when given)."""
    if o is None:
        o = torch.empty((p.B, p.Lq, p.Hq, p.d), dtype=torch.bfloat16, device=q.device)
    st = _lib.hyb_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(kc), _ptr(vc), _ptr(idx), _ptr(k_raw),
                           _ptr(v_raw), _ptr(o), _ptr(lse), _stream(stream))
    _check(st, "hyb_attn_fwd")
    return o


def hyb_fused_fwd(p: HybProblem, q, k_raw, v_raw, wk=None, wv=None, qi=None, wi=None, ki_raw=None,
                  wib=None, kc=None, vc=None, kic=None, idx=None, o=None, lse=None, ws=None,
                  stream=None):
    """Whole forward pass.  Returns dict(o, kc, vc, kic, idx)."""
    dev = q.device
    if kc is None:
        kc = torch.empty((p.B, p.Nc, p.Hkv, p.d), dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
    if p.topk > 0:
        if kic is None:
            kic = torch.empty((p.B, p.Nc, p.di), dtype=torch.bfloat16, device=dev)
        if idx is None:
            idx = torch.empty((p.B, p.Lq, p.topk), dtype=torch.int32, device=dev)
    if o is None:
        o = torch.empty((p.B, p.Lq, p.Hq, p.d), dtype=torch.bfloat16, device=dev)
    need = hyb_workspace_size(p)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    st = _lib.hyb_fused_fwd(ctypes.byref(p), _ptr(q), _ptr(k_raw), _ptr(v_raw), _ptr(wk), _ptr(wv),
                            _ptr(qi), _ptr(wi), _ptr(ki_raw), _ptr(wib), _ptr(kc), _ptr(vc),
                            _ptr(kic), _ptr(idx), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                            _stream(stream))
    _check(st, "hyb_fused_fwd")
    return dict(o=o, kc=kc, vc=vc, kic=kic, idx=idx)


def hyb_decode_append(p: HybProblem, t_new, k_new, v_new, k_ring, v_ring, kc, vc, wk, wv,
                      ki_new=None, wib=None, ki_ring=None, kic=None, kv_pos0=None, stream=None):
    """Appends one token per sequence: t_new [B] int32, k_new/v_new [B, Hkv, d],
    ki_new [B, di] (CSA); rings k_ring/v_ring [B, 2W, Hkv, d], ki_ring [B, W, di];
    caches kc/vc [B, Nc, Hkv, d], kic [B, Nc, di] updated in place.  Returns the
    kv_pos0 [B] int32 tensor to pass to the attention call (Lkv = 2W)."""
    if kv_pos0 is None:
        kv_pos0 = torch.empty((p.B,), dtype=torch.int32, device=k_new.device)
    st = _lib.hyb_decode_append(ctypes.byref(p), _ptr(t_new), _ptr(k_new), _ptr(v_new), _ptr(ki_new),
                                _ptr(wk), _ptr(wv), _ptr(wib), _ptr(k_ring), _ptr(v_ring),
                                _ptr(ki_ring), _ptr(kc), _ptr(vc), _ptr(kic), _ptr(kv_pos0),
                                _stream(stream))
    _check(st, "hyb_decode_append")
    return kv_pos0


class Fp4Cache:
    """A 4-bit cache: codes [..., dx/2] uint8 and qp [..., 2] fp32 (min, scale) per row."""

    def __init__(self, codes: torch.Tensor, qp: torch.Tensor):
        self.codes = codes
        self.qp = qp

    @staticmethod
    def empty(shape, device):
        """Storage for a cache of bf16 shape [..., dx]."""
        *lead, dx = shape
        return Fp4Cache(torch.zeros((*lead, dx // 2), dtype=torch.uint8, device=device),
                        torch.zeros((*lead, 2), dtype=torch.float32, device=device))


def hyb_fp4_quantize(x: torch.Tensor, out: Optional[Fp4Cache] = None, stream=None) -> Fp4Cache:
    """Per-row 4-bit min/max quantization of a bf16 tensor [..., dx]."""
    if out is None:
        out = Fp4Cache.empty(tuple(x.shape), x.device)
    rows = x.numel() // x.shape[-1]
    st = _lib.hyb_fp4_quantize(_ptr(x), rows, x.shape[-1], _ptr(out.codes), _ptr(out.qp), _stream(stream))
    _check(st, "hyb_fp4_quantize")
    return out


def hyb_fp4_dequantize(c: Fp4Cache, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bf16 values [..., dx] of a 4-bit cache."""
    dx = 2 * c.codes.shape[-1]
    if out is None:
        out = torch.empty((*c.codes.shape[:-1], dx), dtype=torch.bfloat16, device=c.codes.device)
    rows = c.codes.numel() // c.codes.shape[-1]
    st = _lib.hyb_fp4_dequantize(_ptr(c.codes), _ptr(c.qp), rows, dx, _ptr(out), _stream(stream))
    _check(st, "hyb_fp4_dequantize")
    return out


def hyb_fp4_workspace_size(p: HybProblem) -> int:
    return int(_lib.hyb_fp4_workspace_size(ctypes.byref(p)))


def _fp4_ws(p, ws, device):
    need = max(hyb_fp4_workspace_size(p), 256)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws


def hyb_csa_index_topk_fp4(p: HybProblem, qi, wi, kic: Fp4Cache, idx=None, sel_scores=None, ws=None,
                           stream=None):
    """hyb_csa_index_topk over a 4-bit indexer-key cache [B, Nc, di]."""
    if idx is None:
        idx = torch.empty((p.B, p.Lq, p.topk), dtype=torch.int32, device=qi.device)
    ws = _fp4_ws(p, ws, qi.device)
    st = _lib.hyb_csa_index_topk_fp4(ctypes.byref(p), _ptr(qi), _ptr(wi), _ptr(kic.codes), _ptr(kic.qp),
                                     _ptr(idx), _ptr(sel_scores), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "hyb_csa_index_topk_fp4")
    return idx


def hyb_attn_fwd_fp4(p: HybProblem, q, kc: Fp4Cache, vc: Fp4Cache, idx, k_raw, v_raw, o=None, lse=None,
                     ws=None, stream=None):
    """hyb_attn_fwd over 4-bit K / V caches [B, Nc, Hkv, d]."""
    if o is None:
        o = torch.empty((p.B, p.Lq, p.Hq, p.d), dtype=torch.bfloat16, device=q.device)
    ws = _fp4_ws(p, ws, q.device)
    st = _lib.hyb_attn_fwd_fp4(ctypes.byref(p), _ptr(q), _ptr(kc.codes), _ptr(kc.qp), _ptr(vc.codes),
                               _ptr(vc.qp), _ptr(idx), _ptr(k_raw), _ptr(v_raw), _ptr(o), _ptr(lse),
                               _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "hyb_attn_fwd_fp4")
    return o


def hyb_decode_append_fp4(p: HybProblem, t_new, k_new, v_new, k_ring, v_ring, kc: Fp4Cache, vc: Fp4Cache,
                          wk, wv, ki_new=None, wib=None, ki_ring=None, kic: Optional[Fp4Cache] = None,
                          kv_pos0=None, stream=None):
    """hyb_decode_append with 4-bit caches (entries quantized as they close)."""
    if kv_pos0 is None:
        kv_pos0 = torch.empty((p.B,), dtype=torch.int32, device=k_new.device)
    st = _lib.hyb_decode_append_fp4(ctypes.byref(p), _ptr(t_new), _ptr(k_new), _ptr(v_new), _ptr(ki_new),
                                    _ptr(wk), _ptr(wv), _ptr(wib), _ptr(k_ring), _ptr(v_ring), _ptr(ki_ring),
                                    _ptr(kc.codes), _ptr(kc.qp), _ptr(vc.codes), _ptr(vc.qp),
                                    _ptr(kic.codes if kic is not None else None),
                                    _ptr(kic.qp if kic is not None else None), _ptr(kv_pos0),
                                    _stream(stream))
    _check(st, "hyb_decode_append_fp4")
    return kv_pos0


def hyb_attn_bwd(p: HybProblem, q, kc, vc, idx, k_raw, v_raw, o, lse, dout, stream=None):
    """Gradients of sum(dout * o) through hyb_attn_fwd (o, lse: its outputs;
    the selection idx is taken as fixed).  Returns dict(dq, dkc, dvc, dk_raw,
    dv_raw), fp32 tensors shaped like q, kc, vc, k_raw, v_raw."""
    f32 = dict(dtype=torch.float32, device=q.device)
    g = dict(dq=torch.empty(q.shape, **f32), dk_raw=torch.empty(k_raw.shape, **f32),
             dv_raw=torch.empty(v_raw.shape, **f32),
             dkc=torch.empty(kc.shape, **f32) if kc is not None else None,
             dvc=torch.empty(vc.shape, **f32) if vc is not None else None)
    st = _lib.hyb_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(kc), _ptr(vc), _ptr(idx), _ptr(k_raw), _ptr(v_raw),
                           _ptr(o), _ptr(lse), _ptr(dout), _ptr(g["dq"]), _ptr(g["dkc"]), _ptr(g["dvc"]),
                           _ptr(g["dk_raw"]), _ptr(g["dv_raw"]), _stream(stream))
    _check(st, "hyb_attn_bwd")
    return g


def hyb_hca_compress_bwd(x: torch.Tensor, w: torch.Tensor, m: int, dc: torch.Tensor,
                         dx: Optional[torch.Tensor] = None, dw: Optional[torch.Tensor] = None,
                         ws: Optional[torch.Tensor] = None, stream=None):
    """Gradients of sum(dc * hyb_hca_compress(x, w, m)): adds the x gradient
    into dx (fp32, zero-initialised when not given) and returns (dx, dw)."""
    B, L, H, D = x.shape if x.dim() == 4 else (x.shape[0], x.shape[1], 1, x.shape[2])
    if dx is None:
        dx = torch.zeros(x.shape, dtype=torch.float32, device=x.device)
    if dw is None:
        dw = torch.empty((m, D), dtype=torch.float32, device=x.device)
    need = max(int(_lib.hyb_hca_compress_bwd_workspace_size(D, m)), 256)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=x.device)
    st = _lib.hyb_hca_compress_bwd(_ptr(x), B, L, H, D, m, _ptr(w), _ptr(dc), _ptr(dx), _ptr(dw), _ptr(ws),
                                   ws.numel(), _stream(stream))
    _check(st, "hyb_hca_compress_bwd")
    return dx, dw


def hyb_gated_workspace_size(p: HybProblem) -> int:
    return int(_lib.hyb_gated_workspace_size(ctypes.byref(p)))


def hyb_gated_fwd(p: HybProblem, q, kc, vc, idx, k_raw, v_raw, gate, o=None, ws=None, stream=None):
    """Gated three-branch attention; gate [B, Lq, Hq, 3] fp32 logits."""
    if o is None:
        o = torch.empty((p.B, p.Lq, p.Hq, p.d), dtype=torch.bfloat16, device=q.device)
    need = int(_lib.hyb_gated_workspace_size(ctypes.byref(p)))
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = _lib.hyb_gated_fwd(ctypes.byref(p), _ptr(q), _ptr(kc), _ptr(vc), _ptr(idx), _ptr(k_raw),
                            _ptr(v_raw), _ptr(gate), _ptr(o), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "hyb_gated_fwd")
    return o


def hyb_get_device_status(stream=None) -> int:
    return int(_lib.hyb_get_device_status(_stream(stream)))


# ---------------------------------------------------------------- timeline
TRACE_ROLES = {1: "gather", 2: "mma", 3: "softmax"}


def hyb_trace_attach(buf: Optional[torch.Tensor]) -> None:
    """Attach (or, with None, detach) a device buffer for the per-role timeline
    of CTA 0 of the kernels that record one (see hyb_trace_attach in the C
    header).  The record counts in the buffer's first four words are cleared
    here."""
    if buf is None:
        st = _lib.hyb_trace_attach(None, 0)
    else:
        if buf.device.type != "cuda" or not buf.is_contiguous():
            raise ValueError("trace buffer: a contiguous CUDA tensor")
        buf.view(torch.uint8)[:32].zero_()
        st = _lib.hyb_trace_attach(_ptr(buf), buf.numel() * buf.element_size())
    if st != HYB_OK:
        raise HybError(st, "hyb_trace_attach")


def trace_records(buf: torch.Tensor):
    """The records of an attached buffer as a list of dicts (clock, role,
    event, item, tile), all roles merged in clock order."""
    words = buf.view(torch.int64).cpu().numpy().view("uint64")
    cap = (words.size - 4) // 8
    out = []
    for role in range(4):
        n = min(int(words[role] & 0xFFFFFFFF), cap)
        base = 4 + 2 * role * cap
        for r in range(n):
            clk, tag = int(words[base + 2 * r]), int(words[base + 2 * r + 1])
            out.append(dict(clock=clk, role=tag >> 56, event=(tag >> 48) & 0xFF,
                            item=(tag >> 16) & 0xFFFFFFFF, tile=tag & 0xFFFF))
    out.sort(key=lambda d: d["clock"])
    return out


def hyb_probe_l2_gather(table: torch.Tensor, rows_per_sm: int, stages: int, sink: torch.Tensor,
                        stream=None) -> None:
    """One launch of the L2-resident random-row gather probe (see the C header)."""
    st = _lib.hyb_probe_l2_gather(_ptr(table), table.numel() * table.element_size(), int(rows_per_sm),
                                  int(stages), _ptr(sink), _stream(stream))
    if st != HYB_OK:
        raise HybError(st, "hyb_probe_l2_gather")


def hyb_probe_l2_gather_tma(table: torch.Tensor, rows_per_sm: int, stages: int, sink: torch.Tensor,
                            stream=None) -> None:
    """The same probe with tile::gather4 copies; sink holds 257 words, sink[256]
    counting misplaced 16-byte chunks (see the C header)."""
    if sink.numel() * sink.element_size() < 257 * 4:
        raise ValueError("sink must hold 257 uint32 words")
    st = _lib.hyb_probe_l2_gather_tma(_ptr(table), table.numel() * table.element_size(), int(rows_per_sm),
                                      int(stages), _ptr(sink), _stream(stream))
    if st != HYB_OK:
        raise HybError(st, "hyb_probe_l2_gather_tma")


def hyb_set_wait_limit_ns(ns: int) -> None:
    """Bound of the kernels' waits for later launches (0: the default 200 ms)."""
    st = _lib.hyb_set_wait_limit_ns(int(ns))
    if st != HYB_OK:
        raise HybError(st, "hyb_set_wait_limit_ns")
