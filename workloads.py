"""Seeded synthetic workloads for hybrid compressed/sparse/sliding attention.

This module only draws random inputs with the shapes, dtypes and value
distributions of the five workloads the method is measured on.  It holds none
of the method's arithmetic (no compression, visibility, scoring or attention):
both the CPU oracle and the CUDA path consume what it produces, and neither
imports the other.

Workloads (sizes as the method's description gives them):
  1 csa_swa_tiny      CSA+SWA, B=1, L=1024, 4 query heads / 1 KV head, d=64,
                      m=4, top-K=16, W=128, indexer 2 heads x 32
  2 hca_swa           HCA+SWA, B=2, L=8192, 16/16 heads, d=128, m=128, W=128
  3 csa_swa_prefill   CSA+SWA, B=1, L=32768, 32/1 heads (MQA), d=128, m=4,
                      top-K=512, W=128, indexer 4 heads x 64
  4 hca_swa_long      HCA+SWA, B=1, L=131072, 64/8 heads (GQA), d=128, m=128,
                      W=128, inputs N(0,1) scaled by 0.5
  5 csa_swa_decode    64 sequences x 1 query token at position 65535, caches of
                      16384 compressed entries (m=4), 128 raw window rows,
                      64/1 heads, d=128, top-K=1024, indexer 4 heads x 64

Distributions: q, k, v, indexer queries/keys ~ N(0,1) (config 4: x0.5) drawn in
fp32 and rounded to bf16; block weights ~ N(0,1) fp32 of shape [m, d]; indexer
head weights ~ U(0,1) fp32 per query token and head.  Seeds are 20260 + config.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    no: int
    name: str
    mode: str            # "csa" | "hca" | "csa_decode"
    B: int
    L: int               # prefill: tokens per sequence; decode: context length
    Hq: int
    Hkv: int
    d: int
    m: int
    W: int
    topk: int = 0        # 0 => HCA dense over all visible compressed entries
    Hi: int = 0
    di: int = 0
    input_scale: float = 1.0
    Nc_cache: int = 0    # decode: compressed-cache capacity per sequence

    @property
    def is_decode(self) -> bool:
        return self.mode == "csa_decode"

    @property
    def Lq(self) -> int:
        return 1 if self.is_decode else self.L

    @property
    def Lkv(self) -> int:
        return self.W if self.is_decode else self.L

    @property
    def Nc(self) -> int:
        return self.Nc_cache if self.is_decode else self.L // self.m

    def describe(self) -> str:
        s = (f"{self.name}: B={self.B} L={self.L} Hq={self.Hq} Hkv={self.Hkv} d={self.d} "
             f"m={self.m} W={self.W}")
        if self.topk:
            s += f" topk={self.topk} Hi={self.Hi} di={self.di}"
        return s


WORKLOADS: Dict[int, Workload] = {
    1: Workload(1, "csa_swa_tiny", "csa", B=1, L=1024, Hq=4, Hkv=1, d=64, m=4, W=128,
                topk=16, Hi=2, di=32),
    2: Workload(2, "hca_swa", "hca", B=2, L=8192, Hq=16, Hkv=16, d=128, m=128, W=128),
    3: Workload(3, "csa_swa_prefill", "csa", B=1, L=32768, Hq=32, Hkv=1, d=128, m=4, W=128,
                topk=512, Hi=4, di=64),
    4: Workload(4, "hca_swa_long", "hca", B=1, L=131072, Hq=64, Hkv=8, d=128, m=128, W=128,
                input_scale=0.5),
    5: Workload(5, "csa_swa_decode", "csa_decode", B=64, L=65536, Hq=64, Hkv=1, d=128, m=4,
                W=128, topk=1024, Hi=4, di=64, Nc_cache=16384),
}


def custom(**kw) -> Workload:
    """A workload with explicit sizes (used for small parity cases)."""
    base = dict(no=0, name="custom", mode="csa", B=1, L=256, Hq=4, Hkv=1, d=64, m=4, W=32)
    base.update(kw)
    return Workload(**base)


def _normal_bf16(gen: torch.Generator, shape, scale: float, device) -> torch.Tensor:
    """N(0,1)*scale drawn in fp32 in chunks, rounded to bf16."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    chunk = 1 << 26
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        t = torch.randn(e - s, generator=gen, dtype=torch.float32, device=device)
        if scale != 1.0:
            t.mul_(scale)
        flat[s:e].copy_(t)
    return out


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw one batch of inputs for workload `w` on `device`.

    Prefill workloads return raw q/k/v, block weights wk/wv and (CSA) indexer
    queries qi, head weights wi, raw indexer keys ki and their block weight wib.
    The decode workload returns ready caches (kc, vc, kic), the raw window
    rows (k_raw, v_raw) and the query-side tensors, plus positions.
    """
    if seed is None:
        seed = 20260 + w.no
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    sc = w.input_scale
    t: Dict[str, torch.Tensor] = {}
    B, Hq, Hkv, d = w.B, w.Hq, w.Hkv, w.d
    t["q"] = _normal_bf16(gen, (B, w.Lq, Hq, d), sc, device)
    if w.is_decode:
        Nc = w.Nc
        t["kc"] = _normal_bf16(gen, (B, Nc, Hkv, d), sc, device)
        t["vc"] = _normal_bf16(gen, (B, Nc, Hkv, d), sc, device)
        t["k_raw"] = _normal_bf16(gen, (B, w.W, Hkv, d), sc, device)
        t["v_raw"] = _normal_bf16(gen, (B, w.W, Hkv, d), sc, device)
        t["qi"] = _normal_bf16(gen, (B, 1, w.Hi, w.di), sc, device)
        t["wi"] = torch.rand((B, 1, w.Hi), generator=gen, dtype=torch.float32, device=device)
        t["kic"] = _normal_bf16(gen, (B, Nc, w.di), sc, device)
        t["q_pos"] = torch.full((B, 1), w.L - 1, dtype=torch.int32, device=device)
        t["kv_pos0"] = torch.full((B,), w.L - w.W, dtype=torch.int32, device=device)
        # decode step with cache maintenance: the new token is position L - 1
        # (its K / V rows are the window's last rows); the window's rows sit in
        # a 2W-row ring at rows p mod W and p mod W + W; block weights and the
        # window's indexer keys are drawn after everything above, so the
        # tensors above do not change
        W = w.W
        pos = torch.arange(w.L - W, w.L, device=device)
        slot = pos % W
        for name, raw in (("k_ring", t["k_raw"]), ("v_ring", t["v_raw"])):
            ring = torch.zeros((B, 2 * W, Hkv, d), dtype=torch.bfloat16, device=device)
            ring[:, slot] = raw
            ring[:, slot + W] = raw
            t[name] = ring
        t["k_new"] = t["k_raw"][:, W - 1].contiguous()
        t["v_new"] = t["v_raw"][:, W - 1].contiguous()
        t["t_new"] = torch.full((B,), w.L - 1, dtype=torch.int32, device=device)
        t["wk"] = torch.randn((w.m, d), generator=gen, dtype=torch.float32, device=device)
        t["wv"] = torch.randn((w.m, d), generator=gen, dtype=torch.float32, device=device)
        t["wib"] = torch.randn((w.m, w.di), generator=gen, dtype=torch.float32, device=device)
        ki_win = _normal_bf16(gen, (B, W, w.di), sc, device)
        t["ki_ring"] = torch.zeros((B, W, w.di), dtype=torch.bfloat16, device=device)
        t["ki_ring"][:, slot] = ki_win
        t["ki_new"] = ki_win[:, W - 1].contiguous()
        return t
    L = w.L
    t["k"] = _normal_bf16(gen, (B, L, Hkv, d), sc, device)
    t["v"] = _normal_bf16(gen, (B, L, Hkv, d), sc, device)
    t["wk"] = torch.randn((w.m, d), generator=gen, dtype=torch.float32, device=device)
    t["wv"] = torch.randn((w.m, d), generator=gen, dtype=torch.float32, device=device)
    if w.topk:
        t["qi"] = _normal_bf16(gen, (B, L, w.Hi, w.di), sc, device)
        t["wi"] = torch.rand((B, L, w.Hi), generator=gen, dtype=torch.float32, device=device)
        t["ki"] = _normal_bf16(gen, (B, L, w.di), sc, device)
        t["wib"] = torch.randn((w.m, w.di), generator=gen, dtype=torch.float32, device=device)
    return t
