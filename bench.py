#!/usr/bin/env python
"""Benchmark of the hybrid compressed / sparse / sliding attention forward pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl reference]

One step = one pass of the whole forward path over one batch of the workload:
block_merge of K, V (and indexer keys for CSA) -> indexer scores + exact top-K
(CSA) -> hybrid attention.  A decode step starts instead with the cache
maintenance of the new token (window ring append; the block it closes becomes
a compressed entry) and reads the window from the ring.  Default workload: the
CSA+SWA prefill (B=1, L=32768, 32 query heads sharing one KV head, d=128, m=4,
top-K=512, W=128, indexer 4 heads x 64).  Inputs are synthetic, seeded and
resident in HBM before the timed region; L2 is flushed between timed steps
(a 256 MiB write, then a read of a separate 256 MiB buffer so that the step
does not pay for writing back the flush's dirty lines), outside the per-step
CUDA events.  Rank 0 prints one JSON
line.  With N > 1 (torchrun) every rank runs an independent replica of the
workload (the path shards by sequence with no exchange): weak scaling, value =
all ranks' query tokens / max-over-ranks time.

--impl reference times the CPU oracle (fp64 C, OpenMP) on a bounded sample of
the same workload on the host cores; rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "query-tokens/s"
DEFAULT_CONFIG = 3


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm_gbs=float(pk["hbm_gbs"]), bf16_tflops=float(pk["bf16_tflops"]),
                    bf16_tflops_sustained=float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                    source="fallback")


# ----------------------------------------------------------------- work counts
def n_visible(t, m, W, Nc):
    a = t - W + 1
    return 0 if a <= 0 else min(a // m, Nc)


def algorithmic_counts(w, gated=False, fp4=False):
    """Per step: attention keys and FLOP, indexer FLOP, unique bytes per stage.
    gated: the three-branch variant (all blocks ending at or before t, the
    selected ones among them, the window; the selection sees the same blocks).
    fp4: decode over 4-bit compressed caches (a row of dx channels is dx/2
    bytes of codes and 8 bytes of (min, scale))."""
    if gated:
        t = np.arange(w.L, dtype=np.int64)
        nv0 = np.minimum((t + 1) // w.m, w.Nc)
        win = np.minimum(w.W, t + 1)
        attn_keys = int(w.B * (nv0 + np.minimum(nv0, w.topk) + win).sum())
        bf = 2
        q_o = 2 * w.B * w.Lq * w.Hq * w.d * bf
        return dict(attn_keys=attn_keys, attn_flop=4 * w.d * w.Hq * attn_keys,
                    idx_flop=2 * w.Hi * w.di * int(w.B * nv0.sum()),
                    attn_bytes=q_o + 2 * w.B * w.L * w.Hkv * w.d * bf + 2 * w.B * w.Nc * w.Hkv * w.d * bf
                    + w.B * w.Lq * w.topk * 4 + w.B * w.Lq * w.Hq * 3 * 4,
                    compress_bytes=2 * w.B * w.L * w.Hkv * w.d * bf + 2 * w.B * w.Nc * w.Hkv * w.d * bf
                    + w.B * w.L * w.di * bf + w.B * w.Nc * w.di * bf,
                    idx_bytes=0)
    if w.is_decode:
        t = w.L - 1
        nv = n_visible(t, w.m, w.W, w.Nc)
        sel = min(w.topk, nv)
        keys_per_tok = sel + min(w.W, t + 1)
        attn_keys = w.B * keys_per_tok
        idx_pairs = w.B * nv
    else:
        t = np.arange(w.L, dtype=np.int64)
        nv = np.clip((t - w.W + 1) // w.m, 0, w.Nc)
        nv[t - w.W + 1 <= 0] = 0
        sel = np.minimum(nv, w.topk) if w.topk else nv
        win = np.minimum(w.W, t + 1)
        attn_keys = int(w.B * (sel + win).sum())
        idx_pairs = int(w.B * nv.sum()) if w.topk else 0
    attn_flop = 4 * w.d * w.Hq * attn_keys
    idx_flop = 2 * w.Hi * w.di * idx_pairs
    bf = 2
    B, Lq, Hq, Hkv, d, Nc = w.B, w.Lq, w.Hq, w.Hkv, w.d, w.Nc
    q_o = 2 * B * Lq * Hq * d * bf
    if w.is_decode:
        # unique bytes: q/o, the selected compressed rows, the raw window rows, the indexer keys
        row_c = (d // 2 + 8) if fp4 else d * bf             # one compressed K or V row
        row_i = (w.di // 2 + 8) if fp4 else w.di * bf       # one compressed indexer key
        win = min(w.W, t + 1)
        attn_bytes = q_o + w.B * (sel * row_c + win * d * bf) * Hkv * 2 + w.B * w.topk * 4
        compress_bytes = 0
        idx_bytes = B * nv * row_i + B * w.Hi * w.di * bf + B * w.topk * 4
    else:
        attn_bytes = q_o + 2 * B * w.L * Hkv * d * bf + 2 * B * Nc * Hkv * d * bf
        if w.topk:
            attn_bytes += B * Lq * w.topk * 4
        compress_bytes = 2 * B * w.L * Hkv * d * bf + 2 * B * Nc * Hkv * d * bf
        if w.topk:
            compress_bytes += B * w.L * w.di * bf + B * Nc * w.di * bf
        idx_bytes = (B * Lq * (w.Hi * w.di * bf + w.Hi * 4) + B * Nc * w.di * bf +
                     B * Lq * w.topk * 4) if w.topk else 0
    return dict(attn_keys=attn_keys, attn_flop=attn_flop, idx_flop=idx_flop, attn_bytes=attn_bytes,
                compress_bytes=compress_bytes, idx_bytes=idx_bytes)


# ----------------------------------------------------------------- GPU arm
def problem_for(hb, w, inp, kv_pos0=None):
    """Decode reads the window from the 2W-row ring that hyb_decode_append
    maintains (kv_pos0: the [B] tensor that call writes)."""
    if w.is_decode:
        return hb.problem(B=w.B, Lq=1, Lkv=2 * w.W, Hq=w.Hq, Hkv=w.Hkv, d=w.d, m=w.m, W=w.W,
                          topk=w.topk, Hi=w.Hi, di=w.di, Nc=w.Nc, q_pos=inp["q_pos"],
                          kv_pos0=kv_pos0)
    return hb.problem(B=w.B, Lq=w.L, Lkv=w.L, Hq=w.Hq, Hkv=w.Hkv, d=w.d, m=w.m, W=w.W,
                      topk=w.topk, Hi=w.Hi, di=w.di, Nc=w.Nc)


class Step:
    """One forward pass as the three C-ABI stages on one stream, with CUDA
    events between the stages (the same kernels hyb_fused_fwd launches)."""

    def __init__(self, hb, w, inp, gated=False, fp4=False, train=False):
        self.hb, self.w, self.inp, self.gated, self.fp4, self.train = hb, w, inp, gated, fp4, train
        dev = inp["q"].device
        self.kv0 = torch.empty((w.B,), dtype=torch.int32, device=dev)
        self.p = problem_for(hb, w, inp, self.kv0)
        if w.is_decode:
            self.kc, self.vc, self.kic = inp["kc"], inp["vc"], inp["kic"]
            if fp4:
                # the caches as stored in 4 bits (quantized once, before timing)
                self.kq = hb.hyb_fp4_quantize(self.kc)
                self.vq = hb.hyb_fp4_quantize(self.vc)
                self.kiq = hb.hyb_fp4_quantize(self.kic)
                self.fws = torch.empty(max(hb.hyb_fp4_workspace_size(self.p), 256), dtype=torch.uint8,
                                       device=dev)
        else:
            self.kc = torch.empty((w.B, w.Nc, w.Hkv, w.d), dtype=torch.bfloat16, device=dev)
            self.vc = torch.empty_like(self.kc)
            self.kic = (torch.empty((w.B, w.Nc, w.di), dtype=torch.bfloat16, device=dev)
                        if w.topk else None)
        self.idx = (torch.empty((w.B, w.Lq, w.topk), dtype=torch.int32, device=dev)
                    if w.topk else None)
        self.o = torch.empty((w.B, w.Lq, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
        need = hb.hyb_workspace_size(self.p)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        if gated:
            # the selection sees the same blocks as the compressed branch (W = 0)
            self.p_sel = problem_for(hb, w, inp)
            self.p_sel.W = 0
            gneed = hb.hyb_gated_workspace_size(self.p)
            self.gws = torch.empty(max(gneed, 256), dtype=torch.uint8, device=dev)
        if train:
            # the backward of the step: a seeded output gradient, lse from the forward
            self.lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=dev)
            gen = torch.Generator(device="cpu")
            gen.manual_seed(30260 + w.no)
            self.dout = torch.randn(self.o.shape, generator=gen).to(torch.bfloat16).to(dev)
            self.bws = torch.empty(max(hb._lib.hyb_hca_compress_bwd_workspace_size(w.d, w.m), 256),
                                   dtype=torch.uint8, device=dev)
            self.dwk = torch.empty((w.m, w.d), dtype=torch.float32, device=dev)
            self.dwv = torch.empty_like(self.dwk)
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        self.launches = 0

    def run(self, stream):
        hb, w, inp, ev = self.hb, self.w, self.inp, self.ev
        launches = 0
        ev[0].record(stream)
        if w.is_decode and self.fp4:
            hb.hyb_decode_append_fp4(self.p, inp["t_new"], inp["k_new"], inp["v_new"], inp["k_ring"],
                                     inp["v_ring"], self.kq, self.vq, inp["wk"], inp["wv"],
                                     ki_new=inp["ki_new"], wib=inp["wib"], ki_ring=inp["ki_ring"],
                                     kic=self.kiq, kv_pos0=self.kv0, stream=stream)
            launches += 1
        elif w.is_decode:
            # cache maintenance of the new token: window ring + the closed block
            hb.hyb_decode_append(self.p, inp["t_new"], inp["k_new"], inp["v_new"], inp["k_ring"],
                                 inp["v_ring"], self.kc, self.vc, inp["wk"], inp["wv"],
                                 ki_new=inp["ki_new"], wib=inp["wib"], ki_ring=inp["ki_ring"],
                                 kic=self.kic, kv_pos0=self.kv0, stream=stream)
            launches += 1
        else:
            hb.hyb_hca_compress(inp["k"], inp["wk"], w.m, out=self.kc, stream=stream)
            hb.hyb_hca_compress(inp["v"], inp["wv"], w.m, out=self.vc, stream=stream)
            launches += 2
            if w.topk:
                hb.hyb_hca_compress(inp["ki"], inp["wib"], w.m, out=self.kic, stream=stream)
                launches += 1
        ev[1].record(stream)
        if self.fp4:
            hb.hyb_csa_index_topk_fp4(self.p, inp["qi"], inp["wi"], self.kiq, idx=self.idx, ws=self.fws,
                                      stream=stream)
            launches += 2
        elif w.topk:
            hb.hyb_csa_index_topk(self.p_sel if self.gated else self.p, inp["qi"], inp["wi"], self.kic,
                                  idx=self.idx, ws=self.ws, stream=stream)
            launches += 2
        ev[2].record(stream)
        if self.train:
            hb.hyb_attn_fwd(self.p, inp["q"], self.kc, self.vc, self.idx, inp["k"], inp["v"], o=self.o,
                            lse=self.lse, stream=stream)
            launches += 1
            ev[3].record(stream)
            # backward: attention (window and compressed paths), then block_merge of K and V,
            # whose x gradients add into the raw K / V gradients
            self.grads = hb.hyb_attn_bwd(self.p, inp["q"], self.kc, self.vc, self.idx, inp["k"], inp["v"],
                                         self.o, self.lse, self.dout, stream=stream)
            hb.hyb_hca_compress_bwd(inp["k"], inp["wk"], w.m, self.grads["dkc"], dx=self.grads["dk_raw"],
                                    dw=self.dwk, ws=self.bws, stream=stream)
            hb.hyb_hca_compress_bwd(inp["v"], inp["wv"], w.m, self.grads["dvc"], dx=self.grads["dv_raw"],
                                    dw=self.dwv, ws=self.bws, stream=stream)
            # dense problems with d = 128: three tensor-core launches; CSA with
            # d = 128: those three for the window keys plus the CUDA-core one
            # for the selected entries; else the CUDA-core one alone
            launches += 4 + (3 if (w.topk == 0 and w.d == 128) else (4 if w.d == 128 else 1))
            ev[4].record(stream)
            self.launches = launches
            return
        if self.fp4:
            hb.hyb_attn_fwd_fp4(self.p, inp["q"], self.kq, self.vq, self.idx, inp["k_ring"], inp["v_ring"],
                                o=self.o, ws=self.fws, stream=stream)
            launches += 2
        elif self.gated:
            hb.hyb_gated_fwd(self.p, inp["q"], self.kc, self.vc, self.idx, inp["k"], inp["v"],
                             inp["gate"], o=self.o, ws=self.gws, stream=stream)
            launches += 4
        else:
            hb.hyb_attn_fwd(self.p, inp["q"], self.kc, self.vc, self.idx,
                            inp["k_ring"] if w.is_decode else inp["k"],
                            inp["v_ring"] if w.is_decode else inp["v"], o=self.o, stream=stream)
            launches += 1
        ev[3].record(stream)
        self.launches = launches

    def times_ms(self):
        e = self.ev
        last = e[4] if self.train else e[3]
        return (e[0].elapsed_time(last), e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]),
                e[2].elapsed_time(e[3]), e[3].elapsed_time(e[4]) if self.train else 0.0)


class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, polled through
    NVML from a background thread while the timed region runs (nvidia-smi's
    loop is far coarser than a timed region of a few milliseconds)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(torch.cuda.current_device())
        bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.sm, self.mask = [], 0
        self.stop_ev = threading.Event()
        self.th = threading.Thread(target=self._run, daemon=True)
        self.th.start()

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                self.mask |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                return
            time.sleep(0.0002)

    def stop(self):
        self.stop_ev.set()
        self.th.join(timeout=5)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass
        if not self.sm:
            return None
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for bit, n in self.REASONS.items() if self.mask & bit),
                "samples": len(self.sm), "source": "nvml"}


def sample_clocks_start():
    try:
        return ClockSampler()
    except Exception:
        pass
    try:
        return subprocess.Popen(
            ["nvidia-smi", "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,"
             "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits", "-lms", "100",
             "-i", str(torch.cuda.current_device())],
            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
    except Exception:
        return None


def sample_clocks_stop(proc):
    if proc is None:
        return None
    if isinstance(proc, ClockSampler):
        return proc.stop()
    proc.terminate()
    try:
        out, _ = proc.communicate(timeout=5)
    except Exception:
        proc.kill()
        return None
    sm, mx, reasons = [], 0.0, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in out.strip().splitlines():
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            mx = max(mx, float(f[2]))
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm), "source": "nvidia-smi"}


def attention_kernel(w):
    """Name and source file of the attention kernel the library dispatches to
    for this workload (the stage the roofline object describes)."""
    if not w.topk and not w.is_decode:
        return "hca_attn_kernel", "attn_dense.cu"
    if w.topk and w.d == 128:
        return "csa_attn_kernel", "attn_sparse.cu"
    return "hybrid_attn_kernel", "attn.cu"


def kernel_traffic(kernel: str, config_no: int):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            tab = json.load(f)
        ent = tab[f"{kernel}@{config_no}"]
        src = os.path.join(ROOT, "compressed_sparse_sliding_b200", "csrc", ent["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return int(ent["bytes_per_launch"]) if h == ent["source_sha"] else None
    except Exception:
        return None


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest value of x over all ranks (each rank's time is its own
    device time; the job takes as long as its slowest replica)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_seed(w, rank: int) -> int:
    """Seed of a replica's synthetic inputs: every rank its own batch."""
    return 20260 + w.no + 1000 * rank


def gate_logits(w, device, rank=0):
    """Seeded gate logits [B, L, Hq, 3] for the gated variant (N(0, 2^2))."""
    g = torch.Generator(device="cpu")
    g.manual_seed(20360 + w.no + 1000 * rank)
    return (torch.randn((w.B, w.Lq, w.Hq, 3), generator=g) * 2).to(device)


def workload_of(args):
    """The workload of --config, with --seq-len (prefill only) shortening its
    sequences for small profiler captures; the full sizes otherwise."""
    import dataclasses
    w = WORKLOADS[args.config]
    if getattr(args, "seq_len", None) and not w.is_decode:
        w = dataclasses.replace(w, L=int(args.seq_len), name=f"{w.name}_l{int(args.seq_len)}")
    return w


def run_gpu(args, rank, world):
    import compressed_sparse_sliding_b200 as hb
    w = workload_of(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_inputs(w, device=dev, seed=replica_seed(w, rank))
    if not w.is_decode:
        inp["k_raw"], inp["v_raw"] = inp["k"], inp["v"]
    gated = args.variant == "gated"
    fp4 = args.variant == "fp4"
    train = args.variant == "train"
    if gated:
        inp["gate"] = gate_logits(w, dev, rank)
    stream = torch.cuda.current_stream()
    step = Step(hb, w, inp, gated, fp4, train)
    # L2 flush: write 256 MiB, then read another 256 MiB so that no dirty line
    # of the flush buffer is left for the timed step to write back
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.int32, device=dev)

    def flush_l2():
        flush.fill_(1)
        flush_rd.sum()

    counts = algorithmic_counts(w, gated, fp4)

    for _ in range(args.warmup):
        flush_l2()
        step.run(stream)
    torch.cuda.synchronize()
    st = hb.hyb_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {hb.hyb_error_string(st)}")

    clk = sample_clocks_start()
    if not isinstance(clk, ClockSampler):
        time.sleep(0.3)  # nvidia-smi needs a moment before its first sample
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    tot, comp, idx, att, back = [], [], [], [], []
    launches = 0
    for _ in range(args.steps):
        flush_l2()  # outside the step's events
        step.run(stream)
        torch.cuda.synchronize()
        a, b, c, d, e = step.times_ms()
        tot.append(a); comp.append(b); idx.append(c); att.append(d); back.append(e)
        launches += step.launches
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sample_clocks_stop(clk)
    st = hb.hyb_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {hb.hyb_error_string(st)}")

    total_ms = max_over_ranks(float(sum(tot)), world, dev)
    ms_per_step = total_ms / args.steps
    tokens = w.B * w.Lq * world
    value = tokens / (ms_per_step / 1e3)

    # ---- end to end through the public C-ABI calls with host buffers ----
    # Prefill: every input of the step crosses from pinned host memory.  Decode:
    # the step's own inputs do (the query, the indexer query and head weights,
    # the new token's K / V / indexer-key rows and positions); the caches,
    # rings and block weights are device-resident state the step maintains.
    if w.is_decode:
        per_step = ("q", "qi", "wi", "k_new", "v_new", "ki_new", "t_new", "q_pos")
    else:
        per_step = ("q", "k", "v", "wk", "wv", "qi", "wi", "ki", "wib", "gate")
    host = {k: inp[k].cpu().pin_memory() for k in per_step if k in inp}
    # Two sets of device inputs and outputs: while step n runs, the inputs of
    # step n + 1 come in on one copy stream and the output of step n - 1 goes
    # out on another (every step still moves all of its bytes both ways; the
    # timed region runs from before the first input copy to after the last
    # output copy).
    bufs = []
    for b in range(2):
        din = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
        if w.is_decode:
            for k in ("k_ring", "v_ring", "ki_ring", "kc", "vc", "kic", "wk", "wv", "wib"):
                din[k] = inp[k]
        odev = step.o if b == 0 else torch.empty_like(step.o)
        ohost = torch.empty(step.o.shape, dtype=step.o.dtype).pin_memory()
        bufs.append((din, odev, ohost))
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = bufs[0][2].numel() * bufs[0][2].element_size()

    kv0_e2e = torch.empty((w.B,), dtype=torch.int32, device=dev)

    def e2e_compute(dev_in, odev):
        """The step's public calls on device inputs already in place, output into odev."""
        if train:
            # the training step through the public calls, on the copied inputs
            saved = step.inp
            step.inp = dict(saved, **dev_in)
            step.run(stream)
            step.inp = saved
            odev.copy_(step.grads["dq"])
            return
        p = problem_for(hb, w, dev_in, kv0_e2e)
        if gated:
            # the public calls of the gated variant: compression, the selection
            # (W = 0 visibility) and the three-branch attention
            hb.hyb_hca_compress(dev_in["k"], dev_in["wk"], w.m, out=step.kc, stream=stream)
            hb.hyb_hca_compress(dev_in["v"], dev_in["wv"], w.m, out=step.vc, stream=stream)
            hb.hyb_hca_compress(dev_in["ki"], dev_in["wib"], w.m, out=step.kic, stream=stream)
            hb.hyb_csa_index_topk(step.p_sel, dev_in["qi"], dev_in["wi"], step.kic, idx=step.idx,
                                  ws=step.ws, stream=stream)
            hb.hyb_gated_fwd(p, dev_in["q"], step.kc, step.vc, step.idx, dev_in["k"], dev_in["v"],
                             dev_in["gate"], o=odev, ws=step.gws, stream=stream)
            return
        if fp4:
            # the public calls over the 4-bit caches
            hb.hyb_decode_append_fp4(p, dev_in["t_new"], dev_in["k_new"], dev_in["v_new"],
                                     dev_in["k_ring"], dev_in["v_ring"], step.kq, step.vq, dev_in["wk"],
                                     dev_in["wv"], ki_new=dev_in["ki_new"], wib=dev_in["wib"],
                                     ki_ring=dev_in["ki_ring"], kic=step.kiq, kv_pos0=kv0_e2e,
                                     stream=stream)
            hb.hyb_csa_index_topk_fp4(p, dev_in["qi"], dev_in["wi"], step.kiq, idx=step.idx, ws=step.fws,
                                      stream=stream)
            hb.hyb_attn_fwd_fp4(p, dev_in["q"], step.kq, step.vq, step.idx, dev_in["k_ring"],
                                dev_in["v_ring"], o=odev, ws=step.fws, stream=stream)
            return
        if w.is_decode:
            hb.hyb_decode_append(p, dev_in["t_new"], dev_in["k_new"], dev_in["v_new"],
                                 dev_in["k_ring"], dev_in["v_ring"], dev_in["kc"], dev_in["vc"],
                                 dev_in["wk"], dev_in["wv"], ki_new=dev_in["ki_new"],
                                 wib=dev_in["wib"], ki_ring=dev_in["ki_ring"], kic=dev_in["kic"],
                                 kv_pos0=kv0_e2e, stream=stream)
            raw_k, raw_v = dev_in["k_ring"], dev_in["v_ring"]
        else:
            raw_k, raw_v = dev_in["k"], dev_in["v"]
        hb.hyb_fused_fwd(p, dev_in["q"], raw_k, raw_v,
                         wk=None if w.is_decode else dev_in.get("wk"),
                         wv=None if w.is_decode else dev_in.get("wv"), qi=dev_in.get("qi"),
                         wi=dev_in.get("wi"), ki_raw=dev_in.get("ki"),
                         wib=None if w.is_decode else dev_in.get("wib"), kc=dev_in.get("kc"),
                         vc=dev_in.get("vc"), kic=dev_in.get("kic"), o=odev, ws=step.ws,
                         stream=stream)

    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n, after=None):
        """n end-to-end steps; copies wait for `after` (an event on `stream`)."""
        if after is not None:
            h2d_s.wait_event(after)
            d2h_s.wait_event(after)
        for s in range(n):
            b = s & 1
            din, odev, ohost = bufs[b]
            if s >= 2:
                h2d_s.wait_event(ev_done[b])     # step s - 2 has read these inputs
            with torch.cuda.stream(h2d_s):
                for k, v in host.items():
                    din[k].copy_(v, non_blocking=True)
            ev_in[b].record(h2d_s)
            stream.wait_event(ev_in[b])
            if s >= 2:
                stream.wait_event(ev_out[b])     # step s - 2's output has left
            with torch.cuda.stream(stream):
                e2e_compute(din, odev)
            ev_done[b].record(stream)
            d2h_s.wait_event(ev_done[b])
            with torch.cuda.stream(d2h_s):
                ohost.copy_(odev, non_blocking=True)
            ev_out[b].record(d2h_s)
        stream.wait_event(ev_out[(n - 1) & 1])

    e2e_steps(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, min(args.steps, 6))
    e0.record(stream)
    e2e_steps(n_e2e, after=e0)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, dev)

    peaks = load_peaks()
    att_ms = statistics.mean(att)
    hbm_bound = w.is_decode or w.no == 2
    bwd_tc = train and w.topk == 0 and w.d == 128
    if train:
        # the attention backward: 10 d FLOP per (query head, key) (the scores
        # again, dP, dq, dk, dv).  Dense problems with d = 128 run on the tensor
        # cores (bf16 peak); the others on CUDA cores, whose peak is 148 SMs x
        # 128 fp32 lanes x 2 FLOP x the clock measured during the run
        bwd_ms = statistics.mean(back)
        achieved = 2.5 * counts["attn_flop"] / (bwd_ms / 1e3) / 1e12
        if bwd_tc:
            peak = peaks["bf16_tflops"]
            bound = "tensor"
        else:
            mhz = (clocks or {}).get("sm_mhz") or 1965.0
            peak = round(148 * 128 * 2 * mhz * 1e6 / 1e12, 1)
            bound = "alu"
        roof = {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4)}
    elif hbm_bound:
        achieved = counts["attn_bytes"] / (att_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4)}
    else:
        achieved = counts["attn_flop"] / (att_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4)}
    kname, ksrc = attention_kernel(w)
    if gated:
        kname = "hyb_gated_fwd (three attention kernels + combine)"
    if fp4:
        kname = "hyb_attn_fwd_fp4 (fp4_gather_kernel + csa_attn_kernel)"
    if train:
        kname = ("bwd_delta_kernel + attn_bwd_kv_kernel + attn_bwd_q_kernel" if bwd_tc
                 else "attn_bwd_kernel (selected entries) + tensor-core window passes" if w.d == 128
                 else "attn_bwd_kernel")
    roof["kernel"] = kname
    roof["peak_source"] = ("derived (unit counts x measured clock)" if train and not bwd_tc
                           else peaks["source"])
    roof["traffic"] = kernel_traffic(kname, w.no)
    stages = {("append_ms" if w.is_decode else "compress_ms"): round(statistics.mean(comp), 4),
              "index_topk_ms": round(statistics.mean(idx), 4),
              "attention_ms": round(att_ms, 4)}
    if counts["compress_bytes"] and statistics.mean(comp) > 0:
        stages["compress_GBps"] = round(counts["compress_bytes"] / (statistics.mean(comp) / 1e3) / 1e9, 1)
    if w.topk and statistics.mean(idx) > 0:
        stages["index_topk_TFLOPs"] = round(counts["idx_flop"] / (statistics.mean(idx) / 1e3) / 1e12, 2)
    stages["attention_TFLOPs"] = round(counts["attn_flop"] / (att_ms / 1e3) / 1e12, 1)
    if train:
        stages["backward_ms"] = round(statistics.mean(back), 4)
    stages["attention_GBps"] = round(counts["attn_bytes"] / (att_ms / 1e3) / 1e9, 1)

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "query-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 inputs, N(0,1) block weights, U(0,1) head weights)",
        "config": {"workload": w.name, "desc": w.describe(), "global_batch": w.B * world,
                   "seq_len": w.L, "parallelism": f"replicas{world}",
                   "variant": args.variant,
                   "l2": "flushed between steps (256 MiB written, then a separate 256 MiB read)"},
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "query-tokens/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "overlap": "double-buffered: step n+1's inputs in and step n-1's output out "
                           "on two copy streams while step n runs"},
        "gpu_launches": int(launches),
        "roofline": roof,
        "stages": stages,
        "clocks": clocks,
    }
    return res


# ----------------------------------------------------------------- CPU oracle
def run_oracle(w, budget_s=12.0, rows_hint=None, gated=False, fp4=False, train=False):
    """Times the oracle on a bounded sample of the workload.  Compression of
    the whole batch is timed once and charged per query token; indexer, top-K
    and attention are timed on a sample of query rows.  fp4: the decode caches
    are the 4-bit round trip of the inputs (the stored form, made before
    timing)."""
    import oracle
    inp = make_inputs(w, device="cpu")
    cores = os.cpu_count()
    bits = {k: oracle.bf16_bits(v) for k, v in inp.items() if v.dtype == torch.bfloat16}
    if fp4:
        for n in ("kc", "vc", "kic"):
            bits[n] = oracle.fp4_dequantize(*oracle.fp4_quantize(bits[n]))
    t0 = time.perf_counter()
    kv0_ring = None
    if w.is_decode:
        # the decode step's cache maintenance of the new token, then the ring
        # holds the window
        state = {n: bits[n] for n in ("k_ring", "v_ring", "ki_ring", "kc", "vc", "kic")}
        kv0_ring = oracle.decode_append(state, inp["t_new"].numpy(), bits["k_new"], bits["v_new"],
                                        inp["wk"].numpy(), inp["wv"].numpy(), w.m, w.W,
                                        ki_new_bits=bits["ki_new"], wib=inp["wib"].numpy())
        kc, vc, kic = state["kc"], state["vc"], state["kic"]
        t_comp = time.perf_counter() - t0
    else:
        _, kc = oracle.block_merge(bits["k"], inp["wk"].numpy(), w.m)
        _, vc = oracle.block_merge(bits["v"], inp["wv"].numpy(), w.m)
        kic = None
        if w.topk:
            _, kic = oracle.block_merge(bits["ki"][:, :, None, :], inp["wib"].numpy(), w.m)
            kic = kic[:, :, 0, :]
        t_comp = time.perf_counter() - t0
    total_rows = w.B * w.Lq
    gate_np = gate_logits(w, "cpu").numpy() if gated else None

    def rows_work(rows):
        t1 = time.perf_counter()
        qp = inp["q_pos"].numpy() if w.is_decode else None
        idx = None
        if w.topk:
            sc, nv = oracle.index_scores(bits["qi"], inp["wi"].numpy(), kic, w.m, 0 if gated else w.W,
                                         q_pos=qp,
                                         rows=rows)
            sel = oracle.topk(sc, nv, w.topk)
            idx = np.full((total_rows, w.topk), -1, np.int32)
            idx[rows] = sel
            idx = idx.reshape(w.B, w.Lq, w.topk)
        if gated:
            oracle.gated_attention(bits["q"], kc, vc, idx, bits["k"], bits["v"], w.m, w.W,
                                   gate_np, rows=rows)
        elif w.is_decode:
            oracle.hybrid_attention(bits["q"], kc, vc, idx, bits["k_ring"], bits["v_ring"], w.m, w.W,
                                    q_pos=qp, kv_pos0=kv0_ring, rows=rows)
        else:
            oracle.hybrid_attention(bits["q"], kc, vc, idx, bits["k"], bits["v"], w.m, w.W,
                                    rows=rows)
        return time.perf_counter() - t1

    rng = np.random.default_rng(0)
    n = 8 if rows_hint is None else rows_hint
    while True:
        rows = np.sort(rng.choice(total_rows, size=min(n, total_rows), replace=False))
        dt = rows_work(rows)
        if dt > budget_s / 4 or n >= total_rows:
            break
        n = min(total_rows, int(n * max(2.0, (budget_s / 2) / max(dt, 1e-3))))
    per_row = t_comp / total_rows + dt / len(rows)
    note = ""
    if train:
        # the backward oracle works on one whole sequence (dense masked form)
        if w.L * (w.Nc + w.L) * 8 <= (1 << 28):
            from oracle import backward as bwd
            f64 = lambda t: t.double().numpy()
            t1 = time.perf_counter()
            bwd.attention_bwd(f64(inp["q"][0]), kc_f64(kc, 0), kc_f64(vc, 0), f64(inp["k"][0]), f64(inp["v"][0]),
                              w.m, w.W, np.ones((w.L, w.Hq, w.d)), idx=None)
            for x, wt in ((inp["k"], inp["wk"]), (inp["v"], inp["wv"])):
                bwd.block_merge_bwd(f64(x[:1]), wt.double().numpy(), w.m, np.ones((1, w.Nc, w.Hkv, w.d)))
            per_row += (time.perf_counter() - t1) / w.Lq
            note = "; backward of one sequence (dense masked oracle) charged per token"
        else:
            note = "; backward not sampled (the dense backward oracle is too large for this sequence length)"
    return {"value": round(1.0 / per_row, 3), "unit": "query-tokens/s", "cores": cores,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": (f"{len(rows)} of {total_rows} query rows (indexer, top-K, attention) + " +
                       (f"cache maintenance of the new tokens ({t_comp:.2f} s)" if w.is_decode else
                        f"compression of the whole batch ({t_comp:.2f} s)") + " charged per token" + note)}


def cpu_model() -> str:
    """The host CPU's model name (for the oracle baseline's record)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def kc_f64(bits, b):
    """One sequence of a bf16-bits cache as fp64."""
    import oracle
    return oracle.bf16_to_f64(bits[b])


def run_reference_arm(args):
    w = workload_of(args)
    per_step = []
    base = None
    gated = args.variant == "gated"
    fp4 = args.variant == "fp4"
    train = args.variant == "train"
    for _ in range(args.warmup):
        run_oracle(w, budget_s=2.0, rows_hint=4, gated=gated, fp4=fp4, train=train)
    for _ in range(args.steps):
        base = run_oracle(w, budget_s=6.0, rows_hint=8, gated=gated, fp4=fp4, train=train)
        per_step.append(1.0 / base["value"])
    value = 1.0 / statistics.mean(per_step)
    cpu = dict(base)
    cpu["value"] = round(value, 3)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "query-tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * statistics.mean(per_step) * w.B * w.Lq, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": w.name, "desc": w.describe(), "global_batch": w.B, "seq_len": w.L,
                   "parallelism": "host cores (OpenMP)", "variant": args.variant},
        "cpu_baseline": cpu,
        "e2e": {"value": round(value, 3), "unit": "query-tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_micro(args):
    """The measured roofline denominators on this GPU: an HBM copy, the
    L2-resident random-row gather (the CSA attention's data path, through the
    library's probe kernel) and a cuBLAS bf16 GEMM.  CUDA events, best of N."""
    import compressed_sparse_sliding_b200 as hb
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def best_ms(fn, reps):
        fn()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return best

    clk = sample_clocks_start()
    a = torch.ones(1 << 30, dtype=torch.bfloat16, device=dev)
    b = torch.empty_like(a)
    ms = best_ms(lambda: b.copy_(a), 10)
    hbm = 2 * a.numel() * 2 / (ms / 1e3) / 1e9
    del a, b
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    table = torch.randint(0, 1 << 30, ((4 << 20) // 4,), dtype=torch.int32, device=dev)
    sink = torch.zeros(256, dtype=torch.int32, device=dev)
    rows = 128 * 2048
    gather = {}
    for stages in range(2, 7):
        ms = best_ms(lambda: hb.hyb_probe_l2_gather(table, rows, stages, sink, stream), 10)
        gather[str(stages)] = round(sms * rows * 256 / (ms / 1e3) / 1e9, 1)
    # the same rows by the tensor memory accelerator's four-row gather
    sink_t = torch.zeros(257, dtype=torch.int32, device=dev)
    gather_tma = {}
    for stages in range(2, 7):
        ms = best_ms(lambda: hb.hyb_probe_l2_gather_tma(table, rows, stages, sink_t, stream), 10)
        gather_tma[str(stages)] = round(sms * rows * 256 / (ms / 1e3) / 1e9, 1)
    misplaced = int(sink_t[256].item())
    n = 8192
    x = torch.randn((n, n), dtype=torch.bfloat16, device=dev)
    y = torch.randn((n, n), dtype=torch.bfloat16, device=dev)
    ms = best_ms(lambda: torch.matmul(x, y), 10)
    gemm = 2 * n ** 3 / (ms / 1e3) / 1e12
    clocks = sample_clocks_stop(clk)
    return {"metric": "roofline denominators", "hbm_copy_GBps": round(hbm, 1),
            "l2_gather_GBps_by_stages": gather, "l2_gather_GBps": max(gather.values()),
            "l2_gather_B_per_clk_per_sm": round(max(gather.values()) * 1e9 / sms /
                                               (((clocks or {}).get("sm_mhz") or 1965.0) * 1e6), 1),
            "l2_gather_tma_GBps_by_stages": gather_tma, "l2_gather_tma_GBps": max(gather_tma.values()),
            "l2_gather_tma_misplaced_chunks": misplaced,
            "bf16_gemm_TFLOPs": round(gemm, 1), "sms": sms,
            "how": "HBM: 1 GiB bf16 copy (read + write bytes); L2 gather: random 256-byte rows of a 4 MB "
                   "table into 32 KB shared-memory stages with 16-byte cp.async, one CTA per SM, "
                   f"{rows} rows per SM (hyb_probe_l2_gather), and with tile::gather4 TMA copies, one "
                   f"warp per SM (hyb_probe_l2_gather_tma); GEMM: torch.matmul bf16 {n}^3; "
                   "best of 10 with CUDA events",
            "clocks": clocks}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="shorter sequences of a prefill workload (small profiler captures); "
                         "the full workload when absent")
    ap.add_argument("--micro", action="store_true",
                    help="print the measured roofline denominators (HBM copy, L2 gather, bf16 GEMM) and exit")
    ap.add_argument("--variant", default="hybrid", choices=["hybrid", "gated", "fp4", "train"],
                    help="gated: the three-branch variant (CSA workloads with prefill); "
                         "fp4: decode over 4-bit compressed caches (config 5); "
                         "train: forward + backward (prefill workloads)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.variant == "gated" and (not WORKLOADS[args.config].topk or WORKLOADS[args.config].is_decode):
        ap.error("--variant gated needs a CSA prefill workload (configs 1 and 3)")
    if args.variant == "fp4" and not WORKLOADS[args.config].is_decode:
        ap.error("--variant fp4 needs the decode workload (config 5)")
    if args.variant == "train" and WORKLOADS[args.config].is_decode:
        ap.error("--variant train needs a prefill workload (configs 1-4)")

    if args.micro:
        print(json.dumps(run_micro(args)), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference_arm(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    try:
        res = run_gpu(args, rank, world)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = run_oracle(workload_of(args), gated=args.variant == "gated",
                                             fp4=args.variant == "fp4", train=args.variant == "train")
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
