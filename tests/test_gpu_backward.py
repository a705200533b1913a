"""Backward pass on the GPU against the oracle (hyb_attn_bwd, hyb_hca_compress_bwd).

Tolerances, per gradient tensor, relative to its largest oracle magnitude R:
  attention  max-abs <= 1e-2 R, mean-abs <= 5e-4 R.  The dense d = 128 cases
             run the tensor-core kernels, whose P and dS operands are bf16
             (~2^-9 relative per term, below the bar with a factor ~2.5 to
             spare); the others run on CUDA cores in fp32.  The GPU recomputes P from
             the forward's lse, which meets the forward's 2e-3 bound, so P
             carries up to 2e-3 relative error; dS = P (dP - D) multiplies it
             by |dP - D| ~ sqrt(d) |v|, and D = dO . o uses the forward's bf16
             o (2^-9 relative per element); through dq = scale sum dS k this
             reaches ~1e-2 of the largest gradient at the extremes, while the
             mean stays two orders below.  The oracle is exact fp64.
  block_merge  dx max-abs <= 1e-5 R (fp32 softmax weights times dc); dw
             max-abs <= 1e-4 R (fp32 sums over every block, batch and head)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bwd
from tests.test_gpu_kernels import _randn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import compressed_sparse_sliding_b200 as hb
    return hb


def _f64(t):
    return t.double().cpu().numpy()


def _close(name, got, ref, rmax, rmean):
    got = got.double().cpu().numpy() if torch.is_tensor(got) else got
    R = float(np.abs(ref).max(initial=0.0)) or 1.0
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{name}: non-finite"
    assert err.max(initial=0.0) <= rmax * R and err.mean() <= rmean * R, \
        f"{name}: max {err.max():.3e} mean {err.mean():.3e} (R {R:.3e})"


@pytest.mark.parametrize("B,L,Hq,Hkv,d,m,W,K", [
    (2, 150, 8, 2, 64, 4, 32, 8),       # CSA, GQA, d = 64
    (1, 300, 32, 1, 128, 4, 64, 40),    # CSA, MQA, d = 128
    (2, 200, 4, 4, 128, 16, 32, 0),     # HCA, MHA
    (1, 90, 16, 1, 128, 4, 128, 6),     # L < W: window only for every query
    # dense, d = 128: the tensor-core kernels (key-tile and query-tile passes)
    (1, 300, 8, 2, 128, 4, 128, 0),     # GQA, 75 entries, ragged last tiles
    (1, 700, 4, 1, 128, 2, 160, 0),     # MQA, 350 entries (3 key tiles), W > 128
    (2, 260, 2, 2, 128, 8, 0, 0),       # no window: early rows see nothing
    (1, 1100, 2, 1, 128, 4, 128, 0),    # 275 entries: several compressed chunks
    (1, 260, 2, 1, 128, 1, 0, 0),       # m = 1, no window: plain causal attention, all through entries
    (1, 520, 16, 2, 128, 128, 128, 0),  # eight query heads per KV head, 4 entries of 128 tokens
])
def test_attention_gradients_match_oracle(hb, B, L, Hq, Hkv, d, m, W, K):
    g = torch.Generator().manual_seed(100 + L + K)
    rng = np.random.default_rng(100 + L + K)
    Nc = L // m
    q = _randn_bf16(g, (B, L, Hq, d))
    k = _randn_bf16(g, (B, L, Hkv, d))
    v = _randn_bf16(g, (B, L, Hkv, d))
    kc = _randn_bf16(g, (B, Nc, Hkv, d))
    vc = _randn_bf16(g, (B, Nc, Hkv, d))
    dout = _randn_bf16(g, (B, L, Hq, d))
    idx = None
    if K:
        idx = np.full((B, L, K), -1, np.int32)
        for b in range(B):
            for t in range(L):
                nv = oracle.visible_count(t, m, W, Nc)
                if nv:
                    s = np.sort(rng.choice(nv, size=min(K, nv), replace=False))
                    idx[b, t, :len(s)] = s
    p = hb.problem(B=B, Lq=L, Lkv=L, Hq=Hq, Hkv=Hkv, d=d, m=m, W=W, topk=K, Nc=Nc)
    dev = lambda x: x.cuda()
    idx_d = None if idx is None else torch.from_numpy(idx).cuda()
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device="cuda")
    o = hb.hyb_attn_fwd(p, dev(q), dev(kc), dev(vc), idx_d, dev(k), dev(v), lse=lse)
    grads = hb.hyb_attn_bwd(p, dev(q), dev(kc), dev(vc), idx_d, dev(k), dev(v), o, lse, dev(dout))
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    for b in range(B):
        ref = bwd.attention_bwd(_f64(q[b]), _f64(kc[b]), _f64(vc[b]), _f64(k[b]), _f64(v[b]), m, W,
                                _f64(dout[b]), idx=None if idx is None else idx[b])
        for name in ("dq", "dkc", "dvc", "dk_raw", "dv_raw"):
            _close(f"{name}[b={b}]", grads[name][b], ref[name], 1e-2, 5e-4)


@pytest.mark.parametrize("B,L,H,dx,m", [(2, 37, 3, 64, 4), (1, 300, 2, 128, 128), (3, 64, 1, 32, 16)])
def test_block_merge_gradients_match_oracle(hb, B, L, H, dx, m):
    g = torch.Generator().manual_seed(200 + L)
    x = _randn_bf16(g, (B, L, H, dx))
    w = torch.randn((m, dx), generator=g)
    dc = torch.randn((B, L // m, H, dx), generator=g)
    base = torch.randn((B, L, H, dx), generator=g)
    # the x gradient is added to what dx already holds
    gx, gw = hb.hyb_hca_compress_bwd(x.cuda(), w.cuda(), m, dc.cuda(), dx=base.clone().cuda())
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    rx, rw = bwd.block_merge_bwd(_f64(x), w.double().numpy(), m, dc.double().numpy())
    _close("dx", gx.cpu().double().numpy() - base.double().numpy(), rx, 1e-5, 1e-6)
    _close("dw", gw, rw, 1e-4, 1e-5)
