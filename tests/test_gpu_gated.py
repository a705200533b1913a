"""The gated three-branch variant on the GPU against the oracle (hyb_gated_fwd)."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import bits, check_output
from tests.test_gpu_kernels import _randn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import compressed_sparse_sliding_b200 as hb
    return hb


@pytest.mark.parametrize("B,L,Hq,Hkv,d,m,W,K", [
    (1, 700, 32, 1, 128, 4, 128, 160),     # CSA-like: MQA, d = 128
    (2, 300, 4, 2, 64, 8, 32, 24),         # GQA, d = 64
    (1, 1100, 8, 8, 128, 16, 128, 40),     # MHA
])
def test_gated_matches_oracle(hb, B, L, Hq, Hkv, d, m, W, K):
    g = torch.Generator().manual_seed(100 + L)
    q = _randn_bf16(g, (B, L, Hq, d))
    k = _randn_bf16(g, (B, L, Hkv, d))
    v = _randn_bf16(g, (B, L, Hkv, d))
    Nc = L // m
    kc = _randn_bf16(g, (B, Nc, Hkv, d))
    vc = _randn_bf16(g, (B, Nc, Hkv, d))
    gate = torch.randn((B, L, Hq, 3), generator=g) * 2
    rng = np.random.default_rng(L)
    idx = np.full((B, L, K), -1, np.int32)
    for b in range(B):
        for t in range(L):
            nv = min(Nc, (t + 1) // m)          # blocks ending at or before t
            if nv:
                n = min(K, nv)
                idx[b, t, :n] = np.sort(rng.choice(nv, size=n, replace=False))
    p = hb.problem(B=B, Lq=L, Lkv=L, Hq=Hq, Hkv=Hkv, d=d, m=m, W=W, topk=K, Nc=Nc)
    o = hb.hyb_gated_fwd(p, q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(idx).cuda(), k.cuda(),
                         v.cuda(), gate.cuda())
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    rows = sorted(set([0, 1, m - 1, m, W, L - 1] + rng.choice(B * L, size=40, replace=False).tolist()))
    ref = oracle.gated_attention(bits(q), bits(kc), bits(vc), idx, bits(k), bits(v), m, W,
                                 gate.numpy(), rows=rows)
    check_output(o.reshape(B * L, Hq, d)[torch.as_tensor(rows).cuda()], ref["o"])
