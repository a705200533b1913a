"""Decode cache maintenance on the GPU against the oracle (hyb_decode_append)."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import abs_merge, bits, check_bf16_cache, check_output
from tests.test_gpu_kernels import _randn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import compressed_sparse_sliding_b200 as hb
    return hb


def _state(B, W, Hkv, d, di, Nc, dev):
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device=dev)
    st = dict(k_ring=z(B, 2 * W, Hkv, d), v_ring=z(B, 2 * W, Hkv, d), kc=z(B, Nc, Hkv, d),
              vc=z(B, Nc, Hkv, d))
    if di:
        st.update(ki_ring=z(B, W, di), kic=z(B, Nc, di))
    return st


@pytest.mark.parametrize("Hkv,d,di,m,W", [(1, 128, 64, 4, 128), (2, 64, 32, 16, 16), (1, 128, 0, 8, 8)])
def test_append_steps_match_oracle(hb, Hkv, d, di, m, W):
    # T decode steps per sequence from three different start positions; after
    # every step the rings, kv_pos0 and the compressed caches match the oracle
    g = torch.Generator().manual_seed(80 + m)
    B, T, Nc = 3, 3 * m + 5, 64
    offs = np.array([0, m - 1, 5 * m + 2])
    k = _randn_bf16(g, (B, T, Hkv, d))
    v = _randn_bf16(g, (B, T, Hkv, d))
    ki = _randn_bf16(g, (B, T, di)) if di else None
    wk = torch.randn((m, d), generator=g)
    wv = torch.randn((m, d), generator=g)
    wib = torch.randn((m, di), generator=g) if di else None
    dev = torch.device("cuda")
    gst = _state(B, W, Hkv, d, di, Nc, dev)
    ost = {n: bits(x.cpu()).copy() for n, x in gst.items()}
    p = hb.problem(B=B, Lq=1, Lkv=2 * W, Hq=Hkv, Hkv=Hkv, d=d, m=m, W=W, Nc=Nc,
                   topk=4 if di else 0, Hi=1, di=di if di else 64)
    wkd, wvd = wk.cuda(), wv.cuda()
    wibd = wib.cuda() if di else None
    for s in range(T):
        t = torch.from_numpy((offs + s).astype(np.int32))
        kv0 = hb.hyb_decode_append(p, t.cuda(), k[:, s].cuda(), v[:, s].cuda(), gst["k_ring"],
                                   gst["v_ring"], gst["kc"], gst["vc"], wkd, wvd,
                                   ki_new=ki[:, s].cuda() if di else None, wib=wibd,
                                   ki_ring=gst.get("ki_ring"), kic=gst.get("kic"))
        okv0 = oracle.decode_append(ost, offs + s, bits(k[:, s]), bits(v[:, s]), wk.numpy(), wv.numpy(),
                                    m, W, ki_new_bits=bits(ki[:, s]) if di else None,
                                    wib=wib.numpy() if di else None)
        torch.cuda.synchronize()
        assert hb.hyb_get_device_status() == hb.HYB_OK
        np.testing.assert_array_equal(kv0.cpu().numpy(), okv0)
        for ring in ("k_ring", "v_ring", "ki_ring"):
            if ring in gst:
                np.testing.assert_array_equal(bits(gst[ring].cpu()), ost[ring])
    # the caches: every completed block against the oracle's merge of the same rows
    for cache, x, w in (("kc", k, wk), ("vc", v, wv), ("kic", ki, wib)):
        if cache not in gst:
            continue
        for b in range(B):
            done = (offs[b] + T) // m
            first = (offs[b] + m - 1) // m          # blocks entirely inside the appended span
            if done <= first:
                continue
            rows = x[b:b + 1, (first * m - offs[b]):(done * m - offs[b])]
            xr = bits(rows) if rows.dim() == 4 else bits(rows)[:, :, None, :]
            _, ref = oracle.block_merge(xr, w.numpy(), m)
            got = gst[cache][b:b + 1, first:done]
            got = got if got.dim() == 4 else got[:, :, None, :]
            check_bf16_cache(got, ref, cache, abs_merge(xr, w.numpy(), m), m)


def test_attention_reads_the_window_from_the_ring(hb):
    # after the append, hyb_attn_fwd with k_raw = ring, Lkv = 2W and the
    # returned kv_pos0 attends exactly to positions t-W+1 .. t
    g = torch.Generator().manual_seed(90)
    B, Hq, d, m, W, Nc, K = 4, 32, 128, 4, 128, 512, 96
    dev = torch.device("cuda")
    t_end = np.array([W + 20 * m - 1, 3 * W + 7, 5 * W, 2 * W + 100], np.int32)
    T = int(t_end.max()) + 1
    k = _randn_bf16(g, (B, T, 1, d))
    v = _randn_bf16(g, (B, T, 1, d))
    w = torch.randn((m, d), generator=g)
    gst = _state(B, W, 1, d, 0, Nc, dev)
    p = hb.problem(B=B, Lq=1, Lkv=2 * W, Hq=Hq, Hkv=1, d=d, m=m, W=W, Nc=Nc)
    for s in range(T):
        live = np.minimum(s, t_end)                  # each sequence stops at its own end
        idx_b = torch.from_numpy(np.arange(B))
        kv0 = hb.hyb_decode_append(p, torch.from_numpy(live.astype(np.int32)).cuda(),
                                   k[idx_b, torch.from_numpy(live)].cuda(),
                                   v[idx_b, torch.from_numpy(live)].cuda(), gst["k_ring"], gst["v_ring"],
                                   gst["kc"], gst["vc"], w.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    q = _randn_bf16(g, (B, 1, Hq, d))
    rng = np.random.default_rng(90)
    idx = np.full((B, 1, K), -1, np.int32)
    for b in range(B):
        nv = oracle.visible_count(int(t_end[b]), m, W, Nc)
        n = min(K, nv)
        idx[b, 0, :n] = np.sort(rng.choice(nv, size=n, replace=False))
    pa = hb.problem(B=B, Lq=1, Lkv=2 * W, Hq=Hq, Hkv=1, d=d, m=m, W=W, topk=K, Nc=Nc,
                    q_pos=torch.from_numpy(t_end.reshape(B, 1)).cuda(), kv_pos0=kv0)
    o = hb.hyb_attn_fwd(pa, q.cuda(), gst["kc"], gst["vc"], torch.from_numpy(idx).cuda(), gst["k_ring"],
                        gst["v_ring"])
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    # oracle: the raw window taken from the raw sequence itself, positions 0..T-1
    ref = oracle.hybrid_attention(bits(q), bits(gst["kc"].cpu()), bits(gst["vc"].cpu()), idx, bits(k),
                                  bits(v), m, W, q_pos=t_end.reshape(B, 1),
                                  kv_pos0=np.zeros(B, np.int32))
    check_output(o, ref["o"])
