"""4-bit compressed caches on the GPU against the oracle (hyb_fp4_*).

Codes, (min, scale) pairs and dequantized values are compared bit for bit
(both sides take every step in IEEE fp32); the indexer, the top-K and the
attention over a 4-bit cache are compared with the oracle's on the
oracle-dequantized cache, under the usual rules of tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import bits, check_lse, check_output, check_topk, from_bits
from tests.test_gpu_kernels import _randn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import compressed_sparse_sliding_b200 as hb
    return hb


def _fp4(hb, x: torch.Tensor):
    """Quantize on the GPU; check codes and (min, scale) against the oracle;
    return the GPU cache and the oracle's dequantized bf16 bits."""
    c = hb.hyb_fp4_quantize(x.cuda())
    torch.cuda.synchronize()
    codes, qp = oracle.fp4_quantize(bits(x))
    np.testing.assert_array_equal(c.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(c.qp.cpu().numpy().view(np.uint32), qp.view(np.uint32))
    return c, oracle.fp4_dequantize(codes, qp)


@pytest.mark.parametrize("dx", [64, 128, 256])
def test_quantize_and_dequantize_bit_exact(hb, dx):
    g = torch.Generator().manual_seed(dx)
    rows = 1000 + dx // 8     # grid-stride tail
    x = (torch.randn(rows, dx, generator=g) * torch.exp(torch.randn(rows, 1, generator=g) * 2))
    x[0] = 0.75                                         # constant row
    x[1] = torch.arange(dx, dtype=torch.float32) % 16   # exact levels, scale 1
    x[2, : dx // 2] = 0.5 + (torch.arange(dx // 2) % 15)  # halfway values: ties to even
    x[2, dx // 2:] = torch.tensor([0.0, 15.0] * (dx // 4))
    x[3] = -x[3].abs() - 1e-30                          # negative row, tiny magnitudes
    xb = x.to(torch.bfloat16)
    c, ref = _fp4(hb, xb)
    back = hb.hyb_fp4_dequantize(c)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits(back), ref)
    assert hb.hyb_get_device_status() == hb.HYB_OK


def test_cache_shapes_quantize_per_head_row(hb):
    # a [B, Nc, Hkv, d] cache: every (entry, head) row has its own (min, scale)
    g = torch.Generator().manual_seed(11)
    x = _randn_bf16(g, (2, 37, 3, 128))
    x[:, :, 1] *= 50
    c, ref = _fp4(hb, x)
    assert tuple(c.codes.shape) == (2, 37, 3, 64) and tuple(c.qp.shape) == (2, 37, 3, 2)
    np.testing.assert_array_equal(bits(hb.hyb_fp4_dequantize(c)), ref)


def _decode_inputs(g, rng, B, Hq, Hkv, d, m, W, Nc, K, min_vis=40):
    pos = rng.integers(W + 1, Nc * m + W, size=B).astype(np.int32)
    pos[0] = Nc * m + W - 1
    pos[-1] = W + min_vis * m
    q = _randn_bf16(g, (B, 1, Hq, d))
    kr = _randn_bf16(g, (B, W, Hkv, d))
    vr = _randn_bf16(g, (B, W, Hkv, d))
    kc = _randn_bf16(g, (B, Nc, Hkv, d))
    vc = _randn_bf16(g, (B, Nc, Hkv, d))
    idx = np.full((B, 1, K), -1, np.int32)
    for b in range(B):
        nv = oracle.visible_count(int(pos[b]), m, W, Nc)
        n = min(K, nv)
        idx[b, 0, :n] = np.sort(rng.choice(nv, size=n, replace=False))
    return pos, q, kr, vr, kc, vc, idx


@pytest.mark.parametrize("B,Hq,Hkv,K", [(6, 64, 1, 512), (4, 32, 2, 300), (3, 16, 1, 100)])
def test_attention_decode_selected_rows(hb, B, Hq, Hkv, K):
    # Lq * topk < Nc: only the selected rows are dequantized (slot order)
    g = torch.Generator().manual_seed(20 + K)
    rng = np.random.default_rng(20 + K)
    d, m, W, Nc = 128, 4, 128, 2048
    pos, q, kr, vr, kc, vc, idx = _decode_inputs(g, rng, B, Hq, Hkv, d, m, W, Nc, K)
    kq, kref = _fp4(hb, kc)
    vq, vref = _fp4(hb, vc)
    qp = torch.from_numpy(pos.reshape(B, 1)).cuda()
    kv0 = torch.from_numpy(pos - W + 1).cuda()
    p = hb.problem(B=B, Lq=1, Lkv=W, Hq=Hq, Hkv=Hkv, d=d, m=m, W=W, topk=K, Nc=Nc, q_pos=qp,
                   kv_pos0=kv0)
    lse_t = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
    o = hb.hyb_attn_fwd_fp4(p, q.cuda(), kq, vq, torch.from_numpy(idx).cuda(), kr.cuda(), vr.cuda(),
                            lse=lse_t)
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    ref = oracle.hybrid_attention(bits(q), kref, vref, idx, bits(kr), bits(vr), m, W,
                                  q_pos=pos.reshape(B, 1), kv_pos0=(pos - W + 1).astype(np.int32))
    check_output(o, ref["o"])
    check_lse(lse_t.reshape(B, Hq).cpu().numpy(), ref["lse"])


@pytest.mark.parametrize("K,d", [(16, 128), (0, 128), (8, 64)])
def test_attention_prefill_whole_cache(hb, K, d):
    # prefill (Lq * topk >= Nc) and HCA (K = 0): the whole caches are dequantized
    g = torch.Generator().manual_seed(30 + K + d)
    rng = np.random.default_rng(30 + K + d)
    B, L, Hq, Hkv, m, W = 2, 300, 8, 2, 4, 32
    Nc = L // m
    q = _randn_bf16(g, (B, L, Hq, d))
    k = _randn_bf16(g, (B, L, Hkv, d))
    v = _randn_bf16(g, (B, L, Hkv, d))
    kc = _randn_bf16(g, (B, Nc, Hkv, d))
    vc = _randn_bf16(g, (B, Nc, Hkv, d))
    idx = None
    if K:
        idx = np.full((B, L, K), -1, np.int32)
        for b in range(B):
            for t in range(L):
                nv = oracle.visible_count(t, m, W, Nc)
                if nv:
                    s = np.sort(rng.choice(nv, size=min(K, nv), replace=False))
                    idx[b, t, :len(s)] = s
    kq, kref = _fp4(hb, kc)
    vq, vref = _fp4(hb, vc)
    p = hb.problem(B=B, Lq=L, Lkv=L, Hq=Hq, Hkv=Hkv, d=d, m=m, W=W, topk=K, Nc=Nc)
    o = hb.hyb_attn_fwd_fp4(p, q.cuda(), kq, vq, None if idx is None else torch.from_numpy(idx).cuda(),
                            k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    ref = oracle.hybrid_attention(bits(q), kref, vref, idx, bits(k), bits(v), m, W)
    check_output(o, ref["o"])


def _index_fp4_case(hb, B, Lq, Hi, Nc, m, W, K, q_pos, seed, rows=None):
    g = torch.Generator().manual_seed(seed)
    di = 64
    qi = _randn_bf16(g, (B, Lq, Hi, di))
    wi = torch.rand((B, Lq, Hi), generator=g)
    kic = _randn_bf16(g, (B, Nc, di))
    kq, kref = _fp4(hb, kic)
    qp = torch.as_tensor(q_pos, dtype=torch.int32).reshape(B, Lq)
    p = hb.problem(B=B, Lq=Lq, Lkv=max(W, 1), Hq=4, Hkv=1, d=64, m=m, W=W, topk=K, Hi=Hi, di=di,
                   Nc=Nc, q_pos=qp.cuda())
    sel = torch.empty((B, Lq, K), dtype=torch.float32, device="cuda")
    idx = hb.hyb_csa_index_topk_fp4(p, qi.cuda(), wi.cuda(), kq, sel_scores=sel)
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    sc, nv = oracle.index_scores(bits(qi), wi.numpy(), kref, m, W, q_pos=qp.numpy(), rows=rows)
    ref = oracle.topk(sc, nv, K)
    got = idx.reshape(B * Lq, K).cpu().numpy()
    ss = sel.reshape(B * Lq, K).cpu().numpy()
    if rows is not None:
        got, ss = got[np.asarray(rows)], ss[np.asarray(rows)]
    check_topk(got, ref, sc, nv, K)
    for r in range(len(got)):
        s = got[r] >= 0
        np.testing.assert_allclose(ss[r][s], sc[r, got[r][s]], rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("Nc", [2100, 16384])
def test_index_topk_decode_keys_dequantized_on_chip(hb, Nc):
    # decode shapes: key tiles dequantized in the indexer; several chunks and a
    # ragged last tile (2100 = 16 tiles + 52)
    m, W, K = 4, 128, 256
    L = Nc * m + W
    pos = [[L - 1], [L // 2], [W + 300 * m], [L - 1 - 5 * m]]
    _index_fp4_case(hb, 4, 1, 4, Nc, m, W, K, pos, seed=Nc)


def test_index_topk_prefill_cache_dequantized(hb):
    # Lq >= 64: the indexer-key cache is dequantized into the workspace
    B, Lq, Nc, m, W, K = 2, 200, 700, 4, 64, 64
    rng = np.random.default_rng(3)
    pos = rng.integers(0, Nc * m + W, size=(B, Lq)).astype(np.int32)
    _index_fp4_case(hb, B, Lq, 4, Nc, m, W, K, pos, seed=3, rows=list(range(0, B * Lq, 7)))


@pytest.mark.parametrize("Hkv,d,di,m,W", [(1, 128, 64, 4, 128), (2, 64, 32, 16, 16)])
def test_decode_append_quantizes_closed_entries(hb, Hkv, d, di, m, W):
    # rings bit-exact; every closed entry is the oracle's block merge of the
    # same rows, quantized: dequantized values within one code step (the bf16
    # entry itself may differ from the oracle's by the merge's rounding), codes
    # equal almost everywhere
    g = torch.Generator().manual_seed(90 + m)
    B, T, Nc = 3, 3 * m + 5, 64
    offs = np.array([0, m - 1, 5 * m + 2])
    k = _randn_bf16(g, (B, T, Hkv, d))
    v = _randn_bf16(g, (B, T, Hkv, d))
    ki = _randn_bf16(g, (B, T, di))
    wk = torch.randn((m, d), generator=g)
    wv = torch.randn((m, d), generator=g)
    wib = torch.randn((m, di), generator=g)
    dev = torch.device("cuda")
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device=dev)
    rings = dict(k_ring=z(B, 2 * W, Hkv, d), v_ring=z(B, 2 * W, Hkv, d), ki_ring=z(B, W, di))
    kq = hb.Fp4Cache.empty((B, Nc, Hkv, d), dev)
    vq = hb.Fp4Cache.empty((B, Nc, Hkv, d), dev)
    kiq = hb.Fp4Cache.empty((B, Nc, di), dev)
    ost = {n: bits(x.cpu()).copy() for n, x in rings.items()}
    ost.update(kc=np.zeros((B, Nc, Hkv, d), np.uint16), vc=np.zeros((B, Nc, Hkv, d), np.uint16),
               kic=np.zeros((B, Nc, di), np.uint16))
    p = hb.problem(B=B, Lq=1, Lkv=2 * W, Hq=Hkv, Hkv=Hkv, d=d, m=m, W=W, Nc=Nc, topk=4, Hi=1, di=di)
    for s in range(T):
        t = torch.from_numpy((offs + s).astype(np.int32))
        kv0 = hb.hyb_decode_append_fp4(p, t.cuda(), k[:, s].cuda(), v[:, s].cuda(), rings["k_ring"],
                                       rings["v_ring"], kq, vq, wk.cuda(), wv.cuda(), ki_new=ki[:, s].cuda(),
                                       wib=wib.cuda(), ki_ring=rings["ki_ring"], kic=kiq)
        okv0 = oracle.decode_append(ost, offs + s, bits(k[:, s]), bits(v[:, s]), wk.numpy(), wv.numpy(), m,
                                    W, ki_new_bits=bits(ki[:, s]), wib=wib.numpy())
        torch.cuda.synchronize()
        assert hb.hyb_get_device_status() == hb.HYB_OK
        np.testing.assert_array_equal(kv0.cpu().numpy(), okv0)
        for ring in rings:
            np.testing.assert_array_equal(bits(rings[ring].cpu()), ost[ring])
    for cache, name in ((kq, "kc"), (vq, "vc"), (kiq, "kic")):
        for b in range(B):
            first, done = (offs[b] + m - 1) // m, (offs[b] + T) // m
            if done <= first:
                continue
            ref_bits = ost[name][b, first:done]
            rc, rq = oracle.fp4_quantize(ref_bits)
            gc = cache.codes[b, first:done].cpu().numpy()
            gq = cache.qp[b, first:done].cpu().numpy()
            want = oracle.bf16_to_f64(oracle.fp4_dequantize(rc, rq))
            got = oracle.bf16_to_f64(oracle.fp4_dequantize(gc, gq))
            step = rq[..., 1:2].astype(np.float64)
            assert np.all(np.abs(got - want) <= 1.01 * step + 2.0 ** -7 * np.abs(want)), name
            assert (gc == rc).mean() > 0.98, name
