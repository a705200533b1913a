"""The per-role timeline of the CSA and HCA attention kernels (a debug aid):
CTA 0 records, per work item, a load, an MMA and a softmax event for every key
tile, with clocks that never go backwards within a role; with no buffer
attached nothing is recorded and the output is unchanged."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import compressed_sparse_sliding_b200 as hb
    return hb


def _case(hb):
    g = torch.Generator().manual_seed(77)
    B, L, Hq, d, m, W, K, Nc = 1, 600, 32, 128, 4, 128, 256, 400
    q = torch.randn((B, L, Hq, d), generator=g).to(torch.bfloat16).cuda()
    kv = [torch.randn((B, L, 1, d), generator=g).to(torch.bfloat16).cuda() for _ in range(2)]
    kc = [torch.randn((B, Nc, 1, d), generator=g).to(torch.bfloat16).cuda() for _ in range(2)]
    idx = torch.stack([torch.randperm(Nc, generator=g)[:K].sort().values for _ in range(L)])
    idx = idx.to(torch.int32).reshape(B, L, K).cuda()
    p = hb.problem(B=B, Lq=L, Lkv=L, Hq=Hq, Hkv=1, d=d, m=m, W=W, topk=K, Nc=Nc)
    return p, q, kc, idx, kv


def test_csa_attention_timeline(hb):
    p, q, kc, idx, kv = _case(hb)
    ref = hb.hyb_attn_fwd(p, q, kc[0], kc[1], idx, kv[0], kv[1])
    buf = torch.zeros(1 << 20, dtype=torch.int64, device="cuda")
    hb.hyb_trace_attach(buf)
    try:
        out = hb.hyb_attn_fwd(p, q, kc[0], kc[1], idx, kv[0], kv[1])
        torch.cuda.synchronize()
    finally:
        hb.hyb_trace_attach(None)
    assert hb.hyb_get_device_status() == hb.HYB_OK
    assert torch.equal(out, ref)
    rec = hb.trace_records(buf)
    assert rec, "no records"
    items = sorted({r["item"] for r in rec})
    # each role's region in append order: its clocks never go backwards
    words = buf.cpu().numpy().view("uint64")
    cap = (words.size - 4) // 8
    for role in (1, 2, 3):
        n = int(words[role])
        assert 0 < n <= cap, f"role {role}: {n} records"
        base = 4 + 2 * role * cap
        clk = words[base:base + 2 * n:2].astype(np.int64)
        tags = words[base + 1:base + 2 * n:2]
        assert np.all((tags >> 56) == role)
        assert np.all(np.diff(clk) >= 0), f"role {role}: clocks out of order"
    # every item of CTA 0: K and V gathered, QK^T and PV issued for each of its
    # key tiles (2 selected tiles of 128 + the window); the softmax events come
    # from one thread of the first softmax warpgroup, which takes every tile
    # (its half of the heads)
    for it in items:
        ev = {(r["role"], r["event"]) for r in rec if r["item"] == it}
        assert {(1, 1), (1, 2), (1, 3), (1, 4), (2, 1), (2, 2), (3, 3), (3, 4)} <= ev
        n_qk = sum(1 for r in rec if r["item"] == it and r["role"] == 2 and r["event"] == 1)
        n_pv = sum(1 for r in rec if r["item"] == it and r["role"] == 2 and r["event"] == 2)
        n_p = sum(1 for r in rec if r["item"] == it and r["role"] == 3 and r["event"] == 2)
        assert n_qk == n_pv == n_p == 3
    # detached: nothing more is appended
    n0 = buf[:4].clone()
    hb.hyb_attn_fwd(p, q, kc[0], kc[1], idx, kv[0], kv[1])
    torch.cuda.synchronize()
    assert torch.equal(buf[:4], n0)


def test_hca_attention_timeline(hb):
    # dense attention over every visible block plus the window: GQA pairs of
    # heads share an item's K / V tiles (query tiles A and B)
    g = torch.Generator().manual_seed(78)
    B, L, Hq, Hkv, d, m, W = 1, 700, 4, 2, 128, 16, 64
    Nc = L // m
    q = torch.randn((B, L, Hq, d), generator=g).to(torch.bfloat16).cuda()
    kv = [torch.randn((B, L, Hkv, d), generator=g).to(torch.bfloat16).cuda() for _ in range(2)]
    kc = [torch.randn((B, Nc, Hkv, d), generator=g).to(torch.bfloat16).cuda() for _ in range(2)]
    p = hb.problem(B=B, Lq=L, Lkv=L, Hq=Hq, Hkv=Hkv, d=d, m=m, W=W, Nc=Nc)
    ref = hb.hyb_attn_fwd(p, q, kc[0], kc[1], None, kv[0], kv[1])
    buf = torch.zeros(1 << 20, dtype=torch.int64, device="cuda")
    hb.hyb_trace_attach(buf)
    try:
        out = hb.hyb_attn_fwd(p, q, kc[0], kc[1], None, kv[0], kv[1])
        torch.cuda.synchronize()
    finally:
        hb.hyb_trace_attach(None)
    assert hb.hyb_get_device_status() == hb.HYB_OK
    assert torch.equal(out, ref)
    rec = hb.trace_records(buf)
    words = buf.cpu().numpy().view("uint64")
    cap = (words.size - 4) // 8
    for role in (0, 1, 2, 3):
        n = int(words[role])
        assert 0 < n <= cap, f"role {role}: {n} records"
        base = 4 + 2 * role * cap
        clk = words[base:base + 2 * n:2].astype(np.int64)
        assert np.all((words[base + 1:base + 2 * n:2] >> 56) == role)
        assert np.all(np.diff(clk) >= 0), f"role {role}: clocks out of order"
    for it in sorted({r["item"] for r in rec}):
        ev = [(r["role"], r["event"]) for r in rec if r["item"] == it]
        # both query tiles finish the item; every K tile loaded is matched by a
        # V tile, and each tile's scores and P are recorded by both softmaxes
        assert ev.count((3, 4)) == 1 and ev.count((0, 4)) == 1
        assert ev.count((1, 1)) == ev.count((1, 2)) >= 1
        for role, qk, pv in ((3, (2, 1), (2, 2)), (0, (2, 3), (2, 4))):
            assert ev.count(qk) == ev.count(pv) == ev.count((role, 1)) == ev.count((role, 2)) >= 1


def test_attention_backward_timeline(hb):
    # tensor-core backward of a dense problem: the key-tile pass records roles
    # 1-3 (producer, MMA, softmax thread 0), the query-tile pass role 0
    g = torch.Generator().manual_seed(79)
    B, L, Hq, Hkv, d, m, W = 1, 600, 2, 1, 128, 4, 128
    Nc = L // m
    q = torch.randn((B, L, Hq, d), generator=g).to(torch.bfloat16).cuda()
    kv = [torch.randn((B, L, Hkv, d), generator=g).to(torch.bfloat16).cuda() for _ in range(2)]
    kc = [torch.randn((B, Nc, Hkv, d), generator=g).to(torch.bfloat16).cuda() for _ in range(2)]
    dout = torch.randn((B, L, Hq, d), generator=g).to(torch.bfloat16).cuda()
    p = hb.problem(B=B, Lq=L, Lkv=L, Hq=Hq, Hkv=Hkv, d=d, m=m, W=W, Nc=Nc)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device="cuda")
    o = hb.hyb_attn_fwd(p, q, kc[0], kc[1], None, kv[0], kv[1], lse=lse)
    ref = hb.hyb_attn_bwd(p, q, kc[0], kc[1], None, kv[0], kv[1], o, lse, dout)
    buf = torch.zeros(1 << 20, dtype=torch.int64, device="cuda")
    hb.hyb_trace_attach(buf)
    try:
        got = hb.hyb_attn_bwd(p, q, kc[0], kc[1], None, kv[0], kv[1], o, lse, dout)
        torch.cuda.synchronize()
    finally:
        hb.hyb_trace_attach(None)
    assert hb.hyb_get_device_status() == hb.HYB_OK
    for name in ("dq", "dk_raw", "dv_raw"):
        assert torch.equal(got[name], ref[name]), name
    # dkc / dvc take reductions from several blocks: equal up to their order
    for name in ("dkc", "dvc"):
        assert torch.allclose(got[name], ref[name], rtol=1e-5, atol=1e-5), name
    rec = hb.trace_records(buf)
    words = buf.cpu().numpy().view("uint64")
    cap = (words.size - 4) // 8
    for role in (0, 1, 2, 3):
        n = int(words[role])
        assert 0 < n <= cap, f"role {role}: {n} records"
        base = 4 + 2 * role * cap
        clk = words[base:base + 2 * n:2].astype(np.int64)
        assert np.all((words[base + 1:base + 2 * n:2] >> 56) == role)
        assert np.all(np.diff(clk) >= 0), f"role {role}: clocks out of order"
    kv_items = sorted({r["item"] for r in rec if r["role"] in (1, 2, 3)})
    for it in kv_items:
        ev = [(r["role"], r["event"], r["tile"]) for r in rec if r["item"] == it]
        units = sorted({u for role, e, u in ev if role == 2 and e == 1})
        assert units, f"item {it}: no unit issued"
        for u in units:
            # per unit: columns staged, S^T / dP^T, dV and dK issued; P and dS written
            for key in ((1, 2), (2, 1), (2, 2), (2, 3), (3, 1), (3, 2), (3, 3)):
                assert (key[0], key[1], u) in ev, f"item {it} unit {u}: event {key} missing"
        # one epilogue per item, after its last dS
        ep = [r["clock"] for r in rec if r["item"] == it and r["role"] == 3 and r["event"] == 4]
        last_ds = max(r["clock"] for r in rec if r["item"] == it and r["role"] == 3 and r["event"] == 3)
        assert len(ep) == 1 and ep[0] >= last_ds
    # the query-tile pass: every S seen is followed by its dS, and each item
    # closes with one epilogue
    q_rec = [r for r in rec if r["role"] == 0]
    for it in sorted({r["item"] for r in q_rec}):
        ev = [r["event"] for r in q_rec if r["item"] == it]
        assert ev.count(1) == ev.count(3) >= 1 and ev.count(4) == ev.count(5) == 1
