"""Per-stage parity of the CUDA kernels against the oracle, on small shapes that
span several tiles and a ragged tail, plus the method's degenerate cases.
Each stage gets identical inputs on both sides (oracle outputs may feed the
GPU; nothing from the GPU feeds the oracle)."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import (abs_merge, bits, check_bf16_cache, check_lse, check_output, check_topk,
                          from_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import compressed_sparse_sliding_b200 as hb
    return hb


def _randn_bf16(g, shape, scale=1.0):
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


# ----------------------------------------------------------------- block_merge
@pytest.mark.parametrize("B,L,H,dx,m", [
    (2, 37, 3, 64, 4),
    (1, 1000, 2, 128, 128),
    (2, 8192, 16, 128, 128),
    (1, 513, 1, 32, 4),
    (1, 64, 2, 64, 1),
    (3, 130, 1, 64, 3),
    (1, 300, 3, 64, 8),
    (2, 257, 2, 128, 16),
    (1, 1100, 5, 64, 64),
    (1, 700, 2, 256, 128),
    (2, 99, 4, 128, 2),
])
def test_block_merge_matches_oracle(hb, B, L, H, dx, m):
    g = torch.Generator().manual_seed(B * 1000 + L + m)
    x = _randn_bf16(g, (B, L, H, dx))
    w = torch.randn((m, dx), generator=g)
    out = hb.hyb_hca_compress(x.cuda(), w.cuda(), m)
    torch.cuda.synchronize()
    _, ref = oracle.block_merge(bits(x), w.numpy(), m)
    check_bf16_cache(out, ref, "block_merge", abs_merge(bits(x), w.numpy(), m), m)
    assert hb.hyb_get_device_status() == hb.HYB_OK


# ------------------------------------------------------------ indexer + top-K
def _index_case(hb, B, Lq, Hi, di, Nc, m, W, K, q_pos=None, seed=0, rows=None, pool=0, neg_w=False,
                ramp=False, one_kernel=False):
    g = torch.Generator().manual_seed(seed)
    qi = _randn_bf16(g, (B, Lq, Hi, di))
    wi = torch.rand((B, Lq, Hi), generator=g)
    if neg_w:
        wi = wi * 2 - 1          # signed head weights: scores of either sign
    kic = _randn_bf16(g, (B, Nc, di))
    if ramp:
        # every key a scaled copy of one vector: each row's scores grow with
        # the entry index, so its largest scores sit past any sampled entry
        base = torch.randn((B, 1, di), generator=g)
        kic = (base * (0.5 + torch.arange(Nc).reshape(1, Nc, 1) / Nc)).to(torch.bfloat16)
    if pool:
        # entries drawn from `pool` distinct rows: every score value repeats,
        # so the K-th score is an exact tie broken toward the lower index
        pick = torch.randint(0, pool, (B, Nc), generator=g)
        kic = torch.stack([kic[b, pick[b]] for b in range(B)])
    qp = None if q_pos is None else torch.as_tensor(q_pos, dtype=torch.int32).reshape(B, Lq)
    p = hb.problem(B=B, Lq=Lq, Lkv=max(W, 1), Hq=4, Hkv=1, d=64, m=m, W=W, topk=K, Hi=Hi, di=di,
                   Nc=Nc, q_pos=None if qp is None else qp.cuda())
    sel_scores = torch.empty((B, Lq, K), dtype=torch.float32, device="cuda")
    # one_kernel: no workspace, so shapes the one-kernel selection takes run there
    idx = hb.hyb_csa_index_topk(p, qi.cuda(), wi.cuda(), kic.cuda(), sel_scores=sel_scores,
                                ws_bytes=0 if one_kernel else None)
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    sc, nv = oracle.index_scores(bits(qi), wi.numpy(), bits(kic), m, W,
                                 q_pos=None if qp is None else qp.numpy(), rows=rows)
    ref = oracle.topk(sc, nv, K)
    got = idx.reshape(B * Lq, K).cpu().numpy()
    if rows is not None:
        got = got[np.asarray(rows)]
    exact = check_topk(got, ref, sc, nv, K)
    # the selected scores agree with the oracle's fp64 scores
    ss = sel_scores.reshape(B * Lq, K).cpu().numpy()
    if rows is not None:
        ss = ss[np.asarray(rows)]
    for r in range(len(got)):
        sel = got[r] >= 0
        want = sc[r, got[r][sel]]
        np.testing.assert_allclose(ss[r][sel], want, rtol=1e-4, atol=1e-4)
        assert np.all(np.isneginf(ss[r][~sel]))
    return exact


@pytest.mark.parametrize("one_kernel", [False, True])
def test_index_topk_tiny_workload_shape(hb, one_kernel):
    # the tiny CSA workload: L=1024, 2 indexer heads of dim 32, m=4, W=128, K=16
    # (its 1 MB of score rows go to the two-kernel path unless no workspace is given)
    exact = _index_case(hb, 1, 1024, 2, 32, 256, 4, 128, 16, seed=1, one_kernel=one_kernel)
    assert exact.mean() > 0.95


@pytest.mark.parametrize("one_kernel", [False, True])
def test_index_topk_ragged_and_small_K(hb, one_kernel):
    _index_case(hb, 2, 333, 4, 64, 83, 4, 8, 5, seed=2, one_kernel=one_kernel)
    _index_case(hb, 1, 200, 3, 32, 66, 3, 0, 64, seed=3, one_kernel=one_kernel)   # W = 0, K > n_vis early


def test_index_topk_decode_positions(hb):
    # one query per sequence at an absolute position, 2048-entry cache, K = 256
    B, Nc = 4, 2048
    pos = [[8191], [5000], [300], [130]]
    _index_case(hb, B, 1, 4, 64, Nc, 4, 128, 256, q_pos=pos, seed=4)


def test_index_topk_decode_workload_shape(hb):
    # the decode workload's selection: K = 1024 of 16352 visible entries of a
    # 16384-entry cache, one query per sequence at the last context position
    B, Nc = 8, 16384
    pos = [[65535 - 5 * b] for b in range(B)]
    exact = _index_case(hb, B, 1, 4, 64, Nc, 4, 128, 1024, q_pos=pos, seed=6)
    assert exact.sum() >= 1


def test_index_topk_large_rows_sampled(hb):
    # entries per row as in the long CSA prefill (up to 8160 visible), sampled rows
    rows = list(range(0, 32768, 997)) + [32767, 520, 521]
    _index_case(hb, 1, 32768, 4, 64, 8192, 4, 128, 512, seed=5, rows=rows)


@pytest.mark.parametrize("Nc,pool", [(3001, 16), (8192, 7), (12000, 16), (16384, 0), (20000, 16)])
def test_index_topk_exact_ties_and_row_lengths(hb, Nc, pool):
    # one query per sequence near the end of the cache, rows of every length
    # class of the selection kernels; pooled keys make the threshold a tie
    B, m, W, K = 3, 4, 128, 300
    L = Nc * m + W
    pos = [[L - 1], [L // 2], [L - 1 - 7 * m]]
    exact = _index_case(hb, B, 1, 4, 64, Nc, m, W, K, q_pos=pos, seed=Nc + pool, pool=pool)
    if pool:
        assert exact.all()   # exact ties are compared index for index


@pytest.mark.parametrize("one_kernel", [False, True])
@pytest.mark.parametrize("Nc,pool", [(3000, 0), (3000, 16), (8192, 0), (12000, 16)])
def test_index_topk_many_rows(hb, Nc, pool, one_kernel):
    # 1500 query rows at spread positions: the narrow per-row selection CTAs
    B, Lq, m, W, K = 3, 500, 4, 128, 300
    L = Nc * m + W
    rng = np.random.default_rng(Nc)
    pos = rng.integers(0, L, size=(B, Lq)).astype(np.int32)
    pos[0, :4] = [L - 1, W + K * m + 3, W + K * m - 5, 0]
    rows = [0, 1, 2, 3] + sorted(rng.choice(B * Lq, size=40, replace=False).tolist())
    exact = _index_case(hb, B, Lq, 4, 64, Nc, m, W, K, q_pos=pos, seed=Nc + 7 * pool, pool=pool,
                        rows=rows, one_kernel=one_kernel)
    if pool:
        assert exact.all()


@pytest.mark.parametrize("case", ["ramp", "signed", "two_values", "random_pos", "all_visible", "k1",
                                  "short_rows"])
def test_index_topk_selection_paths(hb, case):
    # prefill-shaped problems given no workspace select in one kernel that
    # recomputes the scores pass by pass and moves or narrows a per-row key window until the K-th
    # score is pinned; each case drives one of its paths
    rng = np.random.default_rng(len(case))
    if case == "ramp":          # the K-th score lies above every sampled score
        _index_case(hb, 1, 700, 4, 64, 3000, 4, 128, 300, seed=11, ramp=True, one_kernel=True)
    elif case == "signed":      # negative scores (order keys below +0)
        _index_case(hb, 2, 400, 3, 64, 2500, 4, 64, 200, seed=12, neg_w=True, one_kernel=True)
    elif case == "two_values":  # two distinct keys: the threshold bin is one exact score
        exact = _index_case(hb, 1, 520, 4, 32, 2000, 4, 128, 100, seed=13, pool=2, one_kernel=True)
        assert exact.all()
    elif case == "random_pos":  # rows of one tile with very different visible counts
        L = 4000 * 4 + 128
        pos = rng.integers(0, L, size=(2, 300)).astype(np.int32)
        _index_case(hb, 2, 300, 4, 64, 4000, 4, 128, 256, q_pos=pos, seed=14, one_kernel=True)
    elif case == "all_visible":  # K >= every row's visible count
        _index_case(hb, 1, 777, 2, 64, 190, 4, 16, 200, seed=15, one_kernel=True)
    elif case == "k1":
        _index_case(hb, 1, 300, 4, 64, 500, 4, 32, 1, seed=16, one_kernel=True)
    else:                       # rows shorter than one sampled tile
        _index_case(hb, 1, 200, 2, 32, 60, 2, 64, 7, seed=17, one_kernel=True)


# ----------------------------------------------------------------- attention
def _attn_case(hb, B, L, Hq, Hkv, d, m, W, K=0, seed=0, scale=None, lse=True, rows=None):
    g = torch.Generator().manual_seed(seed)
    q = _randn_bf16(g, (B, L, Hq, d))
    k = _randn_bf16(g, (B, L, Hkv, d))
    v = _randn_bf16(g, (B, L, Hkv, d))
    Nc = L // m
    kc = _randn_bf16(g, (B, Nc, Hkv, d))
    vc = _randn_bf16(g, (B, Nc, Hkv, d))
    idx = None
    if K:
        rng = np.random.default_rng(seed)
        idx = np.full((B, L, K), -1, np.int32)
        for b in range(B):
            for t in range(L):
                nv = oracle.visible_count(t, m, W, Nc)
                if nv:
                    s = np.sort(rng.choice(nv, size=min(K, nv), replace=False))
                    idx[b, t, :len(s)] = s
    p = hb.problem(B=B, Lq=L, Lkv=L, Hq=Hq, Hkv=Hkv, d=d, m=m, W=W, topk=K, Nc=Nc,
                   scale=scale or 0.0)
    lse_t = torch.empty((B, Hq, L), dtype=torch.float32, device="cuda") if lse else None
    o = hb.hyb_attn_fwd(p, q.cuda(), kc.cuda(), vc.cuda(),
                        None if idx is None else torch.from_numpy(idx).cuda(), k.cuda(), v.cuda(),
                        lse=lse_t)
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    ref = oracle.hybrid_attention(bits(q), bits(kc), bits(vc), idx, bits(k), bits(v), m, W,
                                  scale=scale, rows=rows)
    og = o if rows is None else o.reshape(B * L, Hq, d)[torch.as_tensor(rows, device=o.device)]
    check_output(og, ref["o"])
    if lse:
        lg = lse_t.permute(0, 2, 1).reshape(B * L, Hq).cpu().numpy()
        check_lse(lg if rows is None else lg[np.asarray(rows)], ref["lse"])
    return o, ref


@pytest.mark.parametrize("d", [64, 128])
def test_dense_attention_ragged_tiles(hb, d):
    # 300 queries = 2 full 128-row tiles + a ragged one; GQA 4 query heads on 2 KV heads
    _attn_case(hb, 2, 300, 4, 2, d, 8, 32, seed=d)


def test_dense_attention_hca_blocks(hb):
    # m = 128 blocks, W = 128, several compressed tiles per query tile
    _attn_case(hb, 1, 1100, 2, 1, 128, 4, 128, seed=11)
    _attn_case(hb, 1, 700, 2, 2, 64, 128, 128, seed=12)


@pytest.mark.parametrize("d", [64, 128])
def test_sparse_attention_given_indices(hb, d):
    # CSA shape: MQA, K selected entries + 128-token window; several key tiles
    _attn_case(hb, 1, 700, 4, 1, d, 4, 128, K=160, seed=20 + d)


@pytest.mark.parametrize("Hq,Hkv,K,W,L", [
    (32, 1, 300, 128, 1700),     # 32-head group, ragged selection tile
    (40, 2, 200, 64, 1300),      # GQA, 20 heads per group padded to 32
    (32, 1, 768, 128, 3400),     # 6 + 1 tiles: a full 32-head token buffer
    (16, 1, 1792, 128, 7400),    # 14 + 1 tiles: a full 16-head token buffer
    (32, 1, 200, 0, 1000),       # no window
    (32, 1, 1000, 128, 4300),    # 8 + 1 tiles: past the token buffer, lazy-softmax kernel
])
def test_sparse_attention_d128_groups(hb, Hq, Hkv, K, W, L):
    # head dim 128 with every group width and tile count around the kernel limits;
    # early, middle and late tokens plus a spread sample
    rng = np.random.default_rng(L + K)
    rows = sorted(set([0, 5, W + 3, L // 3, L // 2, L - 2, L - 1] +
                      rng.choice(L, size=24, replace=False).tolist()))
    _attn_case(hb, 1, L, Hq, Hkv, 128, 4, W, K=K, seed=60 + K, rows=rows)


def test_sparse_attention_gqa_groups(hb):
    _attn_case(hb, 2, 150, 8, 2, 64, 4, 16, K=24, seed=30)


def test_degenerate_shapes(hb):
    _attn_case(hb, 1, 90, 2, 1, 64, 4, 128, seed=40)          # L < W: window only
    _attn_case(hb, 1, 50, 2, 1, 64, 64, 8, seed=41)           # L < m: no compressed entry
    _attn_case(hb, 1, 77, 2, 1, 64, 4, 0, seed=42)            # W = 0: empty rows t < 3
    _attn_case(hb, 1, 77, 2, 1, 64, 4, 0, K=8, seed=43)       # W = 0, sparse
    _attn_case(hb, 1, 140, 2, 2, 64, 1, 0, seed=44)           # m = 1, W = 0: causal attention
    _attn_case(hb, 1, 64, 4, 1, 64, 4, 16, K=600, seed=45)    # K > every n_vis


def test_decode_form(hb):
    # Lq = 1 per sequence at position t_b; raw buffer of the last W rows
    g = torch.Generator().manual_seed(50)
    B, Hq, d, m, W, Nc, K = 3, 16, 128, 4, 128, 1024, 64
    pos = np.array([4095, 2000, 700], np.int32)
    q = _randn_bf16(g, (B, 1, Hq, d))
    kr = _randn_bf16(g, (B, W, 1, d))
    vr = _randn_bf16(g, (B, W, 1, d))
    kc = _randn_bf16(g, (B, Nc, 1, d))
    vc = _randn_bf16(g, (B, Nc, 1, d))
    rng = np.random.default_rng(50)
    idx = np.full((B, 1, K), -1, np.int32)
    for b in range(B):
        nv = oracle.visible_count(int(pos[b]), m, W, Nc)
        idx[b, 0, :min(K, nv)] = np.sort(rng.choice(nv, size=min(K, nv), replace=False))
    qp = torch.from_numpy(pos.reshape(B, 1))
    kv0 = torch.from_numpy(pos - W + 1)
    for use_idx in (True, False):
        p = hb.problem(B=B, Lq=1, Lkv=W, Hq=Hq, Hkv=1, d=d, m=m, W=W, topk=K if use_idx else 0,
                       Nc=Nc, q_pos=qp.cuda(), kv_pos0=kv0.cuda())
        o = hb.hyb_attn_fwd(p, q.cuda(), kc.cuda(), vc.cuda(),
                            torch.from_numpy(idx).cuda() if use_idx else None, kr.cuda(), vr.cuda())
        torch.cuda.synchronize()
        ref = oracle.hybrid_attention(bits(q), bits(kc), bits(vc), idx if use_idx else None,
                                      bits(kr), bits(vr), m, W, q_pos=pos.reshape(B, 1),
                                      kv_pos0=(pos - W + 1).astype(np.int32))
        check_output(o, ref["o"])


@pytest.mark.parametrize("B,Hq,Hkv,K", [(5, 32, 1, 700), (4, 64, 2, 1024), (64, 64, 1, 1024)])
def test_decode_group_widths(hb, B, Hq, Hkv, K):
    # decode: one query per sequence, 32- and 64-head groups, GQA, selections
    # of up to 1024 entries; early positions leave selection slots empty
    g = torch.Generator().manual_seed(70 + K)
    d, m, W, Nc = 128, 4, 128, 2048
    rng = np.random.default_rng(70 + K)
    pos = rng.integers(W + 1, Nc * m + W, size=B).astype(np.int32)
    pos[0] = Nc * m + W - 1
    pos[-1] = W + 40 * m          # only 40 visible entries
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
    qp = torch.from_numpy(pos.reshape(B, 1))
    kv0 = torch.from_numpy(pos - W + 1)
    p = hb.problem(B=B, Lq=1, Lkv=W, Hq=Hq, Hkv=Hkv, d=d, m=m, W=W, topk=K, Nc=Nc,
                   q_pos=qp.cuda(), kv_pos0=kv0.cuda())
    lse_t = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
    o = hb.hyb_attn_fwd(p, q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(idx).cuda(), kr.cuda(),
                        vr.cuda(), lse=lse_t)
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    ref = oracle.hybrid_attention(bits(q), bits(kc), bits(vc), idx, bits(kr), bits(vr), m, W,
                                  q_pos=pos.reshape(B, 1), kv_pos0=(pos - W + 1).astype(np.int32))
    check_output(o, ref["o"])
    check_lse(lse_t.reshape(B, Hq).cpu().numpy(), ref["lse"])


@pytest.mark.parametrize("d", [64, 128])
def test_out_of_range_index_is_reported_not_read(hb, d):
    g = torch.Generator().manual_seed(60)
    B, L, Hq, m, W, K = 1, 64, 4, 4, 8, 4
    Nc = L // m
    q = _randn_bf16(g, (B, L, Hq, d)).cuda()
    k = _randn_bf16(g, (B, L, 1, d)).cuda()
    kc = _randn_bf16(g, (B, Nc, 1, d)).cuda()
    idx = torch.full((B, L, K), -1, dtype=torch.int32)
    idx[0, 40, 0] = Nc + 5
    p = hb.problem(B=B, Lq=L, Lkv=L, Hq=Hq, Hkv=1, d=d, m=m, W=W, topk=K, Nc=Nc)
    hb.hyb_attn_fwd(p, q, kc, kc, idx.cuda(), k, k)
    assert hb.hyb_get_device_status() == hb.HYB_ERR_DEVICE_BOUNDS
    assert hb.hyb_get_device_status() == hb.HYB_OK  # read clears it


# ------------------------------------------------------------ gather probes
@pytest.mark.parametrize("stages", [2, 6])
def test_l2_gather_probes_land_rows_where_the_attention_reads_them(hb, stages):
    """Both measurement probes run to completion; the tile::gather4 form puts
    every 16-byte chunk of its last stage where the 128-byte swizzle of the
    attention's K / V tiles expects it (sink[256] counts misplaced chunks)."""
    dev = torch.device("cuda")
    table = torch.randint(0, 1 << 30, ((1 << 20) // 4,), dtype=torch.int32, device=dev)
    sink = torch.zeros(257, dtype=torch.int32, device=dev)
    hb.hyb_probe_l2_gather(table, 128 * 8, stages, sink)
    sink.zero_()
    hb.hyb_probe_l2_gather_tma(table, 128 * 8, stages, sink)
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == 0
    assert int(sink[256].item()) == 0
    assert int(sink[:256].abs().sum().item()) != 0   # the copied words reached the checksum
