"""Failure detection without a fault: every wait inside the kernels is
bounded.  With the bound cut to 1 ns the first wait that is not already
satisfied runs out, so the launch must still return, leave
HYB_ERR_DEVICE_TIMEOUT in the device status word, and keep the device usable:
the next launch with the normal bound reproduces the reference output.
Cases: the CSA attention kernel over many items (one CTA per item), the same
kernel on a few decode items (two CTAs of a cluster per item, waiting on each
other through distributed shared memory), and the one-kernel indexer +
top-K."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import compressed_sparse_sliding_b200 as hb
    return hb


def _randn(g, shape):
    return torch.randn(shape, generator=g).to(torch.bfloat16).cuda()


def _attention_case(hb, decode):
    g = torch.Generator().manual_seed(91 + decode)
    if decode:
        B, Lq, Lkv, Nc, K = 8, 1, 256, 1024, 256
        pos = torch.tensor([[1023 * 4 + 127 - b] for b in range(B)], dtype=torch.int32).cuda()
        kv0 = torch.tensor([1023 * 4 + 127 - b - 255 for b in range(B)], dtype=torch.int32).cuda()
    else:
        B, Lq, Lkv, Nc, K = 1, 300, 300, 75, 64
        pos = kv0 = None
    Hq, d = 64 if decode else 32, 128
    q = _randn(g, (B, Lq, Hq, d))
    kr, vr = _randn(g, (B, Lkv, 1, d)), _randn(g, (B, Lkv, 1, d))
    kc, vc = _randn(g, (B, Nc, 1, d)), _randn(g, (B, Nc, 1, d))
    idx = torch.stack([torch.randperm(Nc, generator=g)[:K].sort().values for _ in range(B * Lq)])
    idx = idx.to(torch.int32).reshape(B, Lq, K).cuda()
    p = hb.problem(B=B, Lq=Lq, Lkv=Lkv, Hq=Hq, Hkv=1, d=d, m=4, W=128, topk=K, Nc=Nc, q_pos=pos,
                   kv_pos0=kv0)
    return lambda: hb.hyb_attn_fwd(p, q, kc, vc, idx, kr, vr)


def _index_case(hb):
    g = torch.Generator().manual_seed(93)
    B, Lq, Hi, di, Nc, K = 1, 256, 4, 64, 2000, 64
    qi = _randn(g, (B, Lq, Hi, di))
    wi = torch.rand((B, Lq, Hi), generator=g).cuda()
    kic = _randn(g, (B, Nc, di))
    # m = 1, W = 0: row t sees t + 1 entries, so most rows select (all passes run);
    # no workspace, so the selection runs in the one kernel
    p = hb.problem(B=B, Lq=Lq, Lkv=Lq, Hq=4, Hkv=1, d=64, m=1, W=0, topk=K, Hi=Hi, di=di, Nc=Nc)
    return lambda: hb.hyb_csa_index_topk(p, qi, wi, kic, ws_bytes=0)


@pytest.mark.parametrize("case", ["csa_attention", "csa_attention_decode_split", "index_topk"])
def test_wait_timeout_is_reported_and_the_device_recovers(hb, case):
    run = _index_case(hb) if case == "index_topk" else _attention_case(hb, case.endswith("split"))
    ref = run()
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    hb.hyb_set_wait_limit_ns(1)
    try:
        run()
        torch.cuda.synchronize()
    finally:
        hb.hyb_set_wait_limit_ns(0)
    assert hb.hyb_get_device_status() == hb.HYB_ERR_DEVICE_TIMEOUT
    out = run()
    torch.cuda.synchronize()
    assert hb.hyb_get_device_status() == hb.HYB_OK
    assert torch.equal(out, ref)
