"""hyb_csa_index_topk_noalloc against hyb_csa_index_topk.

Some callers may not allocate device memory themselves -- an engine whose
memory planner owns every buffer, or a decode loop in which cudaMalloc /
cudaFree would synchronise the device -- so they cannot supply the indexer's
workspace.  The no-allocation entry point keeps the score scratch in a fixed
array inside the library instead.  These tests call it through the C ABI and
require exactly the selection (and selected scores) of the workspace entry
point, on two calls in a row with different inputs, so that contents left in
the shared scratch by the first call cannot leak into the second.

This file is named to be collected last.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import compressed_sparse_sliding_b200 as hb
    return hb


def _entry(hb):
    f = hb._lib.hyb_csa_index_topk_noalloc
    f.argtypes = [ctypes.POINTER(hb.HybProblem)] + [ctypes.c_void_p] * 6
    f.restype = ctypes.c_int
    return f


def _vp(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


CASES = {
    # decode: one query per sequence at its absolute position, 16384-entry caches
    "decode": dict(B=16, Lq=1, Nc=16384, Hi=4, di=64, m=4, W=128, K=1024,
                   pos=lambda B: torch.tensor([[65535 - 97 * b] for b in range(B)],
                                              dtype=torch.int32)),
    # prefill of the tiny CSA workload's shape
    "prefill": dict(B=1, Lq=1024, Nc=256, Hi=2, di=32, m=4, W=128, K=16, pos=None),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_the_workspace_entry_point(hb, name):
    c = CASES[name]
    f = _entry(hb)
    for call in range(2):
        g = torch.Generator().manual_seed(1000 * call + len(name))
        qi = torch.randn((c["B"], c["Lq"], c["Hi"], c["di"]), generator=g).to(torch.bfloat16).cuda()
        wi = torch.rand((c["B"], c["Lq"], c["Hi"]), generator=g).cuda()
        kic = torch.randn((c["B"], c["Nc"], c["di"]), generator=g).to(torch.bfloat16).cuda()
        qp = c["pos"](c["B"]).cuda() if c["pos"] else None
        p = hb.problem(B=c["B"], Lq=c["Lq"], Lkv=c["W"], Hq=4, Hkv=1, d=64, m=c["m"], W=c["W"],
                       topk=c["K"], Hi=c["Hi"], di=c["di"], Nc=c["Nc"], q_pos=qp)
        sel_ref = torch.empty((c["B"], c["Lq"], c["K"]), dtype=torch.float32, device="cuda")
        idx_ref = hb.hyb_csa_index_topk(p, qi, wi, kic, sel_scores=sel_ref)
        idx = torch.full_like(idx_ref, 7)
        sel = torch.full_like(sel_ref, 3.0)
        st = f(ctypes.byref(p), _vp(qi), _vp(wi), _vp(kic), _vp(idx), _vp(sel),
               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == hb.HYB_OK, hb.hyb_error_string(st)
        torch.cuda.synchronize()
        assert hb.hyb_get_device_status() == hb.HYB_OK
        assert torch.equal(idx, idx_ref), f"call {call}: selection differs"
        assert torch.equal(sel, sel_ref), f"call {call}: selected scores differ"


def test_noalloc_rejects_problems_beyond_its_scratch(hb):
    f = _entry(hb)
    # 64 rows x 40000 entries x 4 B ~ 10 MB > the 8 MiB scratch: refused, nothing launched (Nc
    # stays under the top-K's shared-memory limit, so only the scratch size refuses it)
    p = hb.problem(B=64, Lq=1, Lkv=128, Hq=4, Hkv=1, d=64, m=4, W=128, topk=64, Hi=4, di=64,
                   Nc=40000)
    buf = torch.empty(256, dtype=torch.uint8, device="cuda")
    st = f(ctypes.byref(p), _vp(buf), _vp(buf), _vp(buf), _vp(buf), None, None)
    assert st == hb.HYB_ERR_UNSUPPORTED
