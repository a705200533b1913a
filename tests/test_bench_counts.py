"""The benchmark's algorithmic counts (the roofline numerators) against the
figures derived independently from the visibility formulas (keys per query
token and attention FLOP per workload) and against hand-counted bytes."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import WORKLOADS  # noqa: E402

# keys per query token (selected or visible compressed + window) and
# attention GFLOP (4 d Hq keys) per workload
EXPECTED = {1: (133.5, 0.14), 2: (157.5, 21.1), 3: (621.7, 333.8), 4: (638.4, 2742.0), 5: (1152.0, 2.42)}


@pytest.mark.parametrize("no", sorted(EXPECTED))
def test_keys_and_flop(no):
    w = WORKLOADS[no]
    c = bench.algorithmic_counts(w)
    keys, gflop = EXPECTED[no]
    assert c["attn_keys"] / (w.B * w.Lq) == pytest.approx(keys, abs=0.05)
    assert c["attn_flop"] / 1e9 == pytest.approx(gflop, rel=5e-3)


def test_decode_bytes_bf16_and_4bit():
    w = WORKLOADS[5]
    q_o = 2 * 64 * 1 * 64 * 128 * 2
    idx = 64 * 1024 * 4
    # 1024 selected compressed rows and 128 window rows of K and V per sequence
    bf16 = q_o + 64 * (1024 * 256 + 128 * 256) * 2 + idx
    assert bench.algorithmic_counts(w)["attn_bytes"] == bf16 == 40_108_032
    # 4-bit compressed rows: 64 bytes of codes + 8 bytes of (min, scale)
    fp4 = q_o + 64 * (1024 * 72 + 128 * 256) * 2 + idx
    assert bench.algorithmic_counts(w, fp4=True)["attn_bytes"] == fp4
    # the indexer streams every visible key once: 16352 per sequence
    assert bench.algorithmic_counts(w)["idx_bytes"] == 64 * 16352 * 128 + 64 * 4 * 64 * 2 + idx
    assert bench.algorithmic_counts(w, fp4=True)["idx_bytes"] == 64 * 16352 * 40 + 64 * 4 * 64 * 2 + idx


def test_hca_prefill_bytes():
    # q and o, raw K and V, compressed K and V: the unique bytes of the step
    w = WORKLOADS[2]
    b = 2 * 8192 * 16 * 128 * 2
    assert bench.algorithmic_counts(w)["attn_bytes"] == 2 * b + 2 * b + 2 * (2 * 64 * 16 * 128 * 2)
