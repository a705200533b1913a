"""Pins of the decode cache maintenance oracle against plain definitions."""
import numpy as np

import oracle


def _bits(rng, shape):
    return (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_append_sequence_matches_whole_sequence_compression():
    # appending tokens one at a time leaves in the caches exactly the block_merge
    # of the whole raw sequence, and the window run of the ring holds the raw
    # rows of positions max(0, t-W+1) .. t at every step
    rng = np.random.default_rng(0)
    B, T, Hkv, d, di, m, W, Nc = 2, 53, 2, 16, 8, 4, 8, 16
    k = _bits(rng, (B, T, Hkv, d))
    v = _bits(rng, (B, T, Hkv, d))
    ki = _bits(rng, (B, T, di))
    wk = rng.standard_normal((m, d)).astype(np.float32)
    wv = rng.standard_normal((m, d)).astype(np.float32)
    wib = rng.standard_normal((m, di)).astype(np.float32)
    st = dict(k_ring=np.zeros((B, 2 * W, Hkv, d), np.uint16), v_ring=np.zeros((B, 2 * W, Hkv, d), np.uint16),
              ki_ring=np.zeros((B, W, di), np.uint16), kc=np.zeros((B, Nc, Hkv, d), np.uint16),
              vc=np.zeros((B, Nc, Hkv, d), np.uint16), kic=np.zeros((B, Nc, di), np.uint16))
    for t in range(T):
        kv0 = oracle.decode_append(st, [t] * B, k[:, t], v[:, t], wk, wv, m, W, ki_new_bits=ki[:, t],
                                   wib=wib)
        lo = max(0, t - W + 1)
        for b in range(B):
            base = int(kv0[b])
            assert base <= lo and lo - base < W and t - base < 2 * W
            np.testing.assert_array_equal(st["k_ring"][b, lo - base:t - base + 1], k[b, lo:t + 1])
            np.testing.assert_array_equal(st["v_ring"][b, lo - base:t - base + 1], v[b, lo:t + 1])
    nb = T // m
    _, kc = oracle.block_merge(k, wk, m)
    _, vc = oracle.block_merge(v, wv, m)
    _, kic = oracle.block_merge(ki[:, :, None, :], wib, m)
    np.testing.assert_array_equal(st["kc"][:, :nb], kc)
    np.testing.assert_array_equal(st["vc"][:, :nb], vc)
    np.testing.assert_array_equal(st["kic"][:, :nb], kic[:, :, 0])
    assert not st["kc"][:, nb:].any()     # no entry before its block completes


def test_block_equal_to_window():
    # m = W: the block that completes at t is exactly the whole window
    rng = np.random.default_rng(1)
    B, T, d, m, W = 1, 24, 8, 8, 8
    k = _bits(rng, (B, T, 1, d))
    w = rng.standard_normal((m, d)).astype(np.float32)
    st = dict(k_ring=np.zeros((B, 2 * W, 1, d), np.uint16), v_ring=np.zeros((B, 2 * W, 1, d), np.uint16),
              kc=np.zeros((B, 4, 1, d), np.uint16), vc=np.zeros((B, 4, 1, d), np.uint16))
    for t in range(T):
        oracle.decode_append(st, [t], k[:, t], k[:, t], w, w, m, W)
    _, kc = oracle.block_merge(k, w, m)
    np.testing.assert_array_equal(st["kc"][:, :3], kc)
