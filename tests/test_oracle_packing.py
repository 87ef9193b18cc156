"""Pins of the 4-bit storage layout and of the int4 draft attention.

The layout is this library's own (the pages fix none); these tests check the
pack/unpack pair against the layout's written rule at hand-picked positions,
the round trip, and that the int4 draft equals draft attention over the
original values when those values sit exactly on the quantisation grid
(dequantisation is then exact)."""
import numpy as np

import oracle
from oracle import packing


def test_k_word_positions_follow_the_rule():
    D, T = 128, 32
    nib = np.zeros((T, D), dtype=np.uint8)
    nib[0, 0], nib[0, 1], nib[0, 8], nib[0, 9] = 1, 2, 3, 4
    nib[5, 34], nib[5, 35] = 7, 9         # e = 34: c = 1, w = 1, j = 0
    words = packing.pack_k(nib)           # [1, 32, 4, 4]
    w = int(words[0, 0, 0, 0])
    # channel 0 -> pair 0 first (nibble 0), channel 1 -> pair 0 second (nibble 4)
    # channel 8 -> pair 1 first (nibble 1), channel 9 -> pair 1 second (nibble 5)
    assert w == (1 << 0) | (2 << 16) | (3 << 4) | (4 << 20)
    assert int(words[0, 5, 1, 1]) == (7 << 0) | (9 << 16)
    assert packing.k_channel_of(3, 3, 3) == 6 + 96 + 16 + 8


def test_v_word_positions_follow_the_rule():
    D, T = 64, 64
    nib = np.zeros((T, D), dtype=np.uint8)
    nib[32 + 2, 7], nib[32 + 3, 7] = 5, 6     # block 1, tokens 2,3: c = 1, j = 0
    nib[32 + 10, 7] = 11                      # token 10: c = 1, j = 1 (first)
    words = packing.pack_v(nib)               # [2, 64, 4]
    assert int(words[1, 7, 1]) == (5 << 0) | (6 << 16) | (11 << 4)
    assert int(words[0, 7, 1]) == 0


def test_round_trips():
    rng = np.random.default_rng(0)
    for D in (64, 128):
        nib = rng.integers(0, 16, size=(2, 3, 96, D), dtype=np.uint8)
        assert np.array_equal(packing.unpack_k(packing.pack_k(nib), D), nib)
        assert np.array_equal(packing.unpack_v(packing.pack_v(nib)), nib)
    bits = rng.integers(0, 65535, size=(2, 96, 4), dtype=np.uint16)
    blk = packing.v_scales_to_blocks(bits)
    assert blk.shape == (2, 3, 4, 32)
    assert blk[1, 2, 3, 5] == bits[1, 2 * 32 + 5, 3]
    assert np.array_equal(packing.v_scales_from_blocks(blk), bits)


def test_int4_draft_equals_exact_draft_on_grid_values():
    rng = np.random.default_rng(1)
    B, Hq, Hkv, D, T, R = 2, 8, 2, 64, 96, 5
    f16 = lambda x: x.astype(np.float16).astype(np.float64)
    ks = f16(rng.uniform(0.05, 0.5, size=(B, Hkv, T // 32, 1, D)))
    kz = f16(rng.uniform(-2, 0, size=(B, Hkv, T // 32, 1, D)))
    kn = rng.integers(0, 16, size=(B, Hkv, T // 32, 32, D))
    kn[:, :, :, 0], kn[:, :, :, 1] = 0, 15
    K = (kn * ks + kz).reshape(B, Hkv, T, D)
    vs = f16(rng.uniform(0.05, 0.5, size=(B, Hkv, T, D // 32, 1)))
    vz = f16(rng.uniform(-2, 0, size=(B, Hkv, T, D // 32, 1)))
    vn = rng.integers(0, 16, size=(B, Hkv, T, D // 32, 32))
    vn[..., 0], vn[..., 1] = 0, 15
    V = (vn * vs + vz).reshape(B, Hkv, T, D)
    q = rng.standard_normal((B, Hq, D))
    kt, vt = rng.standard_normal((B, Hkv, R, D)), rng.standard_normal((B, Hkv, R, D))

    qk, sk, zk = oracle.quantize_k_groups(K)
    qv, sv, zv = oracle.quantize_v_groups(V)
    o4, l4 = oracle.draft_attn_int4(
        q, packing.pack_k(qk), sk, zk, packing.pack_v(qv),
        packing.v_scales_to_blocks(sv), packing.v_scales_to_blocks(zv), kt, vt)
    o, l = oracle.draft_attn(q, K, V, T, None, None, kt, vt)
    np.testing.assert_allclose(o4, o, atol=1e-13)
    np.testing.assert_allclose(l4, l, atol=1e-12)
