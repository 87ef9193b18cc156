"""Pins of the oracle's 4-bit group quantiser (the workload's format: keys per
channel over 32-token groups, values per token over 32-channel groups, fp16
scale and zero).  Checked against values on the group grid (exact round trip),
the worst-case error bound, the degenerate constant group, a hand example, and
the group orientation (a change confined to one group changes only its own
scale and zero)."""
import numpy as np
import pytest

import oracle
from oracle.quant import GROUP


def _f16(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def test_hand_example_k_group():
    # one channel, 32 tokens holding 0..15 twice: min 0, max 15 -> s = 1, z = 0
    x = np.tile(np.arange(16.0), 2).reshape(32, 1)
    q, s, z = oracle.quantize_k_groups(x)
    assert q[:, 0].tolist() == list(range(16)) * 2
    assert s.view(np.float16).astype(float).tolist() == [[1.0]]
    assert z.view(np.float16).astype(float).tolist() == [[0.0]]


def test_hand_example_v_group_negative_range():
    # 32 channels spanning [-3, 4.5]: s = 7.5 / 15 = 0.5, z = -3
    x = np.linspace(-3.0, 4.5, 32).reshape(1, 32)
    q, s, z = oracle.quantize_v_groups(x)
    assert float(s.view(np.float16)[0, 0]) == 0.5
    assert float(z.view(np.float16)[0, 0]) == -3.0
    want = np.clip(np.rint((x + 3.0) / 0.5), 0, 15)
    assert np.array_equal(q, want.astype(np.uint8))
    xh = oracle.dequant_v_groups(q, s, z)
    assert np.abs(xh - x).max() <= 0.25 + 1e-12


@pytest.mark.parametrize("which", ["k", "v"])
def test_grid_values_round_trip_exactly(which):
    rng = np.random.default_rng(0)
    T, D = 64, 64
    if which == "k":
        s = _f16(rng.uniform(0.01, 2.0, size=(T // GROUP, 1, D)))
        z = _f16(rng.uniform(-5, 5, size=(T // GROUP, 1, D)))
        qq = rng.integers(0, 16, size=(T // GROUP, GROUP, D))
        qq[:, 0, :], qq[:, 1, :] = 0, 15        # min and max attained
        x = (qq * s + z).reshape(T, D)
        q, sb, zb = oracle.quantize_k_groups(x)
        xh = oracle.dequant_k_groups(q, sb, zb)
    else:
        s = _f16(rng.uniform(0.01, 2.0, size=(T, D // GROUP, 1)))
        z = _f16(rng.uniform(-5, 5, size=(T, D // GROUP, 1)))
        qq = rng.integers(0, 16, size=(T, D // GROUP, GROUP))
        qq[:, :, 0], qq[:, :, 1] = 0, 15
        x = (qq * s + z).reshape(T, D)
        q, sb, zb = oracle.quantize_v_groups(x)
        xh = oracle.dequant_v_groups(q, sb, zb)
    # (max - min)/15 == s exactly and fp16(min) == z, so every value comes back
    assert np.array_equal(q.reshape(qq.shape), qq.astype(np.uint8))
    assert np.array_equal(xh, x)


@pytest.mark.parametrize("which", ["k", "v"])
def test_error_bound(which):
    """|x_hat - x| <= s/2 + |z - min| + 15 |s - (max-min)/15| for every element."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 96, 64)) * np.where(rng.random((1, 1, 64)) < 0.05, 10, 1)
    if which == "k":
        q, sb, zb = oracle.quantize_k_groups(x)
        xh = oracle.dequant_k_groups(q, sb, zb)
        g = x.reshape(2, 3, GROUP, 64)
        mn, mx = g.min(axis=2), g.max(axis=2)                     # [2,3,64]
        s = sb.view(np.float16).astype(float)
        z = zb.view(np.float16).astype(float)
        bound = s / 2 + np.abs(z - mn) + 15 * np.abs(s - (mx - mn) / 15)
        bound = np.repeat(bound, GROUP, axis=1)
    else:
        q, sb, zb = oracle.quantize_v_groups(x)
        xh = oracle.dequant_v_groups(q, sb, zb)
        g = x.reshape(2, 96, 2, GROUP)
        mn, mx = g.min(axis=3), g.max(axis=3)                     # [2,96,2]
        s = sb.view(np.float16).astype(float)
        z = zb.view(np.float16).astype(float)
        bound = s / 2 + np.abs(z - mn) + 15 * np.abs(s - (mx - mn) / 15)
        bound = np.repeat(bound, GROUP, axis=2)
    assert (np.abs(xh - x) <= bound * (1 + 1e-12) + 1e-15).all()
    assert q.max() <= 15


def test_constant_group_uses_unit_scale():
    x = np.full((32, 3), 0.7)
    q, s, z = oracle.quantize_k_groups(x)
    assert (q == 0).all()
    assert (s.view(np.float16) == 1.0).all()
    xh = oracle.dequant_k_groups(q, s, z)
    assert np.allclose(xh, np.float16(0.7), atol=0)


def test_k_groups_run_along_tokens_v_groups_along_channels():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 64))
    _, sk, zk = oracle.quantize_k_groups(x)
    _, sv, zv = oracle.quantize_v_groups(x)
    assert sk.shape == (2, 64) and sv.shape == (64, 2)
    y = x.copy()
    y[40, 5] = 50.0                          # token 40 (k group 1), channel 5 (v group 0)
    _, sk2, zk2 = oracle.quantize_k_groups(y)
    _, sv2, zv2 = oracle.quantize_v_groups(y)
    changed_k = np.argwhere(sk2 != sk)
    changed_v = np.argwhere(sv2 != sv)
    assert changed_k.tolist() == [[1, 5]]
    assert changed_v.tolist() == [[40, 0]]
