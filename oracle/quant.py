"""Asymmetric 4-bit group quantisation of the compressed cache, float64.

Quantisation is one of the lossy compressors the VeriCache summary plugs into its
uniform compression interface (section "Supporto Architetturale", last
paragraph) and the CentroidKV summary lists it among the known reductions of
the KV cache (section "Problematica").  Neither page fixes a format; the
workload fixes this one: keys per channel over groups of 32 consecutive tokens,
values per token over groups of 32 consecutive channels, each group with an
fp16 scale and an fp16 zero point.

Definition (reading: the zero point is an additive fp16 offset, the group min):

    z = fp16(min G)
    s = fp16((max G - min G) / 15), or 1 when that is 0 (constant group)
    q = clamp(rint((x - z) / s), 0, 15)       (round half to even, in float64)
    dequant:  x_hat = q * s + z

Nibbles are returned unpacked (one uint8 per element); the byte packing the
kernels read is a storage layout, handled in ``oracle.packing``.
"""
from __future__ import annotations

import numpy as np

GROUP = 32


def _fp16(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16)


def _quant_groups(x, axis_group: int):
    """Quantise ``x`` with groups of GROUP consecutive elements along
    ``axis_group`` (last two axes are [tokens, channels])."""
    x = np.asarray(x, dtype=np.float64)
    *lead, T, D = x.shape
    if axis_group == -2:          # groups along tokens, one per channel
        if T % GROUP:
            raise ValueError("token count must be a multiple of 32")
        xg = x.reshape(*lead, T // GROUP, GROUP, D)
        red = -2
    else:                         # groups along channels, one per token
        if D % GROUP:
            raise ValueError("channel count must be a multiple of 32")
        xg = x.reshape(*lead, T, D // GROUP, GROUP)
        red = -1
    mn = xg.min(axis=red, keepdims=True)
    mx = xg.max(axis=red, keepdims=True)
    z16 = _fp16(mn)
    s16 = _fp16((mx - mn) / 15.0)
    s16 = np.where((mx == mn) | (s16 == 0), np.float16(1.0), s16)
    z = z16.astype(np.float64)
    s = s16.astype(np.float64)
    q = np.clip(np.rint((xg - z) / s), 0, 15).astype(np.uint8)
    q = q.reshape(*lead, T, D)
    return q, np.squeeze(s16, axis=red).view(np.uint16), np.squeeze(z16, axis=red).view(np.uint16)


def quantize_k_groups(k):
    """Keys [..., T, D] -> (nibbles [..., T, D], scale bits [..., T/32, D],
    zero bits [..., T/32, D])."""
    return _quant_groups(k, -2)


def quantize_v_groups(v):
    """Values [..., T, D] -> (nibbles [..., T, D], scale bits [..., T, D/32],
    zero bits [..., T, D/32])."""
    return _quant_groups(v, -1)


def _f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def dequant_k_groups(q, scale_bits, zero_bits):
    """Inverse of ``quantize_k_groups``: x_hat [..., T, D] = q * s + z."""
    q = np.asarray(q, dtype=np.float64)
    s = np.repeat(_f16(scale_bits), GROUP, axis=-2)
    z = np.repeat(_f16(zero_bits), GROUP, axis=-2)
    return q * s + z


def dequant_v_groups(q, scale_bits, zero_bits):
    """Inverse of ``quantize_v_groups``: x_hat [..., T, D] = q * s + z."""
    q = np.asarray(q, dtype=np.float64)
    s = np.repeat(_f16(scale_bits), GROUP, axis=-1)
    z = np.repeat(_f16(zero_bits), GROUP, axis=-1)
    return q * s + z
