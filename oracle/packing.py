"""Byte layout of the 4-bit cache (a storage format, not arithmetic).

The format is this library's own: the pages name quantisation as a pluggable
compressor but fix no layout.  Within one (batch, kv head) the quantised tokens
form blocks of 32 (one key group).  Words are little-endian uint32 holding 8
nibbles; nibble p occupies bits 4p..4p+3.  A word carries four element pairs:
pair j (j = 0..3) puts its first element in nibble j and its second in nibble
j + 4.

Keys, words [T/32, 32, 4, D/32] (block, token, c, w): pair j of word (t, c, w)
holds channels e and e + 1 of token t with e = 2c + 32w + 16*(j // 2) + 8*(j % 2).

Values, words [T/32, D, 4] (block, channel, c): pair j of word (d, c) holds
channel d of tokens 2c + 8j and 2c + 8j + 1 of the block.

Key scale / zero: fp16 [T/32, D] (block, channel).
Value scale / zero: fp16 [T/32, D/32, 32] (block, channel group, token in block).
"""
from __future__ import annotations

import numpy as np

G = 32


def _nib_to_word(first, second):
    """first, second: [..., 4] nibble arrays (pair j in slot j) -> uint32 [...]."""
    w = np.zeros(first.shape[:-1], dtype=np.uint32)
    for j in range(4):
        w |= first[..., j].astype(np.uint32) << np.uint32(4 * j)
        w |= second[..., j].astype(np.uint32) << np.uint32(4 * (j + 4))
    return w


def _word_to_nib(w):
    w = np.asarray(w, dtype=np.uint32)
    first = np.stack([(w >> np.uint32(4 * j)) & np.uint32(15) for j in range(4)], axis=-1)
    second = np.stack([(w >> np.uint32(4 * (j + 4))) & np.uint32(15) for j in range(4)], axis=-1)
    return first.astype(np.uint8), second.astype(np.uint8)


def k_channel_of(c: int, w: int, j: int) -> int:
    """First channel of pair j in key word (c, w)."""
    return 2 * c + 32 * w + 16 * (j // 2) + 8 * (j % 2)


def pack_k(nib):
    """Key nibbles [..., T, D] -> words [..., T/32, 32, 4, D/32]."""
    nib = np.asarray(nib, dtype=np.uint8)
    *lead, T, D = nib.shape
    nw = D // 32
    first = np.zeros((*lead, T, 4, nw, 4), dtype=np.uint8)
    second = np.zeros_like(first)
    for c in range(4):
        for w in range(nw):
            for j in range(4):
                e = k_channel_of(c, w, j)
                first[..., c, w, j] = nib[..., e]
                second[..., c, w, j] = nib[..., e + 1]
    words = _nib_to_word(first, second)                  # [..., T, 4, nw]
    return words.reshape(*lead, T // G, G, 4, nw)


def unpack_k(words, D: int):
    words = np.asarray(words, dtype=np.uint32)
    *lead, nb, g, four, nw = words.shape
    first, second = _word_to_nib(words.reshape(*lead, nb * g, 4, nw))
    nib = np.zeros((*lead, nb * g, D), dtype=np.uint8)
    for c in range(4):
        for w in range(nw):
            for j in range(4):
                e = k_channel_of(c, w, j)
                nib[..., e] = first[..., c, w, j]
                nib[..., e + 1] = second[..., c, w, j]
    return nib


def pack_v(nib):
    """Value nibbles [..., T, D] -> words [..., T/32, D, 4]."""
    nib = np.asarray(nib, dtype=np.uint8)
    *lead, T, D = nib.shape
    blk = nib.reshape(*lead, T // G, G, D)
    first = np.zeros((*lead, T // G, D, 4, 4), dtype=np.uint8)
    second = np.zeros_like(first)
    for c in range(4):
        for j in range(4):
            t0 = 2 * c + 8 * j
            first[..., c, j] = blk[..., t0, :]
            second[..., c, j] = blk[..., t0 + 1, :]
    return _nib_to_word(first, second)                   # [..., T/32, D, 4]


def unpack_v(words):
    words = np.asarray(words, dtype=np.uint32)
    *lead, nb, D, four = words.shape
    first, second = _word_to_nib(words)                  # [..., nb, D, 4, 4]
    blk = np.zeros((*lead, nb, G, D), dtype=np.uint8)
    for c in range(4):
        for j in range(4):
            t0 = 2 * c + 8 * j
            blk[..., t0, :] = first[..., c, j]
            blk[..., t0 + 1, :] = second[..., c, j]
    return blk.reshape(*lead, nb * G, D)


def v_scales_to_blocks(bits):
    """Value scale/zero bits [..., T, D/32] -> [..., T/32, D/32, 32]."""
    bits = np.asarray(bits, dtype=np.uint16)
    *lead, T, ng = bits.shape
    return np.ascontiguousarray(np.swapaxes(bits.reshape(*lead, T // G, G, ng), -1, -2))


def v_scales_from_blocks(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    *lead, nb, ng, g = bits.shape
    return np.ascontiguousarray(np.swapaxes(bits, -1, -2)).reshape(*lead, nb * g, ng)
