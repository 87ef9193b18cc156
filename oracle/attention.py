"""Draft and verify attention, float64.

Draft attention (VeriCache summary, section "Algoritmo Principale", step 1: the
model decodes over the compressed cache KV_comp) with the CentroidKV degree term
(CentroidKV summary, "Metodologia: CentroidKV", item 4 "Aggregazione": the
cluster degree n_t enters the softmax as a logarithmic term).  For one query
head h of batch b, with kv head j = h // g and g = Hq / Hkv:

    s_t = (q . k_t) * scale + ln(n_t)      t over the S compressed slots, then
    s_t = (q . k_t) * scale                t over the bf16 tail (degree 1)
    o   = sum_t softmax(s)_t v_t

Readings taken where the pages are silent: natural log (the only base for which a
degree-n slot equals n identical copies of it, which is what "approximating the
original attention output" needs); scale = D^-1/2; GQA head h reads kv head
h // g; the tail holds the tokens appended while drafting.

Verify attention (same page, step 2: one forward over KV_full checks all drafted
tokens in parallel).  Row i (0 <= i <= k) is the token at absolute position P + i
and attends keys [0, P + i] -- causal inside the draft block, no degree term.
"""
from __future__ import annotations

import numpy as np


def _scale(D: int, scale):
    return (1.0 / np.sqrt(D)) if (scale is None or scale <= 0.0) else float(scale)


def draft_attn(q, k, v, S: int, idx=None, deg=None, k_tail=None, v_tail=None,
               scale=None):
    """Decode attention over a compressed cache plus a bf16 tail.

    q      [B, Hq, D]          float64
    k, v   [B, Hkv, T, D]      float64 base rows (full cache for an indexed view,
                               or the compact slot rows when idx is None)
    S      number of compressed slots
    idx    [B, Hkv, >=S] int   slot -> base row (None: slot t is row t)
    deg    [B, Hkv, >=S] int   slot degree n_t >= 1 (None: all 1)
    k_tail, v_tail [B, Hkv, n_tail, D] or None
    Returns (o [B, Hq, D], lse [B, Hq]) with lse = ln sum_t exp(s_t).
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    sc = _scale(D, scale)
    o = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for j in range(Hkv):
            rows = np.arange(S) if idx is None else np.asarray(idx[b, j, :S], dtype=np.int64)
            ks = np.asarray(k[b, j][rows], dtype=np.float64)
            vs = np.asarray(v[b, j][rows], dtype=np.float64)
            bias = np.zeros(S) if deg is None else np.log(np.asarray(deg[b, j, :S], dtype=np.float64))
            if k_tail is not None and k_tail.shape[2] > 0:
                ks = np.concatenate([ks, np.asarray(k_tail[b, j], dtype=np.float64)])
                vs = np.concatenate([vs, np.asarray(v_tail[b, j], dtype=np.float64)])
                bias = np.concatenate([bias, np.zeros(k_tail.shape[2])])
            qh = q[b, j * g:(j + 1) * g]                 # [g, D]
            s = qh @ ks.T * sc + bias[None, :]           # [g, S + n_tail]
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            o[b, j * g:(j + 1) * g] = (p @ vs) / l
            lse[b, j * g:(j + 1) * g] = (m + np.log(l))[:, 0]
    return o, lse


def verify_partial(q, k, v, kv_start: int, P: int, scale=None):
    """Softmax state of the verify rows over one run of keys.

    q     [B, nq, Hq, D]; row i sits at absolute position P + i
    k, v  [B, Hkv, n, D]: keys at absolute positions kv_start .. kv_start+n-1
    Returns (m, l, acc): m [B, nq, Hq] max score over the keys row i may see
    (-inf if none), l = sum exp(s - m), acc [B, nq, Hq, D] = sum exp(s - m) v.
    """
    q = np.asarray(q, dtype=np.float64)
    B, nq, Hq, D = q.shape
    Hkv, n = k.shape[1], k.shape[2]
    g = Hq // Hkv
    sc = _scale(D, scale)
    pos = kv_start + np.arange(n)
    rows = P + np.arange(nq)
    visible = pos[None, :] <= rows[:, None]                      # [nq, n]
    m = np.full((B, nq, Hq), -np.inf)
    l = np.zeros((B, nq, Hq))
    acc = np.zeros((B, nq, Hq, D))
    for b in range(B):
        for j in range(Hkv):
            kk = np.asarray(k[b, j], dtype=np.float64)
            vv = np.asarray(v[b, j], dtype=np.float64)
            qh = q[b, :, j * g:(j + 1) * g, :]                   # [nq, g, D]
            s = np.einsum("igd,td->igt", qh, kk) * sc           # [nq, g, n]
            s = np.where(visible[:, None, :], s, -np.inf)
            mm = s.max(axis=2)                                   # [nq, g]
            safe = np.where(np.isfinite(mm), mm, 0.0)
            p = np.where(visible[:, None, :], np.exp(s - safe[:, :, None]), 0.0)
            m[b, :, j * g:(j + 1) * g] = mm
            l[b, :, j * g:(j + 1) * g] = p.sum(axis=2)
            acc[b, :, j * g:(j + 1) * g] = np.einsum("igt,td->igd", p, vv)
    return m, l, acc


def merge_partials(a, b):
    """Combine two softmax states over disjoint key sets (exact log-sum-exp)."""
    ma, la, aa = a
    mb, lb, ab = b
    m = np.maximum(ma, mb)
    safe = np.where(np.isfinite(m), m, 0.0)
    wa = np.where(np.isfinite(ma), np.exp(ma - safe), 0.0)
    wb = np.where(np.isfinite(mb), np.exp(mb - safe), 0.0)
    return m, la * wa + lb * wb, aa * wa[..., None] + ab * wb[..., None]


def finalize_partial(state):
    m, l, acc = state
    return acc / l[..., None]


def verify_attn(q, k, v, P: int, scale=None, chunk: int = 65536):
    """Verify attention over the full KV, rows causal inside the block.

    q [B, nq, Hq, D]; k, v [B, Hkv, >= P + nq, D] with the block's own keys at
    P .. P + nq - 1.  Returns o [B, nq, Hq, D].  Keys are taken in runs of
    ``chunk`` merged by ``merge_partials`` to bound memory; ``chunk`` does not
    change the result beyond float64 rounding.
    """
    nq = q.shape[1]
    L = P + nq
    state = None
    for s0 in range(0, L, chunk):
        s1 = min(L, s0 + chunk)
        part = verify_partial(q, k[:, :, s0:s1], v[:, :, s0:s1], s0, P, scale)
        state = part if state is None else merge_partials(state, part)
    return finalize_partial(state)


def draft_attn_int4(q, kq, k_scale, k_zero, vq, v_scale, v_zero, k_tail=None, v_tail=None,
                    scale=None):
    """Draft attention over a 4-bit cache plus a bf16 tail.

    kq, vq: packed words (layout in ``oracle.packing``) of T_q quantised tokens
    per (batch, kv head); k_scale/k_zero fp16 bits [B, Hkv, T_q/32, D];
    v_scale/v_zero fp16 bits [B, Hkv, T_q/32, D/32, 32].  Every quantised slot
    has degree 1.  Dequantisation is x_hat = q * s + z (``oracle.quant``).
    """
    from .packing import unpack_k, unpack_v, v_scales_from_blocks
    from .quant import dequant_k_groups, dequant_v_groups
    D = q.shape[-1]
    kn = unpack_k(kq, D)
    vn = unpack_v(vq)
    kh = dequant_k_groups(kn, k_scale, k_zero)
    vh = dequant_v_groups(vn, v_scales_from_blocks(v_scale), v_scales_from_blocks(v_zero))
    return draft_attn(q, kh, vh, kh.shape[2], None, None, k_tail, v_tail, scale)
