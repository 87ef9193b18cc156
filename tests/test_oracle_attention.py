"""Pins of the oracle's draft and verify attention against things other than itself:
brute force on tiny inputs, closed forms, the degree-n == n-copies identity,
and PyTorch's CPU scaled-dot-product attention as a library special case.

Draft attention: VeriCache summary ("Riepilogo Tecnico: VeriCache"), section
"Algoritmo Principale", step 1; degree term: CentroidKV summary ("Riassunto
Tecnico: CentroidKV"), "Metodologia: CentroidKV", item 4 "Aggregazione".
Verify attention: VeriCache summary, "Algoritmo Principale", step 2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import gen


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _brute_draft(q, k, v, S, idx, deg, kt, vt):
    """Pure-Python double loop over heads and slots."""
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    o = np.zeros((B, Hq, D))
    for b in range(B):
        for h in range(Hq):
            j = h // g
            scores, vals = [], []
            for t in range(S):
                r = t if idx is None else int(idx[b, j, t])
                n = 1 if deg is None else int(deg[b, j, t])
                dot = sum(q[b, h, d] * k[b, j, r, d] for d in range(D))
                scores.append(dot / math.sqrt(D) + math.log(n))
                vals.append(v[b, j, r])
            if kt is not None:
                for t in range(kt.shape[2]):
                    dot = sum(q[b, h, d] * kt[b, j, t, d] for d in range(D))
                    scores.append(dot / math.sqrt(D))
                    vals.append(vt[b, j, t])
            mx = max(scores)
            w = [math.exp(s - mx) for s in scores]
            tot = sum(w)
            for d in range(D):
                o[b, h, d] = sum(w[t] * vals[t][d] for t in range(len(w))) / tot
    return o


@pytest.mark.parametrize("S,n_tail,use_idx", [(1, 0, True), (5, 0, True), (9, 3, True),
                                              (4, 2, False), (7, 1, False)])
def test_draft_brute_force(S, n_tail, use_idx):
    rng = np.random.default_rng(S * 10 + n_tail)
    B, Hq, Hkv, D, T = 2, 4, 2, 6, 12
    q, k, v = _rand(rng, B, Hq, D), _rand(rng, B, Hkv, T, D), _rand(rng, B, Hkv, T, D)
    idx = np.stack([np.stack([np.sort(rng.choice(T, S, replace=False)) for _ in range(Hkv)])
                    for _ in range(B)]) if use_idx else None
    deg = rng.integers(1, 9, size=(B, Hkv, S))
    kt = _rand(rng, B, Hkv, n_tail, D) if n_tail else None
    vt = _rand(rng, B, Hkv, n_tail, D) if n_tail else None
    o, _ = oracle.draft_attn(q, k, v, S, idx, deg, kt, vt)
    ob = _brute_draft(q, k, v, S, idx, deg, kt, vt)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)


def test_draft_matches_torch_sdpa_with_log_degree_mask():
    """Library special case: softmax(q k^T / sqrt(D) + mask) v with mask = ln n."""
    rng = np.random.default_rng(7)
    B, Hq, Hkv, D, T, S = 3, 8, 2, 16, 40, 23
    q, k, v = _rand(rng, B, Hq, D), _rand(rng, B, Hkv, T, D), _rand(rng, B, Hkv, T, D)
    idx = np.stack([np.stack([np.sort(rng.choice(T, S, replace=False)) for _ in range(Hkv)])
                    for _ in range(B)])
    deg = rng.integers(1, 17, size=(B, Hkv, S))
    o, _ = oracle.draft_attn(q, k, v, S, idx, deg)
    g = Hq // Hkv
    ks = np.take_along_axis(k, idx[..., None], axis=2)        # [B,Hkv,S,D]
    vs = np.take_along_axis(v, idx[..., None], axis=2)
    kt = torch.from_numpy(ks).repeat_interleave(g, dim=1)      # head h -> kv head h // g
    vt = torch.from_numpy(vs).repeat_interleave(g, dim=1)
    mask = torch.from_numpy(np.log(deg.astype(np.float64))).repeat_interleave(g, dim=1)
    qt = torch.from_numpy(q)[:, :, None, :]                      # [B,Hq,1,D]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask[:, :, None, :])
    np.testing.assert_allclose(o, ref[:, :, 0].numpy(), rtol=0, atol=1e-12)


def test_draft_single_slot_returns_its_value():
    rng = np.random.default_rng(1)
    q, k, v = _rand(rng, 1, 4, 8), _rand(rng, 1, 1, 5, 8), _rand(rng, 1, 1, 5, 8)
    idx = np.array([[[3]]])
    deg = np.array([[[5]]])
    o, lse = oracle.draft_attn(q, k, v, 1, idx, deg)
    for h in range(4):
        np.testing.assert_allclose(o[0, h], v[0, 0, 3], atol=1e-15)
        s = q[0, h] @ k[0, 0, 3] / math.sqrt(8) + math.log(5)
        assert abs(lse[0, h] - s) < 1e-12


def test_draft_zero_query_is_degree_weighted_mean():
    """q = 0: every score is ln n_t, so o = sum n_t v_t / sum n_t (closed form)."""
    rng = np.random.default_rng(2)
    S, D = 6, 5
    q = np.zeros((1, 2, D))
    k, v = _rand(rng, 1, 1, S, D), _rand(rng, 1, 1, S, D)
    deg = np.array([[[1, 2, 3, 4, 5, 16]]])
    o, lse = oracle.draft_attn(q, k, v, S, None, deg)
    n = deg[0, 0].astype(float)
    want = (n[:, None] * v[0, 0]).sum(0) / n.sum()
    np.testing.assert_allclose(o[0, 0], want, atol=1e-14)
    assert abs(lse[0, 0] - math.log(n.sum())) < 1e-12


def test_draft_two_slot_closed_form():
    """o = (n1 e^{s1} v1 + n2 e^{s2} v2) / (n1 e^{s1} + n2 e^{s2}), s = q.k / sqrt(D)."""
    D = 4
    q = np.array([[[1.0, -2.0, 0.5, 3.0]]])
    k = np.array([[[[0.5, 0.0, 1.0, -1.0], [2.0, 1.0, 0.0, 0.25]]]])
    v = np.array([[[[1.0, 0.0, 0.0, 2.0], [0.0, 1.0, -1.0, 0.0]]]])
    deg = np.array([[[3, 2]]])
    s1 = (0.5 + 0.5 - 3.0) / 2.0
    s2 = (2.0 - 2.0 + 0.75) / 2.0
    w1, w2 = 3 * math.exp(s1), 2 * math.exp(s2)
    want = (w1 * v[0, 0, 0] + w2 * v[0, 0, 1]) / (w1 + w2)
    o, _ = oracle.draft_attn(q, k, v, 2, None, deg)
    np.testing.assert_allclose(o[0, 0], want, atol=1e-15)


def test_degree_n_equals_n_copies():
    """A slot of degree n gives the same output as n identical copies of it."""
    rng = np.random.default_rng(3)
    B, Hq, Hkv, D, S = 2, 8, 2, 16, 10
    q, k, v = _rand(rng, B, Hq, D), _rand(rng, B, Hkv, S, D), _rand(rng, B, Hkv, S, D)
    deg = rng.integers(1, 7, size=(B, Hkv, S))
    o, lse = oracle.draft_attn(q, k, v, S, None, deg)
    for b in range(B):
        for j in range(Hkv):
            rows = np.repeat(np.arange(S), deg[b, j])
            kk = k[b:b + 1, j:j + 1][:, :, rows]
            vv = v[b:b + 1, j:j + 1][:, :, rows]
            g = Hq // Hkv
            oc, lc = oracle.draft_attn(q[b:b + 1, j * g:(j + 1) * g], kk, vv, len(rows))
            np.testing.assert_allclose(o[b, j * g:(j + 1) * g], oc[0], atol=1e-12)
            np.testing.assert_allclose(lse[b, j * g:(j + 1) * g], lc[0], atol=1e-12)


def test_tail_is_appended_slots_of_degree_one():
    rng = np.random.default_rng(4)
    B, Hq, Hkv, D, S, R = 1, 4, 1, 8, 7, 3
    q, k, v = _rand(rng, B, Hq, D), _rand(rng, B, Hkv, S, D), _rand(rng, B, Hkv, S, D)
    kt, vt = _rand(rng, B, Hkv, R, D), _rand(rng, B, Hkv, R, D)
    deg = rng.integers(1, 5, size=(B, Hkv, S))
    o, _ = oracle.draft_attn(q, k, v, S, None, deg, kt, vt)
    kk = np.concatenate([k, kt], axis=2)
    vv = np.concatenate([v, vt], axis=2)
    dd = np.concatenate([deg, np.ones((B, Hkv, R), dtype=int)], axis=2)
    o2, _ = oracle.draft_attn(q, kk, vv, S + R, None, dd)
    np.testing.assert_allclose(o, o2, atol=1e-13)


def test_gqa_head_mapping_uses_contiguous_groups():
    """Head h reads kv head h // g: with kv heads made of constant values, each
    output head returns its own kv head's constant."""
    B, Hq, Hkv, D, S = 1, 6, 3, 4, 5
    rng = np.random.default_rng(5)
    q, k = _rand(rng, B, Hq, D), _rand(rng, B, Hkv, S, D)
    v = np.zeros((B, Hkv, S, D))
    for j in range(Hkv):
        v[0, j] = 10.0 * (j + 1)
    o, _ = oracle.draft_attn(q, k, v, S)
    np.testing.assert_allclose(o[0, :, 0], [10, 10, 20, 20, 30, 30], atol=1e-12)


# ------------------------------------------------------------------ verify
def _brute_verify(q, k, v, P):
    B, nq, Hq, D = q.shape
    g = Hq // k.shape[1]
    o = np.zeros_like(q)
    for b in range(B):
        for i in range(nq):
            for h in range(Hq):
                j = h // g
                sc = [sum(q[b, i, h, d] * k[b, j, t, d] for d in range(D)) / math.sqrt(D)
                      for t in range(P + i + 1)]
                mx = max(sc)
                w = [math.exp(s - mx) for s in sc]
                for d in range(D):
                    o[b, i, h, d] = sum(w[t] * v[b, j, t, d] for t in range(len(w))) / sum(w)
    return o


def test_verify_brute_force():
    rng = np.random.default_rng(11)
    B, nq, Hq, Hkv, D, P = 2, 4, 4, 2, 5, 6
    q = _rand(rng, B, nq, Hq, D)
    k, v = _rand(rng, B, Hkv, P + nq + 2, D), _rand(rng, B, Hkv, P + nq + 2, D)
    np.testing.assert_allclose(oracle.verify_attn(q, k, v, P), _brute_verify(q, k, v, P),
                               atol=1e-12)


def test_verify_matches_torch_sdpa_causal_block():
    rng = np.random.default_rng(12)
    B, nq, Hq, Hkv, D, P = 2, 9, 8, 2, 32, 50
    q = _rand(rng, B, nq, Hq, D)
    k, v = _rand(rng, B, Hkv, P + nq, D), _rand(rng, B, Hkv, P + nq, D)
    o = oracle.verify_attn(q, k, v, P)
    g = Hq // Hkv
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                 # [B,Hq,nq,D]
    kt = torch.from_numpy(k).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(g, dim=1)
    allowed = torch.arange(P + nq)[None, :] <= (P + torch.arange(nq))[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=allowed)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)


def test_verify_row_equals_decode_step():
    """Row i equals a plain decode step of that token over keys [0, P+i]
    (no compression, degree 1); the last row is the decode over the whole cache."""
    rng = np.random.default_rng(13)
    B, nq, Hq, Hkv, D, P = 2, 5, 8, 4, 16, 33
    q = _rand(rng, B, nq, Hq, D)
    k, v = _rand(rng, B, Hkv, P + nq, D), _rand(rng, B, Hkv, P + nq, D)
    o = oracle.verify_attn(q, k, v, P)
    for i in range(nq):
        od, _ = oracle.draft_attn(q[:, i], k[:, :, :P + i + 1], v[:, :, :P + i + 1], P + i + 1)
        np.testing.assert_allclose(o[:, i], od, atol=1e-12)


def test_verify_future_keys_do_not_leak():
    rng = np.random.default_rng(14)
    B, nq, Hq, Hkv, D, P = 1, 6, 4, 1, 8, 20
    q = _rand(rng, B, nq, Hq, D)
    k, v = _rand(rng, B, Hkv, P + nq, D), _rand(rng, B, Hkv, P + nq, D)
    o = oracle.verify_attn(q, k, v, P)
    for i in range(nq - 1):
        k2, v2 = k.copy(), v.copy()
        k2[:, :, P + i + 1:] = 100.0 * _rand(rng, B, Hkv, nq - i - 1, D)
        v2[:, :, P + i + 1:] = -7.0
        o2 = oracle.verify_attn(q, k2, v2, P)
        assert np.array_equal(o2[:, :i + 1], o[:, :i + 1])


@pytest.mark.parametrize("chunk", [1, 7, 64])
def test_verify_chunked_equals_unchunked(chunk):
    rng = np.random.default_rng(15)
    B, nq, Hq, Hkv, D, P = 2, 5, 8, 2, 16, 90
    q = _rand(rng, B, nq, Hq, D)
    k, v = _rand(rng, B, Hkv, P + nq, D), _rand(rng, B, Hkv, P + nq, D)
    a = oracle.verify_attn(q, k, v, P, chunk=chunk)
    b = oracle.verify_attn(q, k, v, P, chunk=10 ** 6)
    np.testing.assert_allclose(a, b, atol=1e-12)


def test_verify_on_workload1_inputs_matches_sdpa():
    """The oracle on the seeded tiny 1K-context inputs (bf16 widened exactly)."""
    case = gen.attn_case(1)
    cfg = case["cfg"]
    q = oracle.bf16_to_f64(case["q_verify_bits"])
    k = oracle.bf16_to_f64(case["k_bits"])
    v = oracle.bf16_to_f64(case["v_bits"])
    o = oracle.verify_attn(q, k, v, cfg.P)
    g = cfg.g
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(g, dim=1)
    n = cfg.k + 1
    allowed = torch.arange(cfg.P + n)[None, :] <= (cfg.P + torch.arange(n))[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=allowed)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=1e-11)
