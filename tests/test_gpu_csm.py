"""Parity of vc_csm_compress (Chunked Soft Matching, CentroidKV summary "Riassunto Tecnico:
CentroidKV", section "Metodologia", items 2-4) with the fp64 oracle.

The clustering decisions are argmaxes and a top-m selection over cosines that the GPU
computes from bf16 products with fp32 accumulation, the oracle in fp64: where two
candidates are within the GPU's rounding, either choice is correct.  So the tests check
that every GPU decision is valid against the fp64 cosines (its match is a best match and
its merged set is a top-m set, each to within 1e-4), that the structure is exact (sinks,
recent rows, one B row per centroid, floor(r |A|) merges per chunk, degree mass), that
the decisions equal the oracle's where the margins are clear, and that the output rows
equal the oracle's aggregation of the GPU's own decisions to within one bf16 rounding.
"""
import math

import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
import oracle
from oracle import csm
from tests.gpu_util import dev_bf16, dev_i32, host_f64

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _inputs(B, Hkv, T, D, seed, deg_max=1, ar=0.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((2, B, Hkv, T, D))
    if ar:                                   # neighbouring rows alike, as keys are
        for t in range(1, T):
            x[:, :, :, t] = ar * x[:, :, :, t - 1] + math.sqrt(1 - ar * ar) * x[:, :, :, t]
    bits = np.asarray(torch.from_numpy(x.astype(np.float32)).bfloat16().view(torch.int16)
                      .numpy()).view(np.uint16)
    deg = rng.integers(1, deg_max + 1, size=(B, Hkv, T)).astype(np.int32)
    return bits[0], bits[1], deg


def _run(kb, vb, deg, T, ns, nr, chunk, r, use_deg=True):
    k, v = dev_bf16(kb), dev_bf16(vb)
    B, Hkv, T_cap, D = k.shape
    dest = torch.full((B, Hkv, T_cap), -1, dtype=torch.int32, device="cuda")
    ko, vo, do, n_out = vc.csm_compress(k, v, ns, nr, chunk, r,
                                        deg=dev_i32(deg) if use_deg else None, T=T, dest=dest)
    torch.cuda.synchronize()
    return (host_f64(ko)[:, :, :n_out], host_f64(vo)[:, :, :n_out],
            do.cpu().numpy()[:, :, :n_out].astype(np.int64), dest.cpu().numpy()[:, :, :T], n_out)


def _check_pair(K, V, n, dest, ns, nr, chunk, r, Ko, Vo, no):
    T = K.shape[0]
    # structure: sinks in front, recent at the end, every chunk's merges inside it
    assert np.array_equal(dest[:ns], np.arange(ns))
    n_out = len(no)
    assert np.array_equal(dest[T - nr:], n_out - nr + np.arange(nr))
    assert no.sum() == n.sum()
    for c0 in range(ns, T - nr, chunk):
        c1 = min(c0 + chunk, T - nr)
        rows = np.arange(c0, c1)
        A, B = rows[0::2], rows[1::2]
        S = csm.cosine(K[A], K[B]) if len(B) else np.zeros((len(A), 0))
        best = S.max(axis=1) if len(B) else np.zeros(len(A))
        merged, target = [], {}
        for ia, a in enumerate(A):
            partners = [ib for ib, b in enumerate(B) if dest[b] == dest[a]]
            assert len(partners) <= 1
            if partners:
                merged.append(ia)
                target[ia] = partners[0]
        m = math.floor(r * len(A)) if len(B) else 0
        assert len(merged) == m
        for ia, ib in target.items():
            assert S[ia, ib] >= best[ia] - TOL, "merged into a B row that is not a best match"
        if m and m < len(A):
            lo = min(best[ia] for ia in merged)
            hi = max(best[ia] for ia in range(len(A)) if ia not in target)
            assert lo >= hi - TOL, "merged set is not a top-m set"
        # survivors (B rows and unmerged A rows) keep their order on consecutive rows
        b_dest = {int(dest[b]) for b in B}
        surv = [i for i in rows if (i - c0) % 2 == 1 or int(dest[i]) not in b_dest]
        assert np.all(np.diff([dest[i] for i in surv]) == 1)
    # outputs = the fp64 aggregation of the GPU's own decisions, to one bf16 rounding
    Kr, Vr, nr_ = csm.apply(K, V, n, dest.astype(np.int64))
    assert np.array_equal(nr_, no)
    for got, ref in ((Ko, Kr), (Vo, Vr)):
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("T,ns,nr,chunk,r,deg_max", [
    (40, 4, 4, 8, 0.5, 1), (301, 4, 16, 64, 0.5, 8), (300, 0, 0, 256, 1.0, 3),
    (517, 8, 9, 256, 0.3, 16), (90, 2, 3, 2, 1.0, 1), (64, 4, 4, 16, 0.0, 4),
    (20, 10, 10, 8, 0.5, 1)])
def test_shapes(D, T, ns, nr, chunk, r, deg_max):
    kb, vb, deg = _inputs(2, 2, T, D, seed=T + D, deg_max=deg_max, ar=0.8)
    Ko, Vo, no, dest, n_out = _run(kb, vb, deg, T, ns, nr, chunk, r)
    assert n_out == csm.out_len(T, ns, nr, chunk, r)
    f = oracle.bf16_to_f64
    for b in range(2):
        for j in range(2):
            _check_pair(f(kb[b, j]), f(vb[b, j]), deg[b, j].astype(np.int64), dest[b, j], ns, nr,
                        chunk, r, Ko[b, j], Vo[b, j], no[b, j])


def test_degrees_default_to_one_and_capacity_beyond_T():
    kb, vb, deg = _inputs(1, 3, 200, 128, seed=7, ar=0.5)
    T = 150                                   # rows [150, 200) are capacity, not cache
    Ko, Vo, no, dest, n_out = _run(kb, vb, deg, T, 4, 8, 32, 0.5, use_deg=False)
    f = oracle.bf16_to_f64
    for j in range(3):
        _check_pair(f(kb[0, j, :T]), f(vb[0, j, :T]), np.ones(T, np.int64), dest[0, j], 4, 8, 32,
                    0.5, Ko[0, j], Vo[0, j], no[0, j])


def test_clear_margins_give_the_oracle_decisions():
    """Keys built so that every best match and the top-m cut have margins far above the
    GPU's rounding: the decisions are then unique and must equal the oracle's."""
    rng = np.random.default_rng(11)
    D, T = 128, 256
    K = np.zeros((T, D))
    for i in range(T // 2):                   # pair (2i, 2i+1) share a direction
        u = rng.standard_normal(D)
        u /= np.linalg.norm(u)
        K[2 * i] = u
        w = rng.standard_normal(D)
        w -= (w @ u) * u
        w /= np.linalg.norm(w)
        c = 0.6 + 0.35 * ((5 * i) % 8) / 8.0   # 8 distinct cosines in every chunk of 16
        K[2 * i + 1] = c * u + math.sqrt(1 - c * c) * w
    kb = np.asarray(torch.from_numpy(K[None, None].astype(np.float32)).bfloat16()
                    .view(torch.int16).numpy()).view(np.uint16)
    vb = kb.copy()
    deg = np.ones((1, 1, T), np.int32)
    Ko, Vo, no, dest, n_out = _run(kb, vb, deg, T, 0, 0, 16, 0.5)
    want = csm.decide(oracle.bf16_to_f64(kb[0, 0]), 0, 0, 16, 0.5)
    assert np.array_equal(dest[0, 0], want)


def test_32k_context_size_sampled_pairs():
    """B 8 x 8 kv heads x 32768 rows, D 128, chunk 256, r = 0.5, degrees 1..16: structure
    and decisions checked on sampled pairs."""
    kb, vb, deg = _inputs(8, 8, 32768, 128, seed=2, deg_max=16, ar=0.9)
    Ko, Vo, no, dest, n_out = _run(kb, vb, deg, 32768, 4, 512, 256, 0.5)
    assert n_out == csm.out_len(32768, 4, 512, 256, 0.5)
    f = oracle.bf16_to_f64
    for b, j in ((0, 0), (3, 5), (7, 7)):
        _check_pair(f(kb[b, j]), f(vb[b, j]), deg[b, j].astype(np.int64), dest[b, j], 4, 512,
                    256, 0.5, Ko[b, j], Vo[b, j], no[b, j])


def test_compressed_identical_rows_keep_draft_attention():
    """End to end on the GPU: rows that come in identical pairs, compressed by CSM at
    r = 1 and read back by vc_draft_attn as a compact cache with the degrees, give the
    same attention as the uncompressed rows (each merged pair is one centroid of
    degree 2)."""
    rng = np.random.default_rng(13)
    B, Hkv, Hq, D, T = 2, 2, 8, 128, 512
    base = rng.standard_normal((2, B, Hkv, T // 2, D)).astype(np.float32)
    x = np.repeat(base, 2, axis=3)
    k = torch.from_numpy(x[0]).cuda().bfloat16()
    v = torch.from_numpy(x[1]).cuda().bfloat16()
    ko, vo, do, n_out = vc.csm_compress(k, v, 0, 0, 64, 1.0)
    assert n_out == T // 2
    q = torch.randn(B, Hq, D, device="cuda").bfloat16()
    full = vc.draft_attn(q, vc.IndexedCache(k=k, v=v, S=T, Hq=Hq),
                         out=torch.empty(q.shape, device="cuda"))
    comp = vc.draft_attn(q, vc.IndexedCache(k=ko, v=vo, S=n_out, Hq=Hq, deg=do),
                         out=torch.empty(q.shape, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(do, torch.full_like(do, 2))
    assert (full - comp).abs().max().item() < 2e-3
