"""Pins of the Chunked Soft Matching oracle (CentroidKV summary, "Riassunto Tecnico:
CentroidKV", section "Metodologia", items 2-4).

Each pin follows from the page's description or from mathematics, not from the
oracle's own code: r = 0 changes nothing; the degree mass is conserved; at most half of
a chunk disappears and exactly floor(r |A|) rows merge; merges go from an A row (even
offset) to a B row (odd offset) of the same chunk; the merged A rows are the top-m
by cosine (checked by an exhaustive search over subsets on a tiny chunk); cosine
decisions ignore positive per-row scales; a two-row merge is the degree-weighted mean;
and a centroid of identical rows, with its degree as ln n in the softmax, gives the
attention of the rows it replaced (the purpose of the aggregation, item 4).
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from oracle import csm


def _case(T, D, seed, deg_max=1):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((T, D))
    V = rng.standard_normal((T, D))
    n = rng.integers(1, deg_max + 1, size=T)
    return K, V, n


def test_r_zero_is_the_identity():
    K, V, n = _case(50, 16, 1, deg_max=5)
    Ko, Vo, no, dest = csm.compress(K, V, n, 4, 8, 12, 0.0)
    assert np.array_equal(dest, np.arange(50))
    assert np.allclose(Ko, K, atol=0, rtol=1e-15) and np.allclose(Vo, V, atol=0, rtol=1e-15)
    assert np.array_equal(no, n)


@pytest.mark.parametrize("T,ns,nr,chunk,r", [(64, 4, 8, 16, 0.5), (101, 3, 10, 10, 1.0),
                                            (40, 0, 0, 8, 0.3), (37, 4, 4, 256, 0.75),
                                            (20, 10, 10, 4, 1.0), (90, 2, 3, 2, 1.0),
                                            (31, 0, 0, 10, 1.0)])
def test_mass_count_and_partition(T, ns, nr, chunk, r):
    K, V, n = _case(T, 8, 2, deg_max=4)
    Ko, Vo, no, dest = csm.compress(K, V, n, ns, nr, chunk, r)
    assert no.sum() == n.sum()                         # degree mass conserved
    assert len(no) == csm.out_len(T, ns, nr, chunk, r)
    assert np.array_equal(dest[:ns], np.arange(ns))    # sinks untouched, in front
    assert np.array_equal(dest[T - nr:], len(no) - nr + np.arange(nr))   # recent at the end
    assert np.all(np.diff(dest) >= -chunk)             # order kept up to merges in a chunk
    for c0 in range(ns, T - nr, chunk):
        c1 = min(c0 + chunk, T - nr)
        rows = np.arange(c0, c1)
        A = rows[0::2]
        # rows sharing an output row: exactly one B row plus the A rows merged into it
        groups = {}
        for i in rows:
            groups.setdefault(int(dest[i]), []).append(int(i))
        n_merged = 0
        for members in groups.values():
            if len(members) > 1:
                bs = [i for i in members if (i - c0) % 2 == 1]
                assert len(bs) == 1, "a centroid holds exactly one B row"
                n_merged += len(members) - 1
        # a one-row chunk has no B row to merge into
        assert n_merged == (math.floor(r * len(A)) if c1 - c0 >= 2 else 0)
        assert n_merged <= (c1 - c0 + 1) // 2


def test_merged_rows_are_the_top_m_by_cosine():
    """Exhaustive check on one chunk: among all subsets of A of size m, the merged one
    has the largest sum of best-match cosines, and each merged row sits with its most
    similar B row."""
    K, V, n = _case(12, 6, 3)
    chunk, r = 12, 0.5
    dest = csm.decide(K, 0, 0, chunk, r)
    A, B = np.arange(0, 12, 2), np.arange(1, 12, 2)
    cos = lambda x, y: float(x @ y / np.linalg.norm(x) / np.linalg.norm(y))
    best = {a: max(cos(K[a], K[b]) for b in B) for a in A}
    merged = [a for a in A if any(dest[a] == dest[b] for b in B)]
    m = math.floor(r * len(A))
    assert len(merged) == m
    top = max(itertools.combinations(A, m), key=lambda sub: sum(best[a] for a in sub))
    assert sorted(merged) == sorted(top)
    for a in merged:
        b = [b for b in B if dest[b] == dest[a]][0]
        assert cos(K[a], K[b]) == pytest.approx(best[a], abs=1e-15)


def test_decisions_ignore_positive_row_scales():
    K, V, n = _case(64, 8, 4)
    s = np.random.default_rng(5).uniform(0.1, 10.0, size=(64, 1))
    assert np.array_equal(csm.decide(K, 2, 2, 16, 0.6), csm.decide(K * s, 2, 2, 16, 0.6))


def test_two_row_merge_is_the_degree_weighted_mean():
    K = np.array([[1.0, 2.0, 3.0], [2.0, 4.0, 7.0]])
    V = np.array([[0.5, -1.0, 2.0], [1.5, 1.0, 0.0]])
    n = np.array([3, 1])
    Ko, Vo, no, dest = csm.compress(K, V, n, 0, 0, 2, 1.0)
    assert np.array_equal(dest, [0, 0]) and np.array_equal(no, [4])
    assert np.allclose(Ko[0], (3 * K[0] + K[1]) / 4, rtol=0, atol=1e-15)
    assert np.allclose(Vo[0], (3 * V[0] + V[1]) / 4, rtol=0, atol=1e-15)


def test_equal_cosines_merge_into_the_lowest_b_and_rank_lower_a_first():
    K = np.tile(np.array([[1.0, 1.0, 0.0, 2.0]]), (8, 1))     # every cosine is 1
    V = np.arange(32, dtype=np.float64).reshape(8, 4)
    dest = csm.decide(K, 0, 0, 8, 0.5)                        # |A| = 4, m = 2
    # A rows 0 and 2 (lowest) merge, both into B row 1 (lowest)
    assert dest[0] == dest[1] == dest[2]
    assert len(set(dest.tolist())) == 6


def test_centroid_of_identical_rows_keeps_the_attention():
    """Rows with equal K and V merged into one centroid of degree n: attention over the
    compressed rows with ln n in the softmax equals attention over the originals."""
    rng = np.random.default_rng(6)
    D, T = 8, 24
    base_k, base_v = rng.standard_normal((6, D)), rng.standard_normal((6, D))
    # consecutive pairs share K and V (row 2i and 2i+1), so every A row's best match is
    # its neighbour B row with cosine 1
    K = np.repeat(base_k, 4, axis=0)
    V = np.repeat(base_v, 4, axis=0)
    n = np.ones(T, np.int64)
    Ko, Vo, no, _ = csm.compress(K, V, n, 0, 0, 4, 1.0)
    q = rng.standard_normal((1, 2, D))
    full, _ = oracle.draft_attn(q, K[None, None], V[None, None], T, None, None)
    comp, _ = oracle.draft_attn(q, Ko[None, None], Vo[None, None], len(no), None,
                                no[None, None].astype(np.int64))
    assert np.allclose(full, comp, rtol=0, atol=1e-12)


def test_hand_worked_cases():
    """tests/golden/csm_cases.json: a six-row chunk in 2-D worked by hand (cosines,
    matches, ranking, centroids) at r = 0.5 and r = 1."""
    import json
    import os
    d = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "csm_cases.json")))
    K, V, n = (np.asarray(d[k], dtype=np.float64) for k in ("K", "V", "n"))
    for c in d["cases"]:
        Ko, Vo, no, dest = csm.compress(K, V, n.astype(np.int64), d["n_sinks"], d["n_recent"],
                                        d["chunk"], c["r"])
        assert dest.tolist() == c["dest"], c["note"]
        assert no.tolist() == c["n_out"], c["note"]
        assert np.allclose(Ko, c["K_out"], rtol=0, atol=1e-15), c["note"]
        assert np.allclose(Vo, c["V_out"], rtol=0, atol=1e-15), c["note"]
