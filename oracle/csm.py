"""Chunked Soft Matching (CSM): CentroidKV's one-pass clustering of a KV cache, float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "Riassunto Tecnico: CentroidKV" (gist.science/it/paper/2506.11418), section
"Metodologia", items 2 ("Pipeline di Inferenza": sinks and recent tokens are kept out
of the partition), 3 ("Chunked Soft Matching": chunking, alternating A/B partition,
matching as in bipartite soft matching, merging only the most similar fraction r of
the candidate matches, the progressive schedule of r over rounds) and 4
("Aggregazione": a degree-weighted mean per cluster, the degree n_t counting the
tokens merged into a centroid across rounds).  The page gives no formula; the plainest
readings, one per open point:

* Rows [0, n_sinks) and [T - n_recent, T) pass through unchanged; the middle rows are
  cut into consecutive chunks of ``chunk`` rows (the last one may be shorter).
* Within a chunk, A holds the rows at even offsets and B those at odd offsets.
* Similarity is the cosine of the key rows (0 when either row is all zero).  Each A
  row's match is its most similar B row of the chunk, the lowest on ties.
* The candidate matches of a chunk (one per A row) are ranked by similarity, higher
  first, the lower A row on ties; the first m = floor(r * |A|) merge into their matches
  (at most half of a chunk's rows disappear per round, as the page notes).
* A B row and the A rows merged into it become one centroid: K and V are the
  degree-weighted means, the degree is the sum.  Unmerged A rows and B rows without
  merges are kept as they are.
* Output order: sinks, then each chunk's surviving rows in their original order (a
  centroid takes its B row's place), then the recent rows.
* The schedule r_j = r_init - j * delta_r is the caller's: each call takes one r.
"""
from __future__ import annotations

import math

import numpy as np


def out_len(T: int, n_sinks: int, n_recent: int, chunk: int, r: float) -> int:
    """Rows left after one round over T rows."""
    mid = T - n_sinks - n_recent
    n = n_sinks + n_recent
    for c0 in range(0, mid, chunk):
        ln = min(chunk, mid - c0)
        # a one-row chunk has no B row: nothing merges
        n += ln - (math.floor(r * ((ln + 1) // 2)) if ln >= 2 else 0)
    return n


def cosine(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Cosine similarity matrix of the rows of a [n, D] and b [m, D] (0 for zero rows)."""
    na = np.linalg.norm(a, axis=1)
    nb = np.linalg.norm(b, axis=1)
    dots = a @ b.T
    den = na[:, None] * nb[None, :]
    return np.where(den > 0, dots / np.where(den > 0, den, 1.0), 0.0)


def decide(K: np.ndarray, n_sinks: int, n_recent: int, chunk: int, r: float) -> np.ndarray:
    """Clustering decisions for one (batch, kv head): ``dest[i]`` = the output row of
    input row i (rows merged into a centroid point at the centroid's row).

    K: [T, D] key rows.  Returns int64 [T]."""
    T = K.shape[0]
    mid0, mid1 = n_sinks, T - n_recent
    dest = np.empty(T, np.int64)
    dest[:n_sinks] = np.arange(n_sinks)
    o = n_sinks
    for c0 in range(mid0, mid1, chunk):
        c1 = min(c0 + chunk, mid1)
        rows = np.arange(c0, c1)
        A, B = rows[0::2], rows[1::2]
        m = math.floor(r * len(A))
        merged_into = {}
        if m > 0 and len(B) > 0:
            S = cosine(K[A], K[B])
            best = np.argmax(S, axis=1)               # first maximum: lowest B row
            sim = S[np.arange(len(A)), best]
            order = sorted(range(len(A)), key=lambda i: (-sim[i], i))
            for i in order[:m]:
                merged_into[int(A[i])] = int(B[best[i]])
        for row in rows:                              # survivors in their order
            if row not in merged_into:
                dest[row] = o
                o += 1
        for a, b in merged_into.items():
            dest[a] = dest[b]
    dest[mid1:] = o + np.arange(T - mid1)
    return dest


def apply(K: np.ndarray, V: np.ndarray, n: np.ndarray, dest: np.ndarray):
    """Aggregate rows by ``dest``: per output row the degree-weighted means of K and V
    and the sum of the degrees.  K, V [T, D]; n [T] (>= 1).  Returns (K', V', n')."""
    T_out = int(dest.max()) + 1 if len(dest) else 0
    D = K.shape[1]
    w = n.astype(np.float64)
    Ko = np.zeros((T_out, D))
    Vo = np.zeros((T_out, D))
    no = np.zeros(T_out, np.int64)
    np.add.at(Ko, dest, w[:, None] * K)
    np.add.at(Vo, dest, w[:, None] * V)
    np.add.at(no, dest, n.astype(np.int64))
    return Ko / no[:, None], Vo / no[:, None], no


def compress(K, V, n, n_sinks: int, n_recent: int, chunk: int, r: float):
    """One CSM round for one (batch, kv head).  Returns (K', V', n', dest)."""
    dest = decide(K, n_sinks, n_recent, chunk, r)
    Ko, Vo, no = apply(K, V, n, dest)
    return Ko, Vo, no, dest
