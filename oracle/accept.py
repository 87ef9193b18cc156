"""Greedy acceptance (VeriCache summary, section "Algoritmo Principale", step 3).

Tokens are accepted up to the first disagreement with the full-KV prediction;
when every drafted token agrees, one extra "bonus" token is accepted; the loop
resumes from the last accepted token.

Definition used.  Row i of the verify logits is the full-KV prediction after
the i-th verify input (the pending token for i = 0, draft i for i >= 1):

    y_i = argmax_v logits[b, i, v]         i = 0..k   (ties: lowest v)
    a   = min{ i < k : y_i != d_i }, or k if there is none
    commit = d_0 .. d_{a-1}, y_a            n_commit = a + 1

so a = k commits every draft plus the bonus y_k, and a < k commits the agreeing
prefix plus the full-KV correction y_a (which keeps the stream equal to greedy
full-KV decoding, as the summary's results section states).  Since d_i = y_i
for i < a, commit[i] = y_i for all i <= a.  Unused commit entries are -1.

Reading for NaN logits (pages silent): NaN counts as larger than every number,
the first NaN wins, and the row's error flag is raised.
"""
from __future__ import annotations

import math

import numpy as np


def argmax_row(row) -> tuple:
    """(index, saw_nan) of the greedy choice in one logits row."""
    best = -1
    best_val = None
    for v_idx in range(len(row)):
        x = float(row[v_idx])
        if math.isnan(x):
            return v_idx, True
        if best < 0 or x > best_val:
            best, best_val = v_idx, x
    return best, False


def accept(logits, drafts=None):
    """Acceptance over logits [B, nq, V] (float) and drafts [B, nq - 1] (int).

    Returns dict(target [B, nq], accept_len [B], commit [B, nq], n_commit [B],
    err [B]) as int arrays; with drafts None only target and err are meaningful.
    """
    logits = np.asarray(logits)
    B, nq, V = logits.shape
    target = np.zeros((B, nq), dtype=np.int64)
    err = np.zeros(B, dtype=np.int64)
    for b in range(B):
        for i in range(nq):
            row = logits[b, i]
            if np.isnan(row).any():
                j, nan = int(np.argmax(np.isnan(row))), True
            else:
                # np.argmax returns the first maximal index, i.e. ties -> lowest v
                j, nan = int(np.argmax(row)), False
            target[b, i] = j
            err[b] |= int(nan)
    out = {"target": target, "err": err}
    if drafts is None:
        return out
    drafts = np.asarray(drafts, dtype=np.int64)
    k = nq - 1
    accept_len = np.zeros(B, dtype=np.int64)
    commit = np.full((B, nq), -1, dtype=np.int64)
    n_commit = np.zeros(B, dtype=np.int64)
    for b in range(B):
        a = k
        for i in range(k):
            if target[b, i] != drafts[b, i]:
                a = i
                break
        accept_len[b] = a
        commit[b, :a] = drafts[b, :a]
        commit[b, a] = target[b, a]
        n_commit[b] = a + 1
    out.update(accept_len=accept_len, commit=commit, n_commit=n_commit)
    return out
