"""Pins of the oracle's greedy acceptance (VeriCache summary, section "Algoritmo
Principale", step 3): hand-worked fixtures, exhaustive enumeration on tiny
vocabularies against the "longest agreeing prefix" formulation, and a pure-Python
argmax for ties and NaN."""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
from synth import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "accept_cases.json")


def _load_cases():
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        c["logits"] = np.array([[float(x) for x in row] for row in c["logits"]])
    return cases


@pytest.mark.parametrize("case", _load_cases(), ids=lambda c: c["name"])
def test_golden_cases(case):
    logits = case["logits"][None]
    drafts = np.array(case["drafts"], dtype=np.int64)[None]
    r = oracle.accept(logits, drafts)
    assert r["target"][0].tolist() == case["target"]
    assert int(r["accept_len"][0]) == case["accept_len"]
    assert r["commit"][0].tolist() == case["commit"]
    assert int(r["n_commit"][0]) == case["n_commit"]
    assert int(r["err"][0]) == case["err"]


def _longest_agreeing_prefix(target, drafts):
    best = 0
    for a in range(len(drafts) + 1):
        if list(drafts[:a]) == list(target[:a]):
            best = a
    return best


@pytest.mark.parametrize("V,k", [(2, 3), (3, 2), (4, 1)])
def test_exhaustive_tiny(V, k):
    """Every target pattern and every draft sequence on a tiny vocabulary."""
    for target in itertools.product(range(V), repeat=k + 1):
        logits = np.zeros((1, k + 1, V))
        for i, y in enumerate(target):
            logits[0, i, y] = 1.0
        for drafts in itertools.product(range(V), repeat=k):
            r = oracle.accept(logits, np.array([drafts]))
            a = _longest_agreeing_prefix(target, drafts)
            assert r["accept_len"][0] == a
            assert r["n_commit"][0] == a + 1
            # the committed stream is the full-KV prediction stream, cut after a+1
            assert r["commit"][0, :a + 1].tolist() == list(target[:a + 1])
            assert (r["commit"][0, a + 1:] == -1).all()
            if a == k:  # all drafts agree: the bonus token is the last prediction
                assert r["commit"][0, k] == target[k]


def test_argmax_matches_python_scan_with_ties():
    rng = np.random.default_rng(0)
    logits = rng.integers(-3, 3, size=(3, 7, 11)).astype(np.float64)  # many ties
    r = oracle.accept(logits)
    for b in range(3):
        for i in range(7):
            j, nan = oracle.argmax_row(logits[b, i])
            assert r["target"][b, i] == j and not nan


def test_drafts_none_gives_argmax_only():
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((2, 1, 50))
    r = oracle.accept(logits)
    assert set(r) == {"target", "err"}
    assert r["target"][:, 0].tolist() == np.argmax(logits[:, 0], axis=1).tolist()


def test_tiny_inputs_construction_accepts_five():
    """The tiny 1K-context inputs lift the draft logit on rows 0-4 and break row 5."""
    case = gen.attn_case(1)
    r = oracle.accept(case["logits"], case["drafts"])
    assert r["accept_len"].tolist() == [5]
    assert r["n_commit"].tolist() == [6]
    assert r["commit"][0, :5].tolist() == case["drafts"][0, :5].tolist()
