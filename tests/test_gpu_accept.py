"""vc_accept is bit-exact with the oracle's greedy acceptance when both see the same
logits (VeriCache summary, "Riepilogo Tecnico: VeriCache", section "Algoritmo
Principale", step 3)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import lossless_kv_compressed_b200 as vc
from synth import gen

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "accept_cases.json")


def _gpu(logits, drafts):
    lg = torch.from_numpy(np.ascontiguousarray(logits, dtype=np.float32)).cuda()
    dr = None if drafts is None else torch.from_numpy(np.ascontiguousarray(drafts, np.int32)).cuda()
    r = vc.accept(lg, dr)
    torch.cuda.synchronize()
    return {k: (None if v is None else v.cpu().numpy()) for k, v in r.items()}


def _check(logits, drafts):
    g = _gpu(logits, drafts)
    want = oracle.accept(np.asarray(logits, dtype=np.float32), drafts)
    assert np.array_equal(g["target"], want["target"])
    assert np.array_equal(g["err"], want["err"])
    if drafts is not None:
        for k in ("accept_len", "commit", "n_commit"):
            assert np.array_equal(g[k], want[k]), k
    return g


def test_tiny_1k_context_inputs():
    case = gen.attn_case(1)
    g = _check(case["logits"], case["drafts"])
    assert g["accept_len"].tolist() == [5] and g["n_commit"].tolist() == [6]


def test_golden_cases():
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        lg = np.array([[float(x) for x in row] for row in c["logits"]], dtype=np.float32)[None]
        g = _gpu(lg, np.array([c["drafts"]], dtype=np.int32))
        assert g["target"][0].tolist() == c["target"], c["name"]
        assert int(g["accept_len"][0]) == c["accept_len"], c["name"]
        assert g["commit"][0].tolist() == c["commit"], c["name"]
        assert int(g["err"][0]) == c["err"], c["name"]


@pytest.mark.parametrize("B,n_q,V", [(8, 33, 128256), (1, 33, 8192), (3, 41, 1000),
                                     (2, 1, 128256), (5, 70, 33)])
def test_random_with_agreeing_prefixes(B, n_q, V):
    r = gen.children(77 + V, 3)
    drafts = r[0].integers(0, V, size=(B, n_q - 1), dtype=np.int32)
    n_agree = r[1].integers(0, n_q, size=(B,))
    logits = gen.agreeing_logits(r[2], B, n_q, V, drafts, n_agree)
    g = _check(logits, drafts)
    assert (g["accept_len"] == np.minimum(n_agree, n_q - 1)).all()


def test_ties_and_nan_rows():
    rng = np.random.default_rng(3)
    logits = rng.integers(-2, 2, size=(4, 9, 5000)).astype(np.float32)   # heavy ties
    logits[1, 3, 4095] = np.nan
    logits[1, 3, 17] = np.nan
    logits[2, 0, :] = -np.inf
    drafts = rng.integers(0, 3, size=(4, 8)).astype(np.int32)
    g = _check(logits, drafts)
    assert g["err"].tolist() == [0, 1, 0, 0]
    assert g["target"][1, 3] == 17


def test_argmax_only():
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((8, 1, 128256)).astype(np.float32)
    _check(logits, None)


@pytest.mark.parametrize("V", [5000, 33, 128256])
def test_one_position_rows_ties_nan_and_minus_inf(V):
    """One-position rows (a draft step) finish in the argmax launch itself: ties to the
    lowest index, the first NaN wins and flags the row, an all -inf row gives 0; in
    acceptance mode accept_len 0, commit [target], n_commit 1."""
    rng = np.random.default_rng(V)
    logits = rng.integers(-2, 2, size=(5, 1, V)).astype(np.float32)
    logits[1, 0, V - 2] = np.nan
    logits[1, 0, V // 3] = np.nan
    logits[2, 0, :] = -np.inf
    logits[3, 0, V - 1] = 7.0
    g = _check(logits, None)
    assert g["err"].tolist() == [0, 1, 0, 0, 0]
    assert g["target"][1, 0] == V // 3 and g["target"][2, 0] == 0 and g["target"][3, 0] == V - 1
    g = _check(logits, np.zeros((5, 0), np.int32))
    assert g["accept_len"].tolist() == [0] * 5 and g["n_commit"].tolist() == [1] * 5
    assert np.array_equal(g["commit"][:, 0], g["target"][:, 0])
