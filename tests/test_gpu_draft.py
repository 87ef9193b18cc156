"""Parity of vc_draft_attn (indexed bf16 cache + degree + tail) with the fp64 oracle.

Draft attention: VeriCache summary ("Riepilogo Tecnico: VeriCache"), section
"Algoritmo Principale", step 1; the log-degree term: CentroidKV summary
("Riassunto Tecnico: CentroidKV"), item 4 "Aggregazione".
Tolerance: max-abs 1e-2 and rel-L2 2e-3 (bf16 in, fp32 accumulate, bf16 out)."""
import numpy as np
import pytest
import torch

import oracle
import lossless_kv_compressed_b200 as vc
from synth import gen
from tests.gpu_util import assert_close_attn, both_outputs, dev_bf16, dev_i32, host_f64

pytestmark = pytest.mark.gpu


def _run(case, S, n_tail, use_idx=True, use_deg=True, check_lse=True):
    cfg = case["cfg"]
    B, Hq, Hkv, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.D
    k_bits, v_bits = case["k_bits"], case["v_bits"]
    idx = case["idx"][:, :, :S] if use_idx else None
    deg = case["deg"][:, :, :S] if use_deg else None
    kt_bits = gen.bf16_block_rows(case, "k", max(n_tail, 1))
    vt_bits = gen.bf16_block_rows(case, "v", max(n_tail, 1))
    q_bits = case["q_draft_bits"]
    cache = vc.IndexedCache(
        k=dev_bf16(k_bits), v=dev_bf16(v_bits), S=S, Hq=Hq,
        idx=dev_i32(np.ascontiguousarray(idx)) if idx is not None else None,
        deg=dev_i32(np.ascontiguousarray(deg)) if deg is not None else None,
        k_tail=dev_bf16(kt_bits), v_tail=dev_bf16(vt_bits), n_tail=n_tail,
        err_flag=torch.zeros(1, dtype=torch.int32, device="cuda"))
    q = dev_bf16(q_bits)
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    out = both_outputs(lambda dt: vc.draft_attn(q, cache, lse=lse, out=torch.empty(
        q.shape, dtype=dt, device="cuda")))
    assert int(cache.err_flag.item()) == 0
    f = oracle.bf16_to_f64
    o_ref, lse_ref = oracle.draft_attn(
        f(q_bits), f(k_bits), f(v_bits), S, idx, deg,
        f(kt_bits[:, :, :n_tail]) if n_tail else None,
        f(vt_bits[:, :, :n_tail]) if n_tail else None)
    got = host_f64(out)
    res = assert_close_attn(got, o_ref, f"draft S={S} tail={n_tail}")
    if check_lse:
        np.testing.assert_allclose(host_f64(lse), lse_ref, atol=2e-3, rtol=0)
    return res


def test_tiny_1k_context_full():
    case = gen.attn_case(1)
    for n_tail in (0, 1, 9):
        _run(case, case["cfg"].S, n_tail)


@pytest.mark.parametrize("D,Hq,Hkv", [(64, 8, 2), (128, 32, 8), (128, 8, 8), (64, 16, 2)])
@pytest.mark.parametrize("S,n_tail", [(1, 0), (15, 1), (17, 0), (100, 5), (1000, 3), (3000, 31)])
def test_shapes_and_ragged_tails(D, Hq, Hkv, S, n_tail):
    case = gen.attn_case(1, B=2, Hq=Hq, Hkv=Hkv, D=D, P=4096, S=max(S, 2 + 8), n_sinks=1,
                         n_recent=1, deg_max=16, k=max(n_tail, 8))
    _run(case, S, n_tail)


def test_tail_only():
    case = gen.attn_case(1, B=2, P=512, S=64, n_recent=8)
    assert case["k_bits"].shape[2] >= 512 + 7
    _run(case, 0, 7, check_lse=True)


def test_compact_cache_and_unit_degrees():
    case = gen.attn_case(1, B=3, Hq=32, Hkv=8, D=128, P=2000, S=1500, n_recent=16)
    _run(case, 1500, 4, use_idx=False, use_deg=False)
    _run(case, 1500, 4, use_idx=False, use_deg=True)


def test_out_of_range_index_sets_flag_without_faulting():
    case = gen.attn_case(1)
    cfg = case["cfg"]
    idx = case["idx"].copy()
    idx[0, 1, 17] = cfg.L_cap + 1000          # beyond T_cap: clamped in-kernel, flagged
    deg = case["deg"].copy()
    deg[0, 0, 3] = 0                          # degree < 1: flagged
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = vc.IndexedCache(k=dev_bf16(case["k_bits"]), v=dev_bf16(case["v_bits"]), S=cfg.S,
                            Hq=cfg.Hq, idx=dev_i32(idx), deg=dev_i32(deg), err_flag=flag)
    vc.draft_attn(dev_bf16(case["q_draft_bits"]), cache)
    torch.cuda.synchronize()
    assert int(flag.item()) == 1


@pytest.fixture(scope="module")
def case2():
    return gen.attn_case(2)


def test_32k_context_full_size(case2):
    """Full 32K-context sizes (B 8, 32/8 heads, D 128, 8192 slots of a 32K context,
    degrees 1..16) with the longest draft tail of a round (k = 32)."""
    _run(case2, case2["cfg"].S, case2["cfg"].k)


def test_deterministic_across_calls(case2):
    cfg = case2["cfg"]
    cache = vc.IndexedCache(k=dev_bf16(case2["k_bits"]), v=dev_bf16(case2["v_bits"]), S=cfg.S,
                            Hq=cfg.Hq, idx=dev_i32(case2["idx"]), deg=dev_i32(case2["deg"]))
    q = dev_bf16(case2["q_draft_bits"])
    a = vc.draft_attn(q, cache).clone()
    b = vc.draft_attn(q, cache)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_long_context_drafters_65536_compact_slots():
    """The drafting requests of the 1M-token staggered workload at their own shapes:
    3 requests x 64/8 heads (g = 8), D 128, 65536 compact slots each (idx = NULL),
    degrees 1..16, plus a 17-row bf16 tail; every head of every request against the
    oracle (one request at a time, to bound host memory)."""
    from synth.configs import get_config
    cfg = get_config(4)
    n_tail = 17
    dc = gen.staged_draft_case(cfg, n_tail=n_tail)
    cache = vc.IndexedCache(
        k=dev_bf16(dc["kc_bits"]), v=dev_bf16(dc["vc_bits"]), S=cfg.S, Hq=cfg.Hq,
        deg=dev_i32(dc["deg"]), k_tail=dev_bf16(dc["tail_k_bits"]),
        v_tail=dev_bf16(dc["tail_v_bits"]), n_tail=n_tail,
        err_flag=torch.zeros(1, dtype=torch.int32, device="cuda"))
    q = dev_bf16(dc["q_bits"])
    lse = torch.empty((cfg.n_draft_requests, cfg.Hq), dtype=torch.float32, device="cuda")
    out = both_outputs(lambda dt: vc.draft_attn(q, cache, lse=lse, out=torch.empty(
        q.shape, dtype=dt, device="cuda")))
    assert int(cache.err_flag.item()) == 0
    got, got_lse = host_f64(out), host_f64(lse)
    f = oracle.bf16_to_f64
    for r in range(cfg.n_draft_requests):
        s = slice(r, r + 1)
        o_ref, lse_ref = oracle.draft_attn(f(dc["q_bits"][s]), f(dc["kc_bits"][s]),
                                           f(dc["vc_bits"][s]), cfg.S, None, dc["deg"][s],
                                           f(dc["tail_k_bits"][s]), f(dc["tail_v_bits"][s]))
        assert_close_attn(got[s], o_ref, f"65536-slot drafter {r}")
        np.testing.assert_allclose(got_lse[s], lse_ref, atol=2e-3, rtol=0)
