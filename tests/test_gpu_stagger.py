"""Staggered long-context verification (VeriCache summary, "Riepilogo Tecnico:
VeriCache", sections "Supporto Architetturale" and "Scaglionamento tra Risorse (P1)"):
the full cache streams chunk by chunk from pinned host memory through a device ring
while other requests draft on their own stream.  The staged verify and the concurrent
drafts both match the oracle; the drafts also match the same drafts run alone, bit
for bit."""
import dataclasses

import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
import oracle
from lossless_kv_compressed_b200.stagger import StagedVerify, run_alongside
from synth import gen
from synth.configs import get_config
from tests.gpu_util import assert_close_attn, dev_bf16, dev_i32, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    vc.device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert vc.device_error(clear=True) == 0, "a bounded wait in the verify kernel expired"


def _host_chunks(case, n_chunks, chunk, Hkv, D):
    host = torch.empty((n_chunks, 2, Hkv, chunk, D), dtype=torch.bfloat16, pin_memory=True)
    ks, vs = [], []
    for c, (kb, vb) in enumerate(zip(case["chunks_k"], case["chunks_v"])):
        n = kb.shape[1]
        hk = torch.from_numpy(np.ascontiguousarray(kb).view(np.int16)).view(torch.bfloat16)
        hv = torch.from_numpy(np.ascontiguousarray(vb).view(np.int16)).view(torch.bfloat16)
        host[c, 0, :, :n] = hk
        host[c, 1, :, :n] = hv
        ks.append(kb)
        vs.append(vb)
    return host, np.concatenate(ks, axis=1), np.concatenate(vs, axis=1)


def _oracle_rows(case, K, V, q_bits, P, rows):
    """Oracle rows of the block over the reassembled full cache (prefix + block)."""
    f = oracle.bf16_to_f64
    Kf = np.concatenate([K[None], case["block_k_bits"]], axis=2)
    Vf = np.concatenate([V[None], case["block_v_bits"]], axis=2)
    return {i: oracle.verify_attn(f(q_bits[:, i:i + 1]), f(Kf[:, :, :P + i + 1]),
                                  f(Vf[:, :, :P + i + 1]), P + i) for i in rows}


@pytest.mark.parametrize("P,chunk,slots", [(3 * 4096 + 1000, 4096, 2), (8192, 4096, 3)])
def test_staged_verify_matches_oracle_while_drafting(P, chunk, slots):
    cfg = dataclasses.replace(get_config(4), P=P)
    case = gen.staged_case(cfg, chunk=chunk, P=P)
    n_chunks = (P + chunk - 1) // chunk
    host, K, V = _host_chunks(case, n_chunks, chunk, cfg.Hkv, cfg.D)
    bk, bv = dev_bf16(case["block_k_bits"]), dev_bf16(case["block_v_bits"])
    q = dev_bf16(case["q_verify_bits"])
    st = StagedVerify(host, P, bk, bv, n_slots=slots)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")

    # drafting requests on their own stream: a small compact cache with degrees (g = 8,
    # D = 128, as the long-context workload's drafters) and a 3-row tail
    dcase = gen.attn_case(2, B=3, Hq=64, Hkv=8, P=2048, S=1024, n_recent=64, k=4, vocab=0)
    kt, vt = gen.bf16_block_rows(dcase, "k", 3), gen.bf16_block_rows(dcase, "v", 3)
    dc = vc.IndexedCache(k=dev_bf16(dcase["k_bits"]), v=dev_bf16(dcase["v_bits"]), S=1024,
                         Hq=64, idx=dev_i32(dcase["idx"]), deg=dev_i32(dcase["deg"]),
                         k_tail=dev_bf16(kt), v_tail=dev_bf16(vt), n_tail=3)
    dq = dev_bf16(dcase["q_draft_bits"])
    ref = vc.draft_attn(dq, dc, out=torch.empty(dq.shape, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    outs = []

    def draft_step(stream):
        outs.append(vc.draft_attn(dq, dc, stream=stream, out=torch.empty(
            dq.shape, dtype=torch.float32, device="cuda")))

    n = run_alongside(st, q, out, draft_step)
    torch.cuda.synchronize()
    assert n >= 1
    for o in outs:
        assert torch.equal(o, ref)
    f = oracle.bf16_to_f64
    d_ref, _ = oracle.draft_attn(f(dcase["q_draft_bits"]), f(dcase["k_bits"]),
                                 f(dcase["v_bits"]), 1024, dcase["idx"], dcase["deg"], f(kt),
                                 f(vt))
    assert_close_attn(host_f64(outs[-1]), d_ref, "draft while staging")

    got = host_f64(out)
    for i, want in _oracle_rows(case, K, V, case["q_verify_bits"], P, (0, 20, 40)).items():
        assert_close_attn(got[:, i:i + 1], want, f"staged row {i}")


def test_staged_verify_64k_token_chunks():
    """The long-context workload's own chunking: 64K-token chunks (256 MiB each) through
    a 3-slot ring, four full chunks and a 1000-row remainder, k = 40 (41 rows x 8
    heads).  Rows 0, 20 and 40 on kv heads 0 and 5 against the oracle, which follows the
    same chunks."""
    from tests.long_context import walk_chunks
    cfg = get_config(4)
    chunk = cfg.chunk_tokens
    P = 4 * chunk + 1000
    case = gen.staged_case(cfg, chunk=chunk, P=P)
    n_chunks = (P + chunk - 1) // chunk
    host = torch.empty((n_chunks, 2, cfg.Hkv, chunk, cfg.D), dtype=torch.bfloat16,
                       pin_memory=True)
    as_bf16 = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
        torch.bfloat16)

    def fill(kb, vb, s0):
        c, n = s0 // chunk, kb.shape[1]
        host[c, 0, :, :n] = as_bf16(kb)
        host[c, 1, :, :n] = as_bf16(vb)

    want = walk_chunks(case, (0, 20, 40), (0, 5), fill)
    q = dev_bf16(case["q_verify_bits"])
    st = StagedVerify(host, P, dev_bf16(case["block_k_bits"]), dev_bf16(case["block_v_bits"]),
                      n_slots=3)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    st.launch(q, out)
    st.wait()
    torch.cuda.synchronize()
    got = host_f64(out)
    g = cfg.g
    for (i, j), w in want.items():
        assert_close_attn(got[0, i, j * g:(j + 1) * g], w, f"64K chunks row {i} kv head {j}")


def test_two_launches_back_to_back_without_host_sync():
    """Two staged verifies of different queries enqueued one after the other, each query
    written on the caller's stream just before its launch and no host synchronisation in
    between: the side streams follow the caller's stream, and the second launch's copies
    into the ring wait for the first launch's verify."""
    P, chunk = 3 * 4096 + 1000, 4096
    cfg = dataclasses.replace(get_config(4), P=P)
    case = gen.staged_case(cfg, chunk=chunk, P=P)
    n_chunks = (P + chunk - 1) // chunk
    host, K, V = _host_chunks(case, n_chunks, chunk, cfg.Hkv, cfg.D)
    st = StagedVerify(host, P, dev_bf16(case["block_k_bits"]), dev_bf16(case["block_v_bits"]),
                      n_slots=2)
    q_src = dev_bf16(case["q_verify_bits"])
    outs, qs = [], []
    torch.cuda.synchronize()
    for sign in (1.0, -1.0):
        torch.cuda._sleep(2_000_000)        # the caller's stream is still busy ...
        q = q_src * sign                    # ... when it writes this launch's queries
        out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        st.launch(q, out)
        outs.append(out)
        qs.append(q)
    st.wait()
    torch.cuda.synchronize()
    q_bits = case["q_verify_bits"]
    neg = (q_bits.astype(np.uint16) ^ np.uint16(0x8000)).astype(np.uint16)
    for out, bits, name in zip(outs, (q_bits, neg), ("first", "second")):
        got = host_f64(out)
        for i, want in _oracle_rows(case, K, V, bits, P, (0, 40)).items():
            assert_close_attn(got[:, i:i + 1], want, f"{name} launch row {i}")
