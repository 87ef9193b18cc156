"""Staggered long-context verification (VeriCache summary, "Riepilogo Tecnico:
VeriCache", sections "Supporto Architetturale" and "Scaglionamento tra Risorse (P1)"):
the full cache streams chunk by chunk from pinned host memory through a device ring
while other requests draft on their own stream.  The staged verify matches the
oracle, and the concurrent drafts match the same drafts run alone, bit for bit."""
import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
import oracle
from lossless_kv_compressed_b200.stagger import StagedVerify, run_alongside
from synth import gen
from synth.configs import get_config
import dataclasses
from tests.gpu_util import assert_close_attn, dev_bf16, dev_i32, host_f64

pytestmark = pytest.mark.gpu


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

    # drafting requests on their own stream: a small compact cache
    dcase = gen.attn_case(2, B=3, Hq=64, Hkv=8, P=2048, S=1024, n_recent=64, k=4, vocab=0)
    dc = vc.IndexedCache(k=dev_bf16(dcase["k_bits"]), v=dev_bf16(dcase["v_bits"]), S=1024,
                         Hq=64, idx=dev_i32(dcase["idx"]), deg=dev_i32(dcase["deg"]))
    dq = dev_bf16(dcase["q_draft_bits"])
    ref = vc.draft_attn(dq, dc)
    torch.cuda.synchronize()
    outs = []

    def draft_step(stream):
        outs.append(vc.draft_attn(dq, dc, stream=stream))

    n = run_alongside(st, q, out, draft_step)
    torch.cuda.synchronize()
    assert n >= 1
    for o in outs:
        assert torch.equal(o, ref)

    # oracle over the reassembled full cache (prefix from the chunks + the block)
    f = oracle.bf16_to_f64
    Kf = np.concatenate([K[None], case["block_k_bits"]], axis=2)
    Vf = np.concatenate([V[None], case["block_v_bits"]], axis=2)
    got = host_f64(out)
    for i in (0, 20, 40):
        want = oracle.verify_attn(f(case["q_verify_bits"][:, i:i + 1]), f(Kf[:, :, :P + i + 1]),
                                  f(Vf[:, :, :P + i + 1]), P + i)
        assert_close_attn(got[:, i:i + 1], want, f"staged row {i}")
    assert vc.device_error() == 0
