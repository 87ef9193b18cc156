"""Failure detection without any device fault.

(1) Every pipeline wait in the verify kernel is bounded; a very short limit makes the
waits run out on purpose.  The call still returns, the CTAs let their copies and
tensor-core products in flight land, release TMEM and exit, bit 0 of the library's
device error word is raised, and the next call with the normal limit is correct.
(2) The staging call has a host-side injection point (VC_FAULT_INJECT=stage_fail): the
staged verify driver surfaces the failure as an exception before anything is enqueued.
"""
import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
import oracle
from lossless_kv_compressed_b200._lib import VCError, VC_ERR_CUDA
from lossless_kv_compressed_b200.stagger import StagedVerify
from synth import gen
from synth.configs import get_config
import dataclasses
from tests.gpu_util import assert_close_attn, dev_bf16, host_f64

pytestmark = pytest.mark.gpu


def _verify_case():
    case = gen.attn_case(1, B=2, Hq=32, Hkv=8, D=128, P=8192, k=32, S=0, n_recent=0,
                         n_sinks=0, vocab=0)
    q = dev_bf16(case["q_verify_bits"])
    k, v = dev_bf16(case["k_bits"]), dev_bf16(case["v_bits"])
    return case, q, k, v


def test_expired_verify_wait_raises_the_device_error_and_the_context_survives():
    case, q, k, v = _verify_case()
    P = case["cfg"].P
    vc.device_error(clear=True)
    prev = vc.set_wait_limit(1e-8)           # 10 ns: the first wait that is not already
    try:                                     # satisfied runs out
        vc.verify_attn(q, k, v, P, out=torch.empty(q.shape, dtype=torch.float32,
                                                   device="cuda"))
        torch.cuda.synchronize()
    finally:
        vc.set_wait_limit(prev)
    assert vc.device_error(clear=True) & 1 == 1
    # the context is intact: a normal call is correct and raises nothing
    out = vc.verify_attn(q, k, v, P, out=torch.empty(q.shape, dtype=torch.float32,
                                                     device="cuda"))
    torch.cuda.synchronize()
    assert vc.device_error(clear=True) == 0
    f = oracle.bf16_to_f64
    n_q = q.shape[1]
    want = oracle.verify_attn(f(case["q_verify_bits"]), f(case["k_bits"][:, :, :P + n_q]),
                              f(case["v_bits"][:, :, :P + n_q]), P)
    assert_close_attn(host_f64(out), want, "verify after an expired wait")


def test_injected_stage_failure_surfaces_in_the_staged_verify(monkeypatch):
    P, chunk = 2 * 4096 + 100, 4096
    cfg = dataclasses.replace(get_config(4), P=P)
    case = gen.staged_case(cfg, chunk=chunk, P=P)
    n_chunks = (P + chunk - 1) // chunk
    host = torch.zeros((n_chunks, 2, cfg.Hkv, chunk, cfg.D), dtype=torch.bfloat16,
                       pin_memory=True)
    for c, (kb, vb) in enumerate(zip(case["chunks_k"], case["chunks_v"])):
        n = kb.shape[1]
        host[c, 0, :, :n] = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16)
        host[c, 1, :, :n] = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16)
    q = dev_bf16(case["q_verify_bits"])
    st = StagedVerify(host, P, dev_bf16(case["block_k_bits"]), dev_bf16(case["block_v_bits"]),
                      n_slots=2)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    monkeypatch.setenv("VC_FAULT_INJECT", "stage_fail")
    with pytest.raises(VCError) as ei:
        st.launch(q, out)
    assert ei.value.status == VC_ERR_CUDA and "injected" in str(ei.value)
    monkeypatch.delenv("VC_FAULT_INJECT")
    torch.cuda.synchronize()
    st2 = StagedVerify(host, P, dev_bf16(case["block_k_bits"]), dev_bf16(case["block_v_bits"]),
                       n_slots=2)
    st2.launch(q, out)
    st2.wait()
    torch.cuda.synchronize()
    assert vc.device_error(clear=True) == 0
    assert np.isfinite(host_f64(out)).all()
