"""vc_draft_attn_noalloc: draft attention for callers that cannot give the library any
scratch memory (for example a plugin whose host runtime owns all device memory, or a
path that must not call cudaMalloc).  It keeps its split-K partials in a fixed 8 MiB
array inside the library, so the caller passes only inputs and outputs.

The test calls it through the C ABI three times in a row on different problems (each
call runs over whatever the one before left in the shared array; the third is a 4-bit
cache with a bf16 tail, whose partials fill the array as two sets) and compares each
result with the ordinary vc_draft_attn, which uses a caller-allocated workspace.  It also
checks that a problem too big for the fixed array is refused before anything runs.
"""
import ctypes

import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
from lossless_kv_compressed_b200._lib import CompCache, lib
from synth import gen
from tests.gpu_util import assert_close_attn, dev_bf16, dev_f16, dev_i32, dev_u32, host_f64

pytestmark = pytest.mark.gpu


def _problem(case, n_tail):
    cfg = case["cfg"]
    cache = vc.IndexedCache(
        k=dev_bf16(case["k_bits"]), v=dev_bf16(case["v_bits"]), S=cfg.S, Hq=cfg.Hq,
        idx=dev_i32(case["idx"]), deg=dev_i32(case["deg"]),
        k_tail=dev_bf16(gen.bf16_block_rows(case, "k", n_tail)),
        v_tail=dev_bf16(gen.bf16_block_rows(case, "v", n_tail)), n_tail=n_tail)
    return dev_bf16(case["q_draft_bits"]), cache


def _noalloc(q, cache):
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    s = cache.struct()
    st = lib().vc_draft_attn_noalloc(q.data_ptr(), ctypes.byref(s), 0.0, vc.VC_OUT_F32,
                                     out.data_ptr(), None,
                                     torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib().vc_last_error().decode()
    return out


def _with_workspace(q, cache):
    return vc.draft_attn(q, cache, out=torch.empty(q.shape, dtype=torch.float32, device="cuda"))


def _int4_problem(n_tail):
    """A small 4-bit cache (1024 quantised tokens per pair) with a bf16 tail: its partials
    fill the fixed array as two sets, the quantised blocks' then the tail's."""
    from tests.test_gpu_draft_int4 import _quantised
    case = gen.attn_case(3, B=2, P=1024 + 64, k=4, vocab=0)
    cfg, T_q = case["cfg"], 1024
    qz = _quantised(case, T_q)
    cache = vc.Int4Cache(
        kq=dev_u32(qz["kq"]), k_scale=dev_f16(qz["sk"]), k_zero=dev_f16(qz["zk"]),
        vq=dev_u32(qz["vq"]), v_scale=dev_f16(qz["vs"]), v_zero=dev_f16(qz["vz"]), S=T_q,
        Hq=cfg.Hq, k_tail=dev_bf16(case["k_bits"][:, :, T_q:T_q + n_tail]),
        v_tail=dev_bf16(case["v_bits"][:, :, T_q:T_q + n_tail]), n_tail=n_tail)
    return dev_bf16(case["q_draft_bits"]), cache


def test_calls_in_a_row_match_the_workspace_entry_point():
    first = _problem(gen.attn_case(2, B=4, P=8192, S=3000, n_recent=128), 17)
    second = _problem(gen.attn_case(1), 5)
    third = _int4_problem(19)
    problems = (first, second, third)
    assert all(vc.draft_workspace_size(c) <= (8 << 20) for _, c in problems)
    got = [_noalloc(*p) for p in problems]
    torch.cuda.synchronize()
    want = [_with_workspace(*p) for p in problems]
    torch.cuda.synchronize()
    for g, w, name in zip(got, want, ("first call", "second call", "third call (int4)")):
        assert_close_attn(host_f64(g), host_f64(w), name)


def test_too_large_a_problem_is_refused_before_launch():
    c = CompCache()
    c.kind, c.B, c.Hq, c.Hkv, c.D = 0, 256, 64, 8, 128   # 2048 (batch, kv head) pairs
    c.S, c.T_cap = 4096, 4096
    c.k = c.v = 1 << 20                                   # never dereferenced
    need = lib().vc_draft_workspace_size(ctypes.byref(c))
    assert need > (8 << 20)
    st = lib().vc_draft_attn_noalloc(1 << 20, ctypes.byref(c), 0.0, 0, 1 << 20, None, None)
    assert st == 2                                        # VC_ERR_UNSUPPORTED
    assert b"fixed scratch" in lib().vc_last_error()
