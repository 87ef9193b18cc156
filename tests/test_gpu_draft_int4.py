"""Parity of vc_draft_attn over the 4-bit cache (keys per channel over 32-token groups,
values per token over 32-channel groups, fp16 scale and zero; bf16 tail) with the
fp64 oracle.

Quantisation is one of the lossy compressors the VeriCache summary ("Riepilogo
Tecnico: VeriCache", section "Supporto Architetturale") plugs in; the format is
the workload's.  The packed cache is built by the oracle's quantiser and packing
(setup; the kernels read it through their own reading of the documented layout).
Tolerance: max-abs 1e-2 and rel-L2 2e-3 on the fp32 result."""
import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
import oracle
from oracle import packing
from synth import gen
from tests.gpu_util import (assert_close_attn, both_outputs, dev_bf16, dev_f16, dev_u32,
                            host_f64)

pytestmark = pytest.mark.gpu


def _quantised(case, T_q, cap_extra=0):
    """Quantise tokens [0, T_q) of the case's K/V (bf16 values), one (batch, kv head)
    pair at a time; optional capacity padding of cap_extra garbage blocks."""
    f = oracle.bf16_to_f64
    B, Hkv, _, D = case["k_bits"].shape
    nb = T_q // 32
    out = dict(kq=np.zeros((B, Hkv, nb + cap_extra, 32, 4, D // 32), np.uint32),
               sk=np.zeros((B, Hkv, nb + cap_extra, D), np.uint16),
               zk=np.zeros((B, Hkv, nb + cap_extra, D), np.uint16),
               vq=np.zeros((B, Hkv, nb + cap_extra, D, 4), np.uint32),
               vs=np.zeros((B, Hkv, nb + cap_extra, D // 32, 32), np.uint16),
               vz=np.zeros((B, Hkv, nb + cap_extra, D // 32, 32), np.uint16))
    for b in range(B):
        for j in range(Hkv):
            if nb:
                K = f(case["k_bits"][b, j, :T_q])
                V = f(case["v_bits"][b, j, :T_q])
                qk, sk, zk = oracle.quantize_k_groups(K)
                qv, sv, zv = oracle.quantize_v_groups(V)
                out["kq"][b, j, :nb] = packing.pack_k(qk)
                out["sk"][b, j, :nb], out["zk"][b, j, :nb] = sk, zk
                out["vq"][b, j, :nb] = packing.pack_v(qv)
                out["vs"][b, j, :nb] = packing.v_scales_to_blocks(sv)
                out["vz"][b, j, :nb] = packing.v_scales_to_blocks(zv)
    if cap_extra:
        rng = np.random.default_rng(5)
        for k, a in out.items():
            a[:, :, nb:] = rng.integers(0, 2 ** 15, size=a[:, :, nb:].shape).astype(a.dtype)
    return out


def _run(case, T_q, n_tail, cap_extra=0, check_pairs=None):
    cfg = case["cfg"]
    qz = _quantised(case, T_q, cap_extra=cap_extra)
    tail_k = np.ascontiguousarray(case["k_bits"][:, :, T_q:T_q + max(n_tail, 1)])
    tail_v = np.ascontiguousarray(case["v_bits"][:, :, T_q:T_q + max(n_tail, 1)])
    cache = vc.Int4Cache(
        kq=dev_u32(qz["kq"]), k_scale=dev_f16(qz["sk"]), k_zero=dev_f16(qz["zk"]),
        vq=dev_u32(qz["vq"]), v_scale=dev_f16(qz["vs"]), v_zero=dev_f16(qz["vz"]),
        S=T_q, Hq=cfg.Hq, k_tail=dev_bf16(tail_k), v_tail=dev_bf16(tail_v), n_tail=n_tail)
    q = dev_bf16(case["q_draft_bits"])
    out = both_outputs(lambda dt: vc.draft_attn(q, cache, out=torch.empty(q.shape, dtype=dt,
                                                                        device="cuda")))
    got = host_f64(out)
    f = oracle.bf16_to_f64
    nb = T_q // 32
    lead = (slice(None), slice(None)) if check_pairs is None else check_pairs
    sel = lambda a: a[lead]
    if check_pairs is None:
        o_ref, _ = oracle.draft_attn_int4(
            f(case["q_draft_bits"]), qz["kq"][:, :, :nb], qz["sk"][:, :, :nb], qz["zk"][:, :, :nb],
            qz["vq"][:, :, :nb], qz["vs"][:, :, :nb], qz["vz"][:, :, :nb],
            f(tail_k[:, :, :n_tail]) if n_tail else None,
            f(tail_v[:, :, :n_tail]) if n_tail else None)
        assert_close_attn(got, o_ref, f"int4 T_q={T_q} tail={n_tail}")
        return
    g = cfg.g
    for b, j in check_pairs:
        bs, js = slice(b, b + 1), slice(j, j + 1)
        o_ref, _ = oracle.draft_attn_int4(
            f(case["q_draft_bits"][bs, j * g:(j + 1) * g]),
            qz["kq"][bs, js, :nb], qz["sk"][bs, js, :nb], qz["zk"][bs, js, :nb],
            qz["vq"][bs, js, :nb], qz["vs"][bs, js, :nb], qz["vz"][bs, js, :nb],
            f(tail_k[bs, js, :n_tail]) if n_tail else None,
            f(tail_v[bs, js, :n_tail]) if n_tail else None)
        assert_close_attn(got[bs, j * g:(j + 1) * g], o_ref, f"int4 pair ({b},{j})")


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 32, 8), (64, 8, 2), (128, 8, 8), (64, 16, 2)])
@pytest.mark.parametrize("T_q,n_tail", [(32, 0), (96, 5), (512, 128), (1024, 17)])
def test_shapes(D, Hq, Hkv, T_q, n_tail):
    case = gen.attn_case(3, B=2, Hq=Hq, Hkv=Hkv, D=D, P=T_q + 160, k=4, vocab=0)
    _run(case, T_q, n_tail)


def test_capacity_beyond_live_blocks():
    case = gen.attn_case(3, B=2, P=2048, k=4, vocab=0)
    _run(case, 640, 33, cap_extra=3)


def test_tail_only_and_no_tail():
    case = gen.attn_case(3, B=2, P=512, k=4, vocab=0)
    _run(case, 0, 9, cap_extra=1)   # no live quantised block: the tail alone
    _run(case, 256, 0)


def test_128k_int4_full_size_sampled_pairs():
    """Full 128K int4 sizes: batch 4, 32/8 heads, D 128, 130944 quantised tokens
    (4092 groups, 1% outlier channels x10) plus the 128-token bf16 tail."""
    cfg = gen.get_config(3)
    case = gen.attn_case(3)
    T_q = cfg.P - cfg.tail_bf16
    # the sampled pairs include kv heads that carry outlier channels (x10), so the wide
    # groups those channels make are checked, and one kv head that carries none
    out_heads = sorted({int(f) // cfg.D for f in case["outliers"]})
    clean = [j for j in range(cfg.Hkv) if j not in out_heads]
    pairs = [(0, out_heads[0]), (3, out_heads[-1]), (1, clean[0] if clean else 4)]
    assert any(j in out_heads for _, j in pairs)
    _run(case, T_q, cfg.tail_bf16, check_pairs=pairs)
