"""vc_int4_quantize (the int4 compressor on the GPU) is bit-exact against the oracle's
quantiser and the documented packing.

Quantisation plugs into VeriCache's uniform compression interface ("Riepilogo Tecnico:
VeriCache", section "Supporto Architetturale"); the format (keys per channel over 32
tokens, values per token over 32 channels, fp16 scale and zero) is the 128K-context
workload's.  Bytes must match exactly: nibbles, scales, zeros and words."""
import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
import oracle
from oracle import packing
from synth import gen
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def _oracle_blocks(k_bits, v_bits):
    """Packed arrays of whole 32-token blocks of one pair's rows (bits [T, D])."""
    f = oracle.bf16_to_f64
    qk, sk, zk = oracle.quantize_k_groups(f(k_bits))
    qv, sv, zv = oracle.quantize_v_groups(f(v_bits))
    return dict(kq=packing.pack_k(qk), ks=sk, kz=zk, vq=packing.pack_v(qv),
                vs=packing.v_scales_to_blocks(sv), vz=packing.v_scales_to_blocks(zv))


def _special_rows(rng, T, D):
    """bf16 rows that exercise the quantiser's edge cases: constant groups (scale 1), a
    range too small for fp16 (scale rounds to 0, then 1), exact grid values (ties at
    n + 1/2 after the division), large outliers, negative zero."""
    x = rng.standard_normal((T, D)).astype(np.float32)
    x[:32, :5] = 0.75                               # constant key groups
    x[32:64, 5] = 1e-6 + np.arange(32) * 6e-9       # span whose /15 rounds to fp16 zero
    x[64:96, 6] = np.arange(32) % 16 * 0.5          # grid values: ties at half steps
    x[:, 7] *= 1000.0                               # outlier channel
    x[3, 40:72] = -0.0
    x[4, :] = 2.5                                   # constant value groups
    x[5, 32:64] = np.linspace(-3, 3, 32) + 1.0 / 30.0   # ties after rounding the scale
    return gen.f32_to_bf16_bits(x)


@pytest.mark.parametrize("D", [64, 128])
def test_bit_exact_against_the_oracle(D):
    B, Hkv, T = 2, 3, 256
    rng = np.random.default_rng(D)
    kb = np.stack([np.stack([_special_rows(rng, T, D) for _ in range(Hkv)]) for _ in range(B)])
    vb = np.stack([np.stack([_special_rows(rng, T, D) for _ in range(Hkv)]) for _ in range(B)])
    k, v = dev_bf16(kb), dev_bf16(vb)
    # quantise rows [64, 256) into blocks 3..8 of a 10-block cache; the rest must stay
    # untouched (pre-filled with a sentinel)
    cache = vc.empty_int4_cache(B, Hkv, Hkv, D, 32 * 10)
    for t in (cache.kq, cache.vq):
        t.fill_(0x5A5A5A5A)
    for t in (cache.k_scale, cache.k_zero, cache.v_scale, cache.v_zero):
        t.view(torch.int16).fill_(0x1234)
    vc.int4_quantize(k, v, cache, n_blocks=6, src_t0=64, blk0=3)
    torch.cuda.synchronize()
    got = {"kq": cache.kq.cpu().numpy().view(np.uint32),
           "vq": cache.vq.cpu().numpy().view(np.uint32),
           "ks": cache.k_scale.cpu().numpy().view(np.uint16),
           "kz": cache.k_zero.cpu().numpy().view(np.uint16),
           "vs": cache.v_scale.cpu().numpy().view(np.uint16),
           "vz": cache.v_zero.cpu().numpy().view(np.uint16)}
    for b in range(B):
        for j in range(Hkv):
            want = _oracle_blocks(kb[b, j, 64:256], vb[b, j, 64:256])
            for name, w in want.items():
                np.testing.assert_array_equal(got[name][b, j, 3:9], w, err_msg=f"{name} ({b},{j})")
    for name in ("kq", "vq"):
        assert (got[name][:, :, :3] == 0x5A5A5A5A).all() and (got[name][:, :, 9:] == 0x5A5A5A5A).all()
    for name in ("ks", "kz", "vs", "vz"):
        assert (got[name][:, :, :3] == 0x1234).all() and (got[name][:, :, 9:] == 0x1234).all()


def test_blocks_leaving_a_bf16_window_then_draft():
    """The flush a streaming int4 cache makes: 32 tokens at a time leave the bf16 window
    and are appended as the next block; the draft over the result equals the oracle's
    draft over the oracle-packed cache."""
    case = gen.attn_case(3, B=2, P=1024 + 160, k=4, vocab=0)
    cfg = case["cfg"]
    k, v = dev_bf16(case["k_bits"]), dev_bf16(case["v_bits"])
    cache = vc.empty_int4_cache(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, 1024)
    for blk in range(32):                       # one block at a time, as tokens leave
        vc.int4_quantize(k, v, cache, n_blocks=1, src_t0=32 * blk, blk0=blk)
    cache.S = 1024
    n_tail = 128
    cache.k_tail = dev_bf16(case["k_bits"][:, :, 1024:1024 + n_tail])
    cache.v_tail = dev_bf16(case["v_bits"][:, :, 1024:1024 + n_tail])
    cache.n_tail = n_tail
    q = dev_bf16(case["q_draft_bits"])
    out = vc.draft_attn(q, cache, out=torch.empty(q.shape, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    f = oracle.bf16_to_f64
    for b in range(cfg.B):
        for j in range(cfg.Hkv):
            want = _oracle_blocks(case["k_bits"][b, j, :1024], case["v_bits"][b, j, :1024])
            np.testing.assert_array_equal(cache.kq[b, j].cpu().numpy().view(np.uint32), want["kq"])
            np.testing.assert_array_equal(cache.vq[b, j].cpu().numpy().view(np.uint32), want["vq"])
    qz = {n: [] for n in ("kq", "ks", "kz", "vq", "vs", "vz")}
    for b in range(cfg.B):
        rows = [_oracle_blocks(case["k_bits"][b, j, :1024], case["v_bits"][b, j, :1024])
                for j in range(cfg.Hkv)]
        for n in qz:
            qz[n].append(np.stack([r[n] for r in rows]))
    qz = {n: np.stack(a) for n, a in qz.items()}
    want, _ = oracle.draft_attn_int4(f(case["q_draft_bits"]), qz["kq"], qz["ks"], qz["kz"],
                                     qz["vq"], qz["vs"], qz["vz"],
                                     f(case["k_bits"][:, :, 1024:1024 + n_tail]),
                                     f(case["v_bits"][:, :, 1024:1024 + n_tail]))
    from tests.gpu_util import assert_close_attn, host_f64
    assert_close_attn(host_f64(out), want, "draft over the flushed int4 cache")
