"""Parity of vc_verify_attn (tcgen05) with the fp64 oracle.

Verify attention: VeriCache summary ("Riepilogo Tecnico: VeriCache"), section
"Algoritmo Principale", step 2 -- one pass over the full cache checks all drafts;
row i sits at position P + i and sees keys [0, P + i].
Tolerance: max-abs 1e-2 and rel-L2 2e-3 (bf16 in, fp32 accumulate, bf16 out)."""
import numpy as np
import pytest
import torch

import oracle
import lossless_kv_compressed_b200 as vc
from synth import gen
from tests.gpu_util import assert_close_attn, both_outputs, dev_bf16, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error():
    vc.device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert vc.device_error(clear=True) == 0, "a bounded wait in the verify kernel expired"


def _verify(case, P=None, n_q=None):
    cfg = case["cfg"]
    P = cfg.P if P is None else P
    q_bits = case["q_verify_bits"] if n_q is None else case["q_verify_bits"][:, :n_q]
    q = dev_bf16(q_bits)
    k, v = dev_bf16(case["k_bits"]), dev_bf16(case["v_bits"])
    out = both_outputs(lambda dt: vc.verify_attn(q, k, v, P, out=torch.empty(q.shape, dtype=dt,
                                                                              device="cuda")))
    return q_bits, out


def _oracle(case, q_bits, P):
    f = oracle.bf16_to_f64
    n_q = q_bits.shape[1]
    return oracle.verify_attn(f(q_bits), f(case["k_bits"][:, :, :P + n_q]),
                              f(case["v_bits"][:, :, :P + n_q]), P)


def test_tiny_1k_context():
    case = gen.attn_case(1)
    q_bits, out = _verify(case)
    assert_close_attn(host_f64(out), _oracle(case, q_bits, case["cfg"].P), "verify tiny 1K context")


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 32, 8), (64, 8, 2), (128, 8, 8), (64, 16, 2)])
@pytest.mark.parametrize("P,n_q", [(0, 5), (100, 1), (100, 33), (4095, 9), (4096, 41),
                                   (5000, 17), (9000, 33)])
def test_shapes(D, Hq, Hkv, P, n_q):
    case = gen.attn_case(1, B=2, Hq=Hq, Hkv=Hkv, D=D, P=P, k=n_q - 1, S=0, n_recent=0,
                         n_sinks=0, vocab=0)
    q_bits, out = _verify(case)
    assert_close_attn(host_f64(out), _oracle(case, q_bits, P), f"verify D={D} P={P} nq={n_q}")


def test_many_rows_two_row_groups():
    """n_q * g = 328 rows (three M-tiles over two row groups), as in the long-context
    workload's 41 verify positions x 8 heads."""
    case = gen.attn_case(1, B=1, Hq=64, Hkv=8, D=128, P=6000, k=40, S=0, n_recent=0, n_sinks=0,
                         vocab=0)
    q_bits, out = _verify(case)
    assert_close_attn(host_f64(out), _oracle(case, q_bits, 6000), "verify 328 rows")


@pytest.mark.parametrize("D,Hq,Hkv,P", [(128, 32, 8, 8190), (64, 8, 2, 5000)])
def test_row_invariance(D, Hq, Hkv, P):
    """Row i of a verify call over the block equals, bit for bit, the same token
    verified alone at position P + i (n_q = 1): the property that lets the loop's
    committed stream match one-token-at-a-time greedy decoding exactly."""
    n_q = 33
    case = gen.attn_case(1, B=2, Hq=Hq, Hkv=Hkv, D=D, P=P, k=n_q - 1, S=0, n_recent=0, n_sinks=0,
                         vocab=0)
    q = dev_bf16(case["q_verify_bits"])
    k, v = dev_bf16(case["k_bits"]), dev_bf16(case["v_bits"])
    f32 = lambda shape: torch.empty(shape, dtype=torch.float32, device="cuda")
    full = vc.verify_attn(q, k, v, P, out=f32(q.shape))
    for i in (0, 1, 7, 31, 32):
        qi = q[:, i:i + 1].contiguous()
        one = vc.verify_attn(qi, k, v, P + i, out=f32(qi.shape))
        torch.cuda.synchronize()
        assert torch.equal(one[:, 0], full[:, i]), f"row {i} differs"


def test_row_invariance_at_the_32k_geometry():
    """The same bit-exact row invariance on a cache large enough for vc_verify_attn to
    choose a split window other than 4096 keys (64 pairs, 32801 keys of capacity): the
    window depends on the cache only, so the block and each token alone share it."""
    from synth import device as sd
    B, Hq, Hkv, D, P, n_q = 8, 32, 8, 128, 32768, 33
    g = sd.generator(4321, "cuda")
    k = sd.normal_bf16((B, Hkv, P + n_q, D), g, "cuda")
    v = sd.normal_bf16((B, Hkv, P + n_q, D), g, "cuda")
    q = sd.normal_bf16((B, n_q, Hq, D), g, "cuda")
    f32 = lambda shape: torch.empty(shape, dtype=torch.float32, device="cuda")
    full = vc.verify_attn(q, k, v, P, out=f32(q.shape))
    for i in (0, 15, 31, 32):
        qi = q[:, i:i + 1].contiguous()
        one = vc.verify_attn(qi, k, v, P + i, out=f32(qi.shape))
        torch.cuda.synchronize()
        assert torch.equal(one[:, 0], full[:, i]), f"row {i} differs"
    assert torch.isfinite(full).all()


@pytest.mark.parametrize("chunk", [4096, 8192, 12288])
def test_chunked_equals_single_pass(chunk):
    P, n_q = 20000, 41
    case = gen.attn_case(1, B=1, Hq=64, Hkv=8, D=128, P=P, k=n_q - 1, S=0, n_recent=0, n_sinks=0,
                         vocab=0)
    q = dev_bf16(case["q_verify_bits"])
    k_all, v_all = dev_bf16(case["k_bits"]), dev_bf16(case["v_bits"])
    ref = vc.verify_attn(q, k_all, v_all, P, out=torch.empty(q.shape, device="cuda"))
    B, _, Hq, D = q.shape
    m = torch.empty((B, n_q, Hq), dtype=torch.float32, device="cuda")
    l = torch.empty_like(m)
    acc = torch.empty((B, n_q, Hq, D), dtype=torch.float32, device="cuda")
    L = P + n_q
    out = None
    for s0 in range(0, L, chunk):
        s1 = min(L, s0 + chunk)
        # each chunk lives in its own buffer, as a staged slice would
        kc = k_all[:, :, s0:s1].contiguous()
        vc_ = v_all[:, :, s0:s1].contiguous()
        flags = (vc.VC_VERIFY_FIRST if s0 == 0 else 0) | (vc.VC_VERIFY_LAST if s1 == L else 0)
        out = vc.verify_attn(q, kc, vc_, P, kv_start=s0, kv_len=s1 - s0, state=(m, l, acc),
                             flags=flags, out=torch.empty(q.shape, device="cuda"))
    torch.cuda.synchronize()
    got = host_f64(out)
    assert_close_attn(got, _oracle(case, case["q_verify_bits"], P), "chunked")
    assert np.abs(got - host_f64(ref)).max() <= 1e-2


def test_unaligned_chunk_boundaries():
    """Chunks starting off the 64-key tile grid (the block appended after a prefix of
    odd length)."""
    P, n_q = 5003, 17
    case = gen.attn_case(1, B=2, Hq=32, Hkv=8, D=128, P=P, k=n_q - 1, S=0, n_recent=0, n_sinks=0,
                         vocab=0)
    q = dev_bf16(case["q_verify_bits"])
    k_all, v_all = dev_bf16(case["k_bits"]), dev_bf16(case["v_bits"])
    B, _, Hq, D = q.shape
    m = torch.empty((B, n_q, Hq), dtype=torch.float32, device="cuda")
    l, acc = torch.empty_like(m), torch.empty((B, n_q, Hq, D), dtype=torch.float32, device="cuda")
    bounds = [0, 1000, 4100, P, P + n_q]
    for a, c in zip(bounds[:-1], bounds[1:]):
        flags = (vc.VC_VERIFY_FIRST if a == 0 else 0) | (vc.VC_VERIFY_LAST if c == P + n_q else 0)
        out = vc.verify_attn(q, k_all[:, :, a:c].contiguous(), v_all[:, :, a:c].contiguous(), P,
                             kv_start=a, kv_len=c - a, state=(m, l, acc), flags=flags,
                             out=torch.empty(q.shape, device="cuda"))
    torch.cuda.synchronize()
    assert_close_attn(host_f64(out), _oracle(case, case["q_verify_bits"], P), "odd chunks")


@pytest.fixture(scope="module")
def case2():
    return gen.attn_case(2)


def test_32k_context_sampled_rows(case2):
    """Full 32K-context size (B 8, 32/8 heads, D 128, P 32768, k 32) in the bench's
    launch configuration; the oracle recomputes sampled block positions one by one."""
    cfg = case2["cfg"]
    q_bits, out = _verify(case2)
    got = host_f64(out)
    f = oracle.bf16_to_f64
    rng = np.random.default_rng(0)
    for b, i in [(0, 0), (7, 32), (3, 16)] + [tuple(x) for x in rng.integers(0, [8, 33], (3, 2))]:
        P_i = cfg.P + i
        want = oracle.verify_attn(f(q_bits[b:b + 1, i:i + 1]), f(case2["k_bits"][b:b + 1, :, :P_i + 1]),
                                  f(case2["v_bits"][b:b + 1, :, :P_i + 1]), P_i)
        assert_close_attn(got[b:b + 1, i:i + 1], want, f"32K context b={b} i={i}")


def test_device_resident_1m_context_sampled_rows():
    """The long-context workload's verify with the whole full cache resident in HBM:
    P = 1,048,576 keys plus the 41-row block, 64/8 heads, D 128 (2.1 GB per K or V
    tensor, so byte offsets run past 2^31).  The inputs are generated and uploaded in
    64K-token chunks; the oracle follows the chunks for rows 0, 20 and 40 on kv heads
    0 and 7."""
    from synth.configs import get_config
    from tests.long_context import walk_chunks
    cfg = get_config(4)
    P, n_q = cfg.P, cfg.k + 1
    case = gen.staged_case(cfg, chunk=cfg.chunk_tokens, P=P)
    K = torch.empty((1, cfg.Hkv, P + n_q, cfg.D), dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)

    def upload(kb, vb, s0):
        n = kb.shape[1]
        K[0, :, s0:s0 + n] = dev_bf16(kb)
        V[0, :, s0:s0 + n] = dev_bf16(vb)

    want = walk_chunks(case, (0, 20, 40), (0, 7), upload)
    K[0, :, P:] = dev_bf16(case["block_k_bits"][0])
    V[0, :, P:] = dev_bf16(case["block_v_bits"][0])
    q = dev_bf16(case["q_verify_bits"])
    out = vc.verify_attn(q, K, V, P, out=torch.empty(q.shape, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    got = host_f64(out)
    g = cfg.g
    for (i, j), w in want.items():
        assert_close_attn(got[0, i, j * g:(j + 1) * g], w, f"1M context row {i} kv head {j}")
