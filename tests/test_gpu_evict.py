"""Token eviction on the GPU: attention-mass scores against the oracle's causal attention
(within fp32 rounding), and the top-budget selection bit-exact against the oracle's
eviction rule given the same scores.

Eviction by attention score: CentroidKV summary ("Riassunto Tecnico: CentroidKV"),
section "Problematica"; sinks and recent tokens kept: item 2 "Preservazione"."""
import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
import oracle
from oracle import tinylm
from synth import gen
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,W,Hq,Hkv,D", [(2000, 32, 8, 2, 64), (1500, 7, 64, 8, 128),
                                          (33, 32, 4, 4, 64), (2500, 32, 32, 8, 128)])
def test_scores_match_the_oracle(n, W, Hq, Hkv, D):
    rng = gen.children(77 + n, 3)
    qb = gen.f32_to_bf16_bits(gen.normal(rng[0], (n, Hq, D)))
    kb = gen.f32_to_bf16_bits(gen.ar1(rng[1], (Hkv,), n, D, 0.9))
    vb = np.zeros_like(kb)
    k_dev = torch.zeros((1, Hkv, n + 5, D), dtype=torch.bfloat16, device="cuda")
    k_dev[0, :, :n] = dev_bf16(kb)
    q_dev = dev_bf16(qb[None, n - W:])
    score = vc.evict_scores(q_dev, k_dev, n)
    torch.cuda.synchronize()
    f = oracle.bf16_to_f64
    _, want = tinylm.causal_attention(f(qb), f(kb), f(vb), score_window=W)
    got = score[0].double().cpu().numpy()
    np.testing.assert_allclose(got, want, rtol=2e-4, atol=1e-6)
    # total mass: W queries x g heads per kv head
    np.testing.assert_allclose(got.sum(axis=1), W * (Hq // Hkv), rtol=1e-4)


def _select_cases():
    rng = np.random.default_rng(3)
    n = 5000
    smooth = rng.random((4, n)).astype(np.float32)
    ties = np.round(rng.random((4, n)) * 8).astype(np.float32) / 8   # 9 levels: many ties
    zeros = np.zeros((2, n), np.float32)
    zeros[0, ::3] = -0.0
    zeros[1, 100:200] = 1.0
    return [smooth, ties, zeros]


@pytest.mark.parametrize("budget,ns,nr", [(2048, 4, 128), (1000, 0, 0), (132, 4, 128),
                                         (4999, 1, 1), (5000, 4, 128), (6000, 4, 128)])
def test_select_is_bit_exact_against_the_oracle_rule(budget, ns, nr):
    for sc in _select_cases():
        n = sc.shape[1]
        s_dev = torch.from_numpy(sc).cuda()
        idx = vc.evict_select(s_dev, n, budget, ns, nr)
        torch.cuda.synchronize()
        got = idx.cpu().numpy()
        for r in range(sc.shape[0]):
            want = tinylm.evict(sc[r].astype(np.float64), n, budget, ns, nr)
            np.testing.assert_array_equal(got[r, :len(want)], want)
            assert len(want) == min(budget, n)


def test_select_over_gpu_scores_at_the_loop_shape():
    """The tiny decoder's eviction shape: 8192-token prompt, last 32 queries, 8/2 heads of
    64, budget 2048 with 4 sinks and 128 recent; scores from the kernel, selection
    checked against the oracle rule on those scores."""
    n, W, Hq, Hkv, D = 8192, 32, 8, 2, 64
    rng = gen.children(5151, 2)
    q = dev_bf16(gen.f32_to_bf16_bits(gen.normal(rng[0], (1, W, Hq, D))))
    k = dev_bf16(gen.f32_to_bf16_bits(gen.ar1(rng[1], (1, Hkv), n, D, 0.9)))
    score = vc.evict_scores(q, k, n)
    idx = vc.evict_select(score, n, 2048, 4, 128)
    torch.cuda.synchronize()
    sc = score[0].double().cpu().numpy()
    got = idx[0].cpu().numpy()
    for j in range(Hkv):
        np.testing.assert_array_equal(got[j], tinylm.evict(sc[j], n, 2048, 4, 128))
