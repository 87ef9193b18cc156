"""The draft-then-verify loop end to end on the GPU (VeriCache summary, "Riepilogo
Tecnico: VeriCache", sections "Algoritmo Principale" and "Risultati Sperimentali":
outputs identical to full-KV greedy decoding).

* glue kernels: numerics against plain PyTorch fp32, and row invariance (a row's
  result does not depend on the other rows) -- the property the exactness rests on;
* the GPU loop's committed stream equals GPU full-KV greedy decoding bit for bit;
* every round's acceptance is bit-exact with the oracle given the GPU's logits;
* the GPU decoder follows the fp64 oracle decoder on its first tokens (a structural
  pin: a wrong RoPE, norm or head layout diverges at once).
"""
import dataclasses

import ctypes

import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
import oracle
from lossless_kv_compressed_b200._lib import check, lib
from lossless_kv_compressed_b200.loop import (GpuTinyLM, greedy_loop, vericache_loop,
                                              vericache_loop_csm)
from oracle import tinylm
from synth import gen
from synth.configs import LoopConfig, get_config

pytestmark = pytest.mark.gpu
S = lambda: torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("M", [1, 37])
def test_fused_norm_and_swiglu_gemms_equal_the_two_step_forms(M):
    """vc_glue_rmsnorm_gemm == vc_glue_rmsnorm then vc_glue_gemm, and vc_glue_swiglu_gemm ==
    vc_glue_swiglu then vc_glue_gemm, bit for bit (accumulating into a residual too)."""
    torch.manual_seed(M)
    d, F = 512, 1408
    x = torch.randn(M, d, device="cuda") * 3
    w1 = (torch.randn(d, 2 * F, device="cuda") * 0.02).bfloat16()
    h = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    two = torch.empty(M, 2 * F, device="cuda")
    one = torch.empty(M, 2 * F, device="cuda")
    check(lib().vc_glue_rmsnorm(x.data_ptr(), M, d, ctypes.c_float(1e-5), h.data_ptr(), S()), "rmsnorm")
    check(lib().vc_glue_gemm(h.data_ptr(), w1.data_ptr(), M, d, 2 * F, two.data_ptr(), 0, S()), "gemm")
    check(lib().vc_glue_rmsnorm_gemm(x.data_ptr(), ctypes.c_float(1e-5), w1.data_ptr(), M, d,
                                     2 * F, one.data_ptr(), 0, S()), "rmsnorm_gemm")
    torch.cuda.synchronize()
    assert torch.equal(one, two)
    gu = two
    w2 = (torch.randn(F, d, device="cuda") * 0.02).bfloat16()
    act = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
    res = torch.randn(M, d, device="cuda")
    a2, b2 = res.clone(), res.clone()
    check(lib().vc_glue_swiglu(gu.data_ptr(), M, F, act.data_ptr(), S()), "swiglu")
    check(lib().vc_glue_gemm(act.data_ptr(), w2.data_ptr(), M, F, d, a2.data_ptr(), 1, S()), "gemm")
    check(lib().vc_glue_swiglu_gemm(gu.data_ptr(), w2.data_ptr(), M, F, d, b2.data_ptr(), 1, S()),
          "swiglu_gemm")
    torch.cuda.synchronize()
    assert torch.equal(a2, b2)
    assert not torch.equal(a2, res)


@pytest.mark.parametrize("K,N", [(512, 1408 * 2), (1408, 512), (80, 128)])
def test_gemm_matches_fp32_reference_and_is_row_invariant(K, N):
    """K = 80 ends in a part-filled stage of 64 k-rows; K = 1408 runs 22 stages."""
    torch.manual_seed(K)
    a = torch.randn(37, K, device="cuda").bfloat16()
    w = (torch.randn(K, N, device="cuda") * 0.02).bfloat16()
    c = torch.empty(37, N, device="cuda")
    check(lib().vc_glue_gemm(a.data_ptr(), w.data_ptr(), 37, K, N, c.data_ptr(), 0, S()), "gemm")
    ref = a.float() @ w.float()
    torch.cuda.synchronize()
    assert (c - ref).abs().max().item() < 1e-3 * ref.abs().max().item()
    for r in (0, 5, 16, 36):
        c1 = torch.empty(1, N, device="cuda")
        check(lib().vc_glue_gemm(a[r:r + 1].data_ptr(), w.data_ptr(), 1, K, N, c1.data_ptr(), 0,
                                 S()), "gemm")
        torch.cuda.synchronize()
        assert torch.equal(c1[0], c[r]), f"gemm row {r} depends on the batch"
    # accumulate mode adds into c
    c2 = c.clone()
    check(lib().vc_glue_gemm(a.data_ptr(), w.data_ptr(), 37, K, N, c2.data_ptr(), 1, S()), "gemm")
    torch.cuda.synchronize()
    assert torch.allclose(c2, 2 * c, rtol=1e-6, atol=1e-6)


def test_rmsnorm_rope_swiglu_match_reference():
    torch.manual_seed(1)
    n, d, Hq, Hkv, D, F = 9, 512, 8, 2, 64, 1408
    x = torch.randn(n, d, device="cuda")
    h = torch.empty(n, d, dtype=torch.bfloat16, device="cuda")
    check(lib().vc_glue_rmsnorm(x.data_ptr(), n, d, 1e-5, h.data_ptr(), S()), "rmsnorm")
    ref = (x / torch.sqrt((x * x).mean(-1, keepdim=True) + 1e-5)).bfloat16()
    torch.cuda.synchronize()
    assert (h.float() - ref.float()).abs().max().item() <= 1e-2
    qkv = torch.randn(n, (Hq + 2 * Hkv) * D, device="cuda")
    pos = torch.arange(100, 100 + n, dtype=torch.int32, device="cuda")
    q = torch.empty(n, Hq, D, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(Hkv, 200, D, dtype=torch.bfloat16, device="cuda")
    vcc = torch.zeros_like(kc)
    check(lib().vc_glue_rope_store(qkv.data_ptr(), pos.data_ptr(), pos.data_ptr(), n, Hq, Hkv, D,
                                   10000.0, q.data_ptr(), kc.data_ptr(), vcc.data_ptr(), 200, S()),
          "rope")
    torch.cuda.synchronize()
    qr = tinylm.rope(qkv[:, :Hq * D].view(n, Hq, D).double().cpu().numpy(),
                     np.arange(100, 100 + n), 10000.0)
    assert np.abs(q.float().cpu().numpy() - qr).max() < 2e-2
    kr = tinylm.rope(qkv[:, Hq * D:(Hq + Hkv) * D].view(n, Hkv, D).double().cpu().numpy(),
                     np.arange(100, 100 + n), 10000.0)
    assert np.abs(kc[:, 100:100 + n].float().cpu().numpy().transpose(1, 0, 2) - kr).max() < 2e-2
    gu = torch.randn(n, 2 * F, device="cuda")
    out = torch.empty(n, F, dtype=torch.bfloat16, device="cuda")
    check(lib().vc_glue_swiglu(gu.data_ptr(), n, F, out.data_ptr(), S()), "swiglu")
    torch.cuda.synchronize()
    g, u = gu[:, :F], gu[:, F:]
    assert (out.float() - torch.nn.functional.silu(g) * u).abs().max().item() < 2e-2


SMALL = LoopConfig(n_layers=2, d_model=256, Hq=8, Hkv=2, D=64, ffn=256, vocab=512,
                   prompt_len=300, gen_tokens=64, k=8, budget=96, n_sinks=4, n_recent=16,
                   score_window=8, init_std=0.3)


def _model(cfg, weights):
    max_len = cfg.prompt_len + cfg.gen_tokens + cfg.k + 2
    return GpuTinyLM(weights, cfg, max_len, cfg.k, cfg.budget + cfg.gen_tokens + cfg.k + 2)


@pytest.mark.parametrize("cfg", [SMALL, dataclasses.replace(SMALL, init_std=0.05, k=16)])
def test_loop_commits_equal_greedy_and_accept_is_exact(cfg):
    w = gen.tinylm_weights(cfg)
    prompt = gen.tinylm_prompt(cfg)
    greedy = greedy_loop(_model(cfg, w), prompt, cfg.gen_tokens)
    rec = []
    vc_tokens, alens = vericache_loop(_model(cfg, w), prompt, cfg.gen_tokens, cfg.k, cfg.budget,
                                      cfg.n_sinks, cfg.n_recent, cfg.score_window, record=rec)
    assert vc_tokens == greedy
    assert len(alens) >= 2
    for logits, drafts, got in rec:
        want = oracle.accept(logits[None], drafts)
        for key in ("target", "accept_len", "commit", "n_commit", "err"):
            assert np.array_equal(got[key], want[key]), key
    assert vc.device_error() == 0


def test_gpu_decoder_follows_the_fp64_oracle():
    cfg = SMALL
    w = gen.tinylm_weights(cfg)
    prompt = gen.tinylm_prompt(cfg)
    n = 12
    gpu = greedy_loop(_model(cfg, w), prompt, n)
    ref = tinylm.greedy_loop(tinylm.TinyLM({k: oracle.bf16_to_f64(v) for k, v in w.items()}, cfg),
                             prompt, n)
    assert gpu == ref


def test_no_compression_accepts_every_draft():
    """Budget above the prompt: the drafter sees the whole context, so every round
    accepts all k drafts plus the bonus (VeriCache summary, step 3)."""
    cfg = dataclasses.replace(SMALL, budget=400, gen_tokens=37)
    w = gen.tinylm_weights(cfg)
    prompt = gen.tinylm_prompt(cfg)
    toks, alens = vericache_loop(_model(cfg, w), prompt, cfg.gen_tokens, cfg.k, cfg.budget,
                                 cfg.n_sinks, cfg.n_recent, cfg.score_window)
    full = (cfg.gen_tokens - 1) // (cfg.k + 1)
    assert alens[:full] == [cfg.k] * full
    assert toks == greedy_loop(_model(cfg, w), prompt, cfg.gen_tokens)


def test_tinylm_loop_full_size():
    """The tiny-decoder loop at full size: 4 layers, d 512, 8/2 heads of 64, SwiGLU
    1408, vocab 8192, N(0, 0.02) weights; 8192-token prompt, 512 generated, k = 32,
    2048-slot budget."""
    cfg = get_config(5)
    w = gen.tinylm_weights(cfg)
    prompt = gen.tinylm_prompt(cfg)
    greedy = greedy_loop(_model(cfg, w), prompt, cfg.gen_tokens)
    toks, alens = vericache_loop(_model(cfg, w), prompt, cfg.gen_tokens, cfg.k, cfg.budget,
                                 cfg.n_sinks, cfg.n_recent, cfg.score_window)
    assert toks == greedy
    assert sum(a + 1 for a in alens) >= cfg.gen_tokens - 1


def test_tinylm_loop_greedy_follows_oracle_to_a_near_tie():
    """The tiny-decoder loop model: the GPU decoder's logits stay within the
    bf16-activation error of the fp64 oracle's on the GPU's own greedy stream (the
    oracle is fed the same tokens), and
    wherever the two argmaxes differ, the oracle's margin between its pick and the GPU's
    is inside that error -- a near-tie, where either token is a correct rounding.  (The
    random N(0, 0.02) logits are near-flat: top-2 gaps of 1e-4 occur within 16 tokens.)"""
    cfg = get_config(5)
    w = gen.tinylm_weights(cfg)
    prompt = gen.tinylm_prompt(cfg)
    n = 16
    m = _model(cfg, w)
    om = tinylm.TinyLM({k: oracle.bf16_to_f64(v) for k, v in w.items()}, cfg)
    g = m.prefill(prompt).double().cpu().numpy()[0]
    o, Ks, Vs, _ = om.prefill(prompt, cfg.prompt_len + n + 1)
    p = len(prompt)
    for step in range(n):
        err = np.abs(g - o).max()
        assert err < 3e-2, f"step {step}: logit error {err:.3e}"
        tg, to = int(np.argmax(g)), int(np.argmax(o))
        if tg != to:
            margin = o[to] - o[tg]
            assert margin <= 2 * err, f"step {step}: margin {margin:.3e} > 2 x {err:.3e}"
        ids = torch.tensor([tg], dtype=torch.int32, device="cuda")
        g = m.forward(ids, 1, p, "full").double().cpu().numpy()[0]
        o = tinylm._decode_full(om, tg, p, Ks, Vs)
        p += 1


CSM_ARGS = dict(chunk=32, r_init=1.0, delta_r=0.2, r_floor=0.2, recluster_every=16)


def test_csm_loop_commits_equal_greedy_and_accept_is_exact():
    """CentroidKV's pipeline in the loop on the GPU: vc_csm_compress clusters the prompt's
    cache until it fits the budget (r_j = r_init - j delta_r), the drafts attend the
    centroids with ln n_t, accepted tokens join with degree 1 and the cache is
    re-clustered as it grows; the committed stream still equals full-KV greedy decoding
    and every round's acceptance is exact against the oracle."""
    from oracle import csm
    cfg = SMALL
    w = gen.tinylm_weights(cfg)
    prompt = gen.tinylm_prompt(cfg)
    greedy = greedy_loop(_model(cfg, w), prompt, cfg.gen_tokens)
    cap = cfg.prompt_len + cfg.gen_tokens + cfg.k + 2
    m = GpuTinyLM(w, cfg, cap, cfg.k, cap)
    rec = []
    toks, alens, sizes = vericache_loop_csm(m, prompt, cfg.gen_tokens, cfg.k, cfg.budget,
                                            cfg.n_sinks, cfg.n_recent, record=rec, **CSM_ARGS)
    assert toks == greedy
    # clustering after prefill: the sizes follow the schedule exactly (they depend on the
    # row counts only), down to the budget; then at least one re-clustering
    T, j, want = cfg.prompt_len, 0, []
    while T > cfg.budget:
        r = max(CSM_ARGS["r_floor"], CSM_ARGS["r_init"] - j * CSM_ARGS["delta_r"])
        T = csm.out_len(T, cfg.n_sinks, cfg.n_recent, CSM_ARGS["chunk"], r)
        want.append(T)
        j += 1
    assert sizes[:len(want)] == want
    assert len(sizes) > len(want)
    for logits, drafts, got in rec:
        ref = oracle.accept(logits[None], drafts)
        for key in ("target", "accept_len", "commit", "n_commit", "err"):
            assert np.array_equal(got[key], ref[key]), key
    assert vc.device_error() == 0


def test_csm_loop_full_size():
    """The tiny-decoder loop at full size with the Chunked Soft Matching cache: 8192-token
    prompt clustered to the 2048-slot budget (chunk 256), 512 tokens, k = 32."""
    cfg = get_config(5)
    w = gen.tinylm_weights(cfg)
    prompt = gen.tinylm_prompt(cfg)
    greedy = greedy_loop(_model(cfg, w), prompt, cfg.gen_tokens)
    cap = cfg.prompt_len + cfg.gen_tokens + cfg.k + 2
    m = GpuTinyLM(w, cfg, cap, cfg.k, cap)
    toks, alens, sizes = vericache_loop_csm(
        m, prompt, cfg.gen_tokens, cfg.k, cfg.budget, cfg.n_sinks, cfg.n_recent,
        chunk=cfg.csm_chunk, r_init=cfg.csm_r_init, delta_r=cfg.csm_delta_r,
        r_floor=cfg.csm_r_floor, recluster_every=cfg.csm_recluster_every)
    assert toks == greedy
    assert sizes and sizes[0] < cfg.prompt_len
