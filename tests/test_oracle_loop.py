"""Pins of the oracle's tiny decoder and its two loops.

* The decoder's prefill logits equal HuggingFace transformers' Llama model run in
  float64 with the same weights (a third-party implementation of the same
  architecture: pre-norm RMSNorm, rotate-half RoPE, SwiGLU, GQA h -> h // g).
* The VeriCache loop commits exactly the tokens of full-KV greedy decoding
  (VeriCache summary, "Riepilogo Tecnico: VeriCache", section "Risultati
  Sperimentali": identical outputs under greedy decoding).
* With no compression every draft is accepted plus the bonus (same page,
  "Algoritmo Principale", step 3).
* Eviction keeps sinks and recent tokens (CentroidKV summary, item 2).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle import tinylm
from synth import gen
from synth.configs import LoopConfig

SMALL = LoopConfig(n_layers=2, d_model=64, Hq=4, Hkv=2, D=16, ffn=96, vocab=97,
                   prompt_len=40, gen_tokens=30, k=5, budget=16, n_sinks=2, n_recent=4,
                   score_window=6, init_std=0.3)


def _model(cfg):
    w = {k: oracle.bf16_to_f64(v) for k, v in gen.tinylm_weights(cfg).items()}
    return tinylm.TinyLM(w, cfg), w


def test_prefill_matches_transformers_llama():
    from transformers import LlamaConfig, LlamaForCausalLM
    cfg = SMALL
    model, w = _model(cfg)
    hf_cfg = LlamaConfig(vocab_size=cfg.vocab, hidden_size=cfg.d_model,
                         intermediate_size=cfg.ffn, num_hidden_layers=cfg.n_layers,
                         num_attention_heads=cfg.Hq, num_key_value_heads=cfg.Hkv,
                         head_dim=cfg.D, rms_norm_eps=cfg.rms_eps, rope_theta=cfg.rope_theta,
                         tie_word_embeddings=False, attention_bias=False, mlp_bias=False,
                         max_position_embeddings=1024)
    hf = LlamaForCausalLM(hf_cfg).double().eval()
    sd = {"model.embed_tokens.weight": w["embed"], "lm_head.weight": w["lm_head"].T,
          "model.norm.weight": np.ones(cfg.d_model)}
    for l in range(cfg.n_layers):
        p = f"model.layers.{l}."
        sd[p + "self_attn.q_proj.weight"] = w[f"{l}.wq"].T
        sd[p + "self_attn.k_proj.weight"] = w[f"{l}.wk"].T
        sd[p + "self_attn.v_proj.weight"] = w[f"{l}.wv"].T
        sd[p + "self_attn.o_proj.weight"] = w[f"{l}.wo"].T
        sd[p + "mlp.gate_proj.weight"] = w[f"{l}.w_gate"].T
        sd[p + "mlp.up_proj.weight"] = w[f"{l}.w_up"].T
        sd[p + "mlp.down_proj.weight"] = w[f"{l}.w_down"].T
        sd[p + "input_layernorm.weight"] = np.ones(cfg.d_model)
        sd[p + "post_attention_layernorm.weight"] = np.ones(cfg.d_model)
    hf.load_state_dict({k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in sd.items()},
                       strict=True)
    def rope64(x, position_ids):
        # HF builds its rotary table in float32; give it the float64 one
        D = cfg.D
        inv = 1.0 / (cfg.rope_theta ** (torch.arange(0, D, 2, dtype=torch.float64) / D))
        ang = position_ids.to(torch.float64)[..., None] * inv
        emb = torch.cat([ang, ang], dim=-1)
        return emb.cos(), emb.sin()

    hf.model.rotary_emb.forward = rope64

    def make_rms64(mod):
        # HF's RMSNorm upcasts to float32; keep float64 throughout
        def fwd(x):
            return mod.weight * (x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + cfg.rms_eps))
        return fwd

    for mod in hf.modules():
        if type(mod).__name__ == "LlamaRMSNorm":
            mod.forward = make_rms64(mod)
    prompt = gen.tinylm_prompt(cfg)
    with torch.no_grad():
        ref = hf(torch.from_numpy(prompt)[None]).logits[0, -1].numpy()
    logits, _, _, _ = model.prefill(prompt, len(prompt) + 1)
    np.testing.assert_allclose(logits, ref, atol=1e-10, rtol=0)


def test_causal_attention_matches_verify_attention():
    rng = np.random.default_rng(0)
    n, Hq, Hkv, D = 23, 4, 2, 8
    q = rng.standard_normal((n, Hq, D))
    K, V = rng.standard_normal((Hkv, n, D)), rng.standard_normal((Hkv, n, D))
    out, _ = tinylm.causal_attention(q, K, V, block=5)
    ref = oracle.verify_attn(q[None], K[None], V[None], 0)[0]
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_eviction_scores_sum_probabilities():
    rng = np.random.default_rng(1)
    n, Hq, Hkv, D, W = 30, 4, 2, 8, 5
    q = rng.standard_normal((n, Hq, D))
    K, V = rng.standard_normal((Hkv, n, D)), rng.standard_normal((Hkv, n, D))
    _, sc = tinylm.causal_attention(q, K, V, score_window=W, block=7)
    # each of the g*W query rows is a distribution over keys: total mass g*W
    np.testing.assert_allclose(sc.sum(axis=1), [2 * W, 2 * W], atol=1e-12)
    # brute force for one key
    g = Hq // Hkv
    j, t = 1, 11
    want = 0.0
    for h in range(j * g, (j + 1) * g):
        for r in range(n - W, n):
            s = q[r, h] @ K[j, :r + 1].T / np.sqrt(D)
            p = np.exp(s - s.max())
            want += p[t] / p.sum()
    assert abs(sc[j, t] - want) < 1e-12


def test_evict_keeps_sinks_recent_and_top_scores():
    scores = np.array([0.0, 0.0, 5.0, 1.0, 3.0, 3.0, 9.0, 2.0, 0.5, 0.1])
    kept = tinylm.evict(scores, 10, budget=6, n_sinks=2, n_recent=2)
    # sinks 0,1; recent 8,9; middle 2..7 top-2 by score: 6 (9.0) then 2 (5.0)
    assert kept.tolist() == [0, 1, 2, 6, 8, 9]
    # tie on 3.0 between positions 4 and 5 goes to the lower position
    kept = tinylm.evict(scores, 10, budget=7, n_sinks=2, n_recent=2)
    assert kept.tolist() == [0, 1, 2, 4, 6, 8, 9]


def test_vericache_commits_equal_greedy():
    cfg = SMALL
    model, _ = _model(cfg)
    prompt = gen.tinylm_prompt(cfg)
    greedy = tinylm.greedy_loop(model, prompt, cfg.gen_tokens)
    vc, alens = tinylm.vericache_loop(model, prompt, cfg.gen_tokens, cfg.k, cfg.budget,
                                      cfg.n_sinks, cfg.n_recent, cfg.score_window)
    assert vc == greedy
    assert len(alens) >= 1 and all(0 <= a <= cfg.k for a in alens)
    # the compressed drafter must actually disagree somewhere for this to be a test
    assert min(alens) < cfg.k


def test_no_compression_accepts_every_draft_plus_bonus():
    cfg = dataclasses.replace(SMALL, gen_tokens=25)
    model, _ = _model(cfg)
    prompt = gen.tinylm_prompt(cfg)
    n = len(prompt)
    keep_all = [[np.arange(n) for _ in range(cfg.Hkv)] for _ in range(cfg.n_layers)]
    vc, alens = tinylm.vericache_loop(model, prompt, cfg.gen_tokens, cfg.k, n, 0, 0, 0,
                                      slots_override=keep_all)
    full_rounds = (cfg.gen_tokens - 1) // (cfg.k + 1)
    assert alens[:full_rounds] == [cfg.k] * full_rounds
    assert vc == tinylm.greedy_loop(model, prompt, cfg.gen_tokens)


def _csm_loop(cfg, **kw):
    model, _ = _model(cfg)
    prompt = gen.tinylm_prompt(cfg)
    args = dict(budget=20, n_sinks=2, n_recent=4, chunk=8, r_init=1.0, delta_r=0.25,
                r_floor=0.25, recluster_every=6)
    args.update(kw)
    return model, prompt, tinylm.vericache_loop_csm(model, prompt, cfg.gen_tokens, cfg.k,
                                                    **args)


def test_csm_loop_commits_equal_greedy_and_reclusters():
    """CentroidKV's pipeline inside the loop: clustering after prefill until within the
    budget, re-clustering as the cache grows, drafting over centroids with ln n; the
    committed stream is still full-KV greedy decoding (VeriCache summary, "Risultati
    Sperimentali")."""
    cfg = SMALL
    model, prompt, (toks, alens, sizes) = _csm_loop(cfg)
    assert toks == tinylm.greedy_loop(model, prompt, cfg.gen_tokens)
    assert len(sizes) >= 3                      # prefill rounds plus at least one re-cluster
    assert sizes[0] < cfg.prompt_len
    # the schedule's first rounds halve every full chunk of the middle
    from oracle import csm
    assert sizes[0] == csm.out_len(cfg.prompt_len, 2, 4, 8, 1.0)


def test_csm_loop_without_merging_accepts_every_draft():
    """r = 0 merges nothing and a budget above the prompt never clusters: the drafter
    sees the whole context, so every round accepts all k drafts plus the bonus."""
    cfg = dataclasses.replace(SMALL, gen_tokens=19)
    model, prompt, (toks, alens, sizes) = _csm_loop(cfg, budget=1000, r_init=0.0, delta_r=0.0,
                                                    r_floor=0.0)
    assert sizes == []
    full = (cfg.gen_tokens - 1) // (cfg.k + 1)
    assert alens[:full] == [cfg.k] * full
    assert toks == tinylm.greedy_loop(model, prompt, cfg.gen_tokens)
