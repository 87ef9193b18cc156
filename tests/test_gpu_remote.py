"""Remote prefix caching with the real kernels (VeriCache summary, "Riepilogo Tecnico:
VeriCache", section "Supporto Architetturale", second scenario): a drafting side that
holds only the compact (Chunked Soft Matching) cache it was handed, and a verifying side
with the full cache, driven through the in-process transport on one GPU.

The split must change nothing: the committed stream equals full-KV greedy decoding, and
the accept lengths and cache sizes equal the one-GPU CentroidKV loop's round for round
(the drafter extends its own copy of the compact cache with the rows the verifier
returns, which are the rows the one-GPU loop appends from its own full cache).
"""
import numpy as np
import pytest

import lossless_kv_compressed_b200 as vc
from lossless_kv_compressed_b200.loop import GpuTinyLM, greedy_loop, vericache_loop_csm
from lossless_kv_compressed_b200.remote import DrafterSide, VerifierSide, run_local
from synth import gen
from synth.configs import get_config
from tests.test_gpu_loop import CSM_ARGS, SMALL, _model

pytestmark = pytest.mark.gpu


def _remote(cfg, w, prompt, chunk, r_init, delta_r, r_floor, recluster_every):
    cap = cfg.prompt_len + cfg.gen_tokens + cfg.k + 2
    sched = (cfg.budget, cfg.n_sinks, cfg.n_recent, chunk, r_init, delta_r, r_floor)
    v = VerifierSide(GpuTinyLM(w, cfg, cap, cfg.k, cap), cfg.k, sched)
    d = DrafterSide(GpuTinyLM(w, cfg, cap, cfg.k, cap), cfg.k, sched, recluster_every)
    toks, alens, link = run_local(d, v, prompt, cfg.gen_tokens)
    return toks, alens, d, link


@pytest.mark.parametrize("full", [False, True])
def test_remote_drafting_equals_the_one_gpu_loop(full):
    if full:
        cfg = get_config(5)
        args = dict(chunk=cfg.csm_chunk, r_init=cfg.csm_r_init, delta_r=cfg.csm_delta_r,
                    r_floor=cfg.csm_r_floor, recluster_every=cfg.csm_recluster_every)
    else:
        cfg, args = SMALL, CSM_ARGS
    w = gen.tinylm_weights(cfg)
    prompt = gen.tinylm_prompt(cfg)
    greedy = greedy_loop(_model(cfg, w), prompt, cfg.gen_tokens)
    cap = cfg.prompt_len + cfg.gen_tokens + cfg.k + 2
    one = GpuTinyLM(w, cfg, cap, cfg.k, cap)
    toks1, alens1, sizes1 = vericache_loop_csm(one, prompt, cfg.gen_tokens, cfg.k, cfg.budget,
                                               cfg.n_sinks, cfg.n_recent, **args)
    toks, alens, d, link = _remote(cfg, w, prompt, **args)
    assert toks == greedy == toks1
    assert alens == alens1
    # the drafter's re-clusterings are the one-GPU loop's after its prefill rounds
    assert d.sizes == sizes1[len(sizes1) - len(d.sizes):]
    assert d.m.S == one.S
    # link bytes: the compact cache once, then small messages per round
    c = cfg
    S0 = sizes1[len(sizes1) - len(d.sizes) - 1]
    assert link["setup"] == c.n_layers * c.Hkv * S0 * (2 * c.D * 2 + 4) + 32
    assert link["to_verifier"] == len(alens) * (c.k + 1) * 4
    rows = sum(a + 1 for a in alens)
    assert link["to_drafter"] == len(alens) * (c.k + 3) * 4 + rows * c.n_layers * 2 * c.Hkv * c.D * 2
    assert vc.device_error() == 0
