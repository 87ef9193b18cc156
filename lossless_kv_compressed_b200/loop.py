"""The draft-then-verify loop end to end on the GPU (tiny decoder-only transformer).

VeriCache summary ("Riepilogo Tecnico: VeriCache", section "Algoritmo Principale"):
the same model drafts k tokens over the compressed cache, one forward pass over the
full cache verifies them, tokens are accepted up to the first disagreement (plus the
bonus when all agree) and the loop resumes from the last accepted token.  The
compressed cache keeps attention sinks and recent tokens and fills the budget by
attention score (CentroidKV summary, "Riassunto Tecnico: CentroidKV", item 2 and
section "Problematica").

Everything per token runs in libvericache.so: glue kernels (vericache_glue.h) for
embedding, RMSNorm, fused QKV / O / gate-up / down / LM-head GEMMs, RoPE with the cache
store and SwiGLU; vc_draft_attn / vc_verify_attn / vc_accept for the method.  Token ids
stay on the device between draft steps (each argmax is written straight into the next
step's input); the host reads back only the accepted length and the commits, once per
round.  Eviction after the prefill (attention-mass scores of the last prompt queries and
the top-budget selection) runs in the library too.

Readings (same as the fp64 oracle in oracle/tinylm.py): k+1 verify rows (pending token +
k drafts); on a disagreement the full-KV prediction is committed as the correction; the
full cache keeps the a+1 verified block rows; the compressed cache gains those positions
with degree 1 and the draft tail is dropped; no re-compression during generation.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib
from .api import (IndexedCache, accept, draft_attn, draft_workspace_size, evict_scores,
                  evict_select, verify_attn)
from ._lib import check, lib


def _b16(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


class GpuTinyLM:
    """Weights: dict of bf16 bits (as from synth.gen.tinylm_weights), [in, out] layout."""

    PREFILL_ROWS = 256

    def __init__(self, weights: dict, cfg, max_len: int, k: int, s_cap: int, device="cuda"):
        self.cfg = cfg
        self.dev = torch.device(device)
        d, Hq, Hkv, D, F = cfg.d_model, cfg.Hq, cfg.Hkv, cfg.D, cfg.ffn
        self.nqkv = (Hq + 2 * Hkv) * D
        W = lambda n: _b16(weights[n], self.dev)
        self.embed = W("embed")
        self.lm_head = W("lm_head")
        self.wqkv, self.wo, self.wgu, self.wdown = [], [], [], []
        for l in range(cfg.n_layers):
            self.wqkv.append(_b16(np.concatenate(
                [weights[f"{l}.wq"], weights[f"{l}.wk"], weights[f"{l}.wv"]], axis=1), self.dev))
            self.wo.append(W(f"{l}.wo"))
            self.wgu.append(_b16(np.concatenate([weights[f"{l}.w_gate"], weights[f"{l}.w_up"]],
                                                axis=1), self.dev))
            self.wdown.append(W(f"{l}.w_down"))
        self.max_len, self.k, self.s_cap = max_len, k, s_cap
        bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
        z = lambda *s, dt=bf: torch.zeros(s, dtype=dt, device=self.dev)
        L = cfg.n_layers
        self.K = [z(1, Hkv, max_len, D) for _ in range(L)]
        self.V = [z(1, Hkv, max_len, D) for _ in range(L)]
        self.KT = [z(1, Hkv, k + 1, D) for _ in range(L)]       # draft tails
        self.VT = [z(1, Hkv, k + 1, D) for _ in range(L)]
        self.idx = [z(1, Hkv, s_cap, dt=i32) for _ in range(L)]  # compressed slots
        self.S = 0
        self.arange = torch.arange(max_len + k + 2, dtype=i32, device=self.dev)
        rows = max(self.PREFILL_ROWS, k + 1)
        self._alloc(rows)
        self.stream = torch.cuda.current_stream(self.dev)

    def _alloc(self, rows):
        c = self.cfg
        f32, bf = torch.float32, torch.bfloat16
        e = lambda *s, dt=f32: torch.empty(s, dtype=dt, device=self.dev)
        self.rows = rows
        self.x = e(rows, c.d_model)
        self.h = e(rows, c.d_model, dt=bf)
        self.qkv = e(rows, self.nqkv)
        self.q = e(rows, c.Hq, c.D, dt=bf)
        self.att = e(rows, c.Hq, c.D, dt=bf)
        self.gu = e(rows, 2 * c.ffn)
        self.act = e(rows, c.ffn, dt=bf)
        self.logits = e(rows, c.vocab)
        self.qlast = []                                            # eviction queries

    # ---------------------------------------------------------------- pieces
    def _s(self):
        return torch.cuda.current_stream(self.dev).cuda_stream

    def _gemm(self, a, w, M, c, accumulate=False):
        K, N = w.shape
        check(lib().vc_glue_gemm(a.data_ptr(), w.data_ptr(), M, K, N, c.data_ptr(),
                                 int(accumulate), self._s()), "vc_glue_gemm")

    def _norm(self, x, n, out):
        check(lib().vc_glue_rmsnorm(x.data_ptr(), n, self.cfg.d_model, self.cfg.rms_eps,
                                    out.data_ptr(), self._s()), "vc_glue_rmsnorm")

    def forward(self, ids: torch.Tensor, n: int, pos0: int, mode: str, P: int = 0,
                n_tail: int = 0, keep_last: int = 0) -> torch.Tensor:
        """Logits fp32 [n, V] of n tokens at positions pos0 .. pos0+n-1.

        mode 'full': attention over the full cache (K/V stored at their positions; rows
        attend causally -- prefill, greedy steps and the verify block); 'draft': one token
        over the compressed cache plus the draft tail (its K/V stored at tail row n_tail-1).
        """
        c = self.cfg
        L = lib()
        s = self._s()
        check(L.vc_glue_embed(self.embed.data_ptr(), ids.data_ptr(), n, c.d_model,
                              self.x.data_ptr(), s), "vc_glue_embed")
        pos = self.arange[pos0:]
        for l in range(c.n_layers):
            self._norm(self.x, n, self.h)
            self._gemm(self.h, self.wqkv[l], n, self.qkv)
            if mode == "draft":
                dst, kc, vcache, cap = self.arange[n_tail - 1:], self.KT[l], self.VT[l], self.k + 1
            else:
                dst, kc, vcache, cap = pos, self.K[l], self.V[l], self.max_len
            check(L.vc_glue_rope_store(self.qkv.data_ptr(), pos.data_ptr(), dst.data_ptr(), n,
                                       c.Hq, c.Hkv, c.D, c.rope_theta, self.q.data_ptr(),
                                       kc.data_ptr(), vcache.data_ptr(), cap, s),
                  "vc_glue_rope_store")
            if keep_last:
                self.qlast.append(self.q[n - keep_last:n].clone())
            if mode == "draft":
                cache = IndexedCache(k=self.K[l], v=self.V[l], S=self.S, Hq=c.Hq,
                                     idx=self.idx[l], k_tail=self.KT[l], v_tail=self.VT[l],
                                     n_tail=n_tail)
                draft_attn(self.q[:1].view(1, c.Hq, c.D), cache,
                           out=self.att[:1].view(1, c.Hq, c.D))
            else:
                for r0 in range(0, n, self.PREFILL_ROWS):
                    r1 = min(n, r0 + self.PREFILL_ROWS)
                    verify_attn(self.q[r0:r1].view(1, r1 - r0, c.Hq, c.D), self.K[l],
                                self.V[l], pos0 + r0, out=self.att[r0:r1].view(1, r1 - r0,
                                                                                c.Hq, c.D))
            self._gemm(self.att.view(self.rows, -1), self.wo[l], n, self.x, accumulate=True)
            self._norm(self.x, n, self.h)
            self._gemm(self.h, self.wgu[l], n, self.gu)
            check(L.vc_glue_swiglu(self.gu.data_ptr(), n, c.ffn, self.act.data_ptr(), s),
                  "vc_glue_swiglu")
            self._gemm(self.act, self.wdown[l], n, self.x, accumulate=True)
        self._norm(self.x, n, self.h)
        self._gemm(self.h, self.lm_head, n, self.logits)
        return self.logits[:n]

    # ---------------------------------------------------------------- prefill
    def prefill(self, prompt: np.ndarray, score_window: int = 0):
        n = len(prompt)
        if n > self.rows:
            self._alloc(n)
        ids = torch.from_numpy(np.asarray(prompt, dtype=np.int32)).to(self.dev)
        self.qlast = []
        logits = self.forward(ids, n, 0, "full", keep_last=score_window)
        return logits[n - 1:n]

    def evict(self, n: int, budget: int, n_sinks: int, n_recent: int):
        """Per layer and kv head keep sinks, the recent window and the middle positions
        with the highest attention mass from the last prompt queries (ties to the lower
        position); positions ascending, degree 1.  Scores and selection run in the
        library (vc_evict_scores, vc_evict_select)."""
        c = self.cfg
        for l in range(c.n_layers):
            q = self.qlast[l].view(1, *self.qlast[l].shape)      # [1, W, Hq, D]
            score = evict_scores(q, self.K[l], n)
            evict_select(score, n, budget, n_sinks, n_recent, idx=self.idx[l])
        self.S = min(budget, n)


def greedy_loop(model: GpuTinyLM, prompt: np.ndarray, n_gen: int) -> list:
    """Full-KV greedy decoding on the GPU: one token per step through the verify
    attention (n_q = 1), argmax on the device, one read-back at the end."""
    logits = model.prefill(prompt)
    out = torch.empty(n_gen, dtype=torch.int32, device=model.dev)
    accept(logits.view(1, 1, -1), target=out[0:1].view(1, 1))
    p = len(prompt)
    for t in range(1, n_gen):
        lg = model.forward(out[t - 1:t], 1, p, "full")
        accept(lg.view(1, 1, -1), target=out[t:t + 1].view(1, 1))
        p += 1
    return out.cpu().tolist()


def vericache_loop(model: GpuTinyLM, prompt: np.ndarray, n_gen: int, k: int, budget: int,
                   n_sinks: int, n_recent: int, score_window: int, record=None):
    """Draft-then-verify decoding on the GPU.  Returns (tokens, accept lengths).
    ``record`` (a list) receives (verify logits, drafts, accept outputs) per round."""
    n = len(prompt)
    logits = model.prefill(prompt, score_window)
    model.evict(n, budget, n_sinks, n_recent)
    dev = model.dev
    first = torch.empty((1, 1), dtype=torch.int32, device=dev)
    accept(logits.view(1, 1, -1), target=first)
    out = [int(first.item())]
    P = n
    vids = torch.empty(k + 1, dtype=torch.int32, device=dev)   # pending + drafts
    alens = []
    while len(out) < n_gen:
        vids[0] = out[-1]
        for j in range(k):
            lg = model.forward(vids[j:j + 1], 1, P + j, "draft", n_tail=j + 1)
            accept(lg.view(1, 1, -1), target=vids[j + 1:j + 2].view(1, 1))
        lg = model.forward(vids, k + 1, P, "full")
        drafts = vids[1:].view(1, k)
        r = accept(lg.view(1, k + 1, -1), drafts)
        a = int(r["accept_len"].item())
        commit = r["commit"][0, :a + 1].cpu().tolist()
        if record is not None:
            record.append((lg.detach().cpu().numpy().copy(), drafts.cpu().numpy().copy(),
                           {key: v.cpu().numpy().copy() for key, v in r.items() if v is not None}))
        alens.append(a)
        out.extend(commit)
        for l in range(model.cfg.n_layers):
            check(lib().vc_glue_append_slots(model.idx[l].data_ptr(), None, model.cfg.Hkv,
                                             model.s_cap, model.S, P, a + 1, model._s()),
                  "vc_glue_append_slots")
        model.S += a + 1
        P += a + 1
    return out[:n_gen], alens
