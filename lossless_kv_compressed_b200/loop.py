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
store and SwiGLU; vc_draft_attn / vc_verify_attn / vc_accept for the method.  A round is
three library calls from the host -- vc_glue_draft_steps (the k draft steps, each argmax
written straight into the next step's input on the device), vc_glue_forward_full (the
verify pass) and vc_accept -- and the host reads back only the accepted length and the
commits.  Eviction after the prefill (attention-mass scores of the last prompt queries
and the top-budget selection) and CentroidKV's clustering run in the library too.

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
from .api import (IndexedCache, accept, csm_compress, draft_attn, draft_workspace_size,
                  evict_scores, evict_select, verify_attn, verify_workspace_size)
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
        # Chunked Soft Matching caches (compact rows + degrees), two buffers per layer:
        # a clustering round reads one and writes the other (allocated on first use)
        self.csm = None
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
            if mode == "draft" and self.csm is not None:
                kc, vcc, dc = self.csm["cur"][l]
                cache = IndexedCache(k=kc, v=vcc, S=self.S, Hq=c.Hq, deg=dc,
                                     k_tail=self.KT[l], v_tail=self.VT[l], n_tail=n_tail)
            elif mode == "draft":
                cache = IndexedCache(k=self.K[l], v=self.V[l], S=self.S, Hq=c.Hq,
                                     idx=self.idx[l], k_tail=self.KT[l], v_tail=self.VT[l],
                                     n_tail=n_tail)
            if mode == "draft":
                draft_attn(self.q[:1].view(1, c.Hq, c.D), cache,
                           out=self.att[:1].view(1, c.Hq, c.D))
            else:
                self._attend_full(n, pos0, l)
            self._gemm(self.att.view(self.rows, -1), self.wo[l], n, self.x, accumulate=True)
            self._norm(self.x, n, self.h)
            self._gemm(self.h, self.wgu[l], n, self.gu)
            check(L.vc_glue_swiglu(self.gu.data_ptr(), n, c.ffn, self.act.data_ptr(), s),
                  "vc_glue_swiglu")
            self._gemm(self.act, self.wdown[l], n, self.x, accumulate=True)
        self._norm(self.x, n, self.h)
        self._gemm(self.h, self.lm_head, n, self.logits)
        return self.logits[:n]

    PREFILL_STREAMS = 4

    def _attend_full(self, n: int, pos0: int, l: int) -> None:
        """Causal attention of rows [0, n) at positions pos0.. over layer l's full cache, in
        blocks of PREFILL_ROWS positions.  The blocks are independent (disjoint rows of q
        and att, the cache only read), so a long prompt's blocks run on a few side streams
        at once, each with its own workspace; the caller's stream waits for all of them."""
        c = self.cfg
        blocks = list(range(0, n, self.PREFILL_ROWS))
        def one(r0, ws=None):
            r1 = min(n, r0 + self.PREFILL_ROWS)
            verify_attn(self.q[r0:r1].view(1, r1 - r0, c.Hq, c.D), self.K[l], self.V[l],
                        pos0 + r0, out=self.att[r0:r1].view(1, r1 - r0, c.Hq, c.D), ws=ws)
        if len(blocks) == 1:
            one(0)
            return
        if getattr(self, "_pf", None) is None:
            need = verify_workspace_size(1, self.PREFILL_ROWS, c.Hq, c.Hkv, c.D, 0, self.max_len)
            self._pf = [(torch.cuda.Stream(device=self.dev),
                         torch.empty(need, dtype=torch.uint8, device=self.dev))
                        for _ in range(self.PREFILL_STREAMS)]
        cur = torch.cuda.current_stream(self.dev)
        for st, _ in self._pf:
            st.wait_stream(cur)
        for i, r0 in enumerate(blocks):
            st, ws = self._pf[i % len(self._pf)]
            with torch.cuda.stream(st):
                one(r0, ws)
        for st, _ in self._pf:
            cur.wait_stream(st)

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


    # ---------------------------------------------------------------- C-side drivers
    def _native(self):
        """The model descriptor of the C drivers (vericache_glue.h), rebuilt when the work
        buffers change; its workspace covers every attention call of the loop."""
        key = (self.x.data_ptr(), self.rows)
        if getattr(self, "_nat_key", None) == key:
            return self._nat
        c = self.cfg
        P = ctypes.c_void_p
        arr = lambda ts: (P * len(ts))(*[t.data_ptr() for t in ts])
        self._nat_arrays = [arr(self.wqkv), arr(self.wo), arr(self.wgu), arr(self.wdown),
                            arr(self.K), arr(self.V), arr(self.KT), arr(self.VT)]
        a = self._nat_arrays
        m = _lib.TinyLM()
        m.n_layers, m.d_model, m.Hq, m.Hkv, m.D = c.n_layers, c.d_model, c.Hq, c.Hkv, c.D
        m.ffn, m.vocab, m.rms_eps, m.rope_theta = c.ffn, c.vocab, c.rms_eps, c.rope_theta
        m.embed, m.lm_head = self.embed.data_ptr(), self.lm_head.data_ptr()
        m.wqkv, m.wo, m.wgu, m.wdown = a[0], a[1], a[2], a[3]
        m.k_full, m.v_full, m.cap = a[4], a[5], self.max_len
        m.k_tail, m.v_tail, m.tail_cap = a[6], a[7], self.k + 1
        m.positions = self.arange.data_ptr()
        m.x, m.h, m.qkv, m.q = (self.x.data_ptr(), self.h.data_ptr(), self.qkv.data_ptr(),
                                self.q.data_ptr())
        m.att, m.gu, m.act, m.logits = (self.att.data_ptr(), self.gu.data_ptr(),
                                        self.act.data_ptr(), self.logits.data_ptr())
        m.rows_cap = self.rows
        probe = IndexedCache(k=self.K[0], v=self.V[0], S=self.s_cap, Hq=c.Hq,
                             idx=self.idx[0], k_tail=self.KT[0], v_tail=self.VT[0],
                             n_tail=self.k + 1)
        need = max(lib().vc_glue_workspace_size(ctypes.byref(m)), draft_workspace_size(probe))
        self._nat_ws = torch.empty(need, dtype=torch.uint8, device=self.dev)
        m.ws, m.ws_bytes = self._nat_ws.data_ptr(), self._nat_ws.numel()
        self._nat, self._nat_key = m, key
        return m

    def _draft_caches(self):
        c = self.cfg
        out = []
        for l in range(c.n_layers):
            if self.csm is not None:
                kc, vcc, dc = self.csm["cur"][l]
                out.append(IndexedCache(k=kc, v=vcc, S=self.S, Hq=c.Hq, deg=dc).struct())
            else:
                out.append(IndexedCache(k=self.K[l], v=self.V[l], S=self.S, Hq=c.Hq,
                                        idx=self.idx[l]).struct())
        return (_lib.CompCache * len(out))(*out)

    def draft_steps(self, ids: torch.Tensor, k: int, P: int) -> None:
        """k draft steps in one library call: ids[j] at position P + j -> ids[j + 1]."""
        check(lib().vc_glue_draft_steps(ctypes.byref(self._native()), self._draft_caches(),
                                        ids.data_ptr(), k, P, self._s()), "vc_glue_draft_steps")

    def forward_full(self, ids: torch.Tensor, n: int, pos0: int) -> torch.Tensor:
        """n tokens over the full cache in one library call; logits fp32 [n, V]."""
        check(lib().vc_glue_forward_full(ctypes.byref(self._native()), ids.data_ptr(), n, pos0,
                                         self._s()), "vc_glue_forward_full")
        return self.logits[:n]

    def greedy_steps(self, ids: torch.Tensor, n: int, pos0: int) -> None:
        """n greedy steps in one library call: ids[t] at position pos0 + t -> ids[t + 1]."""
        check(lib().vc_glue_greedy_steps(ctypes.byref(self._native()), ids.data_ptr(), n, pos0,
                                         self._s()), "vc_glue_greedy_steps")

    # ---------------------------------------------------------------- CentroidKV
    def _csm_alloc(self, n: int, rounds: int = 0):
        c = self.cfg
        cap = self.s_cap
        if n > cap:
            raise ValueError(f"compressed-cache capacity {cap} < {n} rows")
        bf, i32 = torch.bfloat16, torch.int32
        mk = lambda: [(torch.empty((1, c.Hkv, cap, c.D), dtype=bf, device=self.dev),
                       torch.empty((1, c.Hkv, cap, c.D), dtype=bf, device=self.dev),
                       torch.empty((1, c.Hkv, cap), dtype=i32, device=self.dev))
                      for _ in range(c.n_layers)]
        self.csm = {"cur": mk(), "alt": mk(), "round": rounds}

    def csm_init(self, n: int):
        """The compressed cache starts as the prompt's own rows, degree 1."""
        self._csm_alloc(n)
        for l in range(self.cfg.n_layers):
            kc, vcc, dc = self.csm["cur"][l]
            kc[:, :, :n].copy_(self.K[l][:, :, :n])
            vcc[:, :, :n].copy_(self.V[l][:, :, :n])
            dc[:, :, :n].fill_(1)
        self.S = n

    def csm_export(self):
        """The compact cache as three contiguous tensors: K and V [layers, Hkv, S, D] bf16
        and the degrees [layers, Hkv, S] int32."""
        cur = self.csm["cur"]
        S = self.S
        return (torch.stack([kc[0, :, :S] for kc, _, _ in cur]),
                torch.stack([vcc[0, :, :S] for _, vcc, _ in cur]),
                torch.stack([dc[0, :, :S] for _, _, dc in cur]))

    def csm_load(self, k_rows: torch.Tensor, v_rows: torch.Tensor, deg: torch.Tensor,
                 rounds: int):
        """Take a compact cache built elsewhere (the layout of csm_export) as this model's
        compressed cache; ``rounds`` clustering rounds have already run on it."""
        S = k_rows.shape[2]
        self._csm_alloc(S, rounds)
        for l in range(self.cfg.n_layers):
            kc, vcc, dc = self.csm["cur"][l]
            kc[0, :, :S].copy_(k_rows[l])
            vcc[0, :, :S].copy_(v_rows[l])
            dc[0, :, :S].copy_(deg[l])
        self.S = S

    def csm_round(self, n_sinks: int, n_recent: int, chunk: int, r: float) -> int:
        """One Chunked Soft Matching round (vc_csm_compress) over every layer's compressed
        cache; returns the new size."""
        n_out = 0
        for l in range(self.cfg.n_layers):
            kc, vcc, dc = self.csm["cur"][l]
            ko, vo, do = self.csm["alt"][l]
            _, _, _, n_out = csm_compress(kc, vcc, n_sinks, n_recent, chunk, r, deg=dc,
                                          T=self.S, k_out=ko, v_out=vo, deg_out=do)
        self.csm["cur"], self.csm["alt"] = self.csm["alt"], self.csm["cur"]
        self.csm["round"] += 1
        self.S = n_out
        return n_out

    def csm_append(self, P: int, n: int):
        """The accepted tokens' verify-pass K/V (rows P .. P+n-1 of the full cache) join
        the compressed cache with degree 1."""
        self.csm_append_rows([self.K[l][0, :, P:P + n] for l in range(self.cfg.n_layers)],
                             [self.V[l][0, :, P:P + n] for l in range(self.cfg.n_layers)], n)

    def full_rows(self, P: int, n: int) -> torch.Tensor:
        """Rows P .. P+n-1 of the full cache, every layer: [layers, 2 (K, V), Hkv, n, D]."""
        return torch.stack([torch.stack([self.K[l][0, :, P:P + n], self.V[l][0, :, P:P + n]])
                            for l in range(self.cfg.n_layers)])

    def csm_append_rows(self, k_rows, v_rows, n: int):
        """n rows per layer ([Hkv, n, D] each) join the compressed cache with degree 1."""
        if self.S + n > self.s_cap:
            raise ValueError("compressed cache full")
        for l in range(self.cfg.n_layers):
            kc, vcc, dc = self.csm["cur"][l]
            kc[0, :, self.S:self.S + n].copy_(k_rows[l])
            vcc[0, :, self.S:self.S + n].copy_(v_rows[l])
            dc[:, :, self.S:self.S + n].fill_(1)
        self.S += n


def csm_step(model: GpuTinyLM, n_sinks: int, n_recent: int, chunk: int, r_init: float,
             delta_r: float, r_floor: float) -> int:
    """Clustering round j of the progressive schedule, r_j = max(r_floor, r_init - j
    delta_r) (CentroidKV summary, "Riassunto Tecnico: CentroidKV", section "Metodologia",
    item 3); returns the new cache size."""
    r = max(r_floor, r_init - model.csm["round"] * delta_r)
    return model.csm_round(n_sinks, n_recent, chunk, r)


def csm_fit(model: GpuTinyLM, budget: int, *sched) -> list:
    """Clustering rounds until the cache fits the budget (or a round removes nothing);
    returns the size after each round."""
    sizes = []
    while model.S > budget:
        before = model.S
        sizes.append(csm_step(model, *sched))
        if model.S == before:
            break
    return sizes


def greedy_loop(model: GpuTinyLM, prompt: np.ndarray, n_gen: int) -> list:
    """Full-KV greedy decoding on the GPU: one token per step through the verify
    attention (n_q = 1), argmax on the device, one read-back at the end; the steps after
    the prefill are enqueued by one library call."""
    logits = model.prefill(prompt)
    out = torch.empty(n_gen, dtype=torch.int32, device=model.dev)
    accept(logits.view(1, 1, -1), target=out[0:1].view(1, 1))
    model.greedy_steps(out, n_gen - 1, len(prompt))
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
        model.draft_steps(vids, k, P)
        lg = model.forward_full(vids, k + 1, P)
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


def vericache_loop_csm(model: GpuTinyLM, prompt: np.ndarray, n_gen: int, k: int, budget: int,
                       n_sinks: int, n_recent: int, chunk: int, r_init: float, delta_r: float,
                       r_floor: float, recluster_every: int, record=None):
    """Draft-then-verify decoding over a Chunked Soft Matching cache (CentroidKV summary,
    "Riassunto Tecnico: CentroidKV", section "Metodologia", items 2-4): after prefill the
    prompt's cache is clustered by vc_csm_compress until it fits the budget, with
    r_j = max(r_floor, r_init - j * delta_r) for round j; the drafts attend the centroids
    with their ln n_t bias; the accepted tokens join the cache with degree 1, and after
    every ``recluster_every`` committed tokens one more round runs if the cache is over
    the budget.  The same readings as the fp64 oracle's ``vericache_loop_csm``.
    Returns (tokens, accept lengths, cache sizes after each clustering round)."""
    n = len(prompt)
    logits = model.prefill(prompt)
    model.csm_init(n)
    sched = (n_sinks, n_recent, chunk, r_init, delta_r, r_floor)
    sizes = csm_fit(model, budget, *sched)
    dev = model.dev
    first = torch.empty((1, 1), dtype=torch.int32, device=dev)
    accept(logits.view(1, 1, -1), target=first)
    out = [int(first.item())]
    P = n
    vids = torch.empty(k + 1, dtype=torch.int32, device=dev)
    alens = []
    since = 0
    while len(out) < n_gen:
        vids[0] = out[-1]
        model.draft_steps(vids, k, P)
        lg = model.forward_full(vids, k + 1, P)
        drafts = vids[1:].view(1, k)
        r = accept(lg.view(1, k + 1, -1), drafts)
        a = int(r["accept_len"].item())
        commit = r["commit"][0, :a + 1].cpu().tolist()
        if record is not None:
            record.append((lg.detach().cpu().numpy().copy(), drafts.cpu().numpy().copy(),
                           {key: v.cpu().numpy().copy() for key, v in r.items() if v is not None}))
        alens.append(a)
        out.extend(commit)
        model.csm_append(P, a + 1)
        P += a + 1
        since += a + 1
        if since >= recluster_every:
            since = 0
            if model.S > budget:
                sizes.append(csm_step(model, *sched))
    return out[:n_gen], alens, sizes
