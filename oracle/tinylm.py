"""A tiny random-init decoder and the two decoding loops, float64.

Model (the workload's "decoder-only transformer"; the pages fix no model):
pre-norm layers  x += Attn(RMSNorm(x)) ;  x += W_down(silu(W_gate h) * (W_up h))
with h = RMSNorm(x), a final RMSNorm and an untied LM head.  Readings: RMSNorm
eps 1e-5 with unit weight; rotate-half RoPE with theta 10000 applied to q and k
at absolute positions before caching (eviction never renumbers positions); GQA
head h reads kv head h // g.  Weights are given (bf16 values widened to fp64),
matrices stored [in, out] so that y = x @ W.

Loops:

* ``greedy_loop``: prefill the prompt, then decode one token at a time over the
  full KV (the baseline whose output VeriCache must reproduce).
* ``vericache_loop``: the draft-then-verify loop of the VeriCache summary
  ("Riepilogo Tecnico: VeriCache", section "Algoritmo Principale"): draft k tokens
  with the same model over the compressed cache, verify all of them with one
  forward over the full KV, accept up to the first disagreement (+ bonus), and
  resume from the last accepted token.  The compressed cache is a token-evicted
  subset built once after prefill (CentroidKV summary, "Riassunto Tecnico:
  CentroidKV", item 2: sinks and recent tokens are kept; eviction by attention
  score as in its "Problematica" section).

Readings for what the pages leave open:
the verify pass feeds the pending token plus the k drafts (k + 1 rows); on a
disagreement the full-KV prediction at that row is committed as the correction;
after a round the full cache keeps the a + 1 verified block entries, the draft
tail is dropped and the compressed cache gains the accepted tokens' verify-pass
K/V with degree 1 (no re-compression during generation).
"""
from __future__ import annotations

import numpy as np

from .accept import accept
from .attention import draft_attn, verify_attn


def rmsnorm(x, eps):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def silu(x):
    return x / (1.0 + np.exp(-x))


def rope(x, pos, theta):
    """Rotate-half RoPE.  x [..., n, H, D], pos [n]."""
    D = x.shape[-1]
    inv = theta ** (-np.arange(0, D, 2, dtype=np.float64) / D)       # [D/2]
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]  # [n, D/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


class TinyLM:
    """Weights: dict with 'embed' [V, d], 'lm_head' [d, V] and per layer l the
    keys f'{l}.wq' [d, Hq*D], f'{l}.wk' / f'{l}.wv' [d, Hkv*D], f'{l}.wo'
    [Hq*D, d], f'{l}.w_gate' / f'{l}.w_up' [d, F], f'{l}.w_down' [F, d]."""

    def __init__(self, weights: dict, cfg):
        self.w = {k: np.asarray(v, dtype=np.float64) for k, v in weights.items()}
        self.cfg = cfg

    # ---- pieces of one layer
    def qkv(self, l, x, pos):
        c = self.cfg
        h = rmsnorm(x, c.rms_eps)
        n = x.shape[0]
        q = (h @ self.w[f"{l}.wq"]).reshape(n, c.Hq, c.D)
        k = (h @ self.w[f"{l}.wk"]).reshape(n, c.Hkv, c.D)
        v = (h @ self.w[f"{l}.wv"]).reshape(n, c.Hkv, c.D)
        return rope(q, pos, c.rope_theta), rope(k, pos, c.rope_theta), v

    def finish_layer(self, l, x, attn):
        c = self.cfg
        x = x + attn.reshape(x.shape[0], c.Hq * c.D) @ self.w[f"{l}.wo"]
        h = rmsnorm(x, c.rms_eps)
        return x + (silu(h @ self.w[f"{l}.w_gate"]) * (h @ self.w[f"{l}.w_up"])) @ self.w[f"{l}.w_down"]

    def logits(self, x):
        return rmsnorm(x, self.cfg.rms_eps) @ self.w["lm_head"]

    # ---- prefill over the prompt (causal), filling the full cache
    def prefill(self, tokens, L_cap, score_window=0):
        """Returns (last-position logits [V], K, V caches [layers][Hkv, L_cap, D],
        eviction scores [layers][Hkv, n] or None)."""
        c = self.cfg
        n = len(tokens)
        x = self.w["embed"][np.asarray(tokens)]
        pos = np.arange(n)
        Ks, Vs, scores = [], [], []
        for l in range(c.n_layers):
            q, k, v = self.qkv(l, x, pos)
            Kc = np.zeros((c.Hkv, L_cap, c.D))
            Vc = np.zeros((c.Hkv, L_cap, c.D))
            Kc[:, :n] = k.transpose(1, 0, 2)
            Vc[:, :n] = v.transpose(1, 0, 2)
            attn, sc = causal_attention(q, Kc[:, :n], Vc[:, :n], score_window)
            x = self.finish_layer(l, x, attn)
            Ks.append(Kc)
            Vs.append(Vc)
            scores.append(sc)
        return self.logits(x[-1:])[0], Ks, Vs, (scores if score_window else None)


def causal_attention(q, K, V, score_window=0, block=1024):
    """Causal self-attention of n queries over their own n keys.

    q [n, Hq, D]; K, V [Hkv, n, D].  Returns (out [n, Hq, D], scores [Hkv, n] or
    None) where scores[j, t] sums, over the g heads of kv head j and the last
    ``score_window`` queries, the attention probability each gives to key t."""
    n, Hq, D = q.shape
    Hkv = K.shape[0]
    g = Hq // Hkv
    out = np.zeros((n, Hq, D))
    scores = np.zeros((Hkv, n)) if score_window else None
    for h in range(Hq):
        j = h // g
        for r0 in range(0, n, block):
            r1 = min(n, r0 + block)
            s = q[r0:r1, h] @ K[j, :r1].T / np.sqrt(D)                # [rows, r1]
            allowed = np.arange(r1)[None, :] <= np.arange(r0, r1)[:, None]
            s = np.where(allowed, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            out[r0:r1, h] = p @ V[j, :r1]
            if score_window:
                lo = max(r0, n - score_window)
                if lo < r1:
                    scores[j, :r1] += p[lo - r0:].sum(axis=0)
    return out, scores


def evict(scores, n, budget, n_sinks, n_recent):
    """Kept positions (ascending) of one (layer, kv head): sinks, the recent
    window, and the highest-scoring middle positions (ties to the lower
    position) up to ``budget``.  Degrees are all 1."""
    if budget >= n:
        return np.arange(n)
    lo, hi = n_sinks, n - n_recent
    mid = np.arange(lo, hi)
    order = np.lexsort((mid, -scores[lo:hi]))[: budget - n_sinks - n_recent]
    return np.concatenate([np.arange(n_sinks), np.sort(mid[order]), np.arange(hi, n)])


def _decode_full(model, tok, p, Ks, Vs):
    """One token at position p over the full caches (written in place)."""
    c = model.cfg
    x = model.w["embed"][[tok]]
    for l in range(c.n_layers):
        q, k, v = model.qkv(l, x, [p])
        Ks[l][:, p] = k[0]
        Vs[l][:, p] = v[0]
        o = verify_attn(q[None], Ks[l][None, :, :p + 1], Vs[l][None, :, :p + 1], p)
        x = model.finish_layer(l, x, o[0])
    return model.logits(x)[0]


def greedy_loop(model, prompt, n_gen):
    """Greedy decoding over the full KV; returns the n_gen generated tokens."""
    c = model.cfg
    L_cap = len(prompt) + n_gen + 1
    logits, Ks, Vs, _ = model.prefill(prompt, L_cap)
    out = [int(accept(logits[None, None])["target"][0, 0])]
    p = len(prompt)
    while len(out) < n_gen:
        logits = _decode_full(model, out[-1], p, Ks, Vs)
        out.append(int(accept(logits[None, None])["target"][0, 0]))
        p += 1
    return out


def vericache_loop(model, prompt, n_gen, k, budget, n_sinks, n_recent, score_window,
                   slots_override=None):
    """Draft-then-verify decoding.  Returns (generated tokens, accept lengths a
    per round).  ``slots_override`` (list per layer of [Hkv] position arrays)
    replaces the eviction choice, e.g. to keep every position."""
    c = model.cfg
    n = len(prompt)
    L_cap = n + n_gen + k + 2
    logits, Ks, Vs, scores = model.prefill(prompt, L_cap, score_window)
    if slots_override is not None:
        slots = [[np.asarray(s, dtype=np.int64) for s in layer] for layer in slots_override]
    else:
        slots = [[evict(scores[l][j], n, budget, n_sinks, n_recent) for j in range(c.Hkv)]
                 for l in range(c.n_layers)]
    out = [int(accept(logits[None, None])["target"][0, 0])]
    P = n
    accept_lens = []
    while len(out) < n_gen:
        pending = out[-1]
        # ---- draft k tokens over the compressed cache + the draft tail
        tails_k = [np.zeros((c.Hkv, 0, c.D)) for _ in range(c.n_layers)]
        tails_v = [np.zeros((c.Hkv, 0, c.D)) for _ in range(c.n_layers)]
        drafts = []
        x_tok = pending
        for j in range(k):
            x = model.w["embed"][[x_tok]]
            for l in range(c.n_layers):
                q, kk, vv = model.qkv(l, x, [P + j])
                tails_k[l] = np.concatenate([tails_k[l], kk.transpose(1, 0, 2)], axis=1)
                tails_v[l] = np.concatenate([tails_v[l], vv.transpose(1, 0, 2)], axis=1)
                S = len(slots[l][0])
                idx = np.stack(slots[l])[None]                       # [1, Hkv, S]
                o, _ = draft_attn(q, Ks[l][None], Vs[l][None], S, idx, None,
                                  tails_k[l][None], tails_v[l][None])
                x = model.finish_layer(l, x, o)
            d = int(accept(model.logits(x)[None])["target"][0, 0])
            drafts.append(d)
            x_tok = d
        # ---- verify the pending token + k drafts over the full cache
        toks = [pending] + drafts
        pos = np.arange(P, P + k + 1)
        x = model.w["embed"][toks]
        for l in range(c.n_layers):
            q, kk, vv = model.qkv(l, x, pos)
            Ks[l][:, P:P + k + 1] = kk.transpose(1, 0, 2)
            Vs[l][:, P:P + k + 1] = vv.transpose(1, 0, 2)
            o = verify_attn(q[None], Ks[l][None, :, :P + k + 1], Vs[l][None, :, :P + k + 1], P)
            x = model.finish_layer(l, x, o[0])
        r = accept(model.logits(x)[None], np.array([drafts]))
        a = int(r["accept_len"][0])
        accept_lens.append(a)
        commit = [int(t) for t in r["commit"][0, :a + 1]]
        out.extend(commit)
        # ---- cache update: keep a+1 block rows, append them to the compressed cache
        for l in range(c.n_layers):
            Ks[l][:, P + a + 1:P + k + 1] = 0.0
            Vs[l][:, P + a + 1:P + k + 1] = 0.0
            for j in range(c.Hkv):
                slots[l][j] = np.concatenate([slots[l][j], np.arange(P, P + a + 1)])
        P += a + 1
    return out[:n_gen], accept_lens


def vericache_loop_csm(model, prompt, n_gen, k, budget, n_sinks, n_recent, chunk, r_init,
                       delta_r, r_floor, recluster_every):
    """Draft-then-verify decoding whose compressed cache is built by CentroidKV's Chunked
    Soft Matching ("Riassunto Tecnico: CentroidKV", section "Metodologia": item 2, the
    inference pipeline -- a clustering round after prefill when the cache exceeds the
    budget, re-clustering every g decoding steps, sinks and recent tokens preserved;
    item 3, the progressive schedule r_j = r_init - j * delta_r; item 4, drafting over
    degree-weighted centroids with ln n_t in the softmax).  Returns (generated tokens,
    accept lengths, cache sizes after each clustering round).

    Readings: after prefill, rounds run until the cache is within the budget (each round
    can at most halve a chunk, so one may not suffice); r_j never drops below r_floor;
    the accepted tokens' verify-pass K/V join the compressed cache with degree 1 (the
    draft tail is dropped, as in ``vericache_loop``); after every ``recluster_every``
    committed tokens one more round runs if the cache is over the budget."""
    from . import csm
    c = model.cfg
    n = len(prompt)
    L_cap = n + n_gen + k + 2
    logits, Ks, Vs, _ = model.prefill(prompt, L_cap)
    comp = [[[Ks[l][j, :n].copy(), Vs[l][j, :n].copy(), np.ones(n, np.int64)]
             for j in range(c.Hkv)] for l in range(c.n_layers)]
    state = {"j": 0}
    sizes = []

    def cluster_round():
        r = max(r_floor, r_init - state["j"] * delta_r)
        for l in range(c.n_layers):
            for j in range(c.Hkv):
                Kc, Vc, nc = comp[l][j]
                Ko, Vo, no, _ = csm.compress(Kc, Vc, nc, n_sinks, n_recent, chunk, r)
                comp[l][j] = [Ko, Vo, no]
        state["j"] += 1
        sizes.append(len(comp[0][0][2]))

    while len(comp[0][0][2]) > budget:
        before = len(comp[0][0][2])
        cluster_round()
        if len(comp[0][0][2]) == before:       # nothing left to merge
            break
    out = [int(accept(logits[None, None])["target"][0, 0])]
    P = n
    accept_lens = []
    since = 0
    while len(out) < n_gen:
        pending = out[-1]
        tails_k = [np.zeros((c.Hkv, 0, c.D)) for _ in range(c.n_layers)]
        tails_v = [np.zeros((c.Hkv, 0, c.D)) for _ in range(c.n_layers)]
        drafts = []
        x_tok = pending
        for jd in range(k):
            x = model.w["embed"][[x_tok]]
            for l in range(c.n_layers):
                q, kk, vv = model.qkv(l, x, [P + jd])
                tails_k[l] = np.concatenate([tails_k[l], kk.transpose(1, 0, 2)], axis=1)
                tails_v[l] = np.concatenate([tails_v[l], vv.transpose(1, 0, 2)], axis=1)
                Kc = np.stack([comp[l][j][0] for j in range(c.Hkv)])[None]
                Vc = np.stack([comp[l][j][1] for j in range(c.Hkv)])[None]
                deg = np.stack([comp[l][j][2] for j in range(c.Hkv)])[None]
                o, _ = draft_attn(q, Kc, Vc, Kc.shape[2], None, deg, tails_k[l][None],
                                  tails_v[l][None])
                x = model.finish_layer(l, x, o)
            d = int(accept(model.logits(x)[None])["target"][0, 0])
            drafts.append(d)
            x_tok = d
        toks = [pending] + drafts
        pos = np.arange(P, P + k + 1)
        x = model.w["embed"][toks]
        for l in range(c.n_layers):
            q, kk, vv = model.qkv(l, x, pos)
            Ks[l][:, P:P + k + 1] = kk.transpose(1, 0, 2)
            Vs[l][:, P:P + k + 1] = vv.transpose(1, 0, 2)
            o = verify_attn(q[None], Ks[l][None, :, :P + k + 1], Vs[l][None, :, :P + k + 1], P)
            x = model.finish_layer(l, x, o[0])
        r = accept(model.logits(x)[None], np.array([drafts]))
        a = int(r["accept_len"][0])
        accept_lens.append(a)
        out.extend(int(t) for t in r["commit"][0, :a + 1])
        for l in range(c.n_layers):
            Ks[l][:, P + a + 1:P + k + 1] = 0.0
            Vs[l][:, P + a + 1:P + k + 1] = 0.0
            for j in range(c.Hkv):
                comp[l][j][0] = np.concatenate([comp[l][j][0], Ks[l][j, P:P + a + 1]])
                comp[l][j][1] = np.concatenate([comp[l][j][1], Vs[l][j, P:P + a + 1]])
                comp[l][j][2] = np.concatenate([comp[l][j][2], np.ones(a + 1, np.int64)])
        P += a + 1
        since += a + 1
        if since >= recluster_every:
            since = 0
            if len(comp[0][0][2]) > budget:
                cluster_round()
    return out[:n_gen], accept_lens, sizes
