"""Seeded generators: random draws and their layout, nothing else.

Every tensor comes from its own child of ``SeedSequence(seed)`` (NumPy PCG64),
so adding a tensor never changes the others.  Floating-point tensors are
returned as float32 plus, where the kernels consume bf16 / fp16, the exact
storage bits (uint16) obtained by round-to-nearest-even.

Recipe (shapes and distributions of the pages' workloads, see the workload
table in ``synth.configs``):

* Keys and values: AR(1) along the sequence per (batch, kv head, channel),
  x_0 = e_0, x_t = rho * x_{t-1} + sqrt(1 - rho^2) * e_t with e ~ N(0, 1), so the
  correlation rho^|dt| decays monotonically and convexly with distance, which is
  the shape the CentroidKV summary reports for key similarity (section
  "Metodologia: CentroidKV", item 1, "Osservazioni").  rho = 0 gives i.i.d. N(0,1).
* Compressed slots: sinks [0, n_sinks) and the recent window [P - n_recent, P)
  are always kept (CentroidKV summary, item 2 "Pipeline di Inferenza",
  "Preservazione"); the remaining budget takes the top scores of i.i.d. U(0,1)
  draws over the middle positions (ties to the lower position), sorted ascending.
  Degrees n_t ~ U{1..deg_max} on those kept middle slots and 1 on sinks / recent.
* Queries: i.i.d. N(0, 1).
* Acceptance logits: i.i.d. N(0, 1); where a workload asks for agreement with
  the drafts on a prefix, the draft token's logit is lifted above the row max.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
from numpy.random import PCG64, Generator, SeedSequence
from scipy.signal import lfilter

from .configs import AttnConfig, get_config


# ---------------------------------------------------------------- storage bits
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); return the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


# ---------------------------------------------------------------- draws
def children(seed: int, n: int) -> list:
    return [Generator(PCG64(s)) for s in SeedSequence(seed).spawn(n)]


def normal(rng: Generator, shape) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32)


def ar1(rng: Generator, lead: tuple, L: int, D: int, rho: float) -> np.ndarray:
    """AR(1) along axis -2 of a [*lead, L, D] float32 array (see module doc)."""
    e = rng.standard_normal((*lead, L, D), dtype=np.float32)
    if rho == 0.0:
        return e
    b0 = math.sqrt(1.0 - rho * rho)
    e[..., 0, :] /= b0  # so that x_0 = e_0 after the filter's b0 gain
    return lfilter([b0], [1.0, -rho], e, axis=-2).astype(np.float32)


def slot_indices(rng: Generator, lead: tuple, P: int, S: int, n_sinks: int,
                 n_recent: int) -> np.ndarray:
    """Ascending kept positions [*lead, S] (int32): sinks + recent + top random scores."""
    n_mid = S - n_sinks - n_recent
    lo, hi = n_sinks, P - n_recent
    if n_mid < 0 or n_mid > hi - lo:
        raise ValueError("slot budget does not fit the context")
    n_rows = int(np.prod(lead)) if lead else 1
    scores = rng.random((n_rows, hi - lo))
    out = np.empty((n_rows, S), dtype=np.int32)
    sinks = np.arange(n_sinks, dtype=np.int32)
    recent = np.arange(hi, P, dtype=np.int32)
    pos = np.arange(lo, hi, dtype=np.int64)
    for r in range(n_rows):
        # highest score first, ties to the lower position
        order = np.lexsort((pos, -scores[r]))[:n_mid]
        mid = np.sort(pos[order]).astype(np.int32)
        out[r] = np.concatenate([sinks, mid, recent])
    return out.reshape(*lead, S)


def slot_degrees(rng: Generator, lead: tuple, S: int, n_sinks: int, n_recent: int,
                 deg_max: int) -> np.ndarray:
    """Degrees [*lead, S] (int32): U{1..deg_max} on middle slots, 1 on sinks and recent."""
    deg = rng.integers(1, deg_max + 1, size=(*lead, S), dtype=np.int32)
    deg[..., :n_sinks] = 1
    if n_recent:
        deg[..., S - n_recent:] = 1
    return deg


def agreeing_logits(rng: Generator, B: int, nq: int, V: int, drafts: np.ndarray,
                    n_agree) -> np.ndarray:
    """Logits [B, nq, V] whose argmax equals drafts[b, i] for i < n_agree[b] and,
    at i == n_agree[b] < nq - 1, differs from drafts[b, i]."""
    logits = normal(rng, (B, nq, V))
    n_agree = np.broadcast_to(np.asarray(n_agree), (B,))
    for b in range(B):
        a = int(n_agree[b])
        for i in range(min(a, nq - 1)):
            logits[b, i, drafts[b, i]] = logits[b, i].max() + 1.0
        if a < nq - 1 and int(np.argmax(logits[b, a])) == int(drafts[b, a]):
            logits[b, a, drafts[b, a]] = logits[b, a].min() - 1.0
    return logits


# ---------------------------------------------------------------- workloads
def outlier_channels(cfg: AttnConfig, rng: Generator | None = None) -> np.ndarray:
    """The (kv head, channel) pairs scaled x10 in the int4 workload, as flat indices
    kvh * D + d (unsorted draw order): round(outlier_frac * Hkv * D) distinct pairs."""
    if rng is None:
        rng = children(cfg.seed, 12)[2]
    n_out = int(round(cfg.outlier_frac * cfg.Hkv * cfg.D))
    return rng.choice(cfg.Hkv * cfg.D, size=n_out, replace=False)


def attn_case(cfg: AttnConfig | int, **override) -> dict:
    """Seeded inputs for one attention-layer workload (optionally resized).

    Returns a dict of numpy arrays; bf16 tensors appear as ``*_bits`` (uint16).
    Keys: k_bits, v_bits [B,Hkv,L_cap,D] (full KV incl. the k+1 block rows at
    P..P+k); q_draft_bits [B,Hq,D]; q_verify_bits [B,k+1,Hq,D]; idx, deg
    [B,Hkv,S] (indexed caches; idx is None for compact caches, whose rows are
    ``kc_bits``/``vc_bits`` [B,Hkv,S,D]); drafts [B,k]; logits [B,k+1,V].
    """
    if isinstance(cfg, int):
        cfg = get_config(cfg)
    if override:
        cfg = dataclasses.replace(cfg, **override)
    r = children(cfg.seed, 12)
    B, Hq, Hkv, D, P, k = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.P, cfg.k
    out: dict = {"cfg": cfg}
    Kf = ar1(r[0], (B, Hkv), cfg.L_cap, D, cfg.rho)
    Vf = ar1(r[1], (B, Hkv), cfg.L_cap, D, cfg.rho)
    if cfg.outlier_frac > 0.0:
        flat = outlier_channels(cfg, r[2])
        for f in flat:
            Kf[:, f // D, :, f % D] *= 10.0
            Vf[:, f // D, :, f % D] *= 10.0
        out["outliers"] = np.sort(flat)
    out["k_f32"], out["v_f32"] = Kf, Vf
    out["k_bits"], out["v_bits"] = f32_to_bf16_bits(Kf), f32_to_bf16_bits(Vf)
    out["q_draft_bits"] = f32_to_bf16_bits(normal(r[3], (B, Hq, D)))
    out["q_verify_bits"] = f32_to_bf16_bits(normal(r[4], (B, k + 1, Hq, D)))
    if cfg.cache == "indexed" and cfg.S > 0:
        if cfg.compact:
            ck = ar1(r[5], (B, Hkv), cfg.S, D, cfg.rho)
            cv = ar1(r[6], (B, Hkv), cfg.S, D, cfg.rho)
            out["kc_bits"], out["vc_bits"] = f32_to_bf16_bits(ck), f32_to_bf16_bits(cv)
            out["idx"] = None
        else:
            out["idx"] = slot_indices(r[5], (B, Hkv), P, cfg.S, cfg.n_sinks, cfg.n_recent)
        out["deg"] = slot_degrees(r[7], (B, Hkv), cfg.S, cfg.n_sinks, cfg.n_recent,
                                  cfg.deg_max)
    V = cfg.vocab
    if V:
        drafts = r[8].integers(0, V, size=(B, k), dtype=np.int32)
        n_agree = r[9].integers(0, k + 1, size=(B,))
        if cfg.num == 1:
            n_agree = np.full((B,), 5)
        out["drafts"] = drafts
        out["n_agree"] = n_agree
        out["logits"] = agreeing_logits(r[10], B, k + 1, V, drafts, n_agree)
    return out


def bf16_block_rows(case: dict, which: str, n: int) -> np.ndarray:
    """Rows P..P+n-1 of the full K or V (bits), used as the draft tail: the
    pending token plus the drafts appended so far."""
    cfg = case["cfg"]
    src = case["k_bits"] if which == "k" else case["v_bits"]
    return np.ascontiguousarray(src[:, :, cfg.P:cfg.P + n, :])


# ---------------------------------------------------------------- tiny decoder
def tinylm_weights(cfg) -> dict:
    """Random-init weights N(0, init_std) as bf16 bits, matrices [in, out]."""
    shapes = {"embed": (cfg.vocab, cfg.d_model), "lm_head": (cfg.d_model, cfg.vocab)}
    for l in range(cfg.n_layers):
        shapes[f"{l}.wq"] = (cfg.d_model, cfg.Hq * cfg.D)
        shapes[f"{l}.wk"] = (cfg.d_model, cfg.Hkv * cfg.D)
        shapes[f"{l}.wv"] = (cfg.d_model, cfg.Hkv * cfg.D)
        shapes[f"{l}.wo"] = (cfg.Hq * cfg.D, cfg.d_model)
        shapes[f"{l}.w_gate"] = (cfg.d_model, cfg.ffn)
        shapes[f"{l}.w_up"] = (cfg.d_model, cfg.ffn)
        shapes[f"{l}.w_down"] = (cfg.ffn, cfg.d_model)
    rs = children(cfg.seed, len(shapes) + 1)
    out = {}
    for r, (name, shp) in zip(rs, shapes.items()):
        out[name] = f32_to_bf16_bits(normal(r, shp) * np.float32(cfg.init_std))
    return out


def tinylm_prompt(cfg) -> np.ndarray:
    """Prompt of uniform-random token ids."""
    r = children(cfg.seed + 500, 1)[0]
    return r.integers(0, cfg.vocab, size=cfg.prompt_len, dtype=np.int64)


def ar1_chunks(rng: Generator, lead: tuple, L: int, D: int, rho: float, chunk: int):
    """AR(1) along the sequence in pieces of ``chunk`` rows (bf16 bits [*lead, n, D]),
    the filter state carried across pieces, so long sequences never sit in fp32 whole.
    Same process as ``ar1``."""
    b0 = math.sqrt(1.0 - rho * rho)
    state = None
    for s0 in range(0, L, chunk):
        n = min(chunk, L - s0)
        e = rng.standard_normal((*lead, n, D), dtype=np.float32)
        if rho == 0.0:
            yield f32_to_bf16_bits(e)
            continue
        if state is None:
            e[..., 0, :] /= b0
            x = lfilter([b0], [1.0, -rho], e, axis=-2)
        else:
            x, _ = lfilter([b0], [1.0, -rho], e, axis=-2,
                           zi=(rho * state)[..., None, :])
        state = x[..., -1, :].astype(np.float64)
        yield f32_to_bf16_bits(x.astype(np.float32))


def staged_case(cfg=None, chunk: int | None = None, P: int | None = None):
    """1M-token staged inputs: the full cache of one request as chunk-major bf16 bits
    (generator of [2 (K|V), Hkv, chunk, D] pieces), its verify queries and block K/V,
    and the compact compressed caches of the drafting requests."""
    cfg = cfg or get_config(4)
    chunk = chunk or cfg.chunk_tokens
    P = P or cfg.P
    r = children(cfg.seed + 100, 8)
    out = {"cfg": cfg, "chunk": chunk, "P": P}
    out["chunks_k"] = ar1_chunks(r[0], (cfg.Hkv,), P, cfg.D, cfg.rho, chunk)
    out["chunks_v"] = ar1_chunks(r[1], (cfg.Hkv,), P, cfg.D, cfg.rho, chunk)
    n_q = cfg.k + 1
    out["block_k_bits"] = f32_to_bf16_bits(normal(r[2], (1, cfg.Hkv, n_q, cfg.D)))
    out["block_v_bits"] = f32_to_bf16_bits(normal(r[3], (1, cfg.Hkv, n_q, cfg.D)))
    out["q_verify_bits"] = f32_to_bf16_bits(normal(r[4], (1, n_q, cfg.Hq, cfg.D)))
    return out


def staged_draft_case(cfg=None, n_tail: int = 0) -> dict:
    """Inputs of the requests that draft while the long-context request verifies: per
    request and kv head a compact compressed cache of S rows (AR(1) along the rows, as
    the full caches), degrees U{1..deg_max} on the kept middle rows, one query per
    query head, and ``n_tail`` i.i.d. N(0, 1) tail rows (the drafts appended so far).
    Returns bits: kc_bits, vc_bits [R, Hkv, S, D], deg [R, Hkv, S], q_bits [R, Hq, D],
    tail_k_bits, tail_v_bits [R, Hkv, max(n_tail, 1), D]."""
    cfg = cfg or get_config(4)
    R, S = cfg.n_draft_requests, cfg.S
    r = children(cfg.seed + 200, 6)
    out = {"cfg": cfg, "n_tail": n_tail}
    out["kc_bits"] = f32_to_bf16_bits(ar1(r[0], (R, cfg.Hkv), S, cfg.D, cfg.rho))
    out["vc_bits"] = f32_to_bf16_bits(ar1(r[1], (R, cfg.Hkv), S, cfg.D, cfg.rho))
    out["deg"] = slot_degrees(r[2], (R, cfg.Hkv), S, cfg.n_sinks, cfg.n_recent, cfg.deg_max)
    out["q_bits"] = f32_to_bf16_bits(normal(r[3], (R, cfg.Hq, cfg.D)))
    nt = max(n_tail, 1)
    out["tail_k_bits"] = f32_to_bf16_bits(normal(r[4], (R, cfg.Hkv, nt, cfg.D)))
    out["tail_v_bits"] = f32_to_bf16_bits(normal(r[5], (R, cfg.Hkv, nt, cfg.D)))
    return out
