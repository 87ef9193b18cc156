"""Python names for the C ABI, taking torch CUDA tensors.

Argument marshalling only: every step runs in libvericache.so.  torch provides
device memory, streams and events.  Shapes and layouts are those of
include/vericache.h.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import CompCache, check, lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, dtype, name: str, cuda: bool = True):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")


@dataclass
class IndexedCache:
    """Token-evicted compressed cache: bf16 base rows picked by ``idx`` with degrees.

    k, v: [B, Hkv, T_cap, D] bf16; idx, deg: [B, Hkv, S_cap] int32 or None;
    k_tail, v_tail: [B, Hkv, R_cap, D] bf16 or None with n_tail live rows."""

    k: torch.Tensor
    v: torch.Tensor
    S: int
    Hq: int
    idx: Optional[torch.Tensor] = None
    deg: Optional[torch.Tensor] = None
    k_tail: Optional[torch.Tensor] = None
    v_tail: Optional[torch.Tensor] = None
    n_tail: int = 0
    err_flag: Optional[torch.Tensor] = None

    def struct(self) -> CompCache:
        B, Hkv, T_cap, D = self.k.shape
        _need(self.k, torch.bfloat16, "k")
        _need(self.v, torch.bfloat16, "v")
        c = CompCache()
        c.kind = _lib.VC_CACHE_INDEXED
        c.B, c.Hq, c.Hkv, c.D = B, self.Hq, Hkv, D
        c.S, c.T_cap = self.S, T_cap
        c.S_cap = 0
        for t, n in ((self.idx, "idx"), (self.deg, "deg")):
            if t is not None:
                _need(t, torch.int32, n)
                c.S_cap = t.shape[-1]
        c.k, c.v = _ptr(self.k), _ptr(self.v)
        c.idx, c.deg = _ptr(self.idx), _ptr(self.deg)
        _fill_tail(c, self)
        return c


@dataclass
class Int4Cache:
    """4-bit group-quantised cache (layout in include/vericache.h).

    kq: uint32 words as int32 [B, Hkv, T_cap/32, 32, 4, D/32]; k_scale/k_zero fp16
    [B, Hkv, T_cap/32, D]; vq: int32 [B, Hkv, T_cap/32, D, 4]; v_scale/v_zero fp16
    [B, Hkv, T_cap/32, D/32, 32]; S quantised tokens live."""

    kq: torch.Tensor
    k_scale: torch.Tensor
    k_zero: torch.Tensor
    vq: torch.Tensor
    v_scale: torch.Tensor
    v_zero: torch.Tensor
    S: int
    Hq: int
    k_tail: Optional[torch.Tensor] = None
    v_tail: Optional[torch.Tensor] = None
    n_tail: int = 0
    err_flag: Optional[torch.Tensor] = None

    def struct(self) -> CompCache:
        B, Hkv, nb, D = self.k_scale.shape
        _need(self.kq, torch.int32, "kq")
        _need(self.vq, torch.int32, "vq")
        for t, n in ((self.k_scale, "k_scale"), (self.k_zero, "k_zero"),
                     (self.v_scale, "v_scale"), (self.v_zero, "v_zero")):
            _need(t, torch.float16, n)
        c = CompCache()
        c.kind = _lib.VC_CACHE_INT4
        c.B, c.Hq, c.Hkv, c.D = B, self.Hq, Hkv, D
        c.S, c.T_cap, c.S_cap = self.S, nb * 32, 0
        c.kq, c.vq = _ptr(self.kq), _ptr(self.vq)
        c.k_scale, c.k_zero = _ptr(self.k_scale), _ptr(self.k_zero)
        c.v_scale, c.v_zero = _ptr(self.v_scale), _ptr(self.v_zero)
        _fill_tail(c, self)
        return c


def _fill_tail(c: CompCache, cache) -> None:
    if cache.k_tail is not None:
        _need(cache.k_tail, torch.bfloat16, "k_tail")
        _need(cache.v_tail, torch.bfloat16, "v_tail")
        c.k_tail, c.v_tail = _ptr(cache.k_tail), _ptr(cache.v_tail)
        c.R_cap = cache.k_tail.shape[2]
    c.n_tail = cache.n_tail
    if cache.err_flag is not None:
        _need(cache.err_flag, torch.int32, "err_flag")
        c.err_flag = _ptr(cache.err_flag)


# ------------------------------------------------------------------ draft
def draft_workspace_size(cache) -> int:
    s = cache.struct()
    n = lib().vc_draft_workspace_size(ctypes.byref(s))
    if n == 0:
        check(_lib.VC_ERR_INVALID, "vc_draft_workspace_size")
    return int(n)


def _out_flag(out: torch.Tensor) -> int:
    if out.dtype == torch.float32:
        return _lib.VC_OUT_F32
    if out.dtype != torch.bfloat16:
        raise TypeError("out must be bfloat16 or float32")
    return 0


def draft_attn(q: torch.Tensor, cache, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
               scale: float = 0.0, stream=None) -> torch.Tensor:
    """o[b, h] = softmax_t(q.k_t * scale + ln n_t) . v over KV_comp plus the tail.
    ``out`` may be bfloat16 (default) or float32."""
    _need(q, torch.bfloat16, "q")
    s = cache.struct()
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = torch.empty(draft_workspace_size(cache), dtype=torch.uint8, device=q.device)
    check(lib().vc_draft_attn(q.data_ptr(), ctypes.byref(s), float(scale), _out_flag(out),
                              out.data_ptr(), _ptr(lse), ws.data_ptr(), ws.numel(),
                              _stream(stream)), "vc_draft_attn")
    return out


def draft_attn_noalloc(q: torch.Tensor, cache, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, scale: float = 0.0,
                       stream=None) -> torch.Tensor:
    """draft_attn for callers that cannot provide a workspace: the library keeps the
    split-K partials in a fixed 8 MiB per-device array (see vc_draft_attn_noalloc).
    Calls that overlap on the GPU share that array and must be serialised."""
    _need(q, torch.bfloat16, "q")
    s = cache.struct()
    if out is None:
        out = torch.empty_like(q)
    check(lib().vc_draft_attn_noalloc(q.data_ptr(), ctypes.byref(s), float(scale),
                                      _out_flag(out), out.data_ptr(), _ptr(lse),
                                      _stream(stream)), "vc_draft_attn_noalloc")
    return out


# ------------------------------------------------------------------ verify
def verify_workspace_size(B, n_q, Hq, Hkv, D, kv_start, kv_len) -> int:
    return int(lib().vc_verify_workspace_size(B, n_q, Hq, Hkv, D, kv_start, kv_len))


def verify_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, P: int, kv_start: int = 0,
                kv_len: Optional[int] = None, state=None, flags: int = 0,
                out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                scale: float = 0.0, stream=None) -> torch.Tensor:
    """Verify attention of q [B, n_q, Hq, D] over keys [kv_start, kv_start+kv_len) held
    in k, v [B, Hkv, L_cap, D]; ``state`` = (m, l, acc) for the chunked form.
    ``out`` may be bfloat16 (default) or float32."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    _need(v, torch.bfloat16, "v")
    B, n_q, Hq, D = q.shape
    Hkv, L_cap = k.shape[1], k.shape[2]
    if kv_len is None:
        kv_len = P + n_q - kv_start
    m = l = acc = None
    if state is not None:
        m, l, acc = state
        for t, n in ((m, "m"), (l, "l"), (acc, "acc")):
            _need(t, torch.float32, n)
    if out is None and (state is None or flags & _lib.VC_VERIFY_LAST):
        out = torch.empty_like(q)
    if ws is None:
        ws = torch.empty(max(1, verify_workspace_size(B, n_q, Hq, Hkv, D, kv_start, kv_len)),
                         dtype=torch.uint8, device=q.device)
    if out is not None:
        flags |= _out_flag(out)
    check(lib().vc_verify_attn(q.data_ptr(), B, n_q, Hq, Hkv, D, k.data_ptr(), v.data_ptr(),
                               L_cap, kv_start, kv_len, P, _ptr(m), _ptr(l), _ptr(acc),
                               int(flags), float(scale), _ptr(out), ws.data_ptr(), ws.numel(),
                               _stream(stream)), "vc_verify_attn")
    return out


# ------------------------------------------------------------------ accept
def accept(logits: torch.Tensor, drafts: Optional[torch.Tensor] = None, target=None,
           accept_len=None, commit=None, n_commit=None, err_flag=None, stream=None) -> dict:
    """Greedy acceptance over logits [B, n_q, V] fp32 with drafts [B, n_q-1] int32."""
    _need(logits, torch.float32, "logits")
    B, n_q, V = logits.shape
    dev = logits.device
    i32 = dict(dtype=torch.int32, device=dev)
    if target is None:
        target = torch.empty((B, n_q), **i32)
    if err_flag is None:
        err_flag = torch.empty((B,), **i32)
    want_accept = drafts is not None
    if drafts is not None:
        _need(drafts, torch.int32, "drafts")
        if drafts.numel() == 0:
            drafts = None   # n_q == 1: nothing to compare
    if want_accept:
        accept_len = torch.empty((B,), **i32) if accept_len is None else accept_len
        commit = torch.empty((B, n_q), **i32) if commit is None else commit
        n_commit = torch.empty((B,), **i32) if n_commit is None else n_commit
    check(lib().vc_accept(logits.data_ptr(), _ptr(drafts), B, n_q, V, target.data_ptr(),
                          _ptr(accept_len), _ptr(commit), _ptr(n_commit), _ptr(err_flag),
                          _stream(stream)), "vc_accept")
    return {"target": target, "accept_len": accept_len, "commit": commit,
            "n_commit": n_commit, "err": err_flag}


# ------------------------------------------------------------------ staging
def make_events(n: int, stream=None) -> list:
    """n CUDA events (materialised by one record so their handles exist)."""
    s = stream if stream is not None else torch.cuda.current_stream()
    evs = [torch.cuda.Event() for _ in range(n)]
    for e in evs:
        e.record(s)
    return evs


def stage_full_kv(dst: torch.Tensor, src_pinned: torch.Tensor, chunk_bytes: int,
                  copy_stream, events=None, nbytes: Optional[int] = None) -> None:
    """Copy pinned host ``src_pinned`` into device ``dst`` chunk by chunk on
    ``copy_stream``, recording events[i] after chunk i."""
    if not src_pinned.is_pinned():
        raise ValueError("src_pinned must be page-locked")
    n = nbytes if nbytes is not None else src_pinned.numel() * src_pinned.element_size()
    arr = None
    if events:
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    check(lib().vc_stage_full_kv(dst.data_ptr(), src_pinned.data_ptr(), n, chunk_bytes,
                                 _stream(copy_stream), arr, len(events) if events else 0),
          "vc_stage_full_kv")


def event_wait(event, timeout_s: float) -> None:
    check(lib().vc_event_wait(event.cuda_event, float(timeout_s)), "vc_event_wait")


def device_error(clear: bool = True) -> int:
    """The library's device error word (bit 0: a bounded wait in verify expired)."""
    v = ctypes.c_int32(0)
    check(lib().vc_device_error(ctypes.byref(v), int(clear)), "vc_device_error")
    return int(v.value)


def int4_quantize(k: torch.Tensor, v: torch.Tensor, cache: "Int4Cache", n_blocks: int,
                  src_t0: int = 0, blk0: int = 0, stream=None) -> None:
    """Quantise rows [src_t0, src_t0 + 32 n_blocks) of k, v [B, Hkv, src_cap, D] (bf16)
    into blocks [blk0, blk0 + n_blocks) of every pair of ``cache``'s int4 arrays."""
    _need(k, torch.bfloat16, "k")
    _need(v, torch.bfloat16, "v")
    B, Hkv, src_cap, D = k.shape
    blk_cap = cache.k_scale.shape[2]
    check(lib().vc_int4_quantize(k.data_ptr(), v.data_ptr(), B * Hkv, D, src_cap, src_t0,
                                 n_blocks, cache.kq.data_ptr(), cache.k_scale.data_ptr(),
                                 cache.k_zero.data_ptr(), cache.vq.data_ptr(),
                                 cache.v_scale.data_ptr(), cache.v_zero.data_ptr(), blk_cap,
                                 blk0, _stream(stream)), "vc_int4_quantize")


def empty_int4_cache(B: int, Hq: int, Hkv: int, D: int, T_cap: int, device="cuda") -> "Int4Cache":
    """Uninitialised int4 arrays for T_cap tokens per pair (S = 0 live tokens)."""
    nb = T_cap // 32
    i32, f16 = dict(dtype=torch.int32, device=device), dict(dtype=torch.float16, device=device)
    return Int4Cache(kq=torch.empty((B, Hkv, nb, 32, 4, D // 32), **i32),
                     k_scale=torch.empty((B, Hkv, nb, D), **f16),
                     k_zero=torch.empty((B, Hkv, nb, D), **f16),
                     vq=torch.empty((B, Hkv, nb, D, 4), **i32),
                     v_scale=torch.empty((B, Hkv, nb, D // 32, 32), **f16),
                     v_zero=torch.empty((B, Hkv, nb, D // 32, 32), **f16), S=0, Hq=Hq)


def evict_scores(q: torch.Tensor, k: torch.Tensor, n: int, score: Optional[torch.Tensor] = None,
                 ws: Optional[torch.Tensor] = None, scale: float = 0.0, stream=None) -> torch.Tensor:
    """Attention mass per key from the last W prompt queries q [B, W, Hq, D] over keys
    [0, n) of k [B, Hkv, L_cap, D]; returns score fp32 [B, Hkv, >= n]."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    B, W, Hq, D = q.shape
    Hkv, L_cap = k.shape[1], k.shape[2]
    if score is None:
        score = torch.empty((B, Hkv, n), dtype=torch.float32, device=q.device)
    _need(score, torch.float32, "score")
    if ws is None:
        ws = torch.empty(int(lib().vc_evict_workspace_size(B, W, Hq)), dtype=torch.uint8,
                         device=q.device)
    check(lib().vc_evict_scores(q.data_ptr(), B, W, Hq, Hkv, D, k.data_ptr(), L_cap, n,
                                float(scale), score.data_ptr(), score.shape[-1], ws.data_ptr(),
                                ws.numel(), _stream(stream)), "vc_evict_scores")
    return score


def evict_select(score: torch.Tensor, n: int, budget: int, n_sinks: int, n_recent: int,
                 idx: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Kept positions (ascending) per row of score [..., score_cap]: sinks, the top
    middle scores (ties to the lower position) up to the budget, the recent window."""
    _need(score, torch.float32, "score")
    rows = score.numel() // score.shape[-1]
    if idx is None:
        idx = torch.empty(score.shape[:-1] + (min(budget, n),), dtype=torch.int32,
                          device=score.device)
    _need(idx, torch.int32, "idx")
    check(lib().vc_evict_select(score.data_ptr(), rows, score.shape[-1], n, budget, n_sinks,
                                n_recent, idx.data_ptr(), idx.shape[-1], _stream(stream)),
          "vc_evict_select")
    return idx


def set_wait_limit(seconds: float) -> float:
    """Time limit of the verify kernel's pipeline waits for the launches that follow
    (0 restores the 2 s default); returns the previous limit in seconds."""
    prev = ctypes.c_double(0.0)
    check(lib().vc_set_wait_limit(float(seconds), ctypes.byref(prev)), "vc_set_wait_limit")
    return float(prev.value)


def csm_out_len(T: int, n_sinks: int, n_recent: int, chunk: int, r: float) -> int:
    """Rows left by one Chunked Soft Matching round over T rows (-1 if invalid)."""
    return int(lib().vc_csm_out_len(T, n_sinks, n_recent, chunk, r))


def csm_compress(k: torch.Tensor, v: torch.Tensor, n_sinks: int, n_recent: int, chunk: int,
                 r: float, deg: Optional[torch.Tensor] = None, T: Optional[int] = None,
                 k_out=None, v_out=None, deg_out=None, dest=None, stream=None):
    """One Chunked Soft Matching round (CentroidKV) over rows [0, T) of every pair.

    k, v: [B, Hkv, T_cap, D] bf16; deg: [B, Hkv, T_cap] int32 or None (all 1).
    Returns (k_out, v_out, deg_out, n_out): a compact cache of n_out rows per pair."""
    _need(k, torch.bfloat16, "k")
    _need(v, torch.bfloat16, "v")
    B, Hkv, T_cap, D = k.shape
    T = T_cap if T is None else T
    n_out = csm_out_len(T, n_sinks, n_recent, chunk, r)
    if n_out < 0:
        raise ValueError("csm_compress: invalid sizes or ratio")
    if k_out is None:
        k_out = torch.empty((B, Hkv, max(n_out, 1), D), dtype=k.dtype, device=k.device)
    if v_out is None:
        v_out = torch.empty_like(k_out)
    if deg_out is None:
        deg_out = torch.empty(k_out.shape[:3], dtype=torch.int32, device=k.device)
    if deg is not None:
        _need(deg, torch.int32, "deg")
    if dest is not None:
        _need(dest, torch.int32, "dest")
    check(lib().vc_csm_compress(k.data_ptr(), v.data_ptr(), _ptr(deg), B * Hkv, D, T, T_cap,
                                n_sinks, n_recent, chunk, float(r), k_out.data_ptr(),
                                v_out.data_ptr(), deg_out.data_ptr(), k_out.shape[2], _ptr(dest),
                                _stream(stream)), "vc_csm_compress")
    return k_out, v_out, deg_out, n_out

