"""Staggered long-context verification (host-side scheduling over the C ABI).

VeriCache summary ("Riepilogo Tecnico: VeriCache"): in long-context decoding the full
cache lives in CPU memory and verification loads it over PCIe (section "Supporto
Architetturale"); the runtime staggers requests so that while some verify (loading
the full cache, interconnect-bound) others draft (HBM-bound), keeping both busy
(section "Scaglionamento tra Risorse (P1)").

One request's verify streams its full cache, chunk-major in pinned host memory, through
a ring of device slots:

    copy stream    stage chunk c into slot c % n_slots     (after verify of chunk c - n_slots)
    verify stream  wait chunk c; vc_verify_attn over its keys, carrying (m, l, acc)
    draft stream   other requests' vc_draft_attn calls, back to back, untouched by both

Only events order the streams; nothing here waits on the host except the caller.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch

from . import _lib
from .api import make_events, stage_full_kv, verify_attn


class StagedVerify:
    """Chunked verify of one request whose full KV sits in pinned host memory.

    host_kv: pinned bf16 [n_chunks, 2 (K|V), Hkv, chunk, D], chunk-major: chunk c holds
    positions c*chunk .. (c+1)*chunk-1 of the prefix (the last chunk may be partial,
    P % chunk live rows).  block_k / block_v: device bf16 [1, Hkv, n_q, D], the block's
    own keys at positions P .. P+n_q-1.
    """

    def __init__(self, host_kv: torch.Tensor, P: int, block_k: torch.Tensor,
                 block_v: torch.Tensor, n_slots: int = 3, device=None):
        if not host_kv.is_pinned():
            raise ValueError("host_kv must be page-locked")
        self.host = host_kv
        self.P = P
        self.n_chunks, _, self.Hkv, self.chunk, self.D = host_kv.shape
        self.block_k, self.block_v = block_k, block_v
        self.device = device or block_k.device
        self.n_slots = n_slots
        self.ring = torch.empty((n_slots,) + tuple(host_kv.shape[1:]), dtype=host_kv.dtype,
                                device=self.device)
        self.s_copy = torch.cuda.Stream(self.device)
        self.s_verify = torch.cuda.Stream(self.device)
        self.copied = make_events(self.n_chunks, self.s_copy)
        self.verified = make_events(self.n_chunks, self.s_verify)
        self.t_start = torch.cuda.Event(enable_timing=True)
        self.t_staged = torch.cuda.Event(enable_timing=True)
        self.t_done = torch.cuda.Event(enable_timing=True)
        self.chunk_bytes = self.ring[0].numel() * self.ring.element_size()
        self._launched = False

    def _rows(self, c: int) -> int:
        return min(self.chunk, self.P - c * self.chunk)

    def launch(self, q: torch.Tensor, out: torch.Tensor, state=None, ws=None):
        """Enqueue the whole staged verify of q [1, n_q, Hq, D] and return at once;
        ``self.t_done`` completes when ``out`` is written (``wait()`` orders a stream
        after it).

        Ordering: both side streams first wait for the caller's current stream, so q,
        the block's keys and anything else written there before this call are visible;
        the first chunks of this launch reuse ring slots and events of the previous
        launch, so its copies also wait for that launch's last verify (``t_done``)."""
        B, n_q, Hq, D = q.shape
        current = torch.cuda.current_stream(self.device)
        self.s_copy.wait_stream(current)
        self.s_verify.wait_stream(current)
        if self._launched:
            # ring slots 0..n_slots-1 and the per-chunk events are about to be reused
            self.s_copy.wait_event(self.t_done)
            self.s_verify.wait_event(self.t_done)
        self._launched = True
        if state is None:
            state = (torch.empty((B, n_q, Hq), dtype=torch.float32, device=self.device),
                     torch.empty((B, n_q, Hq), dtype=torch.float32, device=self.device),
                     torch.empty((B, n_q, Hq, D), dtype=torch.float32, device=self.device))
        if ws is None:
            from .api import verify_workspace_size
            need = max(verify_workspace_size(B, n_q, Hq, self.Hkv, D, c * self.chunk,
                                             self._rows(c)) for c in range(self.n_chunks))
            need = max(need, verify_workspace_size(B, n_q, Hq, self.Hkv, D, self.P, n_q))
            ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        # the side streams use these after this call returns: keep them alive and tell
        # the caching allocator which streams use them
        self._live = (state, ws, q, out)
        for t in (*state, ws, q, out):
            t.record_stream(self.s_verify)
        self.ring.record_stream(self.s_copy)
        self.ring.record_stream(self.s_verify)
        self.t_start.record(self.s_copy)
        for c in range(self.n_chunks):
            slot = c % self.n_slots
            if c >= self.n_slots:
                self.s_copy.wait_event(self.verified[c - self.n_slots])
            # a partial last chunk is copied whole: rows past its live ones lie outside
            # the key range the verify call is given, which reads them as zero
            stage_full_kv(self.ring[slot], self.host[c], self.chunk_bytes, self.s_copy,
                          [self.copied[c]])
            self.s_verify.wait_event(self.copied[c])
            kc = self.ring[slot, 0].unsqueeze(0)
            vcv = self.ring[slot, 1].unsqueeze(0)
            verify_attn(q, kc, vcv, self.P, kv_start=c * self.chunk, kv_len=self._rows(c),
                        state=state, flags=_lib.VC_VERIFY_FIRST if c == 0 else 0, ws=ws,
                        stream=self.s_verify)
            self.verified[c].record(self.s_verify)
        self.t_staged.record(self.s_copy)
        verify_attn(q, self.block_k, self.block_v, self.P, kv_start=self.P, kv_len=n_q,
                    state=state, flags=_lib.VC_VERIFY_LAST, out=out, ws=ws,
                    stream=self.s_verify)
        self.t_done.record(self.s_verify)
        return out

    def wait(self, stream=None) -> None:
        """Make ``stream`` (default: the current one) wait until the last launch's
        output is written, without blocking the host."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        s.wait_event(self.t_done)


def run_alongside(staged: StagedVerify, q, out, draft_step: Callable[[torch.cuda.Stream], None],
                  draft_stream: Optional[torch.cuda.Stream] = None, max_drafts: int = 100000):
    """Launch the staged verify, then keep issuing ``draft_step`` on the draft stream
    until the verify has finished; returns the number of draft steps issued."""
    s_draft = draft_stream or torch.cuda.Stream(staged.device)
    staged.launch(q, out)
    n = 0
    while not staged.t_done.query() and n < max_drafts:
        with torch.cuda.stream(s_draft):
            draft_step(s_draft)
        n += 1
        if n % 8 == 0:
            # keep the host at most a few launches ahead of the draft stream
            s_draft.synchronize()
    return n
