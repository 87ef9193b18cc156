"""Remote prefix caching: the drafts run on one GPU over the compressed cache, the verify
pass on another over the full cache.

VeriCache summary ("Riepilogo Tecnico: VeriCache"), section "Supporto Architetturale",
second scenario: the compressed KV is streamed over a slow link to a remote GPU that
drafts, while the full KV is loaded over a fast local link into the GPU that verifies,
so the slow transfer is taken off the remote GPU's compute; section "Risultati
Sperimentali" reports up to 2x throughput for this scenario.

Two sides, one protocol:

* ``VerifierSide`` (the local GPU) holds the model and the full cache.  It prefills the
  prompt and clusters the prompt's cache with Chunked Soft Matching down to the budget
  (the same schedule as ``loop.vericache_loop_csm``).  It hands the compact cache (rows
  and degrees) over once.  Each round it runs the k + 1-row verify pass over the full
  cache and the acceptance, and returns the commits with the verify-pass K/V of the
  accepted positions.
* ``DrafterSide`` (the remote GPU) holds the model and the compact cache only.  Each
  round it drafts k tokens over the compact cache, then appends the returned rows with
  degree 1.  It re-clusters on the one-GPU loop's schedule.

The link carries the compact cache once, then per round the k + 1 token ids one way and
the other way k + 3 int32 plus (a + 1) positions x layers x 2 x Hkv x D bf16 values.

Transports: ``run_local`` drives both sides in one process.  The sides may share a device
or sit on two, and the tensors move by device copies.  ``run_verifier`` / ``run_drafter``
run one side per rank of a ``torch.distributed`` group with point-to-point send/recv:
NCCL between GPUs, or gloo on host tensors.  Both ranks exchange the same messages in the
same order.  They stop after the same round, because both count the same committed tokens.

Readings where the pages are silent: the verifier builds the compact cache from the
prompt it prefilled (the pages fetch it from prefix storage), and the drafter's cache is
extended with the verify-pass K/V of the accepted positions, as in the one-GPU loop.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .api import accept
from .loop import GpuTinyLM, csm_fit, csm_step

_I32 = torch.int32


class VerifierSide:
    """The full cache and the verify pass.  ``sched`` = (budget, n_sinks, n_recent,
    chunk, r_init, delta_r, r_floor) of the clustering after the prefill."""

    def __init__(self, model: GpuTinyLM, k: int, sched: tuple):
        self.m, self.k, self.sched = model, k, tuple(sched)
        self.dev = model.dev
        c = model.cfg
        self.L, self.Hkv, self.D = c.n_layers, c.Hkv, c.D
        self.P = 0

    def start(self, prompt):
        """Prefill and clustering; returns (first token, compact cache (K, V, degrees),
        clustering rounds run, cache sizes after each round)."""
        m = self.m
        logits = m.prefill(prompt)
        m.csm_init(len(prompt))
        budget, *rest = self.sched
        sizes = csm_fit(m, budget, *rest)
        first = torch.empty((1, 1), dtype=_I32, device=self.dev)
        accept(logits.view(1, 1, -1), target=first)
        self.P = len(prompt)
        return int(first.item()), m.csm_export(), m.csm["round"], sizes

    def verify(self, vids: torch.Tensor):
        """vids int32 [k + 1] (pending token, drafts) on this side's device -> (res int32
        [k + 3] = accept length a, n_commit, commit tokens padded; rows bf16 [layers, 2,
        Hkv, a + 1, D] of positions P .. P + a)."""
        m, k = self.m, self.k
        lg = m.forward_full(vids, k + 1, self.P)
        r = accept(lg.view(1, k + 1, -1), vids[1:].view(1, k))
        res = torch.cat([r["accept_len"].view(1), r["n_commit"].view(1), r["commit"].view(-1)])
        a = int(res[0].item())
        rows = m.full_rows(self.P, a + 1)
        self.P += a + 1
        return res, rows


class DrafterSide:
    """The compact cache and the drafts.  ``sched`` as for VerifierSide; the cache is
    re-clustered after every ``recluster_every`` committed tokens while it is over the
    budget."""

    def __init__(self, model: GpuTinyLM, k: int, sched: tuple, recluster_every: int):
        self.m, self.k, self.sched = model, k, tuple(sched)
        self.every = recluster_every
        self.dev = model.dev
        c = model.cfg
        self.L, self.Hkv, self.D = c.n_layers, c.Hkv, c.D
        self.vids = torch.empty(k + 1, dtype=_I32, device=self.dev)
        self.P = self.pending = self.since = 0
        self.sizes = []

    def load(self, first: int, P: int, cache, rounds: int):
        self.m.csm_load(*cache, rounds)
        self.pending, self.P, self.since = first, P, 0

    def draft(self) -> torch.Tensor:
        self.vids[0] = self.pending
        self.m.draft_steps(self.vids, self.k, self.P)
        return self.vids

    def finish(self, res: list, rows: torch.Tensor) -> list:
        """res as the host list of VerifierSide.verify's res; rows on this side's device.
        Returns the committed tokens."""
        a, n_commit = res[0], res[1]
        commit = res[2:2 + n_commit]
        self.m.csm_append_rows(rows[:, 0], rows[:, 1], a + 1)
        self.P += a + 1
        self.pending = commit[-1]
        self.since += a + 1
        if self.since >= self.every:
            self.since = 0
            budget, *rest = self.sched
            if self.m.S > budget:
                self.sizes.append(csm_step(self.m, *rest))
        return commit


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def run_local(drafter, verifier, prompt, n_gen: int):
    """Both sides in this process.  Returns (tokens, accept lengths, link bytes: setup,
    drafter -> verifier, verifier -> drafter)."""
    first, cache, rounds, _ = verifier.start(prompt)
    drafter.load(first, len(prompt), tuple(t.to(drafter.dev) for t in cache), rounds)
    link = {"setup": sum(_nbytes(t) for t in cache) + 32, "to_verifier": 0, "to_drafter": 0}
    out, alens = [first], []
    while len(out) < n_gen:
        vids = drafter.draft()
        res, rows = verifier.verify(vids.to(verifier.dev))
        link["to_verifier"] += _nbytes(vids)
        link["to_drafter"] += _nbytes(res) + _nbytes(rows)
        res_h = res.cpu().tolist()
        out.extend(drafter.finish(res_h, rows.to(drafter.dev)))
        alens.append(res_h[0])
    return out[:n_gen], alens, link


# ---------------------------------------------------------------- one side per rank
def _wire_dev(side):
    """NCCL moves the side's own device tensors (the rank must have made that device
    current); gloo moves host copies."""
    if dist.get_backend() == "nccl":
        idx = side.dev.index if side.dev.index is not None else torch.cuda.current_device()
        if side.dev.type != "cuda" or torch.cuda.current_device() != idx:
            raise RuntimeError(f"NCCL rank: make {side.dev} the current device first "
                               "(torch.cuda.set_device)")
        return side.dev
    return torch.device("cpu")


def _send(t: torch.Tensor, peer: int, wire) -> None:
    t = t.contiguous().to(wire)
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    dist.send(t, peer)


def _recv(shape, dtype, peer: int, wire, dev) -> torch.Tensor:
    wdt = torch.int16 if dtype == torch.bfloat16 else dtype
    t = torch.empty(shape, dtype=wdt, device=wire)
    dist.recv(t, peer)
    if dtype == torch.bfloat16:
        t = t.view(torch.bfloat16)
    return t.to(dev)


def run_verifier(verifier, prompt, n_gen: int, peer: int):
    """The verifier rank: sends the compact cache, then serves one verify per round.
    Returns the accept lengths."""
    wire = _wire_dev(verifier)
    first, cache, rounds, _ = verifier.start(prompt)
    K, V, deg = cache
    _send(torch.tensor([K.shape[2], len(prompt), first, rounds], dtype=torch.int64), peer, wire)
    for t in (K, V, deg):
        _send(t, peer, wire)
    k = verifier.k
    n_out, alens = 1, []
    while n_out < n_gen:
        vids = _recv((k + 1,), _I32, peer, wire, verifier.dev)
        res, rows = verifier.verify(vids)
        _send(res, peer, wire)
        _send(rows, peer, wire)
        res_h = res.cpu().tolist()
        alens.append(res_h[0])
        n_out += res_h[1]
    return alens


def run_drafter(drafter, n_gen: int, peer: int):
    """The drafter rank: receives the compact cache, then drafts every round and takes
    the commits and rows back.  Returns the committed tokens."""
    wire, dev = _wire_dev(drafter), drafter.dev
    L, Hkv, D, k = drafter.L, drafter.Hkv, drafter.D, drafter.k
    S, P, first, rounds = _recv((4,), torch.int64, peer, wire, "cpu").tolist()
    K = _recv((L, Hkv, S, D), torch.bfloat16, peer, wire, dev)
    V = _recv((L, Hkv, S, D), torch.bfloat16, peer, wire, dev)
    deg = _recv((L, Hkv, S), _I32, peer, wire, dev)
    drafter.load(first, P, (K, V, deg), rounds)
    out = [first]
    while len(out) < n_gen:
        _send(drafter.draft(), peer, wire)
        res_h = _recv((k + 3,), _I32, peer, wire, "cpu").tolist()
        rows = _recv((L, 2, Hkv, res_h[0] + 1, D), torch.bfloat16, peer, wire, dev)
        out.extend(drafter.finish(res_h, rows))
    return out[:n_gen]
