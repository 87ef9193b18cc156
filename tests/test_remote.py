"""Remote prefix caching's protocol on CPU (VeriCache summary, "Riepilogo Tecnico:
VeriCache", section "Supporto Architetturale", second scenario): the drafting side and
the verifying side exchange the compact cache once, then token ids one way and commits
plus the accepted positions' K/V rows the other way, every round.

The sides here are stand-ins with toy arithmetic (a fixed next-token rule, drafts that
go wrong at known positions, rows that encode their position), so the tests check the
transports -- one process, and two gloo ranks -- and the round bookkeeping, not the
method's arithmetic (the GPU test in test_gpu_remote.py runs the real sides).
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
VOCAB = 97
L, HKV, D, K = 2, 2, 8, 4


def truth(t: int, pos: int) -> int:
    """The toy verifier's next token after token t at position pos."""
    return (7 * t + 3 * pos + 1) % VOCAB


def row_value(pos: int, layer: int, kv: int) -> float:
    return float((7 * pos + 3 * layer + kv) % 251)      # integers below 256: exact in bf16


class ToyVerifier:
    def __init__(self, S=5):
        self.k, self.dev, self.L, self.Hkv, self.D = K, torch.device("cpu"), L, HKV, D
        self.S = S
        self.P = 0

    def start(self, prompt):
        n = len(prompt)
        self.P = n
        Kc = torch.arange(L * HKV * self.S * D, dtype=torch.float32).view(L, HKV, self.S, D)
        cache = ((Kc % 251).bfloat16(), ((Kc + 1) % 251).bfloat16(),
                 torch.arange(L * HKV * self.S, dtype=torch.int32).view(L, HKV, self.S))
        return truth(int(prompt[-1]), n - 1), cache, 3, [self.S]

    def verify(self, vids):
        v = vids.tolist()
        y = [truth(v[i], self.P + i) for i in range(self.k + 1)]
        a = next((i for i in range(self.k) if y[i] != v[i + 1]), self.k)
        commit = v[1:a + 1] + [y[a]]
        res = torch.tensor([a, a + 1] + commit + [0] * (self.k - a), dtype=torch.int32)
        rows = torch.empty(L, 2, HKV, a + 1, D, dtype=torch.bfloat16)
        for l in range(L):
            for kv in range(2):
                for j in range(a + 1):
                    rows[l, kv, :, j] = row_value(self.P + j, l, kv)
        self.P += a + 1
        return res, rows


class ToyDrafter:
    def __init__(self):
        self.k, self.dev, self.L, self.Hkv, self.D = K, torch.device("cpu"), L, HKV, D
        self.vids = torch.empty(K + 1, dtype=torch.int32)
        self.appended = 0

    def load(self, first, P, cache, rounds):
        Kc, Vc, deg = cache
        S = Kc.shape[2]
        ref = torch.arange(L * HKV * S * D, dtype=torch.float32).view(L, HKV, S, D)
        assert torch.equal(Kc.float(), ref % 251) and torch.equal(Vc.float(), (ref + 1) % 251)
        assert torch.equal(deg, torch.arange(L * HKV * S, dtype=torch.int32).view(L, HKV, S))
        assert rounds == 3
        self.pending, self.P = first, P

    def draft(self):
        t = self.pending
        self.vids[0] = t
        for j in range(self.k):
            pos = self.P + j
            nxt = truth(t, pos)
            t = (nxt + 1) % VOCAB if pos % 5 == 3 else nxt        # wrong at known places
            self.vids[j + 1] = t
        return self.vids

    def finish(self, res, rows):
        a, n = res[0], res[1]
        assert rows.shape == (L, 2, HKV, a + 1, D)
        for l in range(L):
            for kv in range(2):
                for j in range(a + 1):
                    assert torch.all(rows[l, kv, :, j].float() == row_value(self.P + j, l, kv))
        self.appended += a + 1
        self.P += a + 1
        commit = res[2:2 + n]
        self.pending = commit[-1]
        return commit


PROMPT = [5, 11, 3, 40, 2, 9]
N_GEN = 41


def greedy_stream():
    out = [truth(PROMPT[-1], len(PROMPT) - 1)]
    pos = len(PROMPT)
    while len(out) < N_GEN:
        out.append(truth(out[-1], pos))
        pos += 1
    return out


def test_local_transport_commits_the_verifier_stream():
    from lossless_kv_compressed_b200.remote import run_local
    d, v = ToyDrafter(), ToyVerifier()
    toks, alens, link = run_local(d, v, PROMPT, N_GEN)
    assert toks == greedy_stream()
    # drafts go wrong at positions = 3 (mod 5): rounds stop early, and a round whose
    # four positions skip that residue accepts every draft plus the bonus
    assert min(alens) < K and max(alens) == K
    assert d.appended == sum(a + 1 for a in alens)
    assert link["to_verifier"] == len(alens) * (K + 1) * 4
    assert link["to_drafter"] == sum((K + 3) * 4 + L * 2 * HKV * (a + 1) * D * 2 for a in alens)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    from lossless_kv_compressed_b200.remote import run_drafter, run_verifier
    import test_remote as T
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=60))
    try:
        if rank == 0:
            q.put((0, run_verifier(T.ToyVerifier(), T.PROMPT, T.N_GEN, peer=1)))
        else:
            d = T.ToyDrafter()
            q.put((1, (run_drafter(d, T.N_GEN, peer=0), d.appended)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_exchange_the_same_rounds():
    from lossless_kv_compressed_b200.remote import run_local
    toks, alens, _ = run_local(ToyDrafter(), ToyVerifier(), PROMPT, N_GEN)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert got[0] == alens                      # the verifier rank's accept lengths
    assert got[1][0] == toks == greedy_stream()  # the drafter rank's committed stream
    assert got[1][1] == sum(a + 1 for a in alens)


def _rank_dies(rank, port, q):
    """Rank 1 takes the compact cache and exits without drafting (a drafter that died
    between rounds); rank 0 must end with an error from its next receive."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import time
    import torch.distributed as dist
    from lossless_kv_compressed_b200.remote import _recv, run_verifier
    import test_remote as T
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        hdr = _recv((4,), torch.int64, 0, torch.device("cpu"), "cpu").tolist()
        S = hdr[0]
        for shape, dt in (((L, HKV, S, D), torch.bfloat16), ((L, HKV, S, D), torch.bfloat16),
                          ((L, HKV, S), torch.int32)):
            _recv(shape, dt, 0, torch.device("cpu"), "cpu")
        q.put((1, "left"))
        q.close()
        q.join_thread()                               # the message is out before the exit
        os._exit(0)                                   # no teardown: the peer just vanishes
    t0 = time.monotonic()
    try:
        run_verifier(T.ToyVerifier(), T.PROMPT, T.N_GEN, peer=1)
        q.put((0, ("no error", time.monotonic() - t0)))
    except Exception as e:                           # the failure surfaces on the host
        q.put((0, (type(e).__name__, time.monotonic() - t0)))
    q.close()
    q.join_thread()
    os._exit(0)


@pytest.mark.timeout(180)
def test_a_drafter_rank_that_dies_ends_the_verifier_with_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=30)
    assert got[1] == "left"
    kind, seconds = got[0]
    assert kind != "no error"
    assert seconds < 60                               # bounded by the group's timeout
