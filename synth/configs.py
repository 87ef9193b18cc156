"""The five workloads, as frozen dataclasses with explicit seeds.

Shapes follow the public attention geometry of Llama-3.1-8B (32 query heads,
8 KV heads, head dim 128) and Llama-70B (64/8/128), which are the models the
VeriCache and CentroidKV summaries evaluate on (VeriCache summary, section
"Risultati Sperimentali"; CentroidKV summary, section "Contributi Chiave").
Seed of workload n is 1000 + n.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class AttnConfig:
    """One attention-layer workload (workloads 1-4)."""

    num: int
    name: str
    B: int            # batch (requests)
    Hq: int           # query heads
    Hkv: int          # KV heads
    D: int            # head dim
    P: int            # committed context length (prefix before the draft block)
    k: int            # draft length; verify runs k+1 query rows
    cache: str        # "indexed" or "int4"
    S: int = 0        # compressed slots (indexed cache)
    n_sinks: int = 4
    n_recent: int = 0
    deg_max: int = 1  # degrees n_t ~ U{1..deg_max} on the kept (non-sink, non-recent) slots
    compact: bool = False  # indexed cache stored compactly (idx = identity)
    tail_bf16: int = 0     # int4 cache: trailing tokens kept in bf16
    vocab: int = 0         # vocabulary of the acceptance logits
    rho: float = 0.9       # AR(1) coefficient along the sequence (0 = i.i.d.)
    outlier_frac: float = 0.0  # int4 workload: fraction of (kv head, channel) pairs scaled x10
    n_draft_requests: int = 0  # staged verify: other requests drafting meanwhile
    draft_context: int = 0     # staged verify: their context length
    chunk_tokens: int = 0      # staged verify: KV_full streamed in chunks of this many tokens

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def seed(self) -> int:
        return 1000 + self.num

    @property
    def L_cap(self) -> int:
        """Full-KV rows per (batch, kv head): prefix plus the k+1 block rows."""
        return self.P + self.k + 1


@dataclass(frozen=True)
class LoopConfig:
    """The end-to-end loop on a tiny random-init decoder."""

    num: int = 5
    name: str = "tinylm-loop"
    n_layers: int = 4
    d_model: int = 512
    Hq: int = 8
    Hkv: int = 2
    D: int = 64
    ffn: int = 1408
    vocab: int = 8192
    prompt_len: int = 8192
    gen_tokens: int = 512
    k: int = 32
    budget: int = 2048          # compressed slots per (layer, kv head) after prefill
    n_sinks: int = 4
    n_recent: int = 128         # 1/64 of the prompt
    score_window: int = 32      # last prompt queries used for eviction scores
    rope_theta: float = 10000.0
    rms_eps: float = 1e-5
    init_std: float = 0.02
    # Chunked Soft Matching variant of the compressed cache (CentroidKV): chunk size,
    # ratio schedule r_j = max(r_floor, r_init - j * delta_r), re-clustering interval
    csm_chunk: int = 256
    csm_r_init: float = 1.0
    csm_delta_r: float = 0.1
    csm_r_floor: float = 0.1
    csm_recluster_every: int = 128
    extra: dict = field(default_factory=dict)

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def seed(self) -> int:
        return 1000 + self.num


CONFIGS = {
    1: AttnConfig(num=1, name="tiny-indexed", B=1, Hq=8, Hkv=2, D=64, P=1024, k=8,
                  cache="indexed", S=256, n_sinks=4, n_recent=64, deg_max=8, vocab=1024),
    2: AttnConfig(num=2, name="llama3.1-8b-indexed-32k", B=8, Hq=32, Hkv=8, D=128, P=32768,
                  k=32, cache="indexed", S=8192, n_sinks=4, n_recent=512, deg_max=16,
                  vocab=128256),
    3: AttnConfig(num=3, name="llama3.1-8b-int4-128k", B=4, Hq=32, Hkv=8, D=128, P=131072,
                  k=32, cache="int4", tail_bf16=128, rho=0.0, outlier_frac=0.01,
                  vocab=128256),
    4: AttnConfig(num=4, name="llama70b-1m-staged", B=1, Hq=64, Hkv=8, D=128, P=1048576,
                  k=40, cache="indexed", S=65536, n_sinks=4, n_recent=4096, deg_max=16,
                  compact=True, n_draft_requests=3, draft_context=262144,
                  chunk_tokens=65536, vocab=128256),
    5: LoopConfig(),
}


def get_config(n: int):
    return CONFIGS[n]
