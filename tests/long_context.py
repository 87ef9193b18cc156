"""Shared set-up of the long-context verify tests: walk a staged case's full cache
chunk by chunk (host memory stays bounded by one chunk), hand each chunk to the test,
and accumulate the fp64 oracle's softmax state for a few sampled (row, kv head)
pairs as the chunks go by."""
import numpy as np

import oracle


def walk_chunks(case, rows, heads, sink):
    """Calls sink(k_bits [Hkv, n, D], v_bits, kv_start) for every chunk of the prefix and
    returns {(i, j): o [g, D]}: the oracle's verify output of block row i, query heads
    j*g .. j*g+g-1 (kv head j), over the prefix and the block's own keys."""
    f = oracle.bf16_to_f64
    cfg, P = case["cfg"], case["P"]
    g = cfg.Hq // cfg.Hkv
    q = case["q_verify_bits"]
    state = {(i, j): None for i in rows for j in heads}

    def add(kb, vb, s0):
        for j in heads:
            kj, vj = f(kb[None, j:j + 1]), f(vb[None, j:j + 1])
            for i in rows:
                part = oracle.verify_partial(f(q[:, i:i + 1, j * g:(j + 1) * g]), kj, vj, s0,
                                             P + i)
                st = state[(i, j)]
                state[(i, j)] = part if st is None else oracle.merge_partials(st, part)

    s0 = 0
    for kb, vb in zip(case["chunks_k"], case["chunks_v"]):
        sink(kb, vb, s0)
        add(kb, vb, s0)
        s0 += kb.shape[1]
    assert s0 == P
    add(case["block_k_bits"][0], case["block_v_bits"][0], P)
    return {key: oracle.finalize_partial(st)[0, 0] for key, st in state.items()}
