"""fp64 CPU oracle for the VeriCache draft/verify hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run anything in this package.
The product path (the CUDA library and its Python binding) never calls it and
shares no code with it: no kernels, helpers, tables or pre/post-processing.

It is written from two web summaries:

* "Riepilogo Tecnico: VeriCache" (gist.science/it/paper/2605.17613, with its
  Arabic translation gist.science/ar/paper/2605.17613): the draft-then-verify
  loop, greedy acceptance with the bonus token, and the staging of the full KV.
* "Riassunto Tecnico: CentroidKV" (gist.science/it/paper/2506.11418): the per-slot
  degree n_t entering the softmax as a logarithmic term, the preservation of
  attention sinks and recent tokens, and the Chunked Soft Matching compressor
  (``oracle.csm``).

The pages print no formula.  Each function states the plain definition it
implements and the reading taken where the pages are silent.  Everything is
plain NumPy in float64 with no blocking or fusion beyond the definition, so it
can be checked by eye.

Pinned (tests/test_oracle_*.py) against brute force on tiny inputs, closed forms,
the degree-n == n-copies identity, PyTorch's CPU scaled-dot-product attention as
a library special case, exhaustive acceptance on tiny vocabularies, and the
loop invariants (no compression => every draft accepted plus the bonus; the
committed stream equals full-KV greedy decoding).  Parity unpinned: none of the
functions below; acceptance-rate *values* are reported, not checked.
"""
from .numerics import bf16_to_f64, f16_to_f64  # noqa: F401
from .attention import (  # noqa: F401
    draft_attn, draft_attn_int4, verify_attn, verify_partial, merge_partials, finalize_partial,
)
from .accept import argmax_row, accept  # noqa: F401
from .quant import (  # noqa: F401
    quantize_k_groups, quantize_v_groups, dequant_k_groups, dequant_v_groups,
)
from . import csm  # noqa: F401,E402
