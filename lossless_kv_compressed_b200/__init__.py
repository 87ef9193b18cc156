"""VeriCache draft/verify hot path on B200 (sm_100a).

The compute lives in ``libvericache.so`` (C ABI: include/vericache.h); this
package is its thin Python binding over torch tensors.
"""
from ._lib import VCError, lib, LIB_PATH, EXPORTS  # noqa: F401
from ._lib import VC_VERIFY_FIRST, VC_VERIFY_LAST, VC_OUT_F32  # noqa: F401
from .api import (  # noqa: F401
    IndexedCache, Int4Cache, draft_attn, draft_attn_noalloc, draft_workspace_size, verify_attn,
    verify_workspace_size, accept, stage_full_kv, make_events, event_wait, device_error,
    csm_out_len, csm_compress, set_wait_limit, int4_quantize, empty_int4_cache, evict_scores,
    evict_select,
)
