"""ctypes view of libvericache.so (the C ABI in include/vericache.h).

Loading fails loudly: there is no Python or CPU implementation behind these
names, so a missing library is an ImportError, never a silent fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvericache.so")

VC_OK, VC_ERR_INVALID, VC_ERR_UNSUPPORTED, VC_ERR_CUDA, VC_ERR_TIMEOUT = 0, 1, 2, 3, 4
VC_CACHE_INDEXED, VC_CACHE_INT4 = 0, 1
VC_VERIFY_FIRST, VC_VERIFY_LAST = 1, 2
VC_OUT_F32 = 4

# Every exported symbol, in header order.
EXPORTS = (
    "vc_status_string", "vc_last_error", "vc_abi_version",
    "vc_draft_workspace_size", "vc_draft_attn", "vc_draft_attn_noalloc",
    "vc_verify_workspace_size", "vc_verify_attn",
    "vc_accept", "vc_stage_full_kv", "vc_event_wait",
    "vc_csm_out_len", "vc_csm_compress", "vc_int4_quantize", "vc_evict_workspace_size",
    "vc_evict_scores", "vc_evict_select", "vc_device_error", "vc_set_wait_limit",
)
# Model glue of the end-to-end loop (include/vericache_glue.h).
GLUE_EXPORTS = (
    "vc_glue_embed", "vc_glue_rmsnorm", "vc_glue_gemm", "vc_glue_rope_store",
    "vc_glue_swiglu", "vc_glue_append_slots", "vc_glue_forward_full", "vc_glue_draft_steps",
    "vc_glue_greedy_steps", "vc_glue_workspace_size", "vc_glue_rmsnorm_gemm",
    "vc_glue_swiglu_gemm",
)

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t


class CompCache(ctypes.Structure):
    """Mirror of ``vc_comp_cache``."""

    _fields_ = [
        ("kind", _i32), ("B", _i32), ("Hq", _i32), ("Hkv", _i32), ("D", _i32),
        ("S", _i32), ("S_cap", _i32), ("T_cap", _i64),
        ("k", _p), ("v", _p), ("idx", _p), ("deg", _p),
        ("kq", _p), ("k_scale", _p), ("k_zero", _p),
        ("vq", _p), ("v_scale", _p), ("v_zero", _p),
        ("k_tail", _p), ("v_tail", _p), ("R_cap", _i32), ("n_tail", _i32),
        ("err_flag", _p),
    ]


class TinyLM(ctypes.Structure):
    """Mirror of ``vc_tinylm`` (vericache_glue.h)."""

    _fields_ = [
        ("n_layers", _i32), ("d_model", _i32), ("Hq", _i32), ("Hkv", _i32), ("D", _i32),
        ("ffn", _i32), ("vocab", _i32), ("rms_eps", ctypes.c_float),
        ("rope_theta", ctypes.c_float), ("embed", _p), ("lm_head", _p),
        ("wqkv", ctypes.POINTER(_p)), ("wo", ctypes.POINTER(_p)), ("wgu", ctypes.POINTER(_p)),
        ("wdown", ctypes.POINTER(_p)), ("k_full", ctypes.POINTER(_p)),
        ("v_full", ctypes.POINTER(_p)), ("cap", _i32), ("k_tail", ctypes.POINTER(_p)),
        ("v_tail", ctypes.POINTER(_p)), ("tail_cap", _i32), ("positions", _p),
        ("x", _p), ("h", _p), ("qkv", _p), ("q", _p), ("att", _p), ("gu", _p), ("act", _p),
        ("logits", _p), ("rows_cap", _i32), ("ws", _p), ("ws_bytes", _sz),
    ]


class VCError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {status_name(status)}: {detail}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m lossless_kv_compressed_b200.csrc.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        L.vc_status_string.restype = ctypes.c_char_p
        L.vc_status_string.argtypes = [ctypes.c_int]
        L.vc_last_error.restype = ctypes.c_char_p
        L.vc_last_error.argtypes = []
        L.vc_abi_version.restype = ctypes.c_int
        L.vc_draft_workspace_size.restype = _sz
        L.vc_draft_workspace_size.argtypes = [ctypes.POINTER(CompCache)]
        L.vc_draft_attn.restype = ctypes.c_int
        L.vc_draft_attn.argtypes = [_p, ctypes.POINTER(CompCache), ctypes.c_float, ctypes.c_int,
                                    _p, _p, _p, _sz, _p]
        L.vc_draft_attn_noalloc.restype = ctypes.c_int
        L.vc_draft_attn_noalloc.argtypes = [_p, ctypes.POINTER(CompCache), ctypes.c_float,
                                            ctypes.c_int, _p, _p, _p]
        L.vc_verify_workspace_size.restype = _sz
        L.vc_verify_workspace_size.argtypes = [ctypes.c_int] * 5 + [_i64, _i64]
        L.vc_verify_attn.restype = ctypes.c_int
        L.vc_verify_attn.argtypes = ([_p] + [ctypes.c_int] * 5 + [_p, _p] + [_i64] * 4
                                     + [_p, _p, _p, ctypes.c_int, ctypes.c_float, _p, _p, _sz, _p])
        L.vc_accept.restype = ctypes.c_int
        L.vc_accept.argtypes = [_p, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _p, _p, _p, _p,
                                _p, _p]
        L.vc_stage_full_kv.restype = ctypes.c_int
        L.vc_stage_full_kv.argtypes = [_p, _p, _sz, _sz, _p, _p, ctypes.c_int]
        L.vc_event_wait.restype = ctypes.c_int
        L.vc_event_wait.argtypes = [_p, ctypes.c_double]
        L.vc_device_error.restype = ctypes.c_int
        L.vc_device_error.argtypes = [ctypes.POINTER(_i32), ctypes.c_int]
        L.vc_int4_quantize.restype = ctypes.c_int
        L.vc_int4_quantize.argtypes = ([_p, _p, ctypes.c_int, ctypes.c_int, _i64, _i64,
                                        ctypes.c_int] + [_p] * 6 + [_i64, _i64, _p])
        L.vc_evict_workspace_size.restype = _sz
        L.vc_evict_workspace_size.argtypes = [ctypes.c_int] * 3
        L.vc_evict_scores.restype = ctypes.c_int
        L.vc_evict_scores.argtypes = ([_p] + [ctypes.c_int] * 5 + [_p, _i64, _i64, ctypes.c_float,
                                                                   _p, _i64, _p, _sz, _p])
        L.vc_evict_select.restype = ctypes.c_int
        L.vc_evict_select.argtypes = [_p, ctypes.c_int, _i64, _i64, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, _p, _i64, _p]
        L.vc_set_wait_limit.restype = ctypes.c_int
        L.vc_set_wait_limit.argtypes = [ctypes.c_double, ctypes.POINTER(ctypes.c_double)]
        L.vc_csm_out_len.restype = _i64
        L.vc_csm_out_len.argtypes = [_i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_double]
        L.vc_csm_compress.restype = ctypes.c_int
        L.vc_csm_compress.argtypes = ([_p, _p, _p, ctypes.c_int, ctypes.c_int, _i64, _i64,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                       _p, _p, _p, _i64, _p, _p])
        for name in GLUE_EXPORTS:
            getattr(L, name).restype = ctypes.c_int
        L.vc_glue_embed.argtypes = [_p, _p, ctypes.c_int, ctypes.c_int, _p, _p]
        L.vc_glue_rmsnorm.argtypes = [_p, ctypes.c_int, ctypes.c_int, ctypes.c_float, _p, _p]
        L.vc_glue_gemm.argtypes = [_p, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _p,
                                   ctypes.c_int, _p]
        L.vc_glue_rmsnorm_gemm.argtypes = [_p, ctypes.c_float, _p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, _p, ctypes.c_int, _p]
        L.vc_glue_swiglu_gemm.argtypes = [_p, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _p,
                                          ctypes.c_int, _p]
        L.vc_glue_rope_store.argtypes = [_p, _p, _p] + [ctypes.c_int] * 4 + [ctypes.c_float,
                                                                             _p, _p, _p,
                                                                             ctypes.c_int, _p]
        L.vc_glue_swiglu.argtypes = [_p, ctypes.c_int, ctypes.c_int, _p, _p]
        L.vc_glue_append_slots.argtypes = [_p, _p] + [ctypes.c_int] * 5 + [_p]
        L.vc_glue_forward_full.argtypes = [ctypes.POINTER(TinyLM), _p, ctypes.c_int,
                                           ctypes.c_int, _p]
        L.vc_glue_draft_steps.argtypes = [ctypes.POINTER(TinyLM), ctypes.POINTER(CompCache), _p,
                                          ctypes.c_int, ctypes.c_int, _p]
        L.vc_glue_workspace_size.restype = _sz
        L.vc_glue_workspace_size.argtypes = [ctypes.POINTER(TinyLM)]
        L.vc_glue_greedy_steps.argtypes = [ctypes.POINTER(TinyLM), _p, ctypes.c_int,
                                           ctypes.c_int, _p]
        _lib = L
    return _lib


def status_name(st: int) -> str:
    return lib().vc_status_string(int(st)).decode()


def check(st: int, where: str) -> None:
    if st != VC_OK:
        raise VCError(st, where, lib().vc_last_error().decode())
