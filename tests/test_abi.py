"""The C ABI library loads, exports every function include/vericache.h declares, and
rejects bad arguments on the host (these paths make no CUDA call)."""
import ctypes
import os
import re

import pytest

import lossless_kv_compressed_b200 as vc
from lossless_kv_compressed_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("vericache.h", "vericache_glue.h")]


def _declared(path):
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vc_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    L = vc.lib()
    core, glue = _declared(HEADERS[0]), _declared(HEADERS[1])
    assert len(core) >= 10 and len(glue) >= 6
    for n in core + glue:
        assert hasattr(L, n), f"{n} declared in a header but not exported"
    assert set(core) == set(_lib.EXPORTS)
    assert set(glue) == set(_lib.GLUE_EXPORTS)
    assert sorted(os.listdir(os.path.join(ROOT, "include"))) == ["vericache.h", "vericache_glue.h"]


def test_glue_workspace_covers_both_verify_windows():
    """vc_glue_workspace_size is host arithmetic: the prefill's blocks of min(rows_cap,
    1024 / g) rows under any window vc_verify_attn may choose, and the decode blocks'
    smaller windows over tail_cap rows (more splits), whichever is larger; 0 for an
    invalid descriptor."""
    L = vc.lib()
    m = _lib.TinyLM()
    m.n_layers, m.d_model, m.Hq, m.Hkv, m.D = 4, 512, 8, 2, 64
    m.cap, m.rows_cap, m.tail_cap = 8738, 8192, 33
    need = L.vc_glue_workspace_size(ctypes.byref(m))
    prefill = L.vc_verify_workspace_size(1, 256, 8, 2, 64, 0, 8738)
    assert need >= prefill > 0
    # decode blocks: 33 rows x 4 heads over windows of at most 4096 keys
    assert need >= L.vc_verify_workspace_size(1, 33, 8, 2, 64, 0, 8738)
    m.Hkv = 3
    assert L.vc_glue_workspace_size(ctypes.byref(m)) == 0


def test_status_strings_and_version():
    L = vc.lib()
    assert L.vc_abi_version() == 1
    assert _lib.status_name(0) == "VC_OK"
    assert _lib.status_name(2) == "VC_ERR_UNSUPPORTED"
    assert _lib.status_name(99) == "VC_UNKNOWN_STATUS"


def _cache(**kw):
    c = _lib.CompCache()
    c.kind, c.B, c.Hq, c.Hkv, c.D, c.S, c.T_cap = 0, 1, 8, 2, 128, 16, 64
    c.k = c.v = 1 << 20
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), _lib.VC_ERR_UNSUPPORTED),
    (dict(Hq=7), _lib.VC_ERR_INVALID),
    (dict(Hq=32, Hkv=2), _lib.VC_ERR_UNSUPPORTED),       # g = 16
    (dict(S=0, n_tail=0), _lib.VC_ERR_INVALID),
    (dict(n_tail=3), _lib.VC_ERR_INVALID),               # tail pointers missing
    (dict(k=(1 << 20) + 8), _lib.VC_ERR_INVALID),        # misaligned
    (dict(S=100, T_cap=64), _lib.VC_ERR_INVALID),        # compact cache larger than base
    (dict(kind=1, S=40, T_cap=64), _lib.VC_ERR_INVALID), # int4 needs S % 32 == 0
    (dict(kind=7), _lib.VC_ERR_INVALID),
])
def test_draft_rejects_bad_cache(kw, status):
    c = _cache(**kw)
    st = vc.lib().vc_draft_attn(1 << 20, ctypes.byref(c), 0.0, 0, 1 << 20, None, 1 << 20,
                                1 << 20, None)
    assert st == status, vc.lib().vc_last_error()
    assert vc.lib().vc_last_error()


def test_draft_rejects_null_cache():
    assert vc.lib().vc_draft_attn(1 << 20, None, 0.0, 0, 1 << 20, None, 1 << 20, 1, None) == 1


@pytest.mark.parametrize("args,status", [
    (dict(D=80), _lib.VC_ERR_UNSUPPORTED),
    (dict(n_q=0), _lib.VC_ERR_INVALID),
    (dict(Hq=64, Hkv=4), _lib.VC_ERR_UNSUPPORTED),
    (dict(n_q=300), _lib.VC_ERR_UNSUPPORTED),           # n_q * g > 1024
    (dict(kv_len=5000), _lib.VC_ERR_INVALID),           # single pass must cover P + n_q
    (dict(kv_start=3), _lib.VC_ERR_INVALID),
])
def test_verify_rejects_bad_arguments(args, status):
    a = dict(q=1 << 20, B=1, n_q=9, Hq=8, Hkv=2, D=128, k=1 << 20, v=1 << 20, L_cap=4096,
             kv_start=0, kv_len=1033, P=1024, m=None, l=None, acc=None, flags=0, scale=0.0,
             out=1 << 20, ws=1 << 20, ws_bytes=1 << 20, stream=None)
    a.update(args)
    st = vc.lib().vc_verify_attn(*a.values())
    assert st == status, vc.lib().vc_last_error()


def test_accept_and_stage_reject_bad_arguments():
    L = vc.lib()
    assert L.vc_accept(1 << 20, None, 0, 9, 1024, 1 << 20, None, None, None, None, None) == 1
    assert L.vc_accept(None, None, 1, 9, 1024, 1 << 20, None, None, None, None, None) == 1
    assert L.vc_accept(1 << 20, 1 << 20, 1, 9, 1024, 1 << 20, 1 << 20, None, None, None, None) == 1
    assert L.vc_accept(1 << 20, None, 1, 9, 1024, 1 << 20, 1 << 20, 1 << 20, 1 << 20, None, None) == 1
    assert L.vc_stage_full_kv(1 << 20, 1 << 20, 100, 0, None, None, 0) == 1
    assert L.vc_stage_full_kv(None, 1 << 20, 100, 10, None, None, 0) == 1


@pytest.mark.parametrize("T,ns,nr,chunk,r", [(40, 4, 6, 8, 0.5), (90, 2, 3, 2, 1.0),
                                            (32768, 4, 512, 256, 0.5), (517, 8, 9, 256, 0.3),
                                            (31, 0, 0, 10, 1.0), (10, 5, 5, 4, 0.7),
                                            (1000, 0, 0, 7, 0.999), (64, 4, 4, 16, 0.0)])
def test_csm_out_len_matches_the_oracle(T, ns, nr, chunk, r):
    from oracle import csm
    assert vc.lib().vc_csm_out_len(T, ns, nr, chunk, r) == csm.out_len(T, ns, nr, chunk, r)


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), 2), (dict(chunk=1), 2), (dict(chunk=512), 2), (dict(r=1.5), 1),
    (dict(r=-0.1), 1), (dict(n_sinks=60, n_recent=60), 1), (dict(T=300), 1),
    (dict(T_cap_out=10), 1), (dict(pairs=0), 1), (dict(k=3), 1)])
def test_csm_rejects_bad_arguments(kw, status):
    a = dict(k=256, v=256, deg=0, pairs=2, D=128, T=100, T_cap=200, n_sinks=4, n_recent=4,
             chunk=16, r=0.5, k_out=256, v_out=256, deg_out=256, T_cap_out=200, dest=0)
    a.update(kw)
    L = vc.lib()
    st = L.vc_csm_compress(a["k"], a["v"], a["deg"] or None, a["pairs"], a["D"], a["T"],
                           a["T_cap"], a["n_sinks"], a["n_recent"], a["chunk"], a["r"],
                           a["k_out"], a["v_out"], a["deg_out"], a["T_cap_out"],
                           a["dest"] or None, None)
    assert st == status, _lib.status_name(st)
    assert vc.lib().vc_last_error()


def test_stage_fault_injection_fails_before_any_cuda_call(monkeypatch):
    """VC_FAULT_INJECT=stage_fail: the staging call reports a copy failure before it
    enqueues anything (here on a host with no GPU, where any CUDA call would fail
    differently), and works normally once the variable is cleared."""
    L = vc.lib()
    monkeypatch.setenv("VC_FAULT_INJECT", "stage_fail")
    assert L.vc_stage_full_kv(1 << 20, 1 << 20, 100, 10, None, None, 0) == _lib.VC_ERR_CUDA
    assert b"injected" in L.vc_last_error()
    monkeypatch.setenv("VC_FAULT_INJECT", "something_else")
    assert L.vc_stage_full_kv(None, 1 << 20, 100, 10, None, None, 0) == _lib.VC_ERR_INVALID
    monkeypatch.delenv("VC_FAULT_INJECT")
    assert L.vc_stage_full_kv(None, 1 << 20, 100, 10, None, None, 0) == _lib.VC_ERR_INVALID


def test_wait_limit_setting():
    prev = ctypes.c_double(-1.0)
    L = vc.lib()
    assert L.vc_set_wait_limit(-1.0, None) == _lib.VC_ERR_INVALID
    assert L.vc_set_wait_limit(61.0, None) == _lib.VC_ERR_INVALID
    assert L.vc_set_wait_limit(float("nan"), None) == _lib.VC_ERR_INVALID
    assert L.vc_set_wait_limit(0.5, ctypes.byref(prev)) == _lib.VC_OK
    assert prev.value == pytest.approx(2.0)
    assert vc.set_wait_limit(0.0) == pytest.approx(0.5)     # 0 restores the default
    assert vc.set_wait_limit(0.0) == pytest.approx(2.0)
