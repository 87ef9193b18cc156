"""vc_stage_full_kv copies pinned host bytes to HBM chunk by chunk (VeriCache summary,
"Riepilogo Tecnico: VeriCache", sections "Supporto Architetturale" and
"Scaglionamento tra Risorse (P1)"): device bytes == host bytes, the per-chunk
events complete, and a pageable source is refused."""
import numpy as np
import pytest
import torch

import lossless_kv_compressed_b200 as vc
from lossless_kv_compressed_b200._lib import VCError

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes,chunk", [(64 << 20, 16 << 20), ((48 << 20) + 4096, 16 << 20),
                                          (12345, 4096)])
def test_bytes_arrive_intact(nbytes, chunk):
    rng = np.random.default_rng(nbytes)
    host = torch.from_numpy(rng.integers(0, 256, size=nbytes, dtype=np.uint8)).pin_memory()
    dev = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    n_chunks = (nbytes + chunk - 1) // chunk
    evs = vc.make_events(n_chunks, s)
    vc.stage_full_kv(dev, host, chunk, s, evs)
    for e in evs:
        vc.event_wait(e, 30.0)
    torch.cuda.synchronize()
    assert torch.equal(dev.cpu(), host)


def test_pageable_source_is_refused():
    host = torch.zeros(1 << 20, dtype=torch.uint8)
    dev = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        vc.stage_full_kv(dev, host, 1 << 18, torch.cuda.current_stream())
    from lossless_kv_compressed_b200._lib import lib
    import ctypes
    st = lib().vc_stage_full_kv(dev.data_ptr(), host.data_ptr(), 1 << 20, 1 << 18,
                                torch.cuda.current_stream().cuda_stream, None, 0)
    assert st == 1


def test_event_wait_times_out_then_succeeds():
    """A bounded host wait returns VC_ERR_TIMEOUT instead of hanging: the event sits
    behind torch's fixed-length spin kernel (about a second), then completes."""
    s = torch.cuda.Stream()
    ev = torch.cuda.Event()
    with torch.cuda.stream(s):
        torch.cuda._sleep(int(2e9))
        ev.record(s)
    with pytest.raises(VCError) as ei:
        vc.event_wait(ev, 0.05)
    assert ei.value.status == 4
    vc.event_wait(ev, 60.0)
    torch.cuda.synchronize()
