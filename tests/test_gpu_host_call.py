"""The pipelined host-buffer call (asa_attention_host) against the device-resident
call (asa_attention, itself parity-tested against the oracle): per head, the same
kernels run on the same data, so O must be bit-identical whatever the chunking of
the heads, for pinned and pageable host buffers, batches and ASA_G."""
import pytest
import torch

from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["tiny"]


def _case(name):
    return {
        "tiny": BASE,
        "b2-d128-5heads": BASE.with_(name="h5", B=2, H=5, d=128, T=3, Hg=9, W=11, seed=51, tau=0.95),
        "d64-ragged": BASE.with_(name="h3", B=1, H=3, d=64, T=5, Hg=9, W=11, seed=52),
    }[name]


@pytest.mark.parametrize("name,chunk,gw", [("tiny", 0, 0), ("tiny", 1, 0), ("b2-d128-5heads", 2, 0),
                                           ("b2-d128-5heads", 0, 0), ("b2-d128-5heads", 5, 64),
                                           ("d64-ragged", 1, 16), ("d64-ragged", 7, 0)])
def test_host_call_equals_device_call(name, chunk, gw):
    wl = _case(name)
    x = make_inputs(wl)
    qh, kh, vh = (x[n].contiguous().pin_memory() for n in ("q", "k", "v"))
    out = asa.asa_attention_host(qh, kh, vh, wl.T, wl.Hg, wl.W, wl.tau, global_window=gw,
                                 head_chunk=chunk)
    torch.cuda.current_stream().synchronize()
    asa.asa_check_device_status()
    ref, _, _ = asa.asa_attention(*(x[n].cuda() for n in ("q", "k", "v")), wl.T, wl.Hg, wl.W,
                                  wl.tau, global_window=gw)
    assert torch.equal(out.view(torch.int16), ref.cpu().view(torch.int16))


def test_host_call_pageable_and_repeated():
    wl = _case("b2-d128-5heads")
    x = make_inputs(wl)
    q, k, v = (x[n].contiguous() for n in ("q", "k", "v"))
    assert not q.is_pinned()
    ws = asa.host_workspace(wl.B, wl.T, wl.Hg, wl.W, wl.H, wl.d, head_chunk=2)
    outs = [asa.asa_attention_host(q, k, v, wl.T, wl.Hg, wl.W, wl.tau, head_chunk=2, workspace=ws)
            for _ in range(3)]
    torch.cuda.synchronize()
    ref, _, _ = asa.asa_attention(q.cuda(), k.cuda(), v.cuda(), wl.T, wl.Hg, wl.W, wl.tau)
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.cpu().view(torch.int16))


def test_host_call_rejects_device_tensors():
    x = make_inputs(BASE)
    q = x["q"].cuda()
    with pytest.raises(ValueError):
        asa.asa_attention_host(q, q, q, BASE.T, BASE.Hg, BASE.W, BASE.tau)
