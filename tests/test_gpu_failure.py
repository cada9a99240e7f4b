"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies
gives up, the kernel records it in the device error word and returns, the host reports
ASA_ERR_TIMEOUT at the next status check, and the context keeps working."""
import numpy as np
import pytest
import torch

import oracle
from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa
from gpu_util import check_close, f64, upload_mask

pytestmark = pytest.mark.gpu


def test_forced_wait_timeout_is_reported_and_cleared():
    asa.asa_check_device_status()                 # start clean
    asa.asa_selftest_wait_timeout(1 << 20)        # ~0.5 ms of SM clock
    with pytest.raises(asa.AsaError) as ei:
        asa.asa_check_device_status()
    assert ei.value.code == asa.ASA_ERR_TIMEOUT
    assert "0x10" in str(ei.value)
    asa.asa_check_device_status()                 # the word was cleared


def test_context_usable_after_timeout():
    asa.asa_selftest_wait_timeout(1 << 18)
    asa.asa_selftest_wait_timeout(1 << 18)        # two expiries: one sticky report
    with pytest.raises(asa.AsaError):
        asa.asa_check_device_status()
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    ref = {k: oracle.permute(f64(x[k]), perm) for k in ("q", "k", "v")}
    mask = oracle.build_mask(oracle.estimate_pimp(ref["q"], ref["k"]), wl.tau)
    qp, kp, vp = (torch.from_numpy(ref[k]).to(torch.bfloat16).cuda() for k in ("q", "k", "v"))
    o, _ = asa.asa_sparse_attn_fwd(qp, kp, vp, upload_mask(mask, wl.N))
    asa.asa_check_device_status()
    O_ref, _ = oracle.asa_forward(ref["q"], ref["k"], ref["v"], mask)
    check_close(f64(o), O_ref, what="O after a forced timeout")
