"""The allocation-free estimator entry point (asa_estimate_noalloc).

It exists for callers that cannot allocate device memory (engines that own all GPU
memory in a fixed pool, latency-critical loops that must not risk cudaMalloc's
synchronisation): its scratch is a fixed device array inside the library.  These
tests call it through the C ABI and check, on two calls in a row, that it returns
what the workspace-based asa_estimate returns on the same inputs.  The file sorts
last so that a run stopping at the first failure has already run everything else."""
import ctypes

import numpy as np
import pytest
import torch

from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa
from video_dit_dynamic_gilbert_b200.build import build

pytestmark = pytest.mark.gpu


def _call_noalloc(L, qp, kp, out):
    B, H, N, d = qp.shape
    return L.asa_estimate_noalloc(ctypes.c_void_p(qp.data_ptr()), ctypes.c_void_p(kp.data_ptr()),
                                  B, H, N, d, 128, 16, ctypes.c_void_p(out.data_ptr()),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("case", [
    WORKLOADS["tiny"],
    WORKLOADS["tiny"].with_(name="r1200", B=2, H=2, d=128, T=6, Hg=10, W=20, seed=31),
    # the largest call the fixed array takes at the Wan2.1-1.3B shape: 5 heads
    WORKLOADS["wan2.1-1.3b"].with_(name="wan-5-heads", H=5, seed=32),
])
def test_noalloc_matches_workspace_estimate_twice(case):
    """Both entry points run the same deterministic kernels (no atomics) on the same
    inputs, so the outputs must be bit-identical, on each of two calls in a row."""
    build()
    L = asa.lib()
    x = make_inputs(case)
    T, Hg, W = case.T, case.Hg, case.W
    qp = asa.asa_gilbert_permute(x["q"].cuda(), T, Hg, W)
    kp = asa.asa_gilbert_permute(x["k"].cuda(), T, Hg, W)
    ref = asa.asa_estimate(qp, kp)
    B, H, N, d = qp.shape
    nb = -(-N // 128)
    for _ in range(2):
        out = torch.full((B, H, nb, nb), float("nan"), dtype=torch.float32, device="cuda")
        rc = _call_noalloc(L, qp, kp, out)
        assert rc == asa.ASA_OK, L.asa_last_error_string()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert L.asa_check_device_status(None) == asa.ASA_OK


def test_noalloc_rejects_shapes_above_its_fixed_scratch():
    build()
    L = asa.lib()
    q = torch.zeros((1, 48, 128, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(1, dtype=torch.float32, device="cuda")
    # 48 heads at 75,600 tokens need ~1.1 GB of scratch: refused before any launch
    rc = L.asa_estimate_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(q.data_ptr()),
                                1, 48, 75600, 64, 128, 16, ctypes.c_void_p(out.data_ptr()), None)
    assert rc == asa.ASA_ERR_WORKSPACE
    assert b"scratch" in L.asa_last_error_string()
    # one head more than the largest accepted call at the Wan2.1-1.3B shape
    rc = L.asa_estimate_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(q.data_ptr()),
                                1, 6, 32760, 128, 128, 16, ctypes.c_void_p(out.data_ptr()), None)
    assert rc == asa.ASA_ERR_WORKSPACE
