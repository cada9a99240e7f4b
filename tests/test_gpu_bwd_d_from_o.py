"""The opt-in backward with D = rowsum(dO * O) from the stored bf16 O
(asa_sparse_attn_bwd_d_from_o) against the fp64 oracle.

Tolerance, derived: the rounding of O to bf16 perturbs D by up to 2^-9 relative per
element of the dot product; an fp64 estimate on these inputs puts the resulting dQ
error at 2.7e-3 to 3.4e-3 relative L2 (dK is hit alike through dS), on top of the
~1e-3 of the exact-D backward.  The bar is 1e-2 relative L2 and 4e-2 max-abs, twice
the exact backward's.  dV = P^T dO does not involve D: it must equal the exact
backward's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa
from gpu_util import check_close, f64, upload_mask

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["tiny"]
CASES = {
    "tiny": (BASE, 0),
    "d128-ragged": (BASE.with_(name="r495", B=1, H=2, d=128, T=5, Hg=9, W=11, seed=13, tau=0.95), 0),
    "d64-b2": (BASE.with_(name="r1200", B=2, H=2, d=64, T=6, Hg=10, W=20, seed=14), 0),
    "asa-g": (BASE.with_(name="r1200g", B=1, H=2, d=128, T=6, Hg=10, W=20, seed=15), 64),
}


@pytest.mark.parametrize("name", list(CASES))
def test_d_from_o_backward(name):
    wl, gw = CASES[name]
    x = make_inputs(wl, with_dout=True)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    ref = {k: oracle.permute(f64(x[k]), perm) for k in ("q", "k", "v", "dout")}
    mask = oracle.build_mask(oracle.estimate_pimp(ref["q"], ref["k"]), wl.tau)
    qp, kp, vp, dop = (torch.from_numpy(ref[k]).to(torch.bfloat16).cuda()
                       for k in ("q", "k", "v", "dout"))
    bm = upload_mask(mask, wl.N)
    o, lse = asa.asa_sparse_attn_fwd(qp, kp, vp, bm, global_window=gw)
    fast = asa.asa_sparse_attn_bwd(qp, kp, vp, o, dop, lse, bm, global_window=gw, d_from_o=True)
    exact = asa.asa_sparse_attn_bwd(qp, kp, vp, o, dop, lse, bm, global_window=gw)
    asa.asa_check_device_status()
    assert torch.equal(fast[2].view(torch.int16), exact[2].view(torch.int16)), "dV differs"
    dq_d, dkv_d = oracle.asa_backward(ref["q"], ref["k"], ref["v"], ref["dout"], mask,
                                      global_window=gw)
    exp = [np.zeros(qp.shape) for _ in range(3)]
    for (bb, h, I), blk in dq_d.items():
        exp[0][bb, h, 128 * I:128 * I + blk.shape[0]] = blk
    for (bb, h, J), (gk, gv) in dkv_d.items():
        exp[1][bb, h, 128 * J:128 * J + gk.shape[0]] = gk
        exp[2][bb, h, 128 * J:128 * J + gv.shape[0]] = gv
    for g, e, nm in zip(fast, exp, ("dQ", "dK", "dV")):
        check_close(f64(g), e, max_abs=4e-2, rel_l2=1e-2, what=nm + " (D from O)")
