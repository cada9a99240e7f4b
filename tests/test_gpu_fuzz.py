"""Seeded random small shapes through every step against the oracle: permutation
(bit-exact), P_imp, mask rows (bit-exact unless marginal, then a legal cut), forward
and backward under the oracle's mask (the exact backward and the training pair), the
forward storing O straight to raster order, for ASA and ASA_G.  Shapes cover single tokens, ragged last blocks,
blocks shorter than k = 16, batch 2, several heads, d = 64 and 128."""
import math

import numpy as np
import pytest
import torch

import oracle
from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa
from gpu_util import check_close, compare_masks, f64, mask_from_csr, upload_mask

pytestmark = pytest.mark.gpu


def _cases(n=24, seed=2026):
    g = np.random.default_rng(seed)
    out = []
    for i in range(n):
        T, Hg, W = (int(x) for x in (g.integers(1, 6), g.integers(1, 20), g.integers(1, 24)))
        out.append(dict(B=int(g.integers(1, 3)), H=int(g.integers(1, 5)),
                        d=int(g.choice([64, 128])), T=T, Hg=Hg, W=W,
                        tau=float(g.choice([0.5, 0.8, 0.95, 1.0])),
                        n=int(g.choice([0, 0, 1, 7, 64, 130])), seed=100 + i))
    return out


@pytest.mark.parametrize("c", _cases(), ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}_{c['T']}x{c['Hg']}x{c['W']}_t{c['tau']}_n{c['n']}")
def test_fuzz_whole_path(c):
    wl = WORKLOADS["tiny"].with_(name="fz", B=c["B"], H=c["H"], d=c["d"], T=c["T"], Hg=c["Hg"],
                                 W=c["W"], tau=c["tau"], seed=c["seed"])
    n = c["n"]
    x = make_inputs(wl, with_dout=True)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    ref = {name: oracle.permute(f64(x[name]), perm) for name in ("q", "k", "v", "dout")}
    dev = {name: x[name].cuda() for name in ("q", "k", "v", "dout")}
    qp, kp, vp = asa.asa_gilbert_permute3(dev["q"], dev["k"], dev["v"], wl.T, wl.Hg, wl.W)
    assert np.array_equal(f64(qp), ref["q"])
    # estimate + mask
    pimp = oracle.estimate_pimp(ref["q"], ref["k"])
    np.testing.assert_allclose(f64(asa.asa_estimate(qp, kp)), pimp, rtol=2e-4, atol=1e-9)
    bm = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    mask = oracle.build_mask(pimp, wl.tau)
    marg = oracle.marginal_rows(pimp, wl.tau)
    compare_masks(mask_from_csr(bm), mask, marg, pimp, wl.tau, what=f"fuzz seed {c['seed']}")
    # forward and backward under the oracle's mask
    bmo = upload_mask(mask, wl.N)
    o, lse = asa.asa_sparse_attn_fwd(qp, kp, vp, bmo, global_window=n)
    O_ref, L_ref = oracle.asa_forward(ref["q"], ref["k"], ref["v"], mask, global_window=n)
    check_close(f64(o), O_ref, what="O")
    dq_d, dkv_d = oracle.asa_backward(ref["q"], ref["k"], ref["v"], ref["dout"], mask,
                                      global_window=n)
    peak = max([np.abs(b).max() for b in dq_d.values()] +
               [np.abs(b).max() for pair in dkv_d.values() for b in pair])
    sc = 2.0 ** -math.ceil(math.log2(peak / 2.0)) if peak > 2.0 else 1.0
    dop = torch.from_numpy(ref["dout"] * sc).to(torch.bfloat16).cuda()
    dq, dk, dv = (f64(t) for t in asa.asa_sparse_attn_bwd(qp, kp, vp, o, dop, lse, bmo,
                                                          global_window=n))
    asa.asa_check_device_status()
    rq, rk, rv = np.zeros_like(dq), np.zeros_like(dk), np.zeros_like(dv)
    for (bb, h, I), blk in dq_d.items():
        rq[bb, h, 128 * I:128 * I + blk.shape[0]] = blk * sc
    for (bb, h, J), (gk, gv) in dkv_d.items():
        rk[bb, h, 128 * J:128 * J + gk.shape[0]] = gk * sc
        rv[bb, h, 128 * J:128 * J + gv.shape[0]] = gv * sc
    check_close(dq, rq, what="dQ")
    check_close(dk, rk, what="dK")
    check_close(dv, rv, what="dV")
    # the training pair: D from the training forward's fp32 O
    o_t, lse_t, o32 = asa.asa_sparse_attn_fwd_train(qp, kp, vp, bmo, global_window=n)
    check_close(f64(o_t), O_ref, what="O (training forward)")
    grads_t = asa.asa_sparse_attn_bwd_train(qp, kp, vp, o32, dop, lse_t, bmo, global_window=n)
    asa.asa_check_device_status()
    for g, r, nm in zip(grads_t, (rq, rk, rv), ("dQ", "dK", "dV")):
        check_close(f64(g), r, what=f"{nm} (training pair)")
    # the raster output of the whole call, and the forward that stores it directly
    out = asa.asa_unpermute(o, wl.T, wl.Hg, wl.W)
    check_close(f64(out)[:, perm].transpose(0, 2, 1, 3), O_ref, what="O raster")
    out_r, lse_r = asa.asa_sparse_attn_fwd_raster(qp, kp, vp, bmo, wl.T, wl.Hg, wl.W,
                                                  global_window=n)
    assert torch.equal(out_r, out) and torch.equal(lse_r, lse)
