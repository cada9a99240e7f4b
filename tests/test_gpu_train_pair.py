"""The training pair: asa_sparse_attn_fwd_train (P V with fp16 P, the output also in
fp32) and asa_sparse_attn_bwd_train (D = rowsum(dO * O) from that fp32 output, no pass
of its own over the kept tiles), against the fp64 oracle under the oracle's mask.

Bars: the standard ones (outputs and gradients max-abs <= 2e-2, rel-L2 <= 5e-3; the
ASA_G gradients with dO scaled to keep them O(1), plus the unscaled check at
2e-2 + 2^-8 |ref|).  The fp32 output is checked at rel-L2 <= 1e-3 (fp16 P: ~2^-12
relative per weight), and its bf16 rounding must be the bf16 output bit for bit.
dV = P^T dO does not involve D, and the forward's LSE is the inference forward's, so
dV must equal asa_sparse_attn_bwd's bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
from video_dit_dynamic_gilbert_b200 import asa
from gpu_util import LSE_ABS, check_close, check_close_ulp, f64, upload_mask
from test_gpu_parity import CASES, setup_case

pytestmark = pytest.mark.gpu

RUNS = [(name, 0) for name in CASES] + [("tiny", 64), ("d128-ragged", 16), ("d64-b2", 100),
                                        ("multi-tile", 64)]


def _grads_ref(ref, mask, gw):
    dq_d, dkv_d = oracle.asa_backward(ref["q"], ref["k"], ref["v"], ref["dout"], mask,
                                      global_window=gw)
    shape = ref["q"].shape
    exp = [np.zeros(shape) for _ in range(3)]
    for (bb, h, I), blk in dq_d.items():
        exp[0][bb, h, 128 * I:128 * I + blk.shape[0]] = blk
    for (bb, h, J), (gk, gv) in dkv_d.items():
        exp[1][bb, h, 128 * J:128 * J + gk.shape[0]] = gk
        exp[2][bb, h, 128 * J:128 * J + gv.shape[0]] = gv
    return exp


@pytest.mark.parametrize("name,gw", RUNS)
def test_training_pair_against_oracle(name, gw):
    wl, x, perm, ref, pimp, mask, marg, dev = setup_case(name)
    qp, kp, vp = (torch.from_numpy(ref[k]).to(torch.bfloat16).cuda() for k in ("q", "k", "v"))
    bm = upload_mask(mask, wl.N)
    o, lse, o32 = asa.asa_sparse_attn_fwd_train(qp, kp, vp, bm, global_window=gw)
    o_inf, lse_inf = asa.asa_sparse_attn_fwd(qp, kp, vp, bm, global_window=gw)
    asa.asa_check_device_status()
    O_ref, L_ref = oracle.asa_forward(ref["q"], ref["k"], ref["v"], mask, global_window=gw)
    check_close(f64(o), O_ref, what="O (training forward)")
    check_close(f64(o32), O_ref, rel_l2=1e-3, what="fp32 O (training forward)")
    check_close(f64(lse), L_ref, max_abs=LSE_ABS, rel_l2=1e-4, what="LSE (training forward)")
    assert torch.equal(o32.to(torch.bfloat16).view(torch.int16), o.view(torch.int16))
    assert torch.equal(lse, lse_inf)
    exp = _grads_ref(ref, mask, gw)
    peak = max(np.abs(e).max() for e in exp)
    sc = 2.0 ** -max(0, math.ceil(math.log2(peak / 2.0))) if peak > 2.0 else 1.0
    dop = torch.from_numpy(ref["dout"] * sc).to(torch.bfloat16).cuda()
    got = asa.asa_sparse_attn_bwd_train(qp, kp, vp, o32, dop, lse, bm, global_window=gw)
    exact = asa.asa_sparse_attn_bwd(qp, kp, vp, o_inf, dop, lse_inf, bm, global_window=gw)
    asa.asa_check_device_status()
    assert torch.equal(got[2].view(torch.int16), exact[2].view(torch.int16)), "dV differs"
    for g, e, nm in zip(got, exp, ("dQ", "dK", "dV")):
        err, rel = check_close(f64(g), e * sc, what=f"{nm} (training pair)")
        print(f"{name} n={gw} {nm}: max-abs {err:.2e}, rel-L2 {rel:.2e}")
    if sc != 1.0:
        dop1 = torch.from_numpy(ref["dout"]).to(torch.bfloat16).cuda()
        got1 = asa.asa_sparse_attn_bwd_train(qp, kp, vp, o32, dop1, lse, bm, global_window=gw)
        asa.asa_check_device_status()
        for g, e, nm in zip(got1, exp, ("dQ", "dK", "dV")):
            check_close_ulp(f64(g), e, what=f"{nm} unscaled (training pair)")


def test_training_pair_unkept_key_blocks():
    """Rows keeping only their own block or block 0, a key block nobody keeps (dK = dV = 0
    exactly), the CSR the standard backward test uses."""
    wl, x, perm, ref, pimp, _, marg, dev = setup_case("multi-tile")
    nb = -(-wl.N // 128)
    mask = np.zeros((wl.B, wl.H, nb, nb), dtype=bool)
    for I in range(nb):
        mask[:, :, I, I] = True
    mask[:, :, :, 0] = True
    mask[:, :, 1, :] = False
    mask[:, :, 1, 1] = True
    mask[:, :, nb - 1, nb - 1] = False
    mask[:, :, nb - 1, 0] = True
    qp, kp, vp = (torch.from_numpy(ref[k]).to(torch.bfloat16).cuda() for k in ("q", "k", "v"))
    dop = torch.from_numpy(ref["dout"] / 16).to(torch.bfloat16).cuda()
    bm = upload_mask(mask, wl.N)
    o, lse, o32 = asa.asa_sparse_attn_fwd_train(qp, kp, vp, bm)
    got = asa.asa_sparse_attn_bwd_train(qp, kp, vp, o32, dop, lse, bm)
    asa.asa_check_device_status()
    ref16 = dict(ref, dout=ref["dout"] / 16)
    exp = _grads_ref(ref16, mask, 0)
    for g, e, nm in zip(got, exp, ("dQ", "dK", "dV")):
        check_close(f64(g), e, what=nm)
    assert (f64(got[1])[:, :, 128 * (nb - 1):] == 0).all()
    assert (f64(got[2])[:, :, 128 * (nb - 1):] == 0).all()


def test_training_forward_reports_v_beyond_fp16():
    """A V value beyond fp16 range is reported by the next status check."""
    wl, x, perm, ref, pimp, mask, marg, dev = setup_case("tiny")
    qp, kp, vp = (torch.from_numpy(ref[k]).to(torch.bfloat16).cuda() for k in ("q", "k", "v"))
    bm = upload_mask(mask, wl.N)
    asa.asa_check_device_status()
    vbad = vp.clone()
    vbad[0, 1, 7, 3] = 1e5
    asa.asa_sparse_attn_fwd_train(qp, kp, vbad, bm)
    with pytest.raises(asa.AsaError) as ei:
        asa.asa_check_device_status()
    assert ei.value.code == asa.ASA_ERR_INVALID_ARG
    asa.asa_check_device_status()


def test_training_pair_deterministic():
    wl, x, perm, ref, pimp, mask, marg, dev = setup_case("multi-tile")
    qp, kp, vp, dop = (torch.from_numpy(ref[k]).to(torch.bfloat16).cuda()
                       for k in ("q", "k", "v", "dout"))
    bm = upload_mask(mask, wl.N)
    a = asa.asa_sparse_attn_fwd_train(qp, kp, vp, bm)
    b = asa.asa_sparse_attn_fwd_train(qp, kp, vp, bm)
    for s, t in zip(a, b):
        assert torch.equal(s, t)
    g1 = asa.asa_sparse_attn_bwd_train(qp, kp, vp, a[2], dop, a[1], bm)
    g2 = asa.asa_sparse_attn_bwd_train(qp, kp, vp, a[2], dop, a[1], bm)
    for s, t in zip(g1, g2):
        assert torch.equal(s, t)
