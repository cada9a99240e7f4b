"""The differentiable op (asa.ASAAttention): gradients in raster layout against the
oracle where the mask is fixed by definition (tau = 1 keeps every block, so the
oracle's mask needs nothing from the CUDA path), and bit-identical to the step-by-step
calls at a sparse tau."""
import numpy as np
import pytest
import torch

import oracle
from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa
from gpu_util import check_close, f64

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["tiny"]


def _unperm(xp, perm):
    """[B, H, N, d] permuted -> [B, N, H, d] raster."""
    out = np.empty((xp.shape[0], xp.shape[2], xp.shape[1], xp.shape[3]))
    out[:, perm] = np.transpose(xp, (0, 2, 1, 3))
    return out


@pytest.mark.parametrize("d,grid,n", [(64, (3, 10, 10), 0), (128, (2, 9, 11), 0), (64, (3, 10, 10), 64),
                                      (128, (2, 9, 11), 16)])
def test_autograd_dense_against_oracle(d, grid, n):
    T, Hg, W = grid
    wl = BASE.with_(name="ag", B=1, H=2, d=d, T=T, Hg=Hg, W=W, seed=31 + d + n)
    x = make_inputs(wl, with_dout=True)
    q, k, v = (x[name].cuda().requires_grad_(True) for name in ("q", "k", "v"))
    out = asa.asa_attention_trainable(q, k, v, T, Hg, W, 1.0, global_window=n)
    out.backward(x["dout"].cuda())
    asa.asa_check_device_status()
    perm = oracle.gilbert_order(T, Hg, W)
    ref = {name: oracle.permute(f64(x[name]), perm) for name in ("q", "k", "v", "dout")}
    nb = -(-wl.N // 128)
    mask = np.ones((1, wl.H, nb, nb), dtype=bool)
    O_ref, _ = oracle.asa_forward(ref["q"], ref["k"], ref["v"], mask, global_window=n)
    check_close(f64(out), _unperm(O_ref, perm), what="O")
    dq_d, dkv_d = oracle.asa_backward(ref["q"], ref["k"], ref["v"], ref["dout"], mask,
                                      global_window=n)
    g = {name: np.zeros((1, wl.H, wl.N, d)) for name in ("q", "k", "v")}
    for (bb, h, I), blk in dq_d.items():
        g["q"][bb, h, 128 * I:128 * I + blk.shape[0]] = blk
    for (bb, h, J), (gk, gv) in dkv_d.items():
        g["k"][bb, h, 128 * J:128 * J + gk.shape[0]] = gk
        g["v"][bb, h, 128 * J:128 * J + gv.shape[0]] = gv
    for name, t in (("q", q), ("k", k), ("v", v)):
        check_close(f64(t.grad), _unperm(g[name], perm), what=f"d{name}")


def test_autograd_equals_step_by_step():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, with_dout=True)
    q, k, v = (x[name].cuda().requires_grad_(True) for name in ("q", "k", "v"))
    out = asa.asa_attention_trainable(q, k, v, wl.T, wl.Hg, wl.W, wl.tau)
    out.backward(x["dout"].cuda())
    qp, kp, vp = asa.asa_gilbert_permute3(q.detach(), k.detach(), v.detach(), wl.T, wl.Hg, wl.W)
    m = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    op, lse, o32 = asa.asa_sparse_attn_fwd_train(qp, kp, vp, m)
    dop = asa.asa_gilbert_permute(x["dout"].cuda(), wl.T, wl.Hg, wl.W)
    grads = asa.asa_sparse_attn_bwd_train(qp, kp, vp, o32, dop, lse, m)
    asa.asa_check_device_status()
    assert torch.equal(out.detach(), asa.asa_unpermute(op, wl.T, wl.Hg, wl.W))
    for t, gp in zip((q, k, v), grads):
        assert torch.equal(t.grad, asa.asa_unpermute(gp, wl.T, wl.Hg, wl.W))


def test_autograd_d_from_o_equals_step_by_step():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, with_dout=True)
    q, k, v = (x[name].cuda().requires_grad_(True) for name in ("q", "k", "v"))
    out = asa.asa_attention_trainable(q, k, v, wl.T, wl.Hg, wl.W, wl.tau, d_from_o=True)
    out.backward(x["dout"].cuda())
    qp, kp, vp = asa.asa_gilbert_permute3(q.detach(), k.detach(), v.detach(), wl.T, wl.Hg, wl.W)
    m = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    op, lse = asa.asa_sparse_attn_fwd(qp, kp, vp, m)
    dop = asa.asa_gilbert_permute(x["dout"].cuda(), wl.T, wl.Hg, wl.W)
    grads = asa.asa_sparse_attn_bwd(qp, kp, vp, op, dop, lse, m, d_from_o=True)
    asa.asa_check_device_status()
    for t, gp in zip((q, k, v), grads):
        assert torch.equal(t.grad, asa.asa_unpermute(gp, wl.T, wl.Hg, wl.W))
