"""GPU parity at the full workload sizes, in the launch configuration bench.py times
(all heads of the call in one launch), checked on outputs the fp64 oracle can compute
one by one and on properties that hold at any size:

* permutation: sampled rows bit-exact; unpermute(permute(x)) == x;
* block importance and mask: two sampled heads against the oracle.  The mask kernel
  alone, given the oracle's P_imp in fp32, reproduces the oracle's cut on every row;
  through the library's estimate, rows differ only where the oracle marks them
  marginal and each is a legal cut of the oracle's P_imp (counts reported);
* forward (ASA and ASA_G): sampled query rows of those heads against the oracle run
  with the library's mask (the oracle's, except on the legal marginal rows);
* backward (Wan-14B shape): dQ of sampled query blocks, dK/dV of the sampled head's
  least-shared key block, and the invariants sum_j dV_j = sum_i dO_i and
  sum_j dK_j = 0 per head (rows of P sum to one; rows of dS sum to zero)."""
import math

import numpy as np
import pytest
import torch

import oracle
from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa
from gpu_util import LSE_ABS, check_close, compare_masks, f64, mask_from_csr, upload_mask
from test_gpu_parity import kernel_only_mask

pytestmark = pytest.mark.gpu

FULL = ["wan2.1-1.3b", "cogvideox-5b", "wan2.1-1.3b-asag", "wan-14b-720p"]


def _run(wl, x):
    """The call: permute Q,K,V -> estimate+mask -> forward -> unpermute, and the bench's
    forward that stores O straight to raster order (which must equal it bit for bit)."""
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    qp, kp, vp = asa.asa_gilbert_permute3(q, k, v, wl.T, wl.Hg, wl.W)
    p_imp = asa.asa_estimate(qp, kp)
    bm = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    op, lse = asa.asa_sparse_attn_fwd(qp, kp, vp, bm, global_window=wl.global_window)
    out = asa.asa_unpermute(op, wl.T, wl.Hg, wl.W)
    out_r, lse_r = asa.asa_sparse_attn_fwd_raster(qp, kp, vp, bm, wl.T, wl.Hg, wl.W,
                                                  global_window=wl.global_window)
    torch.cuda.synchronize()
    asa.asa_check_device_status()
    assert torch.equal(out_r, out)
    assert torch.equal(lse_r, lse)
    del out_r, lse_r
    return dict(q=q, k=k, v=v, qp=qp, kp=kp, vp=vp, p_imp=p_imp, bm=bm, op=op, lse=lse, out=out)


def _head(x, name, perm, h):
    """Oracle-permuted rows of one head: [1, 1, N, d] float64."""
    return oracle.permute(x[name][:, :, h:h + 1].double().numpy(), perm)


@pytest.mark.parametrize("name", FULL)
def test_full_size_forward_path(name):
    wl = WORKLOADS[name]
    x = make_inputs(wl, with_dout=False)
    r = _run(wl, x)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    g = np.random.default_rng(7)
    # permutation: sampled rows bit-exact, and the round trip
    hs = g.integers(0, wl.H, 2000)
    iis = g.integers(0, wl.N, 2000)
    got = f64(r["qp"][0, torch.from_numpy(hs), torch.from_numpy(iis)])
    exp = x["q"][0, torch.from_numpy(perm[iis]), torch.from_numpy(hs)].double().numpy()
    assert np.array_equal(got, exp)
    assert torch.equal(asa.asa_unpermute(r["qp"], wl.T, wl.Hg, wl.W), r["q"])
    gm = mask_from_csr(r["bm"])
    nb = gm.shape[-1]
    for h in sorted(set([0, wl.H - 1])):
        qh, kh, vh = (_head(x, n, perm, h) for n in ("q", "k", "v"))
        pimp = oracle.estimate_pimp(qh, kh)
        np.testing.assert_allclose(f64(r["p_imp"][:, h:h + 1]), pimp, rtol=2e-4, atol=1e-9)
        mask = oracle.build_mask(pimp, wl.tau)
        marg = oracle.marginal_rows(pimp, wl.tau)
        kernel_only_mask(pimp, wl.N, wl.tau, f"{name} head {h}")
        gm_h = gm[:, h:h + 1]
        compare_masks(gm_h, mask, marg, pimp, wl.tau, what=f"{name} head {h}")
        differ = (gm_h != mask).any(-1)
        # sampled query rows: blocks whose row agrees, every block whose row differs (at
        # most 8), and the ragged last block
        same = np.nonzero(~differ[0, 0])[0]
        pick = np.unique(np.concatenate([g.choice(same, size=min(6, len(same)), replace=False),
                                         np.nonzero(differ[0, 0])[0][:8], [nb - 1]]))
        rows = np.concatenate([128 * I + g.choice(min(128, wl.N - 128 * I), size=min(24, wl.N - 128 * I),
                                                  replace=False) for I in pick])
        O_ref, L_ref = oracle.asa_forward(qh, kh, vh, gm_h, global_window=wl.global_window,
                                          q_index=rows)
        check_close(f64(r["op"][0, h, torch.from_numpy(rows)]), O_ref[0, 0], what=f"{name} O h{h}")
        check_close(f64(r["lse"][0, h, torch.from_numpy(rows)]), L_ref[0, 0], max_abs=LSE_ABS,
                    rel_l2=1e-4, what=f"{name} LSE h{h}")
        # the raster output holds the same rows
        check_close(f64(r["out"][0, torch.from_numpy(perm[rows]), h]), O_ref[0, 0],
                    what=f"{name} raster O h{h}")
    assert int(r["bm"].nnz.item()) == int(gm.sum())
    assert gm.sum(-1).min() >= 1


@pytest.mark.parametrize("pair", ["exact", "training"])
def test_full_size_backward_wan14b(pair):
    """The backward at the Wan-14B shape: the exact one (D pass) and the training pair
    (the training forward's fp32 O gives D)."""
    wl = WORKLOADS["wan-14b-720p"]
    x = make_inputs(wl, with_dout=True)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "dout"))
    qp, kp, vp, dop = (asa.asa_gilbert_permute(t, wl.T, wl.Hg, wl.W) for t in (q, k, v, do))
    # the oracle's mask for the sampled head, the library's own for the others
    h = 5
    qh, kh, vh, doh = (_head(x, n, perm, h) for n in ("q", "k", "v", "dout"))
    pimp = oracle.estimate_pimp(qh, kh)
    mask_h = oracle.build_mask(pimp, wl.tau)
    bm_gpu = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    full = mask_from_csr(bm_gpu)
    full[:, h] = mask_h[:, 0]
    bm = upload_mask(full, wl.N)
    if pair == "exact":
        o, lse = asa.asa_sparse_attn_fwd(qp, kp, vp, bm)
        dq, dk, dv = asa.asa_sparse_attn_bwd(qp, kp, vp, o, dop, lse, bm)
    else:
        o, lse, o32 = asa.asa_sparse_attn_fwd_train(qp, kp, vp, bm)
        dq, dk, dv = asa.asa_sparse_attn_bwd_train(qp, kp, vp, o32, dop, lse, bm)
    torch.cuda.synchronize()
    asa.asa_check_device_status()
    # invariants at full size, every head
    sum_dv = dv.double().sum(dim=2)
    sum_do = dop.double().sum(dim=2)
    scale = dop.double().abs().sum(dim=2).clamp_min(1.0)
    assert float(((sum_dv - sum_do).abs() / scale).max()) < 2e-2
    sum_dk = dk.double().sum(dim=2)
    kscale = dk.double().abs().sum(dim=2).clamp_min(1.0)
    assert float((sum_dk.abs() / kscale).max()) < 2e-2
    # sampled blocks of head h against the oracle
    g = np.random.default_rng(11)
    nb = mask_h.shape[-1]
    q_blocks = sorted(set(g.choice(nb - 1, 3, replace=False).tolist() + [nb - 1]))
    counts = mask_h[0, 0].sum(axis=0)
    J = int(np.argmin(np.where(counts > 0, counts, 10 ** 9)))
    dq_ref, dkv_ref = oracle.asa_backward(qh, kh, vh, doh, mask_h, heads=[(0, 0)],
                                          q_blocks=q_blocks, kv_blocks=[J])
    for I in q_blocks:
        rows = slice(128 * I, min(128 * I + 128, wl.N))
        check_close(f64(dq[0, h, rows]), dq_ref[(0, 0, I)], what=f"{pair} dQ block {I}")
    rows = slice(128 * J, min(128 * J + 128, wl.N))
    check_close(f64(dk[0, h, rows]), dkv_ref[(0, 0, J)][0], what=f"{pair} dK block {J}")
    check_close(f64(dv[0, h, rows]), dkv_ref[(0, 0, J)][1], what=f"{pair} dV block {J}")


def test_full_size_backward_asa_g_wan():
    """ASA_G backward at the Wan2.1-1.3B shape (n = 64), the bench's launch: the
    invariants sum_j dV_j = sum_i dO_i and sum_j dK_j = 0 per head (rows of P over fine
    and global keys sum to one and a window's rows share its token's gradient equally;
    rows of dS sum to zero), and dQ of sampled query blocks of one head against the
    oracle (a query block's dQ needs only its own row of the mask)."""
    wl = WORKLOADS["wan2.1-1.3b-asag"]
    n = wl.global_window
    x = make_inputs(wl, with_dout=True)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    q, k, v, do = (x[name].cuda() for name in ("q", "k", "v", "dout"))
    qp, kp, vp, dop = (asa.asa_gilbert_permute(t, wl.T, wl.Hg, wl.W) for t in (q, k, v, do))
    h = 3
    qh, kh, vh, doh = (_head(x, name, perm, h) for name in ("q", "k", "v", "dout"))
    mask_h = oracle.build_mask(oracle.estimate_pimp(qh, kh), wl.tau)
    full = mask_from_csr(asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True))
    full[:, h] = mask_h[:, 0]
    bm = upload_mask(full, wl.N)
    o, lse = asa.asa_sparse_attn_fwd(qp, kp, vp, bm, global_window=n)
    dq, dk, dv = asa.asa_sparse_attn_bwd(qp, kp, vp, o, dop, lse, bm, global_window=n)
    torch.cuda.synchronize()
    asa.asa_check_device_status()
    sum_dv = dv.double().sum(dim=2)
    sum_do = dop.double().sum(dim=2)
    scale = dop.double().abs().sum(dim=2).clamp_min(1.0)
    assert float(((sum_dv - sum_do).abs() / scale).max()) < 2e-2
    kscale = dk.double().abs().sum(dim=2).clamp_min(1.0)
    assert float((dk.double().sum(dim=2).abs() / kscale).max()) < 2e-2
    g = np.random.default_rng(13)
    nb = mask_h.shape[-1]
    q_blocks = sorted(set(g.choice(nb - 1, 3, replace=False).tolist() + [nb - 1]))
    dq_ref, _ = oracle.asa_backward(qh, kh, vh, doh, mask_h, heads=[(0, 0)], q_blocks=q_blocks,
                                    kv_blocks=[], global_window=n)
    for I in q_blocks:
        rows = slice(128 * I, min(128 * I + 128, wl.N))
        check_close(f64(dq[0, h, rows]), dq_ref[(0, 0, I)], what=f"ASA_G dQ block {I}")

