"""The largest call the library accepts: N = ASA_MAX_TOKENS = 262,144 tokens (grid
4 x 256 x 256, 2,048 blocks), one head, d = 64, through permute -> estimate + mask ->
forward -> backward, and through the training pair.  Checked on outputs the oracle can
compute one by one: sampled permuted rows, P_imp and mask rows of sampled query blocks
(the oracle computes only those rows; a row that differs must be marginal and a legal
cut), forward rows of those blocks and their dQ under the library's rows, and the
backward's invariants over the whole call."""
import numpy as np
import pytest
import torch

import oracle
from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa
from gpu_util import check_close, compare_masks, f64, mask_from_csr

pytestmark = pytest.mark.gpu

MAX_TOKENS = 262144


def test_max_tokens_end_to_end():
    wl = WORKLOADS["tiny"].with_(name="max", B=1, H=1, d=64, T=4, Hg=256, W=256, seed=41, tau=0.9)
    assert wl.N == MAX_TOKENS
    x = make_inputs(wl, with_dout=True)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    q, k, v, do = (x[name].cuda() for name in ("q", "k", "v", "dout"))
    qp, kp, vp, dop = (asa.asa_gilbert_permute(t, wl.T, wl.Hg, wl.W) for t in (q, k, v, do))
    p_imp = asa.asa_estimate(qp, kp)
    bm = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    o, lse = asa.asa_sparse_attn_fwd(qp, kp, vp, bm)
    dq, dk, dv = asa.asa_sparse_attn_bwd(qp, kp, vp, o, dop, lse, bm)
    o_t, lse_t, o32 = asa.asa_sparse_attn_fwd_train(qp, kp, vp, bm)
    dq_t, dk_t, dv_t = asa.asa_sparse_attn_bwd_train(qp, kp, vp, o32, dop, lse_t, bm)
    torch.cuda.synchronize()
    asa.asa_check_device_status()
    assert torch.equal(asa.asa_unpermute(qp, wl.T, wl.Hg, wl.W), q)
    g = np.random.default_rng(3)
    idx = g.integers(0, wl.N, 4000)
    assert np.array_equal(f64(qp[0, 0, torch.from_numpy(idx)]),
                          f64(q[0, torch.from_numpy(perm[idx]), 0]))
    # P_imp and mask rows of sampled query blocks
    nb = -(-wl.N // 128)
    qh, kh, vh, doh = (oracle.permute(x[name][:, :, 0:1].double().numpy(), perm)
                       for name in ("q", "k", "v", "dout"))
    blocks = sorted(set(g.choice(nb - 1, 3, replace=False).tolist() + [0, nb - 1]))
    pimp_rows = oracle.estimate_pimp(qh, kh, q_blocks=blocks)
    np.testing.assert_allclose(f64(p_imp[:, :, blocks]), pimp_rows, rtol=2e-4, atol=1e-9)
    gm = mask_from_csr(bm)[:, :, blocks]
    mask_rows = oracle.build_mask(pimp_rows, wl.tau)
    marg = oracle.marginal_rows(pimp_rows, wl.tau)
    compare_masks(gm, mask_rows, marg, pimp_rows, wl.tau, what="max size")
    full = np.zeros((1, 1, nb, nb), dtype=bool)
    for I, row in zip(blocks, gm[0, 0]):
        full[0, 0, I] = row
    # forward rows and dQ of the sampled blocks under the library's (legal) rows
    rows = np.concatenate([128 * I + g.choice(min(128, wl.N - 128 * I), 16, replace=False)
                           for I in blocks])
    O_ref, L_ref = oracle.asa_forward(qh, kh, vh, full, q_index=rows)
    check_close(f64(o[0, 0, torch.from_numpy(rows)]), O_ref[0, 0], what="O at max size")
    check_close(f64(o_t[0, 0, torch.from_numpy(rows)]), O_ref[0, 0],
                what="O at max size (training forward)")
    dq_ref, _ = oracle.asa_backward(qh, kh, vh, doh, full, heads=[(0, 0)], q_blocks=blocks,
                                    kv_blocks=[])
    for I in blocks:
        r = slice(128 * I, min(128 * I + 128, wl.N))
        check_close(f64(dq[0, 0, r]), dq_ref[(0, 0, I)], what=f"dQ block {I} at max size")
        check_close(f64(dq_t[0, 0, r]), dq_ref[(0, 0, I)],
                    what=f"dQ block {I} at max size (training pair)")
    assert torch.equal(dv_t.view(torch.int16), dv.view(torch.int16))
    # invariants of the whole backward
    sum_dv, sum_do = dv.double().sum(dim=2), dop.double().sum(dim=2)
    scale = dop.double().abs().sum(dim=2).clamp_min(1.0)
    assert float(((sum_dv - sum_do).abs() / scale).max()) < 2e-2
    kscale = dk.double().abs().sum(dim=2).clamp_min(1.0)
    assert float((dk.double().sum(dim=2).abs() / kscale).max()) < 2e-2


def test_over_max_tokens_rejected():
    assert asa.lib().asa_estimate_mask_workspace_size(1, 1, MAX_TOKENS) > 0
    x = torch.zeros((1, 1, MAX_TOKENS + 128, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(asa.AsaError) as ei:
        asa.asa_estimate(x, x)
    assert ei.value.code == asa.ASA_ERR_UNSUPPORTED


def test_max_tokens_query_pruning():
    """Query pruning at 262,144 tokens (2,048 blocks, r = 0.25, windows of 8, four
    blocks per tile): every block keeps 32 queries; the oracle's decisions for the
    sampled blocks; forward rows of sampled tokens against the oracle (their own row
    or their centre's); the packed backward's invariants, dQ = 0 on pruned rows and dQ
    of sampled blocks against the oracle's pruned backward."""
    wl = WORKLOADS["tiny"].with_(name="max", B=1, H=1, d=64, T=4, Hg=256, W=256, seed=44, tau=0.9)
    x = make_inputs(wl, with_dout=True)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    q, k, v, do = (x[name].cuda() for name in ("q", "k", "v", "dout"))
    qp, kp, vp, dop = (asa.asa_gilbert_permute(t, wl.T, wl.Hg, wl.W) for t in (q, k, v, do))
    bm = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    pr = asa.asa_prune_queries(qp, 0.25, 8)
    assert pr.pack == 4 and pr.Ns == 512 * 128
    tm = asa.asa_prune_mask(bm, pr.pack)
    o, lse = asa.asa_sparse_attn_fwd_pruned(pr, kp, vp, tm)
    dq, dk, dv = asa.asa_sparse_attn_bwd_pruned(pr, kp, vp, dop, lse, tm)
    torch.cuda.synchronize()
    asa.asa_check_device_status()
    nb = -(-wl.N // 128)
    sp = pr.src_pos[0, 0].cpu().numpy()
    kept_g = sp == np.arange(wl.N)
    assert int(kept_g.sum()) == nb * 32
    qh, kh, vh, doh = (oracle.permute(x[name][:, :, 0:1].double().numpy(), perm)
                       for name in ("q", "k", "v", "dout"))
    g = np.random.default_rng(5)
    blocks = sorted(set(g.choice(nb - 1, 3, replace=False).tolist() + [0, nb - 1]))
    # the oracle's pruning of the sampled blocks (no near-ties there for this seed);
    # src_or: each token's source row by the oracle in those blocks, itself elsewhere
    src_or = np.arange(wl.N, dtype=np.int64)
    for I in blocks:
        s = slice(128 * I, 128 * I + 128)
        kb, c, dis = oracle.prune_block(qh[0, 0, s], 0.25, 8)
        assert not oracle.marginal_tokens(kb[None, None], dis[None, None], 8)[0, 0].any()
        np.testing.assert_array_equal(kept_g[s], kb)
        src_or[s] = np.where(kb, np.arange(128), c) + 128 * I
    # forward rows: the mask rows of the sampled blocks from the oracle's estimate
    pimp_rows = oracle.estimate_pimp(qh, kh, q_blocks=blocks)
    gm = mask_from_csr(bm)[:, :, blocks]
    mask_rows = oracle.build_mask(pimp_rows, wl.tau)
    agree = [I for I, dif in zip(blocks, (gm != mask_rows).any(-1)[0, 0]) if not dif]
    assert agree
    full = np.zeros((1, 1, nb, nb), dtype=bool)
    for I, row in zip(blocks, mask_rows[0, 0]):
        full[0, 0, I] = row
    rows = np.concatenate([128 * I + g.choice(128, 16, replace=False) for I in agree])
    O_ref, _ = oracle.asa_forward(qh, kh, vh, full, q_index=src_or[rows])
    check_close(f64(o[0, 0, torch.from_numpy(rows)]), O_ref[0, 0], what="pruned O at max size")
    # backward: pruned rows get no query gradient; gradient conservation as unpruned
    dq_h = f64(dq)[0, 0]
    assert np.all(dq_h[~kept_g] == 0.0)
    sum_dv, sum_do = dv.double().sum(dim=2), dop.double().sum(dim=2)
    scale = dop.double().abs().sum(dim=2).clamp_min(1.0)
    assert float(((sum_dv - sum_do).abs() / scale).max()) < 2e-2
    kscale = dk.double().abs().sum(dim=2).clamp_min(1.0)
    assert float((dk.double().sum(dim=2).abs() / kscale).max()) < 2e-2
    # dQ of a block depends on its own rows' filled gradients only
    dq_ref, _ = oracle.asa_backward_pruned(qh, kh, vh, doh, full, src_or[None, None],
                                           heads=[(0, 0)], q_blocks=agree, kv_blocks=[])
    for I in agree:
        r = slice(128 * I, 128 * I + 128)
        check_close(dq_h[r], dq_ref[(0, 0, I)], what=f"pruned dQ block {I} at max size")
