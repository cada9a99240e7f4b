"""GPU parity of query pruning with token filling ("Bidirectional Sparse Attention for
Faster Video Diffusion Training", "Key designs", item 1) against the fp64 oracle,
through the C ABI.

Bars: the keep/prune decision equals the oracle's on every token the oracle does not
mark marginal (a dissimilarity within 1e-5 of its block's cut), with the exact count
per block; the compact layout is checked for validity (kept rows copied bit for bit,
unused rows zero, every pruned token pointing at its centre's row); the packed-tile
CSR equals the union of the blocks' rows bit for bit; outputs and gradients meet the
forward/backward bars (max-abs 2e-2, rel-L2 5e-3, LSE 1e-3) against the oracle's
pruned forward and backward under the oracle's mask."""
import math

import numpy as np
import pytest
import torch

import oracle
from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa
from gpu_util import LSE_ABS, check_close, f64, mask_from_csr, upload_mask

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["tiny"]
CASES = {
    "tiny": BASE,
    "one-ragged-block": BASE.with_(name="r105", B=2, H=3, d=128, T=3, Hg=5, W=7, seed=11),
    "d128-ragged": BASE.with_(name="r495", B=1, H=2, d=128, T=5, Hg=9, W=11, seed=13, tau=0.95),
    "d64-b2": BASE.with_(name="r1200", B=2, H=2, d=64, T=6, Hg=10, W=20, seed=14),
    "multi-tile": BASE.with_(name="r3072", B=1, H=4, d=128, T=8, Hg=16, W=24, seed=15, tau=0.95),
}
_cache = {}


def setup_case(name):
    if name in _cache:
        return _cache[name]
    wl = CASES[name]
    x = make_inputs(wl, with_dout=True)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    ref = {k: oracle.permute(f64(x[k]), perm) for k in ("q", "k", "v", "dout")}
    mask = oracle.build_mask(oracle.estimate_pimp(ref["q"], ref["k"]), wl.tau)
    dev = {k: torch.from_numpy(ref[k]).to(torch.bfloat16).cuda() for k in ("q", "k", "v", "dout")}
    _cache[name] = (wl, x, perm, ref, mask, dev)
    return _cache[name]


def _centres(N, w):
    c = np.zeros(N, dtype=np.int64)
    for I, L in enumerate(oracle.block_sizes(N)):
        c[I * 128:I * 128 + L] = I * 128 + oracle.window_centres(L, w)
    return c


def _check_layout(pr: asa.QueryPrune, qp_dev, N):
    """Compact layout validity: kept rows copied exactly into their block's slot,
    pruned tokens pointing at their centre's row, every other row zero."""
    B, H = qp_dev.shape[:2]
    S = 128 // pr.pack
    src_pos = pr.src_pos.cpu().numpy()
    src_row = pr.src_row.cpu().numpy()
    q = qp_dev.view(torch.int16).cpu().numpy()
    qs = pr.q_s.view(torch.int16).cpu().numpy()
    idx = np.arange(N)
    blk = idx // 128
    lo = (blk // pr.pack) * 128 + (blk % pr.pack) * S
    for bb in range(B):
        for h in range(H):
            sp, sr = src_pos[bb, h], src_row[bb, h]
            kept = sp == idx
            assert ((sr >= lo) & (sr < lo + S)).all(), "row outside its block's slot"
            np.testing.assert_array_equal(sr[~kept], sr[sp[~kept]])
            assert (sp[sp] == sp).all(), "a pruned token points at a pruned token"
            np.testing.assert_array_equal(qs[bb, h, sr[kept]], q[bb, h, idx[kept]])
            assert len(np.unique(sr[kept])) == kept.sum()
            unused = np.setdiff1d(np.arange(pr.Ns), sr[kept])
            assert (qs[bb, h, unused] == 0).all()
            # kept rows of a block fill its slot from the top, in position order
            for I in range(-(-N // 128)):
                rows = sr[(blk == I) & kept]
                np.testing.assert_array_equal(rows, lo[I * 128] + np.arange(len(rows)))


SELECT = [("tiny", 0.5, 8), ("one-ragged-block", 0.5, 8), ("d128-ragged", 0.3, 8),
          ("d64-b2", 0.25, 4), ("multi-tile", 0.5, 8), ("multi-tile", 0.125, 16),
          ("d128-ragged", 1.0, 8), ("tiny", 0.0, 8), ("d64-b2", 0.5, 1), ("tiny", 0.7, 128)]


@pytest.mark.parametrize("name,r,w", SELECT)
def test_prune_selection_matches_oracle(name, r, w):
    wl, x, perm, ref, mask, dev = setup_case(name)
    pr = asa.asa_prune_queries(dev["q"], r, w)
    kept, src, dis = oracle.prune_queries(ref["q"], r, w)
    marg = oracle.marginal_tokens(kept, dis, w)
    sp = pr.src_pos.cpu().numpy()
    g_kept = sp == np.arange(wl.N)
    bad = (g_kept != kept) & ~marg
    assert not bad.any(), f"{int(bad.sum())} non-marginal decisions differ"
    # exact count per block
    nb = -(-wl.N // 128)
    pad = nb * 128 - wl.N
    cnt = lambda k: np.pad(k, ((0, 0), (0, 0), (0, pad))).reshape(wl.B, wl.H, nb, 128).sum(-1)
    np.testing.assert_array_equal(cnt(g_kept), cnt(kept))
    c = _centres(wl.N, w)
    np.testing.assert_array_equal(sp, np.where(g_kept, np.arange(wl.N), c))
    _check_layout(pr, dev["q"], wl.N)
    asa.asa_check_device_status()


@pytest.mark.parametrize("pack", [1, 2, 4])
def test_prune_mask_is_union_with_quarters(pack):
    B, H, N = 2, 3, 11 * 128 - 40
    nb = 11
    g = np.random.default_rng(pack)
    m = g.random((B, H, nb, nb)) < 0.3
    m[..., np.arange(nb), np.arange(nb)] = True
    m[0, 1, 3] = False                       # an empty row
    bm = upload_mask(m, N)
    tm = asa.asa_prune_mask(bm, pack)
    asa.asa_check_device_status()
    ntile = -(-nb // pack)
    qbits = 4 // pack
    exp_ptr, exp_col, exp_q = [0], [], []
    for bb in range(B):
        for h in range(H):
            for t in range(ntile):
                for J in range(nb):
                    q = 0
                    for s in range(pack):
                        I = t * pack + s
                        if I < nb and m[bb, h, I, J]:
                            q |= ((1 << qbits) - 1) << (s * qbits)
                    if q:
                        exp_col.append(J)
                        exp_q.append(q)
                exp_ptr.append(len(exp_col))
    np.testing.assert_array_equal(tm.tile_ptr.cpu().numpy(), exp_ptr)
    n = exp_ptr[-1]
    assert int(tm.nnz.item()) == n
    np.testing.assert_array_equal(tm.tile_col.cpu().numpy()[:n], exp_col)
    np.testing.assert_array_equal(tm.tile_quarters.cpu().numpy()[:n], exp_q)


def _expected_rows(O_full, L_full, src_or, sp_gpu, marg, centres):
    """Oracle rows for each token: the oracle's source row, except marginal tokens,
    where the GPU's valid choice (itself or its centre) selects between two oracle
    rows."""
    B, H, N = src_or.shape
    idx = np.arange(N)
    O = np.empty(O_full.shape)
    L = np.empty(L_full.shape)
    for bb in range(B):
        for h in range(H):
            s = src_or[bb, h].copy()
            m = marg[bb, h]
            assert ((sp_gpu[bb, h, m] == idx[m]) | (sp_gpu[bb, h, m] == centres[m])).all()
            s[m] = sp_gpu[bb, h, m]
            O[bb, h] = O_full[bb, h, s]
            L[bb, h] = L_full[bb, h, s]
    return O, L


def _run_pruned_forward(name, r, w, gw=0, pack=0, with_tiles=False):
    wl, x, perm, ref, mask, dev = setup_case(name)
    pr = asa.asa_prune_queries(dev["q"], r, w, pack=pack)
    bm = upload_mask(mask, wl.N)
    tm = asa.asa_prune_mask(bm, pr.pack)
    o, lse = asa.asa_sparse_attn_fwd_pruned(pr, dev["k"], dev["v"], tm, global_window=gw)
    asa.asa_check_device_status()
    if with_tiles:
        return wl, ref, mask, dev, pr, bm, tm, o, lse
    return wl, ref, mask, dev, pr, bm, o, lse


@pytest.mark.parametrize("name,r,w,gw", [("tiny", 0.5, 8, 0), ("one-ragged-block", 0.5, 8, 0),
                                         ("d128-ragged", 0.3, 8, 0), ("d64-b2", 0.25, 8, 0),
                                         ("multi-tile", 0.5, 8, 0), ("multi-tile", 0.2, 8, 64),
                                         ("d64-b2", 0.5, 8, 64), ("d128-ragged", 0.5, 4, 16)])
def test_forward_pruned_matches_oracle(name, r, w, gw):
    wl, ref, mask, dev, pr, bm, o, lse = _run_pruned_forward(name, r, w, gw)
    kept, src, dis = oracle.prune_queries(ref["q"], r, w)
    marg = oracle.marginal_tokens(kept, dis, w)
    O_full, L_full = oracle.asa_forward(ref["q"], ref["k"], ref["v"], mask, global_window=gw)
    O_exp, L_exp = _expected_rows(O_full, L_full, src, pr.src_pos.cpu().numpy(), marg,
                                  _centres(wl.N, w))
    check_close(f64(o), O_exp, what="O pruned")
    check_close(f64(lse), L_exp, max_abs=LSE_ABS, rel_l2=1e-4, what="LSE pruned")


@pytest.mark.parametrize("name", ["tiny", "d128-ragged", "multi-tile"])
def test_forward_pruned_pack1_equals_unpruned_rows(name):
    """With one block per tile every kept row runs the same key tiles in the same order
    as in the unpruned kernel: its output is bit-identical, and a pruned row is
    bit-identical to its centre's unpruned row."""
    wl, ref, mask, dev, pr, bm, o, lse = _run_pruned_forward(name, 0.5, 8, pack=1)
    o_std, lse_std = asa.asa_sparse_attn_fwd(dev["q"], dev["k"], dev["v"], bm)
    sp = pr.src_pos.long()
    idx = sp[..., None].expand(*sp.shape, o.shape[-1])
    assert torch.equal(o.view(torch.int16), torch.gather(o_std, 2, idx).view(torch.int16))
    assert torch.equal(lse, torch.gather(lse_std, 2, sp))


def test_forward_keep_all_equals_unpruned():
    wl, ref, mask, dev, pr, bm, o, lse = _run_pruned_forward("d64-b2", 1.0, 8)
    assert pr.pack == 1
    o_std, lse_std = asa.asa_sparse_attn_fwd(dev["q"], dev["k"], dev["v"], bm)
    assert torch.equal(o.view(torch.int16), o_std.view(torch.int16))
    assert torch.equal(lse, lse_std)


@pytest.mark.parametrize("name,r,w,gw,pack", [("tiny", 0.5, 8, 0, 0), ("one-ragged-block", 0.5, 8, 0, 0),
                                              ("d128-ragged", 0.3, 8, 0, 0), ("d64-b2", 0.5, 8, 64, 0),
                                              ("multi-tile", 0.2, 8, 0, 4), ("multi-tile", 0.5, 8, 16, 0),
                                              ("d128-ragged", 0.5, 8, 0, 1), ("d64-b2", 1.0, 8, 0, 1)])
def test_backward_pruned_matches_oracle(name, r, w, gw, pack):
    """Packed backward (pack 1, 2, 4; ASA and ASA_G) against the oracle's pruned
    backward; pruned rows get dQ = 0 exactly."""
    wl, ref, mask, dev, pr, bm, tm, o, lse = _run_pruned_forward(name, r, w, gw, pack=pack,
                                                                 with_tiles=True)
    kept, src, dis = oracle.prune_queries(ref["q"], r, w)
    assert not oracle.marginal_tokens(kept, dis, w).any(), "seeded case has a near-tie"
    # a centre collects up to w output gradients: scale dO by 1/8 (exact) on both sides
    dout = ref["dout"] / 8
    dop = torch.from_numpy(dout).to(torch.bfloat16).cuda()
    got = [f64(t) for t in asa.asa_sparse_attn_bwd_pruned(pr, dev["k"], dev["v"], dop, lse, tm,
                                                            global_window=gw)]
    asa.asa_check_device_status()
    dq_d, dkv_d = oracle.asa_backward_pruned(ref["q"], ref["k"], ref["v"], dout, mask, src,
                                             global_window=gw)
    exp = [np.zeros(got[0].shape) for _ in range(3)]
    for (bb, h, I), blk in dq_d.items():
        exp[0][bb, h, 128 * I:128 * I + blk.shape[0]] = blk
    for (bb, h, J), (gk, gv) in dkv_d.items():
        exp[1][bb, h, 128 * J:128 * J + gk.shape[0]] = gk
        exp[2][bb, h, 128 * J:128 * J + gv.shape[0]] = gv
    check_close(got[0], exp[0], what="dQ pruned")
    check_close(got[1], exp[1], what="dK pruned")
    check_close(got[2], exp[2], what="dV pruned")
    assert np.all(got[0][~kept] == 0.0)


@pytest.mark.parametrize("name", ["tiny", "multi-tile"])
def test_attention_query_keep_end_to_end(name):
    wl, x, perm, ref, mask, dev = setup_case(name)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    out, lse, bm = asa.asa_attention(q, k, v, wl.T, wl.Hg, wl.W, wl.tau, query_keep=0.5)
    gm = mask_from_csr(bm)
    marg = oracle.marginal_rows(oracle.estimate_pimp(ref["q"], ref["k"]), wl.tau)
    assert not ((gm != mask) & ~marg[..., None]).any()
    kept, src, dis = oracle.prune_queries(ref["q"], 0.5, 8)
    assert not oracle.marginal_tokens(kept, dis, 8).any()
    O_ref, _ = oracle.asa_forward_pruned(ref["q"], ref["k"], ref["v"], mask, src)
    agree = ~(gm != mask).any(axis=-1)
    got = f64(out)
    for bb in range(wl.B):
        for h in range(wl.H):
            # a token's output comes from its own block's row of the mask
            rows = np.nonzero(np.repeat(agree[bb, h], 128)[:wl.N])[0]
            check_close(got[bb, perm[rows], h], O_ref[bb, h, rows], what="O end-to-end pruned")
    asa.asa_check_device_status()


def test_trainable_query_keep_gradients():
    """The differentiable op with query pruning; tau = 1 keeps every block, so the
    oracle's mask needs nothing from the CUDA path."""
    wl = BASE.with_(name="agp", B=1, H=2, d=128, T=2, Hg=9, W=11, seed=41)
    x = make_inputs(wl, with_dout=True)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    ref = {n: oracle.permute(f64(x[n]), perm) for n in ("q", "k", "v", "dout")}
    q, k, v = (x[n].cuda().requires_grad_(True) for n in ("q", "k", "v"))
    out = asa.asa_attention_trainable(q, k, v, wl.T, wl.Hg, wl.W, 1.0, query_keep=0.5)
    out.backward(x["dout"].cuda() / 8)
    asa.asa_check_device_status()
    kept, src, dis = oracle.prune_queries(ref["q"], 0.5, 8)
    assert not oracle.marginal_tokens(kept, dis, 8).any()
    nb = -(-wl.N // 128)
    mask = np.ones((1, wl.H, nb, nb), dtype=bool)
    O_ref, _ = oracle.asa_forward_pruned(ref["q"], ref["k"], ref["v"], mask, src)
    check_close(oracle.permute(f64(out), perm), O_ref, what="O trainable pruned")
    dq_d, dkv_d = oracle.asa_backward_pruned(ref["q"], ref["k"], ref["v"], ref["dout"] / 8, mask, src)
    exp = [np.zeros(ref["q"].shape) for _ in range(3)]
    for (bb, h, I), blk in dq_d.items():
        exp[0][bb, h, 128 * I:128 * I + blk.shape[0]] = blk
    for (bb, h, J), (gk, gv) in dkv_d.items():
        exp[1][bb, h, 128 * J:128 * J + gk.shape[0]] = gk
        exp[2][bb, h, 128 * J:128 * J + gv.shape[0]] = gv
    for t, e, nm in zip((q, k, v), exp, ("dQ", "dK", "dV")):
        check_close(oracle.permute(f64(t.grad), perm), e, what=nm + " trainable pruned")


def test_single_token_grid_pruned():
    wl = BASE.with_(name="one", B=1, H=2, d=64, T=1, Hg=1, W=1, seed=21)
    x = make_inputs(wl)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    out, lse, bm = asa.asa_attention(q, k, v, 1, 1, 1, 0.9, query_keep=0.5)
    torch.testing.assert_close(out.float(), v.float(), rtol=0, atol=1e-2)
    ref_lse = (f64(q) * f64(k)).sum(-1)[0, 0] / math.sqrt(64)
    np.testing.assert_allclose(f64(lse)[0, :, 0], ref_lse, atol=LSE_ABS)


def test_bad_indices_are_reported():
    wl, ref, mask, dev, pr, bm, o, lse = _run_pruned_forward("tiny", 0.5, 8)
    bad = asa.QueryPrune(pr.q_s, pr.src_pos, pr.src_row.clone(), pr.pack, pr.r, pr.window, pr.N)
    bad.src_row[0, 0, 5] = pr.Ns + 7
    tm = asa.asa_prune_mask(bm, pr.pack)
    o2, lse2 = asa.asa_sparse_attn_fwd_pruned(bad, dev["k"], dev["v"], tm)
    with pytest.raises(asa.AsaError) as e:
        asa.asa_check_device_status()
    assert e.value.code == asa.ASA_ERR_INVALID_ARG
    assert torch.all(o2[0, 0, 5] == 0) and lse2[0, 0, 5].item() == -math.inf
    # a src_pos pointing outside its block
    bad2 = asa.QueryPrune(pr.q_s, pr.src_pos.clone(), pr.src_row, pr.pack, pr.r, pr.window, pr.N)
    bad2.src_pos[0, 0, 3] = 700
    asa.asa_sparse_attn_bwd_pruned(bad2, dev["k"], dev["v"], dev["dout"], lse, tm)
    with pytest.raises(asa.AsaError) as e:
        asa.asa_check_device_status()
    assert e.value.code == asa.ASA_ERR_INVALID_ARG
    asa.asa_check_device_status()


@pytest.mark.parametrize("name", ["d64-b2", "d128-ragged"])
def test_backward_keep_all_equals_unpruned(name):
    """r = 1 keeps every query: the compact layout is the permuted one, every quarter
    bit is set and the transposed tile CSR lists the same query blocks in the same
    order, so the packed backward computes exactly the unpruned backward."""
    wl, ref, mask, dev, pr, bm, tm, o, lse = _run_pruned_forward(name, 1.0, 8, with_tiles=True)
    assert pr.pack == 1
    got = asa.asa_sparse_attn_bwd_pruned(pr, dev["k"], dev["v"], dev["dout"], lse, tm)
    o_std, lse_std = asa.asa_sparse_attn_fwd(dev["q"], dev["k"], dev["v"], bm)
    std = asa.asa_sparse_attn_bwd(dev["q"], dev["k"], dev["v"], o_std, dev["dout"], lse_std, bm)
    asa.asa_check_device_status()
    for g, e, nm in zip(got, std, ("dQ", "dK", "dV")):
        assert torch.equal(g.view(torch.int16), e.view(torch.int16)), nm
