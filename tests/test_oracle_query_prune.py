"""Pins for the oracle's query pruning with token filling ("Bidirectional Sparse
Attention for Faster Video Diffusion Training", "Key designs", item 1, and "A complete
example").  Independent sides: values worked out by hand from known angles, the
page's printed count, torch's cosine_similarity, brute force over subsets, torch SDPA
and autograd (fp64, CPU)."""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _token_mask(block_mask, N, b):
    tm = np.repeat(np.repeat(block_mask, b, axis=2), b, axis=3)
    return tm[:, :, :N, :N]


def _hand_block():
    """8 tokens, windows of 4 (centres at offsets 2 and 6), d = 2."""
    s3 = math.sqrt(3.0)
    q = np.array([
        [0.0, 1.0],     # 0: 90 deg from centre 2      -> 1 - cos = 1
        [1.0, 1.0],     # 1: 45 deg                    -> 1 - 1/sqrt(2)
        [1.0, 0.0],     # 2: centre of window 0
        [-2.0, 0.0],    # 3: opposite                  -> 2
        [1.0, 0.0],     # 4: 90 deg from centre 6      -> 1
        [0.0, -1.0],    # 5: opposite                  -> 2
        [0.0, 3.0],     # 6: centre of window 1
        [s3, 1.0],      # 7: 60 deg                    -> 1/2
    ])
    return q


def test_hand_block_dissimilarities_and_selection():
    q = _hand_block()
    kept, c, dis = oracle.prune_block(q, 0.625, 4)
    np.testing.assert_array_equal(c, [2, 2, 2, 2, 6, 6, 6, 6])
    expect = [1.0, 1.0 - 1.0 / math.sqrt(2.0), 0.0, 2.0, 1.0, 2.0, 0.0, 0.5]
    np.testing.assert_allclose(dis, expect, rtol=0, atol=1e-15)
    # K = ceil(0.625 * 8) = 5: both centres, the two opposite tokens (3, 5), then the
    # tie at 1 - cos = 1 between tokens 0 and 4 goes to the lower position
    np.testing.assert_array_equal(np.nonzero(kept)[0], [0, 2, 3, 5, 6])
    kept, _, _ = oracle.prune_block(q, 0.5, 4)       # K = 4: centres and 3, 5
    np.testing.assert_array_equal(np.nonzero(kept)[0], [2, 3, 5, 6])
    kept, _, _ = oracle.prune_block(q, 0.1, 4)       # ceil(0.8) = 1 < 2 windows: centres
    np.testing.assert_array_equal(np.nonzero(kept)[0], [2, 6])
    # a zero query has cosine 0 to its centre
    q2 = q.copy()
    q2[1] = 0.0
    _, _, dis2 = oracle.prune_block(q2, 0.5, 4)
    assert dis2[1] == 1.0


def test_hand_block_src_and_ragged_windows():
    q = _hand_block()[None, None]        # B = H = 1, N = 8, b = 8
    kept, src, _ = oracle.prune_queries(q, 0.625, 4, b=8)
    np.testing.assert_array_equal(src[0, 0], [0, 2, 2, 3, 6, 5, 6, 6])
    # windows of 3 over 8 tokens: [0,3) centre 1, [3,6) centre 4, [6,8) centre 7
    np.testing.assert_array_equal(oracle.window_centres(8, 3), [1, 1, 1, 4, 4, 4, 7, 7])
    np.testing.assert_array_equal(oracle.window_centres(5, 8), [2, 2, 2, 2, 2])


def test_worked_example_count():
    """The page's example keeps half of 23,296 queries (r = 0.5, 2x2x2 windows):
    11,648.  With 128-token blocks and windows of 8 every block keeps 64."""
    N = 23296
    q = np.random.default_rng(0).standard_normal((1, 1, N, 4))
    kept, _, _ = oracle.prune_queries(q, 0.5, 8)
    assert int(kept.sum()) == 11648


def test_counts_ragged_and_fp32_r():
    q = np.random.default_rng(1).standard_normal((1, 2, 300, 8))
    kept, _, _ = oracle.prune_queries(q, 0.3, 8)
    # blocks of 128, 128, 44: fp32 0.3 * 128 = 38.400001 -> 39; 0.3 * 44 -> 14 (> 6 windows)
    np.testing.assert_array_equal(kept.sum(axis=2), [[92, 92]])
    # fp32 0.1 is a little above 1/10: ceil(0.1f * 10) = 2, not 1
    assert oracle.kept_count(10, 0.1, 10) == 2
    assert oracle.kept_count(128, 0.0, 8) == 16


def test_cosine_matches_torch():
    g = np.random.default_rng(2)
    a = g.standard_normal((500, 64))
    b = g.standard_normal((500, 64)) * 3
    b[7] = 0.0
    ref = F.cosine_similarity(torch.from_numpy(a), torch.from_numpy(b), dim=1, eps=1e-8)
    np.testing.assert_allclose(oracle.cosine(a, b), ref.numpy(), rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_max_dissimilarity(seed):
    """On tiny blocks the kept non-centres are the subset of the required size with
    the largest total dissimilarity (unique for continuous random queries)."""
    g = np.random.default_rng(100 + seed)
    L, w = int(g.integers(5, 11)), int(g.integers(2, 5))
    r = float(g.choice([0.3, 0.5, 0.7]))
    q = g.standard_normal((L, 3))
    kept, c, dis = oracle.prune_block(q, r, w)
    centres = set(c.tolist())
    others = [i for i in range(L) if i not in centres]
    extra = max(math.ceil(float(np.float32(r)) * L), len(centres)) - len(centres)
    best = max(itertools.combinations(others, extra), key=lambda s: sum(dis[list(s)]))
    np.testing.assert_array_equal(np.nonzero(kept)[0], sorted(centres | set(best)))


def test_keep_all_cases_and_parallel_queries():
    g = np.random.default_rng(3)
    q = g.standard_normal((1, 1, 300, 8))
    for r, w in ((1.0, 8), (0.2, 1)):
        kept, src, _ = oracle.prune_queries(q, r, w)
        assert kept.all()
        np.testing.assert_array_equal(src[0, 0], np.arange(300))
    # every query a power-of-two multiple of one unit vector: every cosine is exactly
    # 1, so the block keeps its centres and then the lowest positions
    base = np.zeros(8)
    base[3] = 1.0
    qp = (2.0 ** g.integers(-2, 3, 128))[:, None] * base[None, :]
    kept, c, dis = oracle.prune_block(qp, 0.5, 8)
    np.testing.assert_array_equal(dis, 0.0)
    noncentre = np.setdiff1d(np.arange(128), np.unique(c))
    np.testing.assert_array_equal(np.nonzero(kept)[0], np.union1d(np.unique(c), noncentre[:48]))


def test_random_invariants():
    g = np.random.default_rng(4)
    q = g.standard_normal((2, 2, 333, 16))
    r, w = 0.4, 8
    kept, src, dis = oracle.prune_queries(q, r, w)
    for bb in range(2):
        for h in range(2):
            for I, L in enumerate(oracle.block_sizes(333)):
                s = I * 128
                c = oracle.window_centres(L, w)
                k_ = kept[bb, h, s:s + L]
                assert k_[np.unique(c)].all()
                assert k_.sum() == oracle.kept_count(L, r, w)
                nc = c != np.arange(L)
                d_ = dis[bb, h, s:s + L]
                if (k_ & nc).any() and (~k_ & nc).any():
                    assert d_[k_ & nc].min() >= d_[~k_ & nc].max()
                exp_src = np.where(k_, np.arange(s, s + L), s + c)
                np.testing.assert_array_equal(src[bb, h, s:s + L], exp_src)
    assert not oracle.marginal_tokens(kept, dis, w).any()


def _pruned_case(N, seed, n=0):
    B, H, d, b = 1, 2, 16, 128
    g = np.random.default_rng(seed)
    q, k, v = (oracle.round_to_bf16(g.standard_normal((B, H, N, d)) * s) for s in (1.2, 1.2, 1.0))
    nb = -(-N // b)
    mask = g.random((B, H, nb, nb)) < 0.5
    mask[..., np.arange(nb), np.arange(nb)] = True
    _, src, _ = oracle.prune_queries(q, 0.5, 8)
    return q, k, v, mask, src


@pytest.mark.parametrize("N,n", [(300, 0), (256, 0), (300, 64)])
def test_forward_pruned_equals_gathered_sdpa(N, n):
    q, k, v, mask, src = _pruned_case(N, 50 + N, n)
    O, L = oracle.asa_forward_pruned(q, k, v, mask, src, global_window=n)
    O_full, L_full = oracle.asa_forward(q, k, v, mask, global_window=n)
    if n == 0:
        tm = torch.from_numpy(_token_mask(mask, N, 128))
        ref = F.scaled_dot_product_attention(*(torch.from_numpy(a) for a in (q, k, v)),
                                             attn_mask=tm).numpy()
        np.testing.assert_allclose(O_full, ref, rtol=1e-10, atol=1e-12)
    for bb in range(q.shape[0]):
        for h in range(q.shape[1]):
            np.testing.assert_allclose(O[bb, h], O_full[bb, h, src[bb, h]], rtol=1e-13, atol=1e-15)
            np.testing.assert_allclose(L[bb, h], L_full[bb, h, src[bb, h]], rtol=1e-13)
    # kept rows are untouched by the pruning
    same = src[0, 0] == np.arange(N)
    np.testing.assert_allclose(O[0, 0, same], O_full[0, 0, same], rtol=1e-13, atol=1e-15)


def _grads_dense(d_dict, dkv_dict, shape, b=128):
    dq, dk, dv = (np.zeros(shape) for _ in range(3))
    for (bb, h, I), blk in d_dict.items():
        dq[bb, h, b * I:b * I + blk.shape[0]] = blk
    for (bb, h, J), (gk, gv) in dkv_dict.items():
        dk[bb, h, b * J:b * J + gk.shape[0]] = gk
        dv[bb, h, b * J:b * J + gv.shape[0]] = gv
    return dq, dk, dv


@pytest.mark.parametrize("N,n", [(300, 0), (300, 64)])
def test_backward_pruned_equals_autograd_of_gather(N, n):
    """Autograd through: masked attention (SDPA, with the global tokens for ASA_G),
    then out[i] = O[src[i]]."""
    q, k, v, mask, src = _pruned_case(N, 70 + N, n)
    B, H, _, d = q.shape
    dout = np.random.default_rng(9).standard_normal(q.shape)
    dq, dk, dv = _grads_dense(*oracle.asa_backward_pruned(q, k, v, dout, mask, src,
                                                          global_window=n, bf16=False), q.shape)
    tq, tk, tv = (torch.from_numpy(a).requires_grad_(True) for a in (q, k, v))
    fine = torch.where(torch.from_numpy(_token_mask(mask, N, 128)), 0.0, -math.inf).double()
    if n > 0:
        def pool(x):
            t = x.reshape(B * H, N, d).transpose(1, 2)
            p = F.avg_pool1d(t, kernel_size=n, stride=n, ceil_mode=True)
            p = p.transpose(1, 2).reshape(B, H, -1, d)
            return p + (p.float().bfloat16().double() - p).detach()
        Kg, Vg = pool(tk), pool(tv)
        bias = torch.cat([fine, torch.full((B, H, N, Kg.shape[2]), math.log(n),
                                           dtype=torch.float64)], dim=3)
        O = F.scaled_dot_product_attention(tq, torch.cat([tk, Kg], 2), torch.cat([tv, Vg], 2),
                                           attn_mask=bias)
    else:
        O = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=fine)
    idx = torch.from_numpy(src)[..., None].expand(B, H, N, d)
    out = torch.gather(O, 2, idx)
    out.backward(torch.from_numpy(dout))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-9, atol=1e-11)
    pruned = src != np.arange(N)[None, None]
    assert pruned.any() and np.all(dq[pruned] == 0.0)


def test_filled_dout_sums_and_rounding():
    src = np.array([[[0, 2, 2, 3, 6, 5, 6, 6]]])
    dout = np.arange(8 * 2, dtype=np.float64).reshape(1, 1, 8, 2) / 8
    f = oracle.filled_dout(dout, src)
    np.testing.assert_array_equal(f[0, 0, 2], dout[0, 0, 1] + dout[0, 0, 2])
    np.testing.assert_array_equal(f[0, 0, 6], dout[0, 0, 4] + dout[0, 0, 6] + dout[0, 0, 7])
    np.testing.assert_array_equal(f[0, 0, [1, 4, 7]], 0.0)
    # 1 + 2^-8 + 2^-9 is not a bf16 value: the stored sum is rounded
    d2 = np.zeros((1, 1, 2, 1))
    d2[0, 0, :, 0] = [1.0, 2 ** -8 + 2 ** -9]
    f2 = oracle.filled_dout(d2, np.array([[[0, 0]]]))
    assert f2[0, 0, 0, 0] == 1.0 + 2 ** -7
    assert oracle.filled_dout(d2, np.array([[[0, 0]]]), bf16=False)[0, 0, 0, 0] == 1 + 2 ** -8 + 2 ** -9
