"""Pins for the oracle's attention (Video-BLADE "Step 2.2: Computation", standard ASA
and ASA_G) and for its backward under a fixed mask.  Library routines that do not
share the oracle's code serve as the independent side: torch's
scaled_dot_product_attention (fp64, CPU), avg_pool1d and autograd."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _rand(B, H, N, d, seed, qk_std=1.2):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, H, N, d)) * qk_std
    k = g.standard_normal((B, H, N, d)) * qk_std
    v = g.standard_normal((B, H, N, d))
    return q, k, v


def _token_mask(block_mask, N, b):
    """Expand a [B, H, nb, nb] block mask to a [B, H, N, N] token mask."""
    tm = np.repeat(np.repeat(block_mask, b, axis=2), b, axis=3)
    return tm[:, :, :N, :N]


def _lse_ref(q, k, bias):
    s = torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) / math.sqrt(q.shape[-1])
    return torch.logsumexp(s + bias, dim=-1).numpy()


def test_tau_one_is_dense_attention():
    B, H, N, d, b = 1, 2, 300, 32, 128
    q, k, v = _rand(B, H, N, d, 1)
    nb = -(-N // b)
    mask = np.ones((B, H, nb, nb), dtype=bool)
    O, L = oracle.asa_forward(q, k, v, mask, b=b)
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(a) for a in (q, k, v)))
    np.testing.assert_allclose(O, ref.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(L, _lse_ref(q, k, 0.0), rtol=1e-12)


@pytest.mark.parametrize("N", [256, 333, 1000])
def test_block_mask_equals_masked_sdpa(N):
    B, H, d, b = 2, 2, 16, 128
    q, k, v = _rand(B, H, N, d, N)
    nb = -(-N // b)
    g = np.random.default_rng(N + 1)
    mask = g.random((B, H, nb, nb)) < 0.45
    mask[..., np.arange(nb), g.integers(0, nb, nb)] = True     # no empty row
    O, L = oracle.asa_forward(q, k, v, mask, b=b)
    tm = torch.from_numpy(_token_mask(mask, N, b))
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(a) for a in (q, k, v)), attn_mask=tm)
    np.testing.assert_allclose(O, ref.numpy(), rtol=1e-10, atol=1e-12)
    bias = torch.where(tm, 0.0, -math.inf).double()
    np.testing.assert_allclose(L, _lse_ref(q, k, bias), rtol=1e-12)
    # a subset of query rows gives the same rows
    sel = [0, 5, N - 1, 128, 129]
    O2, L2 = oracle.asa_forward(q, k, v, mask, b=b, q_index=sel)
    np.testing.assert_allclose(O2, O[:, :, sel], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(L2, L[:, :, sel], rtol=1e-13)


def test_round_to_bf16_matches_torch_and_ties_to_even():
    g = np.random.default_rng(3)
    x = g.standard_normal(10000).astype(np.float32).astype(np.float64) * 7
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(oracle.round_to_bf16(x), ref)
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even significand (1)
    assert oracle.round_to_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert oracle.round_to_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    assert oracle.round_to_bf16(np.array([-(1 + 2 ** -8)]))[0] == -1.0


@pytest.mark.parametrize("N,n", [(1000, 64), (256, 64), (300, 16)])
def test_asa_g_equals_sdpa_over_augmented_keys(N, n):
    """ASA_G: K_aug = Concat(K, MeanPool_n(K)), V likewise; the fine part is masked by
    M and the global part carries a fixed additive ln(n)."""
    B, H, d, b = 1, 2, 16, 128
    q, k, v = _rand(B, H, N, d, N + n)
    # round inputs to bf16 values like the kernels' operands
    q, k, v = (oracle.round_to_bf16(a) for a in (q, k, v))
    nb = -(-N // b)
    g = np.random.default_rng(9)
    mask = g.random((B, H, nb, nb)) < 0.4
    mask[..., np.arange(nb), np.arange(nb)] = True
    O, L = oracle.asa_forward(q, k, v, mask, b=b, global_window=n)

    def pool(x):   # [B, H, N, d] -> [B, H, G, d], ragged last window averaged over its count
        t = torch.from_numpy(x).reshape(B * H, N, d).transpose(1, 2)
        p = F.avg_pool1d(t, kernel_size=n, stride=n, ceil_mode=True)
        p = p.transpose(1, 2).reshape(B, H, -1, d)
        return p.float().bfloat16().double()

    Kg, Vg = pool(k), pool(v)
    G = Kg.shape[2]
    kaug = torch.cat([torch.from_numpy(k), Kg], dim=2)
    vaug = torch.cat([torch.from_numpy(v), Vg], dim=2)
    fine = torch.where(torch.from_numpy(_token_mask(mask, N, b)), 0.0, -math.inf).double()
    glob = torch.full((B, H, N, G), math.log(n), dtype=torch.float64)
    bias = torch.cat([fine, glob], dim=3)
    ref = F.scaled_dot_product_attention(torch.from_numpy(q), kaug, vaug, attn_mask=bias)
    np.testing.assert_allclose(O, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_asa_g_window_one_doubles_kept_keys():
    """n = 1: every token is its own global token and ln(1) = 0, so a kept key counts
    twice and a dropped key once: attention with an additive ln 2 on kept keys."""
    B, H, N, d, b = 1, 1, 384, 16, 128
    q, k, v = (oracle.round_to_bf16(a) for a in _rand(B, H, N, d, 21))
    nb = 3
    mask = np.array([[[[1, 0, 0], [0, 1, 1], [1, 0, 1]]]], dtype=bool)
    O, _ = oracle.asa_forward(q, k, v, mask, b=b, global_window=1)
    bias = torch.from_numpy(np.where(_token_mask(mask, N, b), math.log(2.0), 0.0))
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(a) for a in (q, k, v)), attn_mask=bias)
    np.testing.assert_allclose(O, ref.numpy(), rtol=1e-10, atol=1e-12)


def _full_grads(q, k, v, dout, mask, b, n=0):
    B, H, N, d = q.shape
    nb = mask.shape[2]
    dq_d, dkv_d = oracle.asa_backward(q, k, v, dout, mask, b=b, global_window=n)
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    for (bb, h, I), blk in dq_d.items():
        dq[bb, h, b * I:b * I + blk.shape[0]] = blk
    for (bb, h, J), (gk, gv) in dkv_d.items():
        dk[bb, h, b * J:b * J + gk.shape[0]] = gk
        dv[bb, h, b * J:b * J + gv.shape[0]] = gv
    return dq, dk, dv


@pytest.mark.parametrize("N", [256, 300])
def test_backward_equals_autograd_of_masked_sdpa(N):
    B, H, d, b = 1, 2, 16, 128
    q, k, v = _rand(B, H, N, d, 31 + N)
    dout = np.random.default_rng(5).standard_normal(q.shape)
    nb = -(-N // b)
    mask = np.ones((B, H, nb, nb), dtype=bool)
    mask[0, 0, 0, 1] = False
    mask[0, 1, 1, 0] = False
    dq, dk, dv = _full_grads(q, k, v, dout, mask, b)
    tq, tk, tv = (torch.from_numpy(a).requires_grad_(True) for a in (q, k, v))
    tm = torch.from_numpy(_token_mask(mask, N, b))
    O = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=tm)
    O.backward(torch.from_numpy(dout))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_backward_finite_differences():
    B, H, N, d, b = 1, 1, 200, 8, 128
    q, k, v = _rand(B, H, N, d, 77)
    dout = np.random.default_rng(6).standard_normal(q.shape)
    mask = np.array([[[[1, 0], [1, 1]]]], dtype=bool)
    dq, dk, dv = _full_grads(q, k, v, dout, mask, b)

    def loss(qq, kk, vv):
        O, _ = oracle.asa_forward(qq, kk, vv, mask, b=b)
        return float((O * dout).sum())

    h = 1e-6
    g = np.random.default_rng(8)
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            i, c = int(g.integers(0, N)), int(g.integers(0, d))
            plus, minus = arr.copy(), arr.copy()
            plus[0, 0, i, c] += h
            minus[0, 0, i, c] -= h
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = plus
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = minus
            num = (loss(args_p["q"], args_p["k"], args_p["v"])
                   - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
            assert abs(num - grad[0, 0, i, c]) < 1e-6 * max(1.0, abs(num)), (name, i, c)


@pytest.mark.parametrize("N,n", [(300, 64), (256, 16), (200, 1)])
def test_asa_g_backward_equals_autograd(N, n):
    """ASA_G backward against torch autograd through SDPA over the augmented keys: the
    global tokens are avg_pool1d windows of K and V (ragged last window over its own
    count), rounded to bf16 by a straight-through step (value rounded, gradient
    passed), with the fixed + ln(n) on their logits."""
    B, H, d, b = 1, 2, 16, 128
    q, k, v = (oracle.round_to_bf16(a) for a in _rand(B, H, N, d, 40 + N + n))
    dout = np.random.default_rng(n).standard_normal(q.shape)
    nb = -(-N // b)
    g = np.random.default_rng(N)
    mask = g.random((B, H, nb, nb)) < 0.5
    mask[..., np.arange(nb), np.arange(nb)] = True
    dq, dk, dv = _full_grads(q, k, v, dout, mask, b, n=n)

    tq, tk, tv = (torch.from_numpy(a).requires_grad_(True) for a in (q, k, v))

    def pool(x):
        t = x.reshape(B * H, N, d).transpose(1, 2)
        p = F.avg_pool1d(t, kernel_size=n, stride=n, ceil_mode=True)
        p = p.transpose(1, 2).reshape(B, H, -1, d)
        return p + (p.float().bfloat16().double() - p).detach()

    Kg, Vg = pool(tk), pool(tv)
    G = Kg.shape[2]
    fine = torch.where(torch.from_numpy(_token_mask(mask, N, b)), 0.0, -math.inf).double()
    bias = torch.cat([fine, torch.full((B, H, N, G), math.log(n), dtype=torch.float64)], dim=3)
    O = F.scaled_dot_product_attention(tq, torch.cat([tk, Kg], dim=2), torch.cat([tv, Vg], dim=2),
                                       attn_mask=bias)
    O.backward(torch.from_numpy(dout))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_asa_g_backward_block_selection_matches_full():
    B, H, N, d, b, n = 1, 1, 300, 8, 128, 64
    q, k, v = (oracle.round_to_bf16(a) for a in _rand(B, H, N, d, 93))
    dout = np.random.default_rng(4).standard_normal(q.shape)
    mask = np.array([[[[1, 0, 0], [0, 1, 0], [1, 0, 1]]]], dtype=bool)
    full_q, full_kv = oracle.asa_backward(q, k, v, dout, mask, b=b, global_window=n)
    part_q, part_kv = oracle.asa_backward(q, k, v, dout, mask, b=b, heads=[(0, 0)],
                                          q_blocks=[1], kv_blocks=[1], global_window=n)
    np.testing.assert_allclose(part_q[(0, 0, 1)], full_q[(0, 0, 1)], rtol=1e-13)
    # key block 1 is kept only by query block 1, but every query reaches it through
    # the global tokens
    np.testing.assert_allclose(part_kv[(0, 0, 1)][0], full_kv[(0, 0, 1)][0], rtol=1e-13)
    np.testing.assert_allclose(part_kv[(0, 0, 1)][1], full_kv[(0, 0, 1)][1], rtol=1e-13)
    assert np.abs(full_kv[(0, 0, 1)][1]).max() > 0


def test_backward_block_selection_matches_full():
    B, H, N, d, b = 1, 1, 300, 8, 128
    q, k, v = _rand(B, H, N, d, 91)
    dout = np.random.default_rng(2).standard_normal(q.shape)
    mask = np.array([[[[1, 1, 0], [0, 1, 1], [1, 0, 1]]]], dtype=bool)
    full_q, full_kv = oracle.asa_backward(q, k, v, dout, mask, b=b)
    part_q, part_kv = oracle.asa_backward(q, k, v, dout, mask, b=b, heads=[(0, 0)],
                                          q_blocks=[2], kv_blocks=[0])
    np.testing.assert_allclose(part_q[(0, 0, 2)], full_q[(0, 0, 2)], rtol=1e-13)
    np.testing.assert_allclose(part_kv[(0, 0, 0)][0], full_kv[(0, 0, 0)][0], rtol=1e-13)
    np.testing.assert_allclose(part_kv[(0, 0, 0)][1], full_kv[(0, 0, 0)][1], rtol=1e-13)


def test_permute_round_trip_and_definition():
    g = np.random.default_rng(1)
    T, H_, W = 3, 5, 6
    N = T * H_ * W
    x = g.standard_normal((2, N, 3, 4))
    perm = oracle.gilbert_order(T, H_, W)
    xp = oracle.permute(x, perm)
    for bb in range(2):
        for h in range(3):
            for i in range(N):
                assert (xp[bb, h, i] == x[bb, perm[i], h]).all()
    np.testing.assert_array_equal(oracle.unpermute(xp, perm), x)


def test_attention_flops_dense():
    mask = np.ones((1, 3, 3, 3), dtype=bool)
    assert oracle.attention_flops(mask, 300, 64) == 4 * 64 * 300 * 300 * 3
    assert oracle.attention_flops(mask, 300, 64, global_window=64) == \
        4 * 64 * 300 * 300 * 3 + 4 * 64 * 300 * 5 * 3
