"""Pins for blocking, sampling, block-importance estimation (Video-BLADE "Step 1")
and the threshold mask ("Step 2.1")."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- blocking / sampling

@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 1024, 17550, 32760, 75600])
def test_block_sizes(N):
    L = oracle.block_sizes(N)
    assert sum(L) == N and len(L) == -(-N // 128)
    assert all(x == 128 for x in L[:-1]) and 1 <= L[-1] <= 128


def test_sample_offsets_known_values():
    assert oracle.sample_offsets(128) == list(range(0, 128, 8))
    assert oracle.sample_offsets(120) == [math.floor(7.5 * j) for j in range(16)]
    assert oracle.sample_offsets(14) == list(range(14))      # fewer tokens than k
    assert oracle.sample_offsets(16) == list(range(16))
    for L in range(1, 129):
        s = oracle.sample_offsets(L)
        assert len(s) == min(16, L) and s[0] == 0 and s[-1] < L
        assert all(a < b for a, b in zip(s, s[1:]))


def test_sample_rows_counts():
    # Wan-1.3B: 256 blocks of 16 samples; CogVideoX: last block holds 14 < k tokens
    assert len(oracle.sample_rows(32760)) == 4096
    assert len(oracle.sample_rows(17550)) == 16 * 137 + 14
    assert len(oracle.sample_rows(75600)) == 16 * 591


# ---------------------------------------------------------------- estimation

def _rand_qk(B, H, N, d, seed, std=1.0):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, H, N, d)) * std
    k = g.standard_normal((B, H, N, d)) * std
    return q, k


@pytest.mark.parametrize("N", [256, 300, 77])
def test_k_equal_b_is_maxpool_of_exact_attention_map(N):
    """With every token sampled, P_imp is the b x b max-pool of the dense softmax map.
    The dense map comes from torch's SDPA with V = identity (its own scaling and
    softmax), and the pooling from torch's max_pool2d (ceil mode for the ragged
    block)."""
    B, H, d, b = 1, 2, 32, 64
    q, k = _rand_qk(B, H, N, d, seed=N, std=1.5)
    pimp = oracle.estimate_pimp(q, k, b=b, k=b)
    eye = torch.eye(N, dtype=torch.float64).expand(B, H, N, N)
    P = F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k), eye)
    ref = F.max_pool2d(P, kernel_size=b, stride=b, ceil_mode=True)
    np.testing.assert_allclose(pimp, ref.numpy(), rtol=1e-12, atol=1e-15)


def test_one_sample_per_block_rows_sum_to_one():
    # k = 1: P_approx is nb x nb, so P_imp = P_approx and every row is a distribution
    q, k = _rand_qk(2, 3, 1000, 16, seed=7)
    pimp = oracle.estimate_pimp(q, k, b=128, k=1)
    np.testing.assert_allclose(pimp.sum(-1), 1.0, rtol=1e-12)


def test_k_equal_b_invariant_to_in_block_shuffles():
    N, d, b = 384, 16, 128
    q, k = _rand_qk(1, 1, N, d, seed=3)
    g = np.random.default_rng(4)
    perm = np.concatenate([b * I + g.permutation(b) for I in range(N // b)])
    a = oracle.estimate_pimp(q, k, b=b, k=b)
    c = oracle.estimate_pimp(q[:, :, perm], k[:, :, perm], b=b, k=b)
    np.testing.assert_allclose(a, c, rtol=1e-12)


def test_sampled_estimate_uses_only_sampled_rows():
    # changing an unsampled token of Q or K leaves P_imp unchanged; a sampled one does not
    N, d = 300, 16
    q, k = _rand_qk(1, 1, N, d, seed=5)
    base = oracle.estimate_pimp(q, k)
    q2 = q.copy(); q2[0, 0, 1] += 5.0            # offset 1 of block 0 is not sampled
    np.testing.assert_array_equal(oracle.estimate_pimp(q2, k), base)
    k2 = k.copy(); k2[0, 0, 128 + 8] += 5.0      # offset 8 of block 1 is sampled
    assert not np.allclose(oracle.estimate_pimp(q, k2), base)


# ---------------------------------------------------------------- mask

def _brute_force_cut(row, tau):
    share = row / row.sum()
    nb = len(row)
    for c in range(1, nb + 1):
        best = None
        for sub in itertools.combinations(range(nb), c):
            s = share[list(sub)].sum()
            if best is None or s > best[0] + 1e-15:
                best = (s, sub)
        if best[0] >= tau:
            return c, best
    return nb, None


def test_mask_minimal_by_brute_force():
    g = np.random.default_rng(11)
    rows = g.random((40, 8)) ** 3 + 1e-3
    for tau in [0.5, 0.8, 0.9, 0.95, 0.99]:
        m = oracle.build_mask(rows[None, None, :, :], tau)[0, 0]
        for r in range(rows.shape[0]):
            c, (best_share, best_set) = _brute_force_cut(rows[r], tau)
            kept = np.nonzero(m[r])[0]
            assert len(kept) == c
            share = rows[r] / rows[r].sum()
            assert abs(share[kept].sum() - best_share) < 1e-12
            # no smaller subset reaches tau
            assert max(share[list(s)].sum()
                       for s in itertools.combinations(range(8), c - 1)) < tau if c > 1 else True


def test_mask_golden_rows():
    with open(os.path.join(GOLDEN, "mask_rows.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        row = np.asarray(case["p_imp"], dtype=np.float64)
        sq = np.tile(row, (len(row), 1))[None, None]       # square P_imp, equal rows
        m = oracle.build_mask(sq, case["tau"])[0, 0]
        for r in range(len(row)):
            assert np.nonzero(m[r])[0].tolist() == case["kept"], case["why"]


def test_mask_limits_and_monotone():
    g = np.random.default_rng(12)
    pimp = g.random((1, 2, 16, 16)) ** 2 + 1e-4
    tiny = oracle.build_mask(pimp, 1e-12)
    assert (tiny.sum(-1) == 1).all()
    assert (np.argmax(tiny, -1) == np.argmax(pimp, -1)).all()
    assert oracle.build_mask(pimp, 1.0).all()
    assert oracle.build_mask(pimp, 1.7).all()
    prev = None
    for tau in np.linspace(0.05, 0.999, 30):
        m = oracle.build_mask(pimp, tau)
        if prev is not None:
            assert (m | prev == m).all()          # kept sets are nested
        prev = m


def test_csr_round_trip():
    g = np.random.default_rng(13)
    mask = g.random((2, 3, 5, 5)) < 0.4
    rp, ci = oracle.mask_to_csr(mask)
    back = np.zeros_like(mask).reshape(-1, 5)
    for r in range(back.shape[0]):
        cols = ci[rp[r]:rp[r + 1]]
        assert (np.diff(cols) > 0).all()
        back[r, cols] = True
    assert (back.reshape(mask.shape) == mask).all()
    tp, ti = oracle.mask_to_csr_transposed(mask)
    assert tp[-1] == rp[-1]
    for bh in range(6):
        for J in range(5):
            r = bh * 5 + J
            rows = ti[tp[r]:tp[r + 1]]
            assert rows.tolist() == np.nonzero(mask.reshape(6, 5, 5)[bh, :, J])[0].tolist()


def test_estimate_pimp_block_selection_matches_full():
    """Selecting query blocks only picks rows: each P_imp row needs only its own block's
    sample rows (ragged last block and a block shorter than k included)."""
    g = np.random.default_rng(17)
    N, d = 128 * 5 + 9, 16
    q = g.standard_normal((2, 2, N, d))
    k = g.standard_normal((2, 2, N, d))
    full = oracle.estimate_pimp(q, k)
    sel = [4, 0, 5, 2]
    part = oracle.estimate_pimp(q, k, q_blocks=sel)
    assert part.shape == (2, 2, len(sel), full.shape[-1])
    np.testing.assert_allclose(part, full[:, :, sel], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- statistical threshold

def test_stat_mask_median_quantile_keeps_shares_above_mean():
    """k = n/2: U(1/2) = 0, so the threshold is the mean share 1/n exactly."""
    row = np.array([5.0, 1.0, 1.0, 3.0, 0.5, 2.0, 2.5, 1.0])   # mean 2.0 -> shares >= 1/8
    m = oracle.build_mask_stat(row[None, None, None, :], 4)
    assert m[0, 0, 0].tolist() == [True, False, False, True, False, True, True, False]


def test_stat_mask_keeps_about_k_of_n_for_normal_shares():
    """Shares drawn from a normal distribution: about k of n blocks lie above
    mean + std U(1 - k/n).  A flipped quantile (U(k/n)) would keep n - k."""
    g = np.random.default_rng(5)
    n, k, rows = 2000, 200, 40
    p = 10.0 + g.standard_normal((1, 1, rows, n))
    kept = oracle.build_mask_stat(p, k).sum(-1)
    assert abs(kept.mean() - k) < 15
    assert kept.min() > 140 and kept.max() < 260


def test_stat_mask_fallback_and_keep_all():
    # every share equal except one slightly lower: the threshold sits above the equal
    # ones, so none passes and the largest share (lowest J) is kept
    row = np.full(1000, 1.0)
    row[7] = 0.9
    m = oracle.build_mask_stat(row[None, None, None, :], 1)
    assert m.sum() == 1 and m[0, 0, 0, 0]
    assert oracle.build_mask_stat(row[None, None, None, :], 1000).all()
    assert oracle.build_mask_stat(row[None, None, None, :], 5000).all()


def test_stat_mask_quantile_matches_table_values():
    """The threshold uses the standard normal quantile: U(0.75) = 0.674490 (table)."""
    n, k = 40, 10                     # 1 - k/n = 0.75
    R = np.linspace(1.0, 2.0, n)
    m = oracle.build_mask_stat(R[None, None, None, :], k)
    s = R / R.sum()
    want = s >= s.mean() + s.std() * 0.674490
    assert 0 < want.sum() < n
    assert m[0, 0, 0].tolist() == want.tolist()


# ---------------------------------------------------------------- marginal / legal rows

def _fixture():
    with open(os.path.join(GOLDEN, "marginal_rows.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _fixture()["marginal"], ids=lambda c: c["why"][:40])
def test_marginal_rows_hand_built(case):
    row = np.asarray(case["p_imp"], dtype=np.float64)
    got = oracle.marginal_rows(row[None, None, None, :], case["tau"])
    assert bool(got[0, 0, 0]) is case["marginal"], case["why"]


@pytest.mark.parametrize("case", _fixture()["marginal_stat"], ids=lambda c: c["why"][:40])
def test_marginal_rows_stat_hand_built(case):
    row = np.asarray(case["p_imp"], dtype=np.float64)
    got = oracle.marginal_rows_stat(row[None, None, None, :], case["k"])
    assert bool(got[0, 0, 0]) is case["marginal"], case["why"]


def test_marginal_rows_stat_fallback_row_keeps_lowest_maximum():
    # the tied fallback row of the fixture keeps J0, the lowest of the equal maxima
    m = oracle.build_mask_stat(np.asarray([0.3, 0.3, 0.3, 0.1])[None, None, None, :], 1)
    assert np.nonzero(m[0, 0, 0])[0].tolist() == [0]


@pytest.mark.parametrize("case", _fixture()["legal"], ids=lambda c: c["why"][:40])
def test_legal_mask_rows_hand_built(case):
    row = np.asarray(case["p_imp"], dtype=np.float64)
    S = np.zeros(len(row), dtype=bool)
    S[case["kept"]] = True
    got = oracle.legal_mask_rows(row[None, None, None, :], S[None, None, None, :], case["tau"])
    assert bool(got[0, 0, 0]) is case["legal"], case["why"]


def test_legal_mask_rows_accepts_exact_cut_and_rejects_perturbed_sets():
    """The exact cut is legal on every row; dropping its largest block, or adding the
    largest dropped block when that block is far from a tie and the cut is far from tau,
    is not."""
    g = np.random.default_rng(21)
    pimp = g.random((1, 2, 24, 24)) ** 4 + 1e-4
    for tau in (0.5, 0.8, 0.95):
        m = oracle.build_mask(pimp, tau)
        assert oracle.legal_mask_rows(pimp, m, tau).all()
        marg = oracle.marginal_rows(pimp, tau)
        for h in range(2):
            for I in range(24):
                share = pimp[0, h, I] / pimp[0, h, I].sum()
                bad = m[0, h, I].copy()
                bad[int(np.argmax(share))] = False
                if bad.any():
                    assert not oracle.legal_mask_rows(pimp[:, h:h + 1, I:I + 1],
                                                      bad[None, None, None], tau)[0, 0, 0]
                if not marg[0, h, I] and (~m[0, h, I]).any():
                    extra = m[0, h, I].copy()
                    extra[int(np.argmax(np.where(m[0, h, I], -1.0, share)))] = True
                    cum = share[m[0, h, I]].sum()
                    if cum - tau > 1e-3:
                        assert not oracle.legal_mask_rows(pimp[:, h:h + 1, I:I + 1],
                                                          extra[None, None, None], tau)[0, 0, 0]
