"""Host-side arithmetic of bench.py (no GPU): the near-threshold row count of the
measurement report and the effective-FLOP count of kept tiles."""
import numpy as np

import bench


def test_near_threshold_rows_cases():
    tau = 0.9
    rows = np.array([
        [0.5, 0.3, 0.1, 0.1],            # cumulative 0.5, 0.8, 0.9 (exactly tau): near
        [0.6, 0.35, 0.03, 0.02],         # 0.6, 0.95: far from tau
        [0.45, 0.45, 0.05, 0.05],        # 0.45, 0.9: cut exactly at tau: near
        [0.85, 0.07, 0.07 - 1e-8, 0.01],  # cut after 0.92; last kept and first dropped tie
        [0.25, 0.25, 0.25, 0.25],        # 0.25 .. 1.0: cut at 1.0, far
    ])[None, None]
    near, n = bench._near_threshold_rows(rows, tau)
    assert n == 5
    assert near == 3


def test_near_threshold_scale_invariant():
    g = np.random.default_rng(3)
    p = g.random((2, 3, 40, 40)) ** 4
    a = bench._near_threshold_rows(p, 0.95)
    b = bench._near_threshold_rows(p * 1e-6, 0.95)
    assert a == b


def test_kept_tile_flops_small():
    # N = 300: blocks of 128, 128, 44; one head keeps (0,0), (0,2), (2,1), (2,2)
    row_ptr = np.array([0, 2, 2, 4], dtype=np.int32)
    col_idx = np.array([0, 2, 1, 2], dtype=np.int32)
    flops, nnz, tiles = bench._kept_tile_flops(row_ptr, col_idx, 1, 1, 300, 64)
    L = [128, 128, 44]
    want = 4 * 64 * (L[0] * L[0] + L[0] * L[2] + L[2] * L[1] + L[2] * L[2])
    assert (flops, nnz, tiles) == (want, 4, 9)


def _csr(mask):
    rows = mask.reshape(-1, mask.shape[-1])
    rp = np.concatenate([[0], np.cumsum(rows.sum(1))]).astype(np.int64)
    ci = np.concatenate([np.nonzero(r)[0] for r in rows]).astype(np.int64)
    return rp, ci


def test_pruned_flops_against_kept_tile_flops():
    B, H, N, d = 1, 2, 300, 64            # blocks of 128, 128, 44
    g = np.random.default_rng(3)
    mask = g.random((B, H, 3, 3)) < 0.6
    mask[..., np.arange(3), np.arange(3)] = True
    rp, ci = _csr(mask)
    full, _, _ = bench._kept_tile_flops(rp, ci, B, H, N, d)
    # every query kept: the kept-tile count
    src_all = np.tile(np.arange(N), (B, H, 1))
    f_all, kept_all = bench._pruned_flops(rp, ci, src_all, B, H, N, d)
    assert f_all == full and kept_all == B * H * N
    # every other token points at its left neighbour: half of each even block kept
    src_half = src_all.copy()
    src_half[..., 1::2] -= 1
    f_half, kept_half = bench._pruned_flops(rp, ci, src_half, B, H, N, d)
    assert kept_half == B * H * N // 2
    L = np.array([128, 128, 44])
    K = L // 2
    expect = 0
    for h in range(H):
        for I in range(3):
            expect += 4 * d * K[I] * L[np.nonzero(mask[0, h, I])[0]].sum()
    assert f_half == expect
