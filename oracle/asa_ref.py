"""fp64 reference of the ASA hot path (test infrastructure; see oracle/__init__.py).

Source: "Video-BLADE: Block-Sparse Attention Meets Step Distillation for Efficient
Video Generation" (arXiv 2508.10774), section "Adaptive Block-Sparse Attention":
  * "Preprocessing"            -> permute / unpermute (with gilbert.gilbert_order)
  * "Step 1: Efficient block importance estimation" -> estimate_pimp
  * "Step 2.1: Sparse mask construction"            -> build_mask
  * "Step 2.2: Computation", variant 1 (standard ASA) and variant 2 (ASA_G, global
    tokens with the fixed additive ln(n) mask)      -> asa_forward
  * the block mask applies in training as well as at inference (end of
    Step 2.1)                                    -> asa_backward (fixed mask; ASA
    and ASA_G)
  * "Implementation details": b = 128, k = 16.

Readings taken where the pages are silent:
  * blocks are consecutive runs of b permuted tokens; the last block is ragged,
    nothing is padded;
  * the k "representative tokens" of a block of L tokens are the evenly strided
    offsets floor(j L / k_I), j < k_I = min(k, L) (all tokens when L < k);
  * P_approx is one softmax over all sampled keys of the head (the definition of
    P = softmax(QK^T / sqrt(d)) is global); P_imp[I, J] is the max of the
    k_I x k_J tile of P_approx;
  * each row of P_imp is normalised to shares R = P_imp / sum(P_imp); the kept set
    is the first c* blocks in (R descending, J ascending) order, c* the least c
    whose cumulative share is >= tau; tau >= 1 keeps every block;
  * ASA_G global token g is the mean of K (V) over permuted positions
    [n g, min(n g + n, N)), rounded to bf16 (the kernels store bf16 operands);
    every query sees every global token with logit q.kg / sqrt(d) + ln(n), also
    for the ragged last window;
  * LSE is the natural-log log-sum-exp of the logits a query row attends to;
  * in the ASA_G backward the gradient of a global token reaches the rows of its
    window through the mean (divided by the window's row count); its bf16 rounding
    passes gradients unchanged;
  * the statistical threshold (BSA page) is a threshold on each block's share, not a
    cumulative target: with U(1 - k/n) the normal quantile it keeps about k of n blocks;
    a row that keeps none keeps its largest share.
"""
from __future__ import annotations

import math
from typing import Iterable

import numpy as np


# ----------------------------------------------------------------------------
# blocking and sampling ("Preprocessing", "Step 1", "Implementation details")
# ----------------------------------------------------------------------------

def block_sizes(N: int, b: int = 128) -> list[int]:
    """L_I for each block I: runs of b permuted tokens, the last one ragged."""
    nb = -(-N // b)
    return [min(b, N - b * I) for I in range(nb)]


def sample_offsets(L: int, k: int = 16) -> list[int]:
    """Offsets inside a block of L tokens of its k_I = min(k, L) sampled tokens."""
    kk = min(k, L)
    return [(j * L) // kk for j in range(kk)]


def sample_rows(N: int, b: int = 128, k: int = 16) -> np.ndarray:
    """Permuted positions of all sampled tokens, block by block (length M)."""
    rows = []
    for I, L in enumerate(block_sizes(N, b)):
        rows.extend(b * I + s for s in sample_offsets(L, k))
    return np.asarray(rows, dtype=np.int64)


def _sample_block_starts(N: int, b: int, k: int) -> np.ndarray:
    starts, pos = [], 0
    for L in block_sizes(N, b):
        starts.append(pos)
        pos += min(k, L)
    return np.asarray(starts, dtype=np.int64)


# ----------------------------------------------------------------------------
# token rearrangement ("Preprocessing")
# ----------------------------------------------------------------------------

def permute(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """x [B, N, H, d] in raster order -> xp [B, H, N, d] with xp[b,h,i] = x[b,perm[i],h]."""
    return np.ascontiguousarray(np.transpose(x[:, perm, :, :], (0, 2, 1, 3)))


def unpermute(xp: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Inverse of permute: x[b, perm[i], h] = xp[b, h, i]."""
    B, H, N, d = xp.shape
    x = np.empty((B, N, H, d), dtype=xp.dtype)
    x[:, perm, :, :] = np.transpose(xp, (0, 2, 1, 3))
    return x


# ----------------------------------------------------------------------------
# Step 1: block importance estimation
# ----------------------------------------------------------------------------

def estimate_pimp(qp: np.ndarray, kp: np.ndarray, b: int = 128, k: int = 16,
                  q_blocks=None) -> np.ndarray:
    """P_imp [B, H, nb, nb] from k sampled tokens per block.

    Q_s, K_s = sampled rows; P_approx = softmax(Q_s K_s^T / sqrt(d)) over each row;
    P_imp[I, J] = max of the (rows of block I) x (columns of block J) tile.
    With k >= b every token is sampled and this is the exact max-pool of the full
    attention map that the section describes first.
    q_blocks: compute only these rows of P_imp (each row needs only its own block's
    sample rows against every sampled key); returns [B, H, len(q_blocks), nb].
    """
    B, H, N, d = qp.shape
    rows = sample_rows(N, b, k)
    starts = _sample_block_starts(N, b, k)
    nb = len(starts)
    sel = np.arange(nb) if q_blocks is None else np.asarray(list(q_blocks), dtype=np.int64)
    ends = np.append(starts[1:], len(rows))
    qrows = np.concatenate([np.arange(starts[I], ends[I]) for I in sel])
    qstarts = np.concatenate([[0], np.cumsum(ends[sel] - starts[sel])[:-1]]).astype(np.int64)
    out = np.empty((B, H, len(sel), nb), dtype=np.float64)
    for bb in range(B):
        for h in range(H):
            Qs = np.asarray(qp[bb, h, rows[qrows], :], dtype=np.float64)
            Ks = np.asarray(kp[bb, h, rows, :], dtype=np.float64)
            S = (Qs @ Ks.T) / math.sqrt(d)
            S = S - S.max(axis=1, keepdims=True)
            P = np.exp(S)
            P = P / P.sum(axis=1, keepdims=True)
            tile_max = np.maximum.reduceat(np.maximum.reduceat(P, qstarts, axis=0), starts, axis=1)
            out[bb, h] = tile_max
    return out


# ----------------------------------------------------------------------------
# Step 2.1: threshold mask
# ----------------------------------------------------------------------------

def _row_order(p_row: np.ndarray):
    share = p_row / p_row.sum()
    order = np.lexsort((np.arange(len(p_row)), -share))   # share desc, J asc
    return share, order


def _row_cut(share: np.ndarray, order: np.ndarray, tau: float) -> int:
    nb = len(share)
    if tau >= 1.0:
        return nb
    cum = np.cumsum(share[order])
    hit = np.nonzero(cum >= tau)[0]
    return int(hit[0]) + 1 if len(hit) else nb


def build_mask(pimp: np.ndarray, tau: float) -> np.ndarray:
    """Boolean block mask [B, H, nb, nb]: per row the fewest blocks with share >= tau."""
    B, H, nb, _ = pimp.shape
    mask = np.zeros(pimp.shape, dtype=bool)
    for bb in range(B):
        for h in range(H):
            for I in range(nb):
                share, order = _row_order(pimp[bb, h, I])
                c = _row_cut(share, order, tau)
                mask[bb, h, I, order[:c]] = True
    return mask


def build_mask_stat(pimp: np.ndarray, k_target: int) -> np.ndarray:
    """Statistical-threshold mask [B, H, rows, nb] (BSA's adaptive KV selection,
    p = mean(S_b) + std(S_b) U(1 - k/n), U the standard normal quantile function).

    Per row: shares R = P_imp / sum(P_imp); p = mean(R) + std(R) * U(1 - k/n) with n the
    number of key blocks and the population std; keep every block with R >= p; a row
    that keeps none keeps its largest share (lowest J on ties); k >= n keeps all.
    """
    from scipy.stats import norm
    B, H, nr, nb = pimp.shape
    mask = np.zeros(pimp.shape, dtype=bool)
    if k_target >= nb:
        mask[:] = True
        return mask
    z = norm.ppf(1.0 - k_target / nb)
    for bb in range(B):
        for h in range(H):
            for I in range(nr):
                v = np.maximum(np.asarray(pimp[bb, h, I], dtype=np.float64), 0.0)
                total = v.sum()
                if not total > 0:
                    mask[bb, h, I] = True
                    continue
                R = v / total
                p = R.mean() + R.std() * z
                keep = R >= p
                if not keep.any():
                    keep[int(np.argmax(R))] = True
                mask[bb, h, I] = keep
    return mask


def marginal_rows_stat(pimp: np.ndarray, k_target: int, eps: float = 1e-9) -> np.ndarray:
    """Rows whose statistical-threshold decision an fp32 evaluation may place
    differently: some share within ``eps`` (relative) of the threshold, or a fallback row
    whose largest shares tie within ``eps``."""
    from scipy.stats import norm
    B, H, nr, nb = pimp.shape
    marg = np.zeros((B, H, nr), dtype=bool)
    if k_target >= nb:
        return marg
    z = norm.ppf(1.0 - k_target / nb)
    for bb in range(B):
        for h in range(H):
            for I in range(nr):
                v = np.maximum(np.asarray(pimp[bb, h, I], dtype=np.float64), 0.0)
                if not v.sum() > 0:
                    continue
                R = v / v.sum()
                p = R.mean() + R.std() * z
                m = np.abs(R - p).min() <= eps * max(abs(p), 1e-300)
                if not (R >= p).any():
                    top = np.sort(R)[::-1]
                    m |= len(top) > 1 and top[0] - top[1] <= eps * top[0]
                marg[bb, h, I] = m
    return marg


def marginal_rows(pimp: np.ndarray, tau: float, eps: float = 1e-4,
                  tie_eps: float = 1e-6) -> np.ndarray:
    """Rows whose cut an fp32 evaluation may legitimately place differently.

    A row is marginal when the cumulative share at the cut, or one block before
    it, lies within ``eps`` of tau, or when the last kept share and the first
    dropped share differ by less than ``tie_eps``.
    """
    B, H, nb, _ = pimp.shape
    marg = np.zeros((B, H, nb), dtype=bool)
    if tau >= 1.0:
        return marg
    for bb in range(B):
        for h in range(H):
            for I in range(nb):
                share, order = _row_order(pimp[bb, h, I])
                cum = np.cumsum(share[order])
                c = _row_cut(share, order, tau)
                ncol = len(share)
                m = abs(cum[c - 1] - tau) < eps
                if c >= 2:
                    m |= abs(cum[c - 2] - tau) < eps
                if c < ncol:
                    m |= abs(share[order[c - 1]] - share[order[c]]) < tie_eps
                marg[bb, h, I] = m
    return marg


def legal_mask_rows(pimp: np.ndarray, mask: np.ndarray, tau: float, eps: float = 1e-4,
                    tie_rel: float = 5e-4) -> np.ndarray:
    """Rows of a block mask [B, H, nb, nb] that are a legal threshold cut of ``pimp``
    under a small perturbation of its values ("Step 2.1": the fewest blocks, taken in
    descending order, whose cumulative share reaches tau).

    A row's kept set S is legal when, with the row's exact shares R:
      * tau >= 1: S is every block;
      * |S| differs from the exact cut c* by at most one;
      * S is a leading set of the descending order up to near-ties: the smallest
        share in S is at least (1 - tie_rel) times the largest share left out;
      * S reaches tau within eps: sum_S R >= tau - eps;
      * S is minimal within eps: without its smallest share it stays below
        tau + eps.
    The exact cut of build_mask satisfies all five.  A set evaluated from shares
    that carry a relative error well below tie_rel (an fp32 estimate) can differ
    from it only at a row whose cumulative share at the cut is within eps of tau,
    or by the order of near-equal shares, and still passes.  Returns [B, H, nb] bool.
    """
    B, H, nb, _ = pimp.shape
    ok = np.zeros((B, H, nb), dtype=bool)
    for bb in range(B):
        for h in range(H):
            for I in range(nb):
                S = np.asarray(mask[bb, h, I], dtype=bool)
                if tau >= 1.0:
                    ok[bb, h, I] = bool(S.all())
                    continue
                if not S.any():
                    continue
                share, order = _row_order(pimp[bb, h, I])
                c = _row_cut(share, order, tau)
                if abs(int(S.sum()) - c) > 1:
                    continue
                smin = share[S].min()
                if (~S).any() and smin < (1.0 - tie_rel) * share[~S].max():
                    continue
                cum = share[S].sum()
                ok[bb, h, I] = cum >= tau - eps and cum - smin < tau + eps
    return ok


def mask_to_csr(mask: np.ndarray):
    """row_ptr [B*H*nb + 1], col_idx [nnz]; rows in (b, h, I) order, columns ascending."""
    B, H, nb, _ = mask.shape
    flat = mask.reshape(B * H * nb, nb)
    counts = flat.sum(axis=1)
    row_ptr = np.zeros(B * H * nb + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.nonzero(flat)[1].astype(np.int64)
    return row_ptr, col_idx


def mask_to_csr_transposed(mask: np.ndarray):
    """col_ptr [B*H*nb + 1], row_idx [nnz]: for each (b, h, J) the q-blocks I keeping J."""
    return mask_to_csr(np.swapaxes(mask, 2, 3))


# ----------------------------------------------------------------------------
# Step 2.2: computation (standard ASA and ASA_G), and its backward
# ----------------------------------------------------------------------------

def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                  # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)   # 8 significant bits


def global_tokens(x_head: np.ndarray, n: int) -> np.ndarray:
    """MeanPool_n over permuted positions of one head's [N, d] rows, bf16-rounded."""
    N = x_head.shape[0]
    G = -(-N // n)
    out = np.empty((G, x_head.shape[1]), dtype=np.float64)
    for g in range(G):
        out[g] = np.asarray(x_head[n * g:min(n * g + n, N)], dtype=np.float64).mean(axis=0)
    return round_to_bf16(out)


def _kept_positions(mask_row: np.ndarray, N: int, b: int) -> np.ndarray:
    blocks = np.nonzero(mask_row)[0]
    if len(blocks) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(b * J, min(b * J + b, N)) for J in blocks])


def asa_forward(qp, kp, vp, mask, b: int = 128, global_window: int = 0,
                q_index: Iterable[int] | None = None):
    """O [B, H, nq, d] and natural-log LSE [B, H, nq] for the queries ``q_index``.

    A query in block I attends to every token of the kept blocks of row I (standard
    ASA).  With ``global_window = n > 0`` (ASA_G) it also attends to all
    ceil(N/n) global tokens, whose logits carry the fixed additive ln(n).
    """
    B, H, N, d = qp.shape
    q_index = np.arange(N) if q_index is None else np.asarray(list(q_index), dtype=np.int64)
    nq = len(q_index)
    O = np.zeros((B, H, nq, d), dtype=np.float64)
    LSE = np.zeros((B, H, nq), dtype=np.float64)
    scale = 1.0 / math.sqrt(d)
    qblk = q_index // b
    for bb in range(B):
        for h in range(H):
            if global_window > 0:
                Kg = global_tokens(kp[bb, h], global_window)
                Vg = global_tokens(vp[bb, h], global_window)
            for I in np.unique(qblk):
                sel = np.nonzero(qblk == I)[0]
                q = np.asarray(qp[bb, h, q_index[sel]], dtype=np.float64)
                idx = _kept_positions(mask[bb, h, I], N, b)
                K = np.asarray(kp[bb, h, idx], dtype=np.float64)
                V = np.asarray(vp[bb, h, idx], dtype=np.float64)
                S = (q @ K.T) * scale
                if global_window > 0:
                    S = np.concatenate([S, (q @ Kg.T) * scale + math.log(global_window)], axis=1)
                    V = np.concatenate([V, Vg], axis=0)
                m = S.max(axis=1, keepdims=True)
                E = np.exp(S - m)
                l = E.sum(axis=1, keepdims=True)
                O[bb, h, sel] = (E / l) @ V
                LSE[bb, h, sel] = (m + np.log(l))[:, 0]
    return O, LSE


def asa_backward(qp, kp, vp, dout, mask, b: int = 128, heads=None,
                 q_blocks=None, kv_blocks=None, global_window: int = 0):
    """Gradients of ASA under a fixed mask (the mask is not differentiated).

    For each query block I with kept keys K_I, V_I (and, for ASA_G, the global tokens
    Kg, Vg of global_tokens() with the fixed + ln(n) on their logits):
        P = softmax(logits),  dP = dO_I [V_I; Vg]^T,  dS = P * (dP - rowsum(P * dP)),
        dQ_I = dS [K_I; Kg] / sqrt(d),
        dK_J += dS_J^T Q_I / sqrt(d),  dV_J += P_J^T dO_I   (kept fine blocks J),
        dKg += dS_g^T Q_I / sqrt(d),   dVg += P_g^T dO_I    (global tokens).
    A global token is the mean of the n permuted rows of its window, so its gradient
    reaches each of those rows divided by the window's row count (the bf16 rounding of
    the pooled token passes gradients through unchanged).
    Returns dicts {(b, h, I): dQ block} and {(b, h, J): (dK block, dV block)} for
    the requested heads / blocks (all by default).
    """
    B, H, N, d = qp.shape
    nb = -(-N // b)
    scale = 1.0 / math.sqrt(d)
    n = global_window
    heads = [(bb, h) for bb in range(B) for h in range(H)] if heads is None else list(heads)
    dq_out, dkv_out = {}, {}
    for (bb, h) in heads:
        want_q = set(range(nb)) if q_blocks is None else set(q_blocks)
        want_kv = set(range(nb)) if kv_blocks is None else set(kv_blocks)
        dK = {J: np.zeros((min(b, N - b * J), d)) for J in want_kv}
        dV = {J: np.zeros((min(b, N - b * J), d)) for J in want_kv}
        if n > 0:
            Kg = global_tokens(kp[bb, h], n)
            Vg = global_tokens(vp[bb, h], n)
            dKg = np.zeros_like(Kg)
            dVg = np.zeros_like(Vg)
        for I in range(nb):
            kept = np.nonzero(mask[bb, h, I])[0]
            # every query block reaches every requested key block through the global
            # tokens; without globals only through its kept blocks
            if I not in want_q and not (want_kv if n > 0 else set(kept.tolist()) & want_kv):
                continue
            rows = np.arange(b * I, min(b * I + b, N))
            idx = _kept_positions(mask[bb, h, I], N, b)
            Q = np.asarray(qp[bb, h, rows], dtype=np.float64)
            K = np.asarray(kp[bb, h, idx], dtype=np.float64)
            V = np.asarray(vp[bb, h, idx], dtype=np.float64)
            dO = np.asarray(dout[bb, h, rows], dtype=np.float64)
            S = (Q @ K.T) * scale
            nf = len(idx)
            if n > 0:
                S = np.concatenate([S, (Q @ Kg.T) * scale + math.log(n)], axis=1)
                K = np.concatenate([K, Kg], axis=0)
                V = np.concatenate([V, Vg], axis=0)
            E = np.exp(S - S.max(axis=1, keepdims=True))
            P = E / E.sum(axis=1, keepdims=True)
            dP = dO @ V.T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            if I in want_q:
                dq_out[(bb, h, I)] = (dS @ K) * scale
            off = 0
            for J in kept:
                LJ = min(b, N - b * J)
                if J in want_kv:
                    dK[J] += (dS[:, off:off + LJ].T @ Q) * scale
                    dV[J] += P[:, off:off + LJ].T @ dO
                off += LJ
            if n > 0:
                dKg += (dS[:, nf:].T @ Q) * scale
                dVg += P[:, nf:].T @ dO
        if n > 0:
            # MeanPool_n: row i of window g receives the window's gradient / its count
            cnt = np.array([min(n, N - n * g) for g in range(len(Kg))], dtype=np.float64)
            for J in want_kv:
                r = np.arange(b * J, min(b * J + b, N))
                dK[J] += dKg[r // n] / cnt[r // n, None]
                dV[J] += dVg[r // n] / cnt[r // n, None]
        for J in want_kv:
            dkv_out[(bb, h, J)] = (dK[J], dV[J])
    return dq_out, dkv_out


def attention_flops(mask: np.ndarray, N: int, d: int, b: int = 128,
                    global_window: int = 0) -> int:
    """Effective forward FLOPs: 4 d L_I L_J per kept tile (+ 4 d N G per head for ASA_G)."""
    L = np.asarray(block_sizes(N, b), dtype=np.int64)
    tiles = (mask * (L[:, None] * L[None, :])).sum()
    flops = 4 * d * int(tiles)
    if global_window > 0:
        B, H = mask.shape[:2]
        flops += 4 * d * N * (-(-N // global_window)) * B * H
    return flops
