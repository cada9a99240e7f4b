"""fp64 reference of query pruning with token filling (test infrastructure; see
oracle/__init__.py).

Source: "Bidirectional Sparse Attention for Faster Video Diffusion Training" (BSA),
section "Key designs", item 1 (spatio-temporal query pruning and token filling, the
set Q^s defined by rank_b(1 - cos(q_c, q_i)) <= ceil(r |Q_c|)), and its section "A
complete example" (blocks with 2x2x2 windows, r = 0.5, half of 23,296 queries kept).
Layered on ASA's blocks ("Video-BLADE: Block-Sparse Attention Meets Step
Distillation for Efficient Video Generation", "Preprocessing": runs of b = 128
Gilbert-ordered tokens).

Readings taken where the pages are silent:
  * a query block is a block of b permuted tokens; its windows are runs of w
    consecutive permuted tokens from the block start (the last one ragged);
    the centre of a window of length l starting at s is the token at s + l // 2;
  * cos(a, b) = a.b / (max(|a|, eps) max(|b|, eps)), eps = 1e-8 (a zero vector has
    cosine 0 to everything, so it counts as fully dissimilar);
  * a block of L tokens keeps K = max(ceil(r L), n_c) tokens, n_c its window count:
    every centre (the filling copies the centres' outputs, so they are computed)
    plus the K - n_c other tokens with the largest 1 - cos to their own window's
    centre, ties to the lower position; ceil(r L) is taken on the fp32 value of r;
  * a pruned token's output row and LSE are its centre's; in the backward its output
    gradient is added to the centre's (the copy's derivative) and it gets no gradient
    of its own; the summed output gradient is stored in bf16, the kernels' operand
    type.
"""
from __future__ import annotations

import math

import numpy as np

from .asa_ref import asa_backward, asa_forward, block_sizes, round_to_bf16

COS_EPS = 1e-8


def window_centres(L: int, w: int) -> np.ndarray:
    """Offset of each token's window centre inside a block of L tokens, windows of w."""
    off = np.arange(L)
    start = (off // w) * w
    length = np.minimum(w, L - start)
    return start + length // 2


def kept_count(L: int, r: float, w: int) -> int:
    """K = max(ceil(r L), number of windows) with r read as an fp32 value."""
    r32 = float(np.float32(r))
    return max(int(math.ceil(r32 * L)), -(-L // w))


def cosine(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Row-wise cosine of a [n, d] and b [n, d] with each norm floored at COS_EPS."""
    na = np.maximum(np.linalg.norm(a, axis=-1), COS_EPS)
    nb = np.maximum(np.linalg.norm(b, axis=-1), COS_EPS)
    return np.einsum("nd,nd->n", a, b) / (na * nb)


def prune_block(q: np.ndarray, r: float, w: int):
    """One block's decision.  q [L, d] -> (kept bool [L], centre offset [L],
    dissimilarity 1 - cos(q_centre, q_i) [L])."""
    L = q.shape[0]
    c = window_centres(L, w)
    dis = 1.0 - cosine(np.asarray(q, dtype=np.float64)[c], np.asarray(q, dtype=np.float64))
    is_centre = c == np.arange(L)
    kept = is_centre.copy()
    extra = kept_count(L, r, w) - int(is_centre.sum())
    if extra > 0:
        cand = np.nonzero(~is_centre)[0]
        # most dissimilar first, lower position first among equals
        order = cand[np.lexsort((cand, -dis[cand]))]
        kept[order[:extra]] = True
    return kept, c, dis


def prune_queries(qp: np.ndarray, r: float, w: int, b: int = 128):
    """qp [B, H, N, d] permuted queries -> (kept [B, H, N] bool, src [B, H, N] int64,
    dis [B, H, N] float64).  src[i] is the permuted position whose output token i
    takes: i itself when kept, else its window centre."""
    B, H, N, d = qp.shape
    kept = np.zeros((B, H, N), dtype=bool)
    src = np.zeros((B, H, N), dtype=np.int64)
    dis = np.zeros((B, H, N), dtype=np.float64)
    for bb in range(B):
        for h in range(H):
            for I, L in enumerate(block_sizes(N, b)):
                s = I * b
                k_, c, d_ = prune_block(qp[bb, h, s:s + L], r, w)
                kept[bb, h, s:s + L] = k_
                dis[bb, h, s:s + L] = d_
                src[bb, h, s:s + L] = np.where(k_, np.arange(s, s + L), s + c)
    return kept, src, dis


def marginal_tokens(kept: np.ndarray, dis: np.ndarray, w: int, b: int = 128,
                    eps: float = 1e-5) -> np.ndarray:
    """Tokens whose keep/prune decision an fp32 evaluation of the cosines may take
    the other way.  With lo the smallest kept and hi the largest pruned non-centre
    dissimilarity of a block, errors below eps/2 can only swap tokens across the cut
    when lo - hi <= eps; then every non-centre with dissimilarity in
    [hi - eps, lo + eps] is marginal."""
    B, H, N = kept.shape
    marg = np.zeros_like(kept)
    for bb in range(B):
        for h in range(H):
            for I, L in enumerate(block_sizes(N, b)):
                s = I * b
                c = window_centres(L, w)
                nc = c != np.arange(L)
                k_ = kept[bb, h, s:s + L] & nc
                p_ = ~kept[bb, h, s:s + L] & nc
                if not k_.any() or not p_.any():
                    continue
                d_ = dis[bb, h, s:s + L]
                lo, hi = d_[k_].min(), d_[p_].max()
                if lo - hi <= eps:
                    marg[bb, h, s:s + L] = nc & (d_ >= hi - eps) & (d_ <= lo + eps)
    return marg


def asa_forward_pruned(qp, kp, vp, mask, src, b: int = 128, global_window: int = 0,
                       q_index=None):
    """O [B, H, nq, d] and LSE [B, H, nq] with query pruning and token filling: row i
    is ASA's (or ASA_G's) output and LSE at row src[i]."""
    B, H, N, d = qp.shape
    q_index = np.arange(N) if q_index is None else np.asarray(list(q_index), dtype=np.int64)
    O = np.zeros((B, H, len(q_index), d))
    LSE = np.zeros((B, H, len(q_index)))
    for bb in range(B):
        for h in range(H):
            o, l = asa_forward(qp[bb:bb + 1, h:h + 1], kp[bb:bb + 1, h:h + 1],
                               vp[bb:bb + 1, h:h + 1], mask[bb:bb + 1, h:h + 1], b=b,
                               global_window=global_window, q_index=src[bb, h, q_index])
            O[bb, h] = o[0, 0]
            LSE[bb, h] = l[0, 0]
    return O, LSE


def filled_dout(dout: np.ndarray, src: np.ndarray, bf16: bool = True) -> np.ndarray:
    """dO' [B, H, N, d]: dO'[c] = sum of dO[i] over the tokens i with src[i] = c
    (a kept token's own gradient plus those of the pruned tokens it fills); zero on
    pruned rows.  Rounded to bf16 unless bf16=False."""
    B, H, N, d = dout.shape
    out = np.zeros((B, H, N, d), dtype=np.float64)
    for bb in range(B):
        for h in range(H):
            np.add.at(out[bb, h], src[bb, h], np.asarray(dout[bb, h], dtype=np.float64))
    return round_to_bf16(out) if bf16 else out


def asa_backward_pruned(qp, kp, vp, dout, mask, src, b: int = 128, heads=None,
                        q_blocks=None, kv_blocks=None, global_window: int = 0,
                        bf16: bool = True):
    """Gradients with query pruning and token filling under a fixed mask.  Token i's
    output is row src[i] of the attention, so dL/dO_c collects every dO_i with
    src[i] = c; a pruned row's output is never used, so its gradient terms vanish
    (its dO' row is zero) and its dQ is zero.  Same return format as asa_backward."""
    return asa_backward(qp, kp, vp, filled_dout(dout, src, bf16), mask, b=b, heads=heads,
                        q_blocks=q_blocks, kv_blocks=kv_blocks, global_window=global_window)
