"""fp64 CPU oracle for Adaptive Block-Sparse Attention (ASA / ASA_G).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never imports, links or calls anything here, and nothing here
imports the CUDA library: the two share no code, tables or helpers.  The only
shared module is the seeded input generator in ``inputs/``, which holds none of
the method's arithmetic.

Everything is plain NumPy in float64 (bf16 inputs are read as exact float64
values).  Each function cites the passage of "Video-BLADE: Block-Sparse Attention
Meets Step Distillation for Efficient Video Generation" (arXiv 2508.10774,
section "Adaptive Block-Sparse Attention") it restates.

Parity status per function (how each is pinned is in tests/test_oracle_*.py):
  gilbert_order      pinned: bijection, unit steps, brute force over all grids
                     up to 8x8x8, 1-D identity, textbook Hilbert curve on 2^m
                     squares (up to symmetry), locality vs raster.  The absolute
                     order relative to other Gilbert implementations is
                     "parity unpinned" (the pages do not define the curve).
  permute/unpermute  pinned: round trip, explicit index definition.
  estimate_pimp      pinned: k=b closed form vs the dense softmax map, row sums,
                     in-block permutation invariance.
  build_mask         pinned: brute-force minimality over all subsets (nb=8),
                     tau->0 keeps the argmax, tau=1 keeps all, monotone in tau.
  marginal_rows      pinned: hand-built rows whose cumulative share lands 5e-5 and
                     2e-4 from tau at the cut and one block before it, exact and
                     near ties at the cut, tau = 1 (tests/golden/marginal_rows.json).
  marginal_rows_stat pinned: hand-built rows with a share on the threshold, 4e-4
                     from it, a fallback row with a tied and an untied maximum,
                     k >= n (same fixture).
  legal_mask_rows    pinned: hand-built rows and kept sets (a prefix one block short
                     or long within and beyond 1e-4 of tau, a swap of near-equal and
                     of distinct shares, a size off by more than one, tau = 1); the
                     exact cut is legal on random rows (same fixture).
  asa_forward        pinned: tau=1 equals dense attention (torch SDPA fp64);
                     any mask equals SDPA with the token-expanded block mask.
  asa_g_forward      pinned: SDPA fp64 over Concat(K, MeanPool_n K) with the
                     additive ln(n) mask; n=1 closed form.
  asa_backward       pinned: torch.autograd of masked SDPA fp64; central finite
                     differences on a tiny case.
  build_mask_stat    pinned: k = n/2 keeps exactly the shares >= 1/n (U(1/2) = 0);
                     normal-distributed shares keep about k of n blocks (a flipped
                     quantile keeps n - k); the all-below fallback; k >= n keeps all.
  prune_queries      pinned (BSA query pruning): a hand-computed block with known
                     angles; the printed count of the BSA page's worked example
                     (23,296 queries, r = 0.5 -> 11,648); cosine vs torch's
                     cosine_similarity; brute-force maximal dissimilarity sum on tiny
                     blocks; r = 1 and w = 1 keep all; parallel queries keep the
                     centres and the lowest positions.
  asa_forward_pruned pinned: torch SDPA fp64 with the token mask, rows gathered by src.
  asa_backward_pruned pinned: torch.autograd of (masked SDPA, then the row gather by
                     src), ASA and ASA_G.
"""
from .gilbert import gilbert_order  # noqa: F401
from .asa_ref import (  # noqa: F401
    block_sizes,
    sample_offsets,
    sample_rows,
    permute,
    unpermute,
    estimate_pimp,
    build_mask,
    build_mask_stat,
    marginal_rows_stat,
    mask_to_csr,
    mask_to_csr_transposed,
    marginal_rows,
    legal_mask_rows,
    global_tokens,
    round_to_bf16,
    asa_forward,
    asa_backward,
    attention_flops,
)
from .query_prune import (  # noqa: F401
    window_centres,
    kept_count,
    cosine,
    prune_block,
    prune_queries,
    marginal_tokens,
    asa_forward_pruned,
    filled_dout,
    asa_backward_pruned,
)
