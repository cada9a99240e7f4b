"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/asa.h declares, computes the Gilbert table exactly like the oracle,
and rejects bad arguments with the documented codes before touching a device.

Every call below is built to fail validation (or is pure host code), so nothing is
ever launched with the fake pointers these tests pass."""
import ctypes
import itertools
import os
import re

import numpy as np
import pytest

import oracle
from video_dit_dynamic_gilbert_b200 import asa
from video_dit_dynamic_gilbert_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "asa.h")


@pytest.fixture(scope="module")
def L():
    build()
    return asa.lib()


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(asa_\w+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(asa._SIGNATURES), set(names) ^ set(asa._SIGNATURES)


def test_version_and_error_string(L):
    assert L.asa_version() >= 100
    assert isinstance(L.asa_last_error_string(), bytes)


@pytest.mark.parametrize("shape", list(itertools.product([1, 2, 3, 5, 8], repeat=3)))
def test_gilbert_table_matches_oracle_small(L, shape):
    np.testing.assert_array_equal(asa.asa_gilbert_index(*shape), oracle.gilbert_order(*shape))


@pytest.mark.parametrize("shape", [(21, 30, 52), (13, 30, 45), (21, 45, 80), (4, 16, 16),
                                   (1, 64, 64), (7, 9, 11), (1, 2, 197)])
def test_gilbert_table_matches_oracle_workloads(L, shape):
    np.testing.assert_array_equal(asa.asa_gilbert_index(*shape), oracle.gilbert_order(*shape))


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
MIS = ctypes.c_void_p(0x10008)       # misaligned


def test_gilbert_index_rejects(L):
    buf = np.empty(8, dtype=np.int32)
    p = buf.ctypes.data_as(ctypes.c_void_p)
    assert L.asa_gilbert_index(0, 2, 2, p) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_gilbert_index(2, 2, 2, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_gilbert_index(1, 1, 300000, p) == asa.ASA_ERR_UNSUPPORTED
    assert b"300000" in L.asa_last_error_string()


def test_permute_rejects(L):
    # bad head dim, aliasing, null, misaligned: all fail before any device work
    assert L.asa_gilbert_permute(FAKE, ctypes.c_void_p(0x20000), 1, 2, 2, 2, 3, 96, None) == \
        asa.ASA_ERR_UNSUPPORTED
    assert L.asa_gilbert_permute(FAKE, FAKE, 1, 2, 2, 2, 3, 64, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_gilbert_permute(None, FAKE, 1, 2, 2, 2, 3, 64, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_unpermute(MIS, FAKE, 1, 2, 2, 2, 3, 64, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_gilbert_permute(FAKE, ctypes.c_void_p(0x20000), 0, 2, 2, 2, 3, 64, None) == \
        asa.ASA_ERR_INVALID_ARG
    assert L.asa_gilbert_permute(FAKE, ctypes.c_void_p(0x20000), 1, 0, 2, 2, 3, 64, None) == \
        asa.ASA_ERR_INVALID_ARG


def test_estimate_mask_rejects(L):
    args = lambda d=64, block=128, samples=16, tau=0.9, ws=None, wsb=0: (
        FAKE, FAKE, 1, 2, 1024, d, block, samples, ctypes.c_float(tau), ws, wsb,
        FAKE, FAKE, FAKE, None, None, None)
    assert L.asa_estimate_mask(*args(d=80)) == asa.ASA_ERR_UNSUPPORTED
    assert L.asa_estimate_mask(*args(block=64)) == asa.ASA_ERR_UNSUPPORTED
    assert L.asa_estimate_mask(*args(samples=8)) == asa.ASA_ERR_UNSUPPORTED
    assert L.asa_estimate_mask(*args(tau=0.0)) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_estimate_mask(*args(tau=float("nan"))) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_estimate_mask(*args()) == asa.ASA_ERR_WORKSPACE          # no workspace
    assert L.asa_estimate_mask(*args(ws=ctypes.c_void_p(0x10010), wsb=1 << 30)) == \
        asa.ASA_ERR_WORKSPACE                                               # not 256-aligned
    need = L.asa_estimate_mask_workspace_size(1, 2, 1024)
    assert need > 0
    assert L.asa_estimate_mask(*args(ws=ctypes.c_void_p(0x100000), wsb=need - 1)) == \
        asa.ASA_ERR_WORKSPACE
    # one transposed pointer without the other
    bad = list(args(ws=ctypes.c_void_p(0x100000), wsb=need))
    bad[14] = FAKE
    assert L.asa_estimate_mask(*bad) == asa.ASA_ERR_INVALID_ARG
    # N too large, B*H too large
    assert L.asa_estimate(FAKE, FAKE, 1, 1, 300000, 64, 128, 16, None, 0, FAKE, None) == \
        asa.ASA_ERR_UNSUPPORTED
    assert L.asa_estimate(FAKE, FAKE, 300, 300, 1024, 64, 128, 16, None, 0, FAKE, None) == \
        asa.ASA_ERR_UNSUPPORTED


def test_attention_rejects(L):
    assert L.asa_sparse_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 1024, 96, 128, 0, None, 0,
                                 FAKE, FAKE, None) == asa.ASA_ERR_UNSUPPORTED
    assert L.asa_sparse_attn_fwd(FAKE, FAKE, MIS, FAKE, FAKE, 1, 2, 1024, 64, 128, 0, None, 0,
                                 FAKE, FAKE, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_sparse_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 1024, 64, 128, 64, None, 0,
                                 FAKE, FAKE, None) == asa.ASA_ERR_WORKSPACE
    assert L.asa_sparse_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 1024, 64, 128, -1, None, 0,
                                 FAKE, FAKE, None) == asa.ASA_ERR_INVALID_ARG
    args = [FAKE] * 10 + [1, 2, 1024, 64, 128, 0, None, 0] + [FAKE] * 3 + [None]
    assert L.asa_sparse_attn_bwd(*args) == asa.ASA_ERR_WORKSPACE
    args[15] = -1    # global_window
    assert L.asa_sparse_attn_bwd(*args) == asa.ASA_ERR_INVALID_ARG
    args[15] = 64
    assert L.asa_sparse_attn_bwd(*args) == asa.ASA_ERR_WORKSPACE
    args[15] = 0
    args[9] = None   # row_idx_t
    assert L.asa_sparse_attn_bwd(*args) == asa.ASA_ERR_INVALID_ARG


def test_stat_mask_rejects(L):
    args = lambda k=4, ws=None, wsb=0: (FAKE, 1, 2, 1024, k, ws, wsb, FAKE, FAKE, FAKE, None, None,
                                        None)
    assert L.asa_build_mask_stat(*args(k=0)) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_build_mask_stat(*args()) == asa.ASA_ERR_WORKSPACE
    bad = list(args(ws=ctypes.c_void_p(0x100000), wsb=1 << 30))
    bad[10] = FAKE          # col_ptr_t without row_idx_t
    assert L.asa_build_mask_stat(*bad) == asa.ASA_ERR_INVALID_ARG


def test_selftest_rejects_bad_limits(L):
    assert L.asa_selftest_wait_timeout(0, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_selftest_wait_timeout((1 << 31) + 1, None) == asa.ASA_ERR_INVALID_ARG
    assert b"limit_cycles" in L.asa_last_error_string()


def test_workspace_sizes(L):
    nb = 256
    est = L.asa_estimate_mask_workspace_size(1, 12, 32760)
    assert est >= 12 * nb * nb * (16 * 4 + 4 + 1)
    assert L.asa_fwd_workspace_size(1, 12, 32760, 128, 0) >= 12 * 256 * 4      # launch order
    assert L.asa_fwd_workspace_size(1, 12, 32760, 128, 64) >= 2 * 12 * 512 * 128 * 2
    assert L.asa_bwd_workspace_size(1, 12, 32760, 128, 0) >= 2 * 12 * 32760 * 4
    # ASA_G adds the global tokens (bf16 K, V, fp16 K) and their fp32 gradients
    G = -(-32760 // 64)
    extra = L.asa_bwd_workspace_size(1, 12, 32760, 128, 64) - L.asa_bwd_workspace_size(1, 12, 32760, 128, 0)
    assert extra >= 12 * G * 128 * (3 * 2 + 2 * 4)
    assert L.asa_bwd_workspace_size(1, 12, 32760, 128, -1) == 0
    assert L.asa_estimate_mask_workspace_size(0, 12, 32760) == 0


def test_prune_host_rules(L):
    # pack: 4 while a block keeps at most 32 queries, 2 up to 64, else 1
    assert L.asa_prune_pack(0.5, 8) == 2
    assert L.asa_prune_pack(0.25, 8) == 4
    assert L.asa_prune_pack(0.25, 2) == 2        # 64 centres per block
    assert L.asa_prune_pack(0.51, 8) == 1
    assert L.asa_prune_pack(0.0, 128) == 4
    assert L.asa_prune_pack(1.5, 8) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_prune_pack(float("nan"), 8) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_prune_pack(0.5, 0) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_prune_pack(0.5, 129) == asa.ASA_ERR_INVALID_ARG
    # compact rows: whole tiles of `pack` blocks
    assert L.asa_prune_rows(32760, 2) == 128 * 128
    assert L.asa_prune_rows(300, 4) == 128
    assert L.asa_prune_rows(300, 1) == 3 * 128
    assert L.asa_prune_rows(300, 3) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_prune_rows(0, 1) == asa.ASA_ERR_INVALID_ARG


def test_prune_rejects(L):
    q = lambda pack=2, r=0.5, w=8, qp=FAKE, d=64: L.asa_prune_queries(
        qp, 1, 2, 1024, d, 128, r, w, pack, FAKE, FAKE, FAKE, None)
    assert q(pack=4) == asa.ASA_ERR_INVALID_ARG     # 64 kept rows do not fit 32-row slots
    assert q(pack=3) == asa.ASA_ERR_INVALID_ARG
    assert q(r=-0.1) == asa.ASA_ERR_INVALID_ARG
    assert q(w=0) == asa.ASA_ERR_INVALID_ARG
    assert q(qp=MIS) == asa.ASA_ERR_INVALID_ARG
    assert q(d=96) == asa.ASA_ERR_UNSUPPORTED
    assert b"pack" in (q(pack=4) and L.asa_last_error_string())
    # the tile CSR needs its counts workspace
    assert L.asa_prune_mask(FAKE, FAKE, 1, 2, 1024, 2, None, 0, FAKE, FAKE, FAKE, FAKE,
                            None) == asa.ASA_ERR_WORKSPACE
    assert L.asa_prune_mask(FAKE, FAKE, 1, 2, 1024, 2, None, 0, FAKE, FAKE, None, FAKE,
                            None) == asa.ASA_ERR_INVALID_ARG
    fwd = [FAKE] * 7 + [1, 2, 1024, 64, 128, 2, 0, None, 0, FAKE, FAKE, None]
    assert L.asa_sparse_attn_fwd_pruned(*fwd) == asa.ASA_ERR_WORKSPACE
    fwd[12] = 3      # pack
    assert L.asa_sparse_attn_fwd_pruned(*fwd) == asa.ASA_ERR_INVALID_ARG
    fwd[12] = 2
    fwd[13] = -1     # global_window
    assert L.asa_sparse_attn_fwd_pruned(*fwd) == asa.ASA_ERR_INVALID_ARG
    bwd = [FAKE] * 10 + [1, 2, 1024, 64, 128, 2, 0, None, 0] + [FAKE] * 3 + [None]
    assert L.asa_sparse_attn_bwd_pruned(*bwd) == asa.ASA_ERR_WORKSPACE
    bwd[15] = 3      # pack
    assert L.asa_sparse_attn_bwd_pruned(*bwd) == asa.ASA_ERR_INVALID_ARG
    bwd[15] = 2
    bwd[5] = None    # src_pos
    assert L.asa_sparse_attn_bwd_pruned(*bwd) == asa.ASA_ERR_INVALID_ARG
    bwd[5] = FAKE
    bwd[9] = None    # tile_quarters
    assert L.asa_sparse_attn_bwd_pruned(*bwd) == asa.ASA_ERR_INVALID_ARG


def test_prune_workspace_sizes(L):
    BH, N, d = 12, 32760, 128
    tiles = BH * 128                     # 256 blocks, 2 per tile
    assert L.asa_prune_mask_workspace_size(1, 12, N, 2) >= tiles * 4
    assert L.asa_prune_mask_workspace_size(1, 12, N, 3) == 0
    fw = L.asa_fwd_pruned_workspace_size(1, 12, N, d, 2, 0)
    assert fw >= tiles * 4 + tiles * 128 * (d * 2 + 4)      # order, compact O and LSE
    G = -(-N // 64)
    assert L.asa_fwd_pruned_workspace_size(1, 12, N, d, 2, 64) - fw >= 2 * BH * G * d * 2
    # the packed backward: query side over 2 x 128 compact rows per tile, the compact
    # dO' and dQ, the dense quarter matrix and the transposed tile CSR
    Ns = 128 * 128
    bw = L.asa_bwd_pruned_workspace_size(1, 12, N, d, 2, 0)
    assert bw >= BH * Ns * (2 * 4 + 2 * d * 2) + BH * N * d * 2 + BH * 128 * 256 * 6
    assert bw < L.asa_bwd_workspace_size(1, 12, N, d, 0) + BH * Ns * d * 4 + BH * 128 * 256 * 8
    assert L.asa_bwd_pruned_workspace_size(1, 12, N, 96, 2, 0) == 0
    assert L.asa_bwd_pruned_workspace_size(1, 12, N, d, 3, 0) == 0


def test_host_call_rejects(L):
    ws = ctypes.c_void_p(0x100000)
    args = lambda q=FAKE, chunk=0, tau=0.9, wsb=1 << 40, T=4: (
        q, FAKE, FAKE, 1, T, 16, 16, 2, 64, tau, 0, chunk, ws, wsb, FAKE, None)
    assert L.asa_attention_host(*args(q=None)) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_attention_host(*args(chunk=-1)) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_attention_host(*args(tau=0.0)) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_attention_host(*args(T=0)) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_attention_host(*args(wsb=10)) == asa.ASA_ERR_WORKSPACE


def test_host_call_workspace_sizes(L):
    # two slots of head_chunk heads: 7 raster/permuted tensors of B*hc*N*d bf16 each (Q, K,
    # V in both orders and the raster O, which the forward stores directly), plus the
    # per-chunk estimator, mask and forward workspaces
    B, T, Hg, W, H, d = 1, 21, 30, 52, 12, 128
    N = T * Hg * W
    one = L.asa_attention_host_workspace_size(B, T, Hg, W, H, d, 0, 1)
    three = L.asa_attention_host_workspace_size(B, T, Hg, W, H, d, 0, 3)
    # default: max(ceil(256/d), ceil(H/24)) heads, capped at H
    assert L.asa_attention_host_workspace_size(B, T, Hg, W, H, d, 0, 0) == \
        L.asa_attention_host_workspace_size(B, T, Hg, W, H, d, 0, 2)                # d=128, H=12
    assert L.asa_attention_host_workspace_size(B, T, Hg, W, 48, 64, 0, 0) == \
        L.asa_attention_host_workspace_size(B, T, Hg, W, 48, 64, 0, 4)              # d=64
    assert L.asa_attention_host_workspace_size(B, T, Hg, W, 96, d, 0, 0) == \
        L.asa_attention_host_workspace_size(B, T, Hg, W, 96, d, 0, 4)               # 24 chunks
    assert L.asa_attention_host_workspace_size(B, T, Hg, W, 1, 64, 0, 0) == \
        L.asa_attention_host_workspace_size(B, T, Hg, W, 1, 64, 0, 1)               # capped at H
    assert one >= 2 * 7 * N * d * 2 + 2 * L.asa_estimate_mask_workspace_size(B, 1, N)
    assert one < 2 * 8 * N * d * 2 + 2 * L.asa_estimate_mask_workspace_size(B, 1, N)
    assert 2.5 * one < three < 3.5 * one
    assert L.asa_attention_host_workspace_size(B, T, Hg, W, H, d, 0, 99) == \
        L.asa_attention_host_workspace_size(B, T, Hg, W, H, d, 0, H)
    assert L.asa_attention_host_workspace_size(B, T, Hg, W, H, 96, 0, 0) == 0
    assert L.asa_attention_host_workspace_size(B, T, Hg, W, H, d, 0, -1) == 0


def test_seqpar_rejects(L):
    offs = lambda *v: (ctypes.c_int * len(v))(*v)
    ok_heads = offs(0, 2, 4)
    assert L.asa_seqpar_pack(FAKE, FAKE, 1, 10, 4, 64, offs(0, 2, 5), 2, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_seqpar_pack(FAKE, FAKE, 1, 10, 4, 64, offs(1, 2, 4), 2, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_seqpar_pack(FAKE, FAKE, 1, 10, 4, 64, offs(0, 3, 2, 4), 3, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_seqpar_pack(FAKE, FAKE, 1, 10, 4, 64, ok_heads, 0, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_seqpar_pack(FAKE, FAKE, 1, 10, 4, 64, None, 2, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_seqpar_unpack(MIS, FAKE, 1, 10, 4, 64, ok_heads, 2, None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_seqpar_pack(FAKE, FAKE, 1, 10, 4, 96, ok_heads, 2, None) == asa.ASA_ERR_UNSUPPORTED
    # token offsets must run from 0 to T*Hg*W (here 4*16*16 = 1024)
    assert L.asa_seqpar_permute3(*([FAKE] * 6), 1, 4, 16, 16, 2, 64, offs(0, 500, 1000), 2,
                                 None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_seqpar_unpermute(FAKE, FAKE, 1, 4, 16, 16, 2, 64, offs(0, 600, 500, 1024), 3,
                                  None) == asa.ASA_ERR_INVALID_ARG
    assert L.asa_seqpar_unpermute(FAKE, FAKE, 1, 0, 16, 16, 2, 64, offs(0, 1024), 1,
                                  None) == asa.ASA_ERR_INVALID_ARG


def test_bwd_d_from_o_rejects(L):
    # same contract as asa_sparse_attn_bwd: workspace, window and pointer checks first
    args = [FAKE] * 10 + [1, 2, 1024, 64, 128, 0, None, 0] + [FAKE] * 3 + [None]
    assert L.asa_sparse_attn_bwd_d_from_o(*args) == asa.ASA_ERR_WORKSPACE
    args[15] = -1
    assert L.asa_sparse_attn_bwd_d_from_o(*args) == asa.ASA_ERR_INVALID_ARG
    args[15] = 0
    args[3] = MIS     # o, the operand this variant reads
    assert L.asa_sparse_attn_bwd_d_from_o(*args) == asa.ASA_ERR_INVALID_ARG
    args[3] = FAKE
    args[13] = 96     # d
    assert L.asa_sparse_attn_bwd_d_from_o(*args) == asa.ASA_ERR_UNSUPPORTED


def test_trainable_op_rejects_d_from_o_with_query_pruning():
    """The query-pruned backward always takes the exact D, so asking for both is an
    error, raised before any device work."""
    import torch
    x = torch.zeros((1, 8, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        asa.asa_attention_trainable(x, x, x, 1, 2, 4, 0.9, query_keep=0.5, d_from_o=True)


def test_training_pair_rejects(L):
    # forward: workspace first, then the fp32 output's alignment, then d
    args = [FAKE] * 5 + [1, 2, 1024, 64, 128, 0, None, 0, FAKE, FAKE, FAKE, None]
    assert L.asa_sparse_attn_fwd_train(*args) == asa.ASA_ERR_WORKSPACE
    need = L.asa_fwd_train_workspace_size(1, 2, 1024, 64, 0)
    assert need >= L.asa_fwd_workspace_size(1, 2, 1024, 64, 0) + 2 * 1024 * 64 * 2
    args[11], args[12] = FAKE, need
    args[15] = MIS
    assert L.asa_sparse_attn_fwd_train(*args) == asa.ASA_ERR_INVALID_ARG
    args[15] = FAKE
    args[8] = 96
    assert L.asa_sparse_attn_fwd_train(*args) == asa.ASA_ERR_UNSUPPORTED
    # backward: the asa_sparse_attn_bwd contract with o32 in place of o
    bargs = [FAKE] * 10 + [1, 2, 1024, 64, 128, 0, None, 0] + [FAKE] * 3 + [None]
    assert L.asa_sparse_attn_bwd_train(*bargs) == asa.ASA_ERR_WORKSPACE
    bargs[15] = -1
    assert L.asa_sparse_attn_bwd_train(*bargs) == asa.ASA_ERR_INVALID_ARG
    bargs[15] = 0
    bargs[3] = MIS
    assert L.asa_sparse_attn_bwd_train(*bargs) == asa.ASA_ERR_INVALID_ARG
    assert b"o32" in L.asa_last_error_string()


def test_fwd_raster_rejects(L):
    # grid 4 x 16 x 16 = 1024 tokens, B=1, H=2
    def call(T=4, d=64, o=FAKE, gw=0, ws=None, wsb=0, vp=FAKE):
        return L.asa_sparse_attn_fwd_raster(FAKE, FAKE, vp, FAKE, FAKE, 1, T, 16, 16, 2, d, 128,
                                            gw, ws, wsb, o, FAKE, None)
    assert call(T=0) == asa.ASA_ERR_INVALID_ARG
    assert call(d=96) == asa.ASA_ERR_UNSUPPORTED
    assert call(o=FAKE) == asa.ASA_ERR_INVALID_ARG            # o aliases qp
    other = ctypes.c_void_p(0x20000)
    assert call(o=other, gw=-1) == asa.ASA_ERR_INVALID_ARG
    assert call(o=other) == asa.ASA_ERR_WORKSPACE
    assert call(o=other, vp=MIS) == asa.ASA_ERR_INVALID_ARG


def test_global_pool_kv_rejects(L):
    assert L.asa_global_pool_kv(FAKE, FAKE, FAKE, FAKE, 1, 2, 1024, 64, 0, None) == \
        asa.ASA_ERR_INVALID_ARG
    assert L.asa_global_pool_kv(FAKE, MIS, FAKE, FAKE, 1, 2, 1024, 64, 64, None) == \
        asa.ASA_ERR_INVALID_ARG
    assert L.asa_global_pool_kv(FAKE, FAKE, FAKE, FAKE, 1, 2, 1024, 96, 64, None) == \
        asa.ASA_ERR_UNSUPPORTED
