"""Sequence-parallel ASA over P ranks (one process per GPU, torch.distributed).

Rank r holds the raster tokens [tok_off[r], tok_off[r+1]) of every head (a
sequence-sharded DiT).  ASA needs every token of a head (its estimate, mask and
attention are per head), so the call exchanges sequence shards for head shards:

    pack (head groups)  -> all-to-all -> Gilbert gather straight from the receive
    chunks -> estimate + mask + sparse forward on this rank's heads -> inverse gather
    straight into the send chunks -> all-to-all -> unpack (head groups)

The exchanges are NCCL all-to-alls into local buffers; every data movement around
them runs in the library's kernels (asa_seqpar_* in include/asa.h).  Tokens and heads
are split as evenly as possible (the first ranks take one more); H >= P.
"""
from __future__ import annotations

import ctypes

import torch
import torch.distributed as dist

from . import asa


def shard_offsets(n: int, P: int) -> list[int]:
    """P + 1 offsets splitting n items over P ranks, the first n mod P ranks one more."""
    base, rem = divmod(n, P)
    offs = [0]
    for r in range(P):
        offs.append(offs[-1] + base + (1 if r < rem else 0))
    return offs


def _ints(offs):
    return (ctypes.c_int * len(offs))(*offs)


class KernelOps:
    """The local steps on the library's kernels (CUDA tensors)."""

    def pack(self, x, head_off):
        B, Nr, H, d = x.shape
        send = torch.empty(x.numel(), dtype=x.dtype, device=x.device)
        asa._check(asa.lib().asa_seqpar_pack(asa._ptr(x), asa._ptr(send), B, Nr, H, d,
                                             _ints(head_off), len(head_off) - 1,
                                             asa._stream(None)))
        return send

    def unpack(self, recv, head_off, shape):
        B, Nr, H, d = shape
        x = torch.empty(shape, dtype=recv.dtype, device=recv.device)
        asa._check(asa.lib().asa_seqpar_unpack(asa._ptr(recv), asa._ptr(x), B, Nr, H, d,
                                               _ints(head_off), len(head_off) - 1,
                                               asa._stream(None)))
        return x

    def permute3(self, recvs, tok_off, B, T, Hg, W, Hl, d):
        N = T * Hg * W
        outs = tuple(torch.empty((B, Hl, N, d), dtype=recvs[0].dtype, device=recvs[0].device)
                     for _ in range(3))
        asa._check(asa.lib().asa_seqpar_permute3(*(asa._ptr(t) for t in recvs),
                                                 *(asa._ptr(t) for t in outs), B, T, Hg, W, Hl,
                                                 d, _ints(tok_off), len(tok_off) - 1,
                                                 asa._stream(None)))
        return outs

    def attention(self, qp, kp, vp, T, Hg, W, tau, global_window):
        mask = asa.asa_estimate_mask(qp, kp, tau, transposed=False)
        op, _ = asa.asa_sparse_attn_fwd(qp, kp, vp, mask, global_window=global_window)
        return op

    def unpermute(self, op, tok_off, T, Hg, W):
        B, Hl, N, d = op.shape
        send = torch.empty(op.numel(), dtype=op.dtype, device=op.device)
        asa._check(asa.lib().asa_seqpar_unpermute(asa._ptr(op), asa._ptr(send), B, T, Hg, W, Hl,
                                                  d, _ints(tok_off), len(tok_off) - 1,
                                                  asa._stream(None)))
        return send


def seqpar_attention(q, k, v, T: int, Hg: int, W: int, tau: float, global_window: int = 0,
                     group=None, ops=None):
    """ASA (or ASA_G) self-attention of a sequence-sharded batch: q, k, v [B, N_r, H, d]
    bf16 hold this rank's raster tokens; returns O for the same tokens [B, N_r, H, d]."""
    ops = ops or KernelOps()
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    B, Nr, H, d = q.shape
    N = T * Hg * W
    if H < P:
        raise ValueError(f"{H} heads cannot be split over {P} ranks")
    tok_off, head_off = shard_offsets(N, P), shard_offsets(H, P)
    if Nr != tok_off[r + 1] - tok_off[r]:
        raise ValueError(f"rank {r} holds {Nr} tokens, expected {tok_off[r + 1] - tok_off[r]}")
    Hl = head_off[r + 1] - head_off[r]
    # element counts: what this rank sends to / receives from each rank
    by_heads = [B * Nr * (head_off[s + 1] - head_off[s]) * d for s in range(P)]
    by_tokens = [B * (tok_off[s + 1] - tok_off[s]) * Hl * d for s in range(P)]
    recvs = []
    for x in (q, k, v):
        send = ops.pack(x, head_off)
        recv = torch.empty(sum(by_tokens), dtype=x.dtype, device=x.device)
        dist.all_to_all_single(recv, send, by_tokens, by_heads, group=group)
        recvs.append(recv)
    qp, kp, vp = ops.permute3(recvs, tok_off, B, T, Hg, W, Hl, d)
    op = ops.attention(qp, kp, vp, T, Hg, W, tau, global_window)
    send = ops.unpermute(op, tok_off, T, Hg, W)
    recv = torch.empty(sum(by_heads), dtype=q.dtype, device=q.device)
    dist.all_to_all_single(recv, send, by_heads, by_tokens, group=group)
    return ops.unpack(recv, head_off, (B, Nr, H, d))
