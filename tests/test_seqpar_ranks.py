"""Sequence-parallel exchange logic on two gloo ranks (CPU): the harness's splits and
the order of its two all-to-alls, with the local steps done by torch index operations
(this file's LayoutOps, independent of the kernels) and the attention replaced by an
elementwise stand-in.  The result on each rank must equal the stand-in applied to the
unsharded tensors, restricted to the rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from video_dit_dynamic_gilbert_b200 import seqpar


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class LayoutOps:
    def __init__(self, perm):
        self.perm = torch.from_numpy(perm).long()

    def pack(self, x, head_off):
        P = len(head_off) - 1
        return torch.cat([x[:, :, head_off[s]:head_off[s + 1]].reshape(-1) for s in range(P)])

    def unpack(self, recv, head_off, shape):
        B, Nr, H, d = shape
        out, pos = torch.empty(shape, dtype=recv.dtype), 0
        for s in range(len(head_off) - 1):
            hs = head_off[s + 1] - head_off[s]
            out[:, :, head_off[s]:head_off[s + 1]] = recv[pos:pos + B * Nr * hs * d].view(B, Nr, hs, d)
            pos += B * Nr * hs * d
        return out

    def permute3(self, recvs, tok_off, B, T, Hg, W, Hl, d):
        outs = []
        for recv in recvs:
            parts, pos = [], 0
            for s in range(len(tok_off) - 1):
                ns = tok_off[s + 1] - tok_off[s]
                parts.append(recv[pos:pos + B * ns * Hl * d].view(B, ns, Hl, d))
                pos += B * ns * Hl * d
            full = torch.cat(parts, dim=1)                     # [B, N, Hl, d] raster
            outs.append(full[:, self.perm].permute(0, 2, 1, 3).contiguous())
        return outs

    def attention(self, qp, kp, vp, T, Hg, W, tau, global_window):
        return 2 * qp - kp + 0.5 * vp

    def unpermute(self, op, tok_off, T, Hg, W):
        B, Hl, N, d = op.shape
        raster = torch.empty((B, N, Hl, d), dtype=op.dtype)
        raster[:, self.perm] = op.permute(0, 2, 1, 3)
        return torch.cat([raster[:, tok_off[s]:tok_off[s + 1]].reshape(-1)
                          for s in range(len(tok_off) - 1)])


def _rank(rank, world, port, T, Hg, W, H, B, d, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        N = T * Hg * W
        g = torch.Generator().manual_seed(7)
        full = [torch.randn((B, N, H, d), generator=g, dtype=torch.float64) for _ in range(3)]
        tok = seqpar.shard_offsets(N, world)
        shard = [x[:, tok[rank]:tok[rank + 1]].contiguous() for x in full]
        ops = LayoutOps(oracle.gilbert_order(T, Hg, W))
        out = seqpar.seqpar_attention(*shard, T, Hg, W, 0.9, ops=ops)
        ref = (2 * full[0] - full[1] + 0.5 * full[2])[:, tok[rank]:tok[rank + 1]]
        q.put((rank, bool(torch.equal(out, ref)), tuple(out.shape)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,T,Hg,W,H", [(2, 3, 5, 7, 4), (2, 2, 4, 5, 3), (3, 2, 3, 5, 5)])
def test_seqpar_exchange_round_trip(world, T, Hg, W, H):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, T, Hg, W, H, 2, 8, q), daemon=True)
             for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = [q.get(timeout=120) for _ in procs]
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    finally:
        for p in procs:          # the children this test started, if one is left waiting
            if p.is_alive():
                p.kill()
    N = T * Hg * W
    tok = seqpar.shard_offsets(N, world)
    for rank, ok, shape in res:
        assert ok, f"rank {rank}: output differs from the unsharded stand-in"
        assert shape == (2, tok[rank + 1] - tok[rank], H, 8)


def test_shard_offsets():
    assert seqpar.shard_offsets(10, 3) == [0, 4, 7, 10]
    assert seqpar.shard_offsets(12, 4) == [0, 3, 6, 9, 12]
    assert seqpar.shard_offsets(2, 3) == [0, 1, 2, 2]
