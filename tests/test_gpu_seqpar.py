"""Sequence-parallel kernels on one GPU with P ranks emulated: every rank's send buffer
is built by asa_seqpar_pack, the all-to-all is done by slicing (as NCCL would deliver
the chunks), and each rank's steps run through the C ABI.  Per head the kernels see
the same data as the unsharded call, so every intermediate and the result must be
bit-identical to asa_gilbert_permute3 / asa_attention on the full tensors.  A real
NCCL process group of one rank runs the harness itself."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa, seqpar

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["tiny"]


def _emulated_exchange(sends, splits_from):
    """sends[s]: rank s's send buffer; splits_from[s][r]: elements s sends to r.
    Returns recv[r] = concat over s of s's chunk for r."""
    P = len(sends)
    recv = []
    for r in range(P):
        parts = []
        for s in range(P):
            beg = sum(splits_from[s][:r])
            parts.append(sends[s][beg:beg + splits_from[s][r]])
        recv.append(torch.cat(parts))
    return recv


@pytest.mark.parametrize("P,wl", [
    (2, BASE),
    (3, BASE.with_(name="sp3", B=2, H=5, d=128, T=3, Hg=9, W=11, seed=61, tau=0.95)),
    (4, BASE.with_(name="sp4", B=1, H=4, d=64, T=5, Hg=9, W=11, seed=62)),
])
def test_emulated_ranks_bit_identical(P, wl):
    x = make_inputs(wl)
    full = [x[n].cuda() for n in ("q", "k", "v")]
    B, N, H, d = full[0].shape
    T, Hg, W = wl.T, wl.Hg, wl.W
    tok, heads = seqpar.shard_offsets(N, P), seqpar.shard_offsets(H, P)
    ops = seqpar.KernelOps()
    shards = [[t[:, tok[r]:tok[r + 1]].contiguous() for t in full] for r in range(P)]
    by_heads = [[B * (tok[s + 1] - tok[s]) * (heads[r + 1] - heads[r]) * d for r in range(P)]
                for s in range(P)]
    # first exchange: each tensor separately
    recvs = [[None] * 3 for _ in range(P)]
    for i in range(3):
        sends = [ops.pack(shards[s][i], heads) for s in range(P)]
        for r, buf in enumerate(_emulated_exchange(sends, by_heads)):
            recvs[r][i] = buf
    full_p = asa.asa_gilbert_permute3(*full, T, Hg, W)
    o_full, _, _ = asa.asa_attention(*full, T, Hg, W, wl.tau)
    sends2 = []
    for r in range(P):
        Hl = heads[r + 1] - heads[r]
        xp = ops.permute3(recvs[r], tok, B, T, Hg, W, Hl, d)
        for a, b in zip(xp, full_p):
            assert torch.equal(a.view(torch.int16), b[:, heads[r]:heads[r + 1]].view(torch.int16))
        op = ops.attention(*xp, T, Hg, W, wl.tau, 0)
        sends2.append(ops.unpermute(op, tok, T, Hg, W))
    # second exchange: rank r sends rank s its heads of s's tokens
    by_tokens = [[B * (tok[s + 1] - tok[s]) * (heads[r + 1] - heads[r]) * d for s in range(P)]
                 for r in range(P)]
    for s, recv in enumerate(_emulated_exchange(sends2, by_tokens)):
        Ns = tok[s + 1] - tok[s]
        out = ops.unpack(recv, heads, (B, Ns, H, d))
        assert torch.equal(out.view(torch.int16), o_full[:, tok[s]:tok[s + 1]].view(torch.int16))
    asa.asa_check_device_status()


def test_pack_unpack_round_trip_and_rejects():
    x = torch.randn((2, 37, 7, 64), device="cuda").to(torch.bfloat16)
    ops = seqpar.KernelOps()
    heads = [0, 3, 3, 7]            # an empty head group in the middle
    send = ops.pack(x, heads)
    assert torch.equal(send[:2 * 37 * 3 * 64].view(2, 37, 3, 64), x[:, :, 0:3])
    assert torch.equal(ops.unpack(send, heads, tuple(x.shape)), x)
    with pytest.raises(asa.AsaError):
        ops.pack(x, [0, 3, 8])       # offsets must end at H
    with pytest.raises(asa.AsaError):
        ops.pack(x, [0, 4, 3, 7])    # decreasing


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.timeout(300)
def test_nccl_single_rank_harness():
    wl = BASE.with_(name="sp1", B=1, H=3, d=64, T=3, Hg=9, W=11, seed=63)
    x = make_inputs(wl)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0),
                            timeout=datetime.timedelta(seconds=60))
    try:
        out = seqpar.seqpar_attention(q, k, v, wl.T, wl.Hg, wl.W, wl.tau)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref, _, _ = asa.asa_attention(q, k, v, wl.T, wl.Hg, wl.W, wl.tau)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
