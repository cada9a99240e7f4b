"""Sequence-parallel kernels on one GPU with P ranks emulated: every rank's send buffer
is built by asa_seqpar_pack, the all-to-all is done by slicing (as NCCL would deliver
the chunks), and each rank's steps run through the C ABI.  Per head the kernels see
the same data as the unsharded call, so every intermediate and the result must be
bit-identical to asa_gilbert_permute3 / asa_attention on the full tensors, and the
assembled output is checked against the fp64 oracle.  A real NCCL process group of one
rank runs the harness itself."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

import oracle
from inputs import WORKLOADS, make_inputs
from video_dit_dynamic_gilbert_b200 import asa, seqpar
from gpu_util import check_close, compare_masks, f64, mask_from_csr

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


def _emulated_call(P, wl, x, check=None):
    """One sequence-parallel ASA call over P emulated ranks: pack, first exchange,
    Gilbert gather from the receive chunks, attention on each rank's heads, inverse
    scatter into send chunks, second exchange, unpack.  Returns the raster output
    [B, N, H, d] assembled from the ranks' token shards.  check(r, xp, heads) sees each
    rank's permuted tensors."""
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
    sends2 = []
    for r in range(P):
        Hl = heads[r + 1] - heads[r]
        xp = ops.permute3(recvs[r], tok, B, T, Hg, W, Hl, d)
        if check is not None:
            check(r, xp, heads)
        op = ops.attention(*xp, T, Hg, W, wl.tau, 0)
        sends2.append(ops.unpermute(op, tok, T, Hg, W))
    # second exchange: rank r sends rank s its heads of s's tokens
    by_tokens = [[B * (tok[s + 1] - tok[s]) * (heads[r + 1] - heads[r]) * d for s in range(P)]
                 for r in range(P)]
    outs = []
    for s, recv in enumerate(_emulated_exchange(sends2, by_tokens)):
        Ns = tok[s + 1] - tok[s]
        outs.append(ops.unpack(recv, heads, (B, Ns, H, d)))
    asa.asa_check_device_status()
    return torch.cat(outs, dim=1)


@pytest.mark.parametrize("P,wl", [
    (2, BASE),
    (3, BASE.with_(name="sp3", B=2, H=5, d=128, T=3, Hg=9, W=11, seed=61, tau=0.95)),
    (4, BASE.with_(name="sp4", B=1, H=4, d=64, T=5, Hg=9, W=11, seed=62)),
])
def test_emulated_ranks_bit_identical(P, wl):
    x = make_inputs(wl)
    full = [x[n].cuda() for n in ("q", "k", "v")]
    full_p = asa.asa_gilbert_permute3(*full, wl.T, wl.Hg, wl.W)

    def check(r, xp, heads):
        for a, b in zip(xp, full_p):
            assert torch.equal(a.view(torch.int16), b[:, heads[r]:heads[r + 1]].view(torch.int16))

    out = _emulated_call(P, wl, x, check)
    o_full, _, _ = asa.asa_attention(*full, wl.T, wl.Hg, wl.W, wl.tau)
    assert torch.equal(out.view(torch.int16), o_full.view(torch.int16))


@pytest.mark.parametrize("P,wl", [
    (2, BASE.with_(name="spo2", B=1, H=2, d=128, T=3, Hg=9, W=11, seed=64, tau=0.95)),
    (3, BASE.with_(name="spo3", B=2, H=3, d=64, T=4, Hg=7, W=13, seed=65, tau=0.9)),
])
def test_emulated_ranks_against_oracle(P, wl):
    """The sequence-parallel call's raster output against the fp64 oracle: its mask
    rows (the library's, computed per rank on that rank's heads) against the oracle's
    cut, differing rows only where marginal and then legal cuts; every output row against
    the oracle's forward under that mask."""
    x = make_inputs(wl)
    out = _emulated_call(P, wl, x)
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    ref = {n: oracle.permute(f64(x[n]), perm) for n in ("q", "k", "v")}
    pimp = oracle.estimate_pimp(ref["q"], ref["k"])
    qp, kp, _ = asa.asa_gilbert_permute3(*(x[n].cuda() for n in ("q", "k", "v")),
                                         wl.T, wl.Hg, wl.W)
    gm = mask_from_csr(asa.asa_estimate_mask(qp, kp, wl.tau))
    compare_masks(gm, oracle.build_mask(pimp, wl.tau), oracle.marginal_rows(pimp, wl.tau), pimp,
                  wl.tau, what=f"sequence parallel P={P} {wl.name}")
    O_ref, _ = oracle.asa_forward(ref["q"], ref["k"], ref["v"], gm)
    got = f64(out)
    for bb in range(wl.B):
        for h in range(wl.H):
            check_close(got[bb, perm, h], O_ref[bb, h], what=f"P={P} O b{bb} h{h}")


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
