#!/usr/bin/env python
"""ASA benchmark: one attention call of the Wan2.1-1.3B-shaped workload per step.

A step is the whole hot path of one training-free ASA self-attention call on
resident inputs: Gilbert permute of Q, K, V -> sampled block-importance estimate ->
tau-threshold mask (CSR) -> block-sparse attention forward, which stores O straight
back to raster order (the inverse permutation fused into its store).
Prints ONE JSON line (rank 0).  Metric: effective TFLOP/s counting only kept tiles
(4 d sum_kept L_I L_J per head), whole-job (all ranks) over the max-over-ranks time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own seeded batch on its own GPU (heads and
batches are independent, no collective on the data path: weak scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "wan2.1-1.3b"
METRIC = "ASA ms/call & effective TFLOP/s at 32760 tok, H=12, d=128, τ=0.95"


def count_launches(torch, step):
    """Kernels of this library (namespace asa) that one step launches, counted by CUPTI
    through torch.profiler over one untimed step: (count, sorted distinct names), or
    (None, reason) when the profiler is unavailable."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events()
                 if "asa::" in e.name and str(e.device_type).endswith("CUDA")]
        if not names:  # a step always launches kernels: another profiler holds CUPTI
            return None, "profiler saw no kernels (CUPTI held by another profiler)"
        return len(names), sorted(set(n.split("(")[0][-60:] for n in names))
    except Exception as exc:  # noqa: BLE001 - report, do not fail the bench
        return None, f"profiler unavailable: {type(exc).__name__}"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["bf16_tflops"], d["bf16_tflops_sustained"], d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def _fwd_traffic_bytes():
    """dram read+write bytes per forward launch from the committed ncu summary, or None
    when the kernel source has changed since that capture."""
    import hashlib
    import re
    prof = os.path.join(ROOT, "profiles", "fwd_tc_kernel_wan2.1-1.3b.md")
    src = os.path.join(ROOT, "video_dit_dynamic_gilbert_b200", "csrc", "attn_fwd_tc.cu")
    try:
        txt = open(prof).read()
        want = re.search(r"sha256 prefix\s+([0-9a-f]{16})", txt).group(1)
        have = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if want != have:
            return None
        mb = re.search(r"traffic per launch \(read \+ write\) \| ([0-9.]+) MB", txt).group(1)
        return float(mb) * 1e6
    except (OSError, AttributeError):
        return None


def _kept_tile_flops(row_ptr, col_idx, B, H, N, d):
    """4 d sum over kept (I, J) of L_I L_J, from the CSR the step produced."""
    nb = -(-N // 128)
    L = np.array([min(128, N - 128 * i) for i in range(nb)], dtype=np.int64)
    rp = row_ptr.astype(np.int64)
    counts = np.diff(rp)
    rows_I = np.tile(np.arange(nb), B * H)
    LJ = L[col_idx[:rp[-1]].astype(np.int64)]
    per_row = np.add.reduceat(LJ, rp[:-1]) if rp[-1] > 0 else np.zeros(len(counts), np.int64)
    per_row = np.where(counts > 0, per_row, 0)
    return int(4 * d * (L[rows_I] * per_row).sum()), int(rp[-1]), B * H * nb * nb


def _pruned_flops(row_ptr, col_idx, src_pos, B, H, N, d):
    """Effective forward FLOPs with query pruning: 4 d sum over kept (I, J) of K_I L_J,
    K_I the kept queries of block I."""
    nb = -(-N // 128)
    L = np.array([min(128, N - 128 * i) for i in range(nb)], dtype=np.int64)
    kept = (src_pos.reshape(B * H, N) == np.arange(N)[None]).astype(np.int64)
    K = np.add.reduceat(kept, np.arange(0, N, 128), axis=1).reshape(-1)      # [B*H*nb]
    rp = row_ptr.astype(np.int64)
    counts = np.diff(rp)
    LJ = L[col_idx[:rp[-1]].astype(np.int64)]
    per_row = np.add.reduceat(LJ, rp[:-1]) if rp[-1] > 0 else np.zeros(len(counts), np.int64)
    per_row = np.where(counts > 0, per_row, 0)
    return int(4 * d * (K * per_row).sum()), int(kept.sum())


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU is busy."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(device_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, n = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                clk, mx, pw = float(f[1]), float(f[2]), float(f[3])
            except ValueError:
                continue
            n += 1
            smax = mx
            if pw > 250.0:   # under load
                sm.append(clk)
                for name, val in zip(names, f[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": n, "samples_under_load": len(sm)}


def oracle_setup(wl, x, h=0, with_pimp=False):
    """The oracle's permuted Q, K, V of head h and its estimate + mask, with the time
    the estimate + mask took (and the oracle's P_imp when asked)."""
    import oracle
    perm = oracle.gilbert_order(wl.T, wl.Hg, wl.W)
    t0 = time.perf_counter()
    qp, kp, vp = (oracle.permute(x[n][:, :, h:h + 1].double().numpy(), perm)
                  for n in ("q", "k", "v"))
    pimp = oracle.estimate_pimp(qp, kp)
    mask = oracle.build_mask(pimp, wl.tau)
    out = (qp, kp, vp, mask, time.perf_counter() - t0)
    return out + (pimp,) if with_pimp else out


def mask_rows_vs_oracle(wl, pimp, mask, row_ptr, col_idx, h=0):
    """Rows of head h of the timed call's mask against the oracle's: how many differ,
    how many the oracle marks marginal, and how many differing rows are not a legal cut
    of the oracle's P_imp (a leading set within near-ties, one block from the exact cut
    at most, reaching tau within 1e-4 and minimal within 1e-4)."""
    import oracle
    nb = mask.shape[-1]
    rp = row_ptr.astype(np.int64)
    gm = np.zeros((1, 1, nb, nb), dtype=bool)
    for I in range(nb):
        gm[0, 0, I, col_idx[rp[h * nb + I]:rp[h * nb + I + 1]]] = True
    differ = (gm != mask).any(-1)
    marg = oracle.marginal_rows(pimp, wl.tau)
    legal = oracle.legal_mask_rows(pimp, gm, wl.tau)
    return {"head": h, "differ": int(differ.sum()), "marginal": int(marg.sum()),
            "differ_not_marginal": int((differ & ~marg).sum()), "not_legal": int((~legal).sum()),
            "of": int(nb)}


def cpu_oracle_sample(wl, x, budget_s=15.0, setup=None, seed=0):
    """Time the fp64 oracle on a bounded sample of the workload: estimate + mask of one
    head (or the given `setup` of it), then the sparse forward of as many of its query
    blocks as fit the budget.  The head's estimate + mask is charged in proportion to
    the blocks sampled."""
    import oracle
    import threadpoolctl
    qp, kp, vp, mask, t_mask = setup if setup is not None else oracle_setup(wl, x)
    nb = mask.shape[-1]
    flops, blocks, t_fwd = 0, 0, 0.0
    L = oracle.block_sizes(wl.N)
    order = np.random.default_rng(seed).permutation(nb)
    for I in order:
        t1 = time.perf_counter()
        oracle.asa_forward(qp, kp, vp, mask, q_index=np.arange(128 * I, 128 * I + L[I]))
        t_fwd += time.perf_counter() - t1
        flops += 4 * wl.d * L[I] * sum(L[J] for J in np.nonzero(mask[0, 0, I])[0])
        blocks += 1
        if t_fwd + (t_mask if setup is None else 0.0) > budget_s:
            break
    t_total = t_fwd + t_mask * blocks / nb
    info = threadpoolctl.threadpool_info()
    cores = max([i.get("num_threads", 1) for i in info] or [1])
    return {"value": flops / t_total / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "seconds": t_total,
            "sample": (f"1 of {wl.H} heads: fp64 estimate+mask of the head ({t_mask:.1f} s, charged "
                       f"{blocks}/{nb} of it) + sparse forward of {blocks} of {nb} query blocks "
                       f"({t_fwd:.1f} s)")}


def reference_step_budget(steps, warmup, total_s=150.0, cap_s=10.0):
    """Seconds of oracle work per reference step, so that the whole run stays within a
    few minutes whatever --steps and --warmup are."""
    return max(0.2, min(cap_s, total_s / max(1, steps + warmup)))


def run_reference(args, wl):
    """The reference arm: the fp64 CPU oracle, timed as it stands, on a bounded sample
    per step (rank 0 only; other ranks exit without work)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    from inputs import make_inputs
    x = make_inputs(wl)
    setup = oracle_setup(wl, x)
    budget = reference_step_budget(args.steps, args.warmup, cap_s=args.ref_budget)
    vals = []
    for step in range(args.warmup + args.steps):
        r = cpu_oracle_sample(wl, x, budget_s=budget, setup=setup, seed=step)
        if step >= args.warmup:
            vals.append(r)
    v = statistics.median(r["value"] for r in vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(r["seconds"] for r in vals),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(wl),
        "cpu_baseline": {**{k: vals[-1][k] for k in ("unit", "cores", "kind", "sample")},
                         "value": v},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return line


def rank_seed(wl, rank):
    """Each rank runs its own independent seeded call (weak scaling)."""
    return wl.seed + 1000 * rank


def combine_over_ranks(dist, device, times, work):
    """Max over ranks of each time in `times` and the sum over ranks of `work`: the
    same two collectives on every rank, in the same order."""
    import torch
    t = torch.tensor([float(v) for v in times], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    w = torch.tensor([float(work)], dtype=torch.float64, device=device)
    dist.all_reduce(w)
    return [float(v) for v in t.tolist()], float(w.item())


def _config(wl):
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "d": wl.d, "N": wl.N,
            "grid_THW": [wl.T, wl.Hg, wl.W], "block": 128, "samples": 16, "tau": wl.tau,
            "l2": "inputs larger than L2: raster Q, K, V are 3 x 100.6 MB",
            "parallelism": "one independent call per GPU (weak)"}

# ----------------------------------------------------------------------- measurement report

def _near_threshold_rows(p_imp, tau, eps=1e-4, gap=1e-6):
    """Mask rows whose cut is within `eps` of tau (or whose last kept and first dropped
    shares differ by less than `gap`): the rows where fp32 and fp64 may cut differently."""
    p = np.asarray(p_imp, dtype=np.float64).reshape(-1, p_imp.shape[-1])
    r = -np.sort(-(p / p.sum(axis=1, keepdims=True)), axis=1)
    cum = np.cumsum(r, axis=1)
    c = np.minimum(np.argmax(cum >= tau, axis=1), r.shape[1] - 1)
    rows = np.arange(len(c))
    near = np.abs(cum[rows, c] - tau) < eps
    near |= (c > 0) & (np.abs(cum[rows, np.maximum(c - 1, 0)] - tau) < eps)
    nxt = np.minimum(c + 1, r.shape[1] - 1)
    near |= (c + 1 < r.shape[1]) & (np.abs(r[rows, c] - r[rows, nxt]) < gap)
    return int(near.sum()), int(len(c))


class _Timer:
    """Per-call CUDA-event times on one stream: median and min over `reps` calls after
    `warm` untimed ones; `flush` runs before each call, outside its events.  The flush
    reads a buffer twice the size of L2: it evicts every line (and writes back, before
    the timed call, whatever the previous call left dirty) while leaving only clean
    lines behind, so that the timed call is not charged for someone else's
    write-back (a flush that writes the buffer would add up to 126 MB of it)."""

    def __init__(self, torch, stream, flush_bytes=256 << 20):
        self.torch, self.stream = torch, stream
        self.buf = torch.ones(flush_bytes // 4, dtype=torch.int32, device="cuda")

    def flush(self):
        self.sink = self.buf.sum()

    def __call__(self, fn, reps=20, warm=5, flush=False):
        torch = self.torch
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            if flush:
                self.flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(self.stream)
            fn()
            b.record(self.stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return {"median_ms": float(statistics.median(ts)), "min_ms": float(min(ts))}


def _report_config(asa, torch, wl, timer, dev, peaks):
    """Every stage of one workload, timed separately (permute, estimate, mask,
    attention, pool, backward, unpermute)."""
    from inputs import make_inputs
    x = make_inputs(wl, with_dout=wl.backward)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    B, N, H, d = q.shape
    T, Hg, W = wl.T, wl.Hg, wl.W
    nb = -(-N // 128)
    qp, kp, vp = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    asa.asa_gilbert_permute3(q, k, v, T, Hg, W, outs=(qp, kp, vp))
    ws = asa.estimate_mask_workspace(B, H, N, dev)
    p_imp = torch.empty((B, H, nb, nb), dtype=torch.float32, device=dev)
    gw = wl.global_window
    want_bwd = wl.backward or gw > 0
    mask = asa._alloc_mask(B, H, N, dev, transposed=want_bwd)
    fws = asa.fwd_workspace(B, H, N, d, gw, dev)
    op = torch.empty_like(qp)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    tensor_bytes = q.numel() * q.element_size()
    burst, sustained, hbm, kind = peaks
    r = {"workload": wl.name, "B": B, "H": H, "N": N, "d": d, "tau": wl.tau, "global_window": gw}

    def hbm_stage(name, fn, nbytes):
        for fl in (True, False):
            t = timer(fn, flush=fl)
            t["GB_s"] = nbytes / (t["median_ms"] * 1e-3) / 1e9
            t["frac_of_measured_hbm"] = t["GB_s"] / hbm
            r[name + ("_l2_flushed" if fl else "_l2_warm")] = t

    hbm_stage("permute_qkv", lambda: asa.asa_gilbert_permute3(q, k, v, T, Hg, W, outs=(qp, kp, vp)),
              3 * 2 * tensor_bytes)
    r["estimate"] = timer(lambda: asa.asa_estimate(qp, kp, workspace=ws, out=p_imp))
    r["mask"] = timer(lambda: asa.asa_build_mask(p_imp, N, wl.tau, transposed=want_bwd,
                                                 workspace=ws, mask=mask))
    r["estimate_mask"] = timer(lambda: asa.asa_estimate_mask(qp, kp, wl.tau, transposed=want_bwd,
                                                             workspace=ws, mask=mask))
    torch.cuda.synchronize()
    Ls = np.array([min(128, N - 128 * i) for i in range(nb)])
    M = int(np.minimum(16, Ls).sum())
    est_flops = 2 * M * M * d * B * H
    r["estimate"]["TFLOP_s"] = est_flops / (r["estimate"]["median_ms"] * 1e-3) / 1e12
    r["estimate"]["exp_count"] = M * M * B * H
    # the second mask mode (statistical threshold), about a quarter of the blocks per row
    mstat = asa._alloc_mask(B, H, N, dev, transposed=False)
    r["mask_stat"] = timer(lambda: asa.asa_build_mask_stat(p_imp, N, max(1, nb // 4),
                                                           transposed=False, workspace=ws,
                                                           mask=mstat))
    torch.cuda.synchronize()
    r["mask_stat"]["k_target"] = max(1, nb // 4)
    r["mask_stat"]["kept_fraction"] = int(mstat.nnz.item()) / (B * H * nb * nb)
    near, rows = _near_threshold_rows(p_imp.cpu().numpy(), wl.tau)
    r["near_threshold_rows"] = {"count": near, "of": rows}
    flops, nnz, tiles = _kept_tile_flops(mask.row_ptr.cpu().numpy(), mask.col_idx.cpu().numpy(),
                                         B, H, N, d)
    r["kept_tiles"], r["tiles"], r["kept_fraction"] = nnz, tiles, nnz / tiles
    if gw > 0:
        G = -(-N // gw)
        kg = torch.empty((B, H, G, d), dtype=torch.bfloat16, device=dev)
        hbm_stage("pool_K", lambda: asa.asa_global_pool(kp, gw, out=kg),
                  tensor_bytes + B * H * G * d * 2)
        vg = torch.empty_like(kg)
        hbm_stage("pool_KV", lambda: asa.asa_global_pool_kv(kp, vp, gw, outs=(kg, vg)),
                  2 * (tensor_bytes + B * H * G * d * 2))
        flops += 4 * d * N * G * B * H
    r["effective_flops"] = flops
    r["attn_fwd"] = timer(lambda: asa.asa_sparse_attn_fwd(qp, kp, vp, mask, global_window=gw,
                                                          workspace=fws, out=op, lse=lse))
    t = r["attn_fwd"]["median_ms"] * 1e-3
    r["attn_fwd"].update({"TFLOP_s": flops / t / 1e12, "frac_of_burst": flops / t / 1e12 / burst,
                          "frac_of_sustained": flops / t / 1e12 / sustained,
                          "frac_of_datasheet_2250": flops / t / 1e12 / 2250.0})
    hbm_stage("unpermute_o", lambda: asa.asa_unpermute(op, T, Hg, W, out=out), 2 * tensor_bytes)
    em = r["estimate_mask"]["median_ms"]
    r["estimate_mask_share"] = em / (em + r["attn_fwd"]["median_ms"])
    if want_bwd:
        if wl.backward:
            dop = asa.asa_gilbert_permute(x["dout"].to(dev), T, Hg, W)
        else:
            dop = torch.randn_like(qp)
        bws = asa.bwd_workspace(B, H, N, d, dev, gw)
        grads = tuple(torch.empty_like(qp) for _ in range(3))
        r["attn_bwd"] = timer(lambda: asa.asa_sparse_attn_bwd(qp, kp, vp, op, dop, lse, mask,
                                                              global_window=gw, workspace=bws,
                                                              outs=grads),
                              reps=8, warm=3)
        tb = r["attn_bwd"]["median_ms"] * 1e-3
        r["attn_bwd"]["effective_TFLOP_s"] = 2.5 * flops / tb / 1e12
        r["attn_bwd"]["executed_TFLOP_s"] = 4.5 * flops / tb / 1e12
        # the training pair: its forward (fp16 P V, fp32 O written) and its backward (D
        # from that O, no D pass: 7 executed GEMM units per kept tile, i.e. 3.5 forwards)
        tws = asa.fwd_train_workspace(B, H, N, d, gw, dev)
        o_t, lse_t = torch.empty_like(qp), torch.empty_like(lse)
        o32 = torch.empty(qp.shape, dtype=torch.float32, device=dev)
        r["attn_fwd_train"] = timer(lambda: asa.asa_sparse_attn_fwd_train(
            qp, kp, vp, mask, global_window=gw, workspace=tws, out=o_t, lse=lse_t, out32=o32))
        r["attn_fwd_train"]["TFLOP_s"] = flops / (r["attn_fwd_train"]["median_ms"] * 1e-3) / 1e12
        r["attn_bwd_train"] = timer(lambda: asa.asa_sparse_attn_bwd_train(
            qp, kp, vp, o32, dop, lse_t, mask, global_window=gw, workspace=bws, outs=grads),
            reps=8, warm=3)
        tt = r["attn_bwd_train"]["median_ms"] * 1e-3
        r["attn_bwd_train"]["effective_TFLOP_s"] = 2.5 * flops / tt / 1e12
        r["attn_bwd_train"]["executed_TFLOP_s"] = 3.5 * flops / tt / 1e12
    # BSA query pruning with token filling on the same mask: r = 0.5, windows of 8
    pr = asa.asa_prune_queries(qp, 0.5, 8)
    pmws = asa._workspace(asa.lib().asa_prune_mask_workspace_size(B, H, N, pr.pack), dev)
    ptm = asa.asa_prune_mask(mask, pr.pack, workspace=pmws)
    pfws = asa.fwd_pruned_workspace(B, H, N, d, pr.pack, gw, dev)
    plse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    qpr = {"r": 0.5, "window": 8, "pack": pr.pack}
    qpr["prune"] = timer(lambda: asa.asa_prune_queries(qp, 0.5, 8, out=pr))
    qpr["prune"]["GB_s"] = (tensor_bytes + B * H * pr.Ns * d * 2 + 2 * B * H * N * 4) / (
        qpr["prune"]["median_ms"] * 1e-3) / 1e9
    qpr["prune_mask"] = timer(lambda: asa.asa_prune_mask(mask, pr.pack, workspace=pmws, out=ptm))
    qpr["attn_fwd"] = timer(lambda: asa.asa_sparse_attn_fwd_pruned(pr, kp, vp, ptm, global_window=gw,
                                                                   workspace=pfws, out=op, lse=plse))
    torch.cuda.synchronize()
    pflops, nkept = _pruned_flops(mask.row_ptr.cpu().numpy(), mask.col_idx.cpu().numpy(),
                                  pr.src_pos.cpu().numpy(), B, H, N, d)
    if gw > 0:
        pflops += 4 * d * nkept * (-(-N // gw))
    qpr.update({"kept_queries": nkept, "tile_entries": int(ptm.nnz.item()),
                "block_entries": nnz, "effective_flops": pflops,
                "fwd_speedup": r["attn_fwd"]["median_ms"] / qpr["attn_fwd"]["median_ms"]})
    qpr["attn_fwd"]["TFLOP_s"] = pflops / (qpr["attn_fwd"]["median_ms"] * 1e-3) / 1e12
    if want_bwd:
        pbws = asa.bwd_pruned_workspace(B, H, N, d, pr.pack, dev, gw)
        qpr["attn_bwd"] = timer(lambda: asa.asa_sparse_attn_bwd_pruned(
            pr, kp, vp, dop, plse, ptm, global_window=gw, workspace=pbws, outs=grads), reps=8, warm=3)
        qpr["attn_bwd"]["effective_TFLOP_s"] = 2.5 * pflops / (qpr["attn_bwd"]["median_ms"] * 1e-3) / 1e12
        qpr["bwd_speedup"] = r["attn_bwd"]["median_ms"] / qpr["attn_bwd"]["median_ms"]
    r["query_prune"] = qpr
    asa.asa_check_device_status()
    return r, (qp, kp, vp)


def _seqpar_stages(asa, torch, timer, wl, dev, peaks, P=8):
    """The sequence-parallel local steps of rank 0 of P ranks emulated on this GPU (the
    all-to-alls are replaced by slicing): pack of its token shard, the Gilbert gather
    from its receive chunks, the inverse into its send chunks, the unpack."""
    from inputs import make_inputs
    from video_dit_dynamic_gilbert_b200 import seqpar
    x = make_inputs(wl)
    full = [x[n].to(dev) for n in ("q", "k", "v")]
    B, N, H, d = full[0].shape
    T, Hg, W = wl.T, wl.Hg, wl.W
    tok, heads = seqpar.shard_offsets(N, P), seqpar.shard_offsets(H, P)
    ops = seqpar.KernelOps()
    Hl, N0 = heads[1] - heads[0], tok[1] - tok[0]
    shard0 = [t[:, tok[0]:tok[1]].contiguous() for t in full]
    recv0 = []
    for t in full:        # rank 0's receive buffer: every rank's tokens of heads [0, Hl)
        recv0.append(torch.cat([t[:, tok[s]:tok[s + 1], heads[0]:heads[1]].reshape(-1)
                                for s in range(P)]))
    op0 = torch.randn((B, Hl, N, d), device=dev).to(torch.bfloat16)
    back0 = torch.cat([full[0][:, tok[0]:tok[1], heads[s]:heads[s + 1]].reshape(-1)
                       for s in range(P)])
    hbm = peaks[2]
    r = {"P": P, "rank0_tokens": N0, "rank0_heads": Hl}

    def stage(name, fn, nbytes):
        t = timer(fn)
        t["GB_s"] = nbytes / (t["median_ms"] * 1e-3) / 1e9
        t["frac_of_measured_hbm"] = t["GB_s"] / hbm
        r[name] = t

    shard_bytes = B * N0 * H * d * 2
    recv_bytes = B * N * Hl * d * 2
    stage("pack_q", lambda: ops.pack(shard0[0], heads), 2 * shard_bytes)
    stage("permute3_from_chunks", lambda: ops.permute3(recv0, tok, B, T, Hg, W, Hl, d),
          3 * 2 * recv_bytes)
    stage("unpermute_to_chunks", lambda: ops.unpermute(op0, tok, T, Hg, W), 2 * recv_bytes)
    stage("unpack_o", lambda: ops.unpack(back0, heads, (B, N0, H, d)), 2 * shard_bytes)
    asa.asa_check_device_status()
    return r


def _dense(asa, torch, timer, qp, kp, vp, peaks):
    """Dense attention on the same inputs: our kernel with every tile kept, and torch SDPA."""
    B, H, N, d = qp.shape
    nb = -(-N // 128)
    dense_flops = 4 * d * N * N * B * H
    full = asa.asa_build_mask(torch.ones((B, H, nb, nb), dtype=torch.float32, device=qp.device),
                              N, 1.0, transposed=False)
    ours = timer(lambda: asa.asa_sparse_attn_fwd(qp, kp, vp, full), reps=10, warm=3)
    sdpa = timer(lambda: torch.nn.functional.scaled_dot_product_attention(qp, kp, vp),
                 reps=10, warm=3)
    burst = peaks[0]
    for t in (ours, sdpa):
        t["TFLOP_s"] = dense_flops / (t["median_ms"] * 1e-3) / 1e12
        t["frac_of_burst"] = t["TFLOP_s"] / burst
    return {"ours_tau1": ours, "torch_sdpa": sdpa, "dense_flops": dense_flops}


def run_report(path):
    """Every measurement of the scope table, one JSON file: per-stage times of each
    workload (median and min of 20 CUDA-event-timed calls after 5 warm-up calls; the
    copy kernels with and without an L2 flush), dense comparisons, the tau sweep on the
    CogVideoX-5B shape and the backward on the Wan-14B shape."""
    import torch
    from inputs import WORKLOADS, make_inputs
    from video_dit_dynamic_gilbert_b200 import asa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    timer = _Timer(torch, stream)
    peaks = _peaks()
    rep = {"peaks": {"bf16_burst_tflops": peaks[0], "bf16_sustained_tflops": peaks[1],
                     "hbm_gbs": peaks[2], "kind": peaks[3]},
           "device": torch.cuda.get_device_name(dev), "configs": {}, "dense": {}, "tau_sweep": []}
    clocks = ClockSampler(0)
    for name in ("tiny", "wan2.1-1.3b", "cogvideox-5b", "wan2.1-1.3b-asag", "wan-14b-720p"):
        wl = WORKLOADS[name]
        r, (qp, kp, vp) = _report_config(asa, torch, wl, timer, dev, peaks)
        rep["configs"][name] = r
        if name in ("wan2.1-1.3b", "cogvideox-5b"):
            rep["dense"][name] = _dense(asa, torch, timer, qp, kp, vp, peaks)
        if name == "cogvideox-5b":
            B, H, N, d = qp.shape
            ws = asa.estimate_mask_workspace(B, H, N, dev)
            for tau in (0.80, 0.90, 0.95, 0.99):
                m = asa.asa_estimate_mask(qp, kp, tau, transposed=False, workspace=ws)
                em = timer(lambda: asa.asa_estimate_mask(qp, kp, tau, transposed=False,
                                                         workspace=ws, mask=m))
                fw = timer(lambda: asa.asa_sparse_attn_fwd(qp, kp, vp, m))
                flops, nnz, tiles = _kept_tile_flops(m.row_ptr.cpu().numpy(),
                                                     m.col_idx.cpu().numpy(), B, H, N, d)
                rep["tau_sweep"].append({
                    "workload": name, "tau": tau, "kept_fraction": nnz / tiles,
                    "estimate_mask": em, "attn_fwd": fw,
                    "TFLOP_s": flops / (fw["median_ms"] * 1e-3) / 1e12,
                    "estimate_mask_share": em["median_ms"] / (em["median_ms"] + fw["median_ms"])})
        del qp, kp, vp
        torch.cuda.empty_cache()
    rep["seqpar_emulated"] = {"wan-14b-720p": _seqpar_stages(asa, torch, timer,
                                                             WORKLOADS["wan-14b-720p"], dev, peaks)}
    rep["clocks"] = clocks.stop()
    with open(path, "w") as f:
        json.dump(rep, f, indent=1)
    for name, r in rep["configs"].items():
        line = (f"{name:18s} fwd {r['attn_fwd']['median_ms']:.3f} ms "
                f"{r['attn_fwd']['TFLOP_s']:.0f} TF/s ({r['attn_fwd']['frac_of_burst']:.3f} burst) "
                f"est+mask {r['estimate_mask']['median_ms']:.3f} ms "
                f"({100 * r['estimate_mask_share']:.1f}%) kept {r['kept_fraction']:.3f} "
                f"perm {r['permute_qkv_l2_flushed']['GB_s']:.0f} GB/s")
        if "attn_bwd" in r:
            line += (f" bwd {r['attn_bwd']['median_ms']:.2f} ms "
                     f"{r['attn_bwd']['effective_TFLOP_s']:.0f} TF/s eff")
        if "attn_bwd_train" in r:
            line += (f" bwd_train {r['attn_bwd_train']['median_ms']:.2f} ms "
                     f"{r['attn_bwd_train']['effective_TFLOP_s']:.0f} TF/s eff")
        qpr = r["query_prune"]
        line += (f" | pruned r=0.5: fwd {qpr['attn_fwd']['median_ms']:.3f} ms "
                 f"(x{qpr['fwd_speedup']:.2f})")
        if "attn_bwd" in qpr:
            line += f" bwd {qpr['attn_bwd']['median_ms']:.2f} ms (x{qpr['bwd_speedup']:.2f})"
        print(line)
    for name, sp in rep["seqpar_emulated"].items():
        print(f"{name} seqpar rank 0 of {sp['P']}: " + ", ".join(
            f"{k} {sp[k]['median_ms']:.3f} ms {sp[k]['GB_s']:.0f} GB/s" for k in
            ("pack_q", "permute3_from_chunks", "unpermute_to_chunks", "unpack_o")))
    return rep


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=10.0)
    ap.add_argument("--report", metavar="PATH", default=None,
                    help="run the full measurement set on one GPU, write it to PATH as JSON")
    ap.add_argument("--no-launch-count", action="store_true",
                    help="skip the CUPTI count of the step's kernels (for runs under ncu)")
    ap.add_argument("--only", choices=["bwd_train"], default=None,
                    help="time one stage alone on the workload (training forward once, then "
                         "--steps training backward calls) and print its JSON line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from inputs import WORKLOADS, make_inputs
    wl = WORKLOADS[args.workload]
    if args.report:
        run_report(args.report)
        return
    if args.impl == "reference":
        run_reference(args, wl)
        return
    if args.only == "bwd_train":
        run_bwd_train_only(args, wl)
        return

    import torch
    import torch.distributed as dist
    from video_dit_dynamic_gilbert_b200 import asa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    x = make_inputs(wl.with_(seed=rank_seed(wl, rank)))
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    B, N, H, d = q.shape
    T, Hg, W = wl.T, wl.Hg, wl.W
    qp, kp, vp = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    ws = asa.estimate_mask_workspace(B, H, N, dev)
    fws = asa.fwd_workspace(B, H, N, d, 0, dev)
    mask = asa._alloc_mask(B, H, N, dev, transposed=False)
    stream = torch.cuda.current_stream()

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(marks=None):
        if marks is not None:
            marks[0].record(stream)
        asa.asa_gilbert_permute3(q, k, v, T, Hg, W, outs=(qp, kp, vp))
        if marks is not None:
            marks[1].record(stream)
        asa.asa_estimate_mask(qp, kp, wl.tau, transposed=False, workspace=ws, mask=mask)
        if marks is not None:
            marks[2].record(stream)
        asa.asa_sparse_attn_fwd_raster(qp, kp, vp, mask, T, Hg, W, workspace=fws, out=out,
                                       lse=lse)
        if marks is not None:
            marks[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flops, nnz, tiles = _kept_tile_flops(mask.row_ptr.cpu().numpy(), mask.col_idx.cpu().numpy(),
                                         B, H, N, d)

    clocks = ClockSampler(local)
    time.sleep(0.3)
    marks = [[ev() for _ in range(4)] for _ in range(args.steps)]
    start, stop = ev(), ev()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        step(marks[i])
    stop.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = start.elapsed_time(stop)
    stage = np.array([[m[j].elapsed_time(m[j + 1]) for j in range(3)] for m in marks])
    st_ms = stage.mean(axis=0)
    fwd_ms = float(st_ms[2])

    burst, sustained, hbm, peak_kind = _peaks()
    achieved = flops / (fwd_ms * 1e-3) / 1e12
    result = {
        "metric": METRIC, "value": None, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": _config(wl),
        "stages_ms": {"permute_qkv": float(st_ms[0]), "estimate_mask": float(st_ms[1]),
                      "attn_fwd": fwd_ms},
        "kept_tiles": nnz, "tiles": tiles, "kept_fraction": nnz / tiles,
        "effective_flops_per_call": flops,
        "roofline": {"kernel": "asa sparse attention forward", "bound": "tensor",
                     "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                     "frac": achieved / burst, "traffic": _fwd_traffic_bytes(),
                     "peak_kind": f"{peak_kind} bf16 burst",
                     "frac_of_sustained": achieved / sustained},
        "clocks": clk,
    }
    per_step, names = ((None, "not counted (--no-launch-count)") if args.no_launch_count
                       else count_launches(torch, step))
    result["gpu_launches"] = per_step * args.steps if per_step is not None else None
    result["gpu_launches_how"] = (f"{per_step} kernels of this library per step, counted by "
                                  f"CUPTI (torch.profiler) over one untimed step, x steps"
                                  if per_step is not None else names)

    # ---- end to end through the public host-buffer call (asa_attention_host): pinned
    # raster Q, K, V in, raster O out, the library's copies pipelined against its
    # kernels; device time on the caller's stream, which the call joins at both ends
    qh, kh, vh = (x[n].contiguous().pin_memory() for n in ("q", "k", "v"))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    hws = asa.host_workspace(B, T, Hg, W, H, d)

    def host_call_ms(reps, chunk=0, workspace=hws):
        out = []
        for i in range(reps + 2):
            e0, e1 = ev(), ev()
            torch.cuda.synchronize()
            e0.record(stream)
            asa.asa_attention_host(qh, kh, vh, T, Hg, W, wl.tau, head_chunk=chunk, out=oh,
                                   workspace=workspace, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= 2:
                out.append(e0.elapsed_time(e1))
        return statistics.median(out)

    e_s = host_call_ms(args.e2e_steps) * 1e-3
    asa.asa_check_device_status()

    # whole job: max over ranks of each time, work summed over ranks
    if world > 1:
        (elapsed_ms, e_s), total_flops = combine_over_ranks(dist, dev, [elapsed_ms, e_s], flops)
    else:
        total_flops = float(flops)
    result["ms_per_step"] = elapsed_ms / args.steps
    result["value"] = total_flops * args.steps / (elapsed_ms * 1e-3) / 1e12
    nbytes = q.numel() * q.element_size()
    result["e2e"] = {"value": total_flops / e_s / 1e12, "unit": "TFLOP/s",
                     "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
                     "ms_per_call": e_s * 1e3, "timing": "CUDA events on the stream",
                     "call": "asa_attention_host (pinned host buffers, head chunks pipelined)"}

    if not args.no_extras:
        xclocks = ClockSampler(local)
        result["extras"] = extras(asa, wl, q, k, v, qp, kp, vp, mask, dev, stream)
        result["extras"]["clocks"] = xclocks.stop()
        # the host-buffer call by head chunk, and the unpipelined sequence (copy Q, K, V
        # in, device call, copy O out) for comparison
        by_chunk = {}
        for c in (1, 2, 3, 4, 6, 12):
            if c <= H:
                by_chunk[c] = host_call_ms(3, c, asa.host_workspace(B, T, Hg, W, H, d, 0, c))
        seq = []
        for i in range(5):
            e0, e1 = ev(), ev()
            torch.cuda.synchronize()
            e0.record(stream)
            qd, kd, vd = (t.to(dev, non_blocking=True) for t in (qh, kh, vh))
            o_d, _, _ = asa.asa_attention(qd, kd, vd, T, Hg, W, wl.tau)
            oh.copy_(o_d, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= 2:
                seq.append(e0.elapsed_time(e1))
        result["extras"]["host_call_ms_by_head_chunk"] = by_chunk
        result["extras"]["host_sequential_ms"] = statistics.median(seq)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        *setup, pimp0 = oracle_setup(wl, x, with_pimp=True)
        result["cpu_baseline"] = cpu_oracle_sample(wl, x, setup=tuple(setup))
        result["mask_rows"] = mask_rows_vs_oracle(wl, pimp0, setup[3], mask.row_ptr.cpu().numpy(),
                                                  mask.col_idx.cpu().numpy())
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_bwd_train_only(args, wl):
    """The training backward alone: Gilbert permute and mask of the workload, the
    training forward once, then `warmup` untimed and `steps` timed backward calls
    (CUDA events on the stream); one JSON line with its ms and effective TFLOP/s."""
    import torch
    from inputs import make_inputs
    from video_dit_dynamic_gilbert_b200 import asa
    dev = torch.device("cuda", 0)
    x = make_inputs(wl, with_dout=True)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "dout"))
    qp, kp, vp, dop = (asa.asa_gilbert_permute(t, wl.T, wl.Hg, wl.W) for t in (q, k, v, do))
    m = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    o, lse, o32 = asa.asa_sparse_attn_fwd_train(qp, kp, vp, m, global_window=wl.global_window)
    B, H, N, d = qp.shape
    ws = asa.bwd_workspace(B, H, N, d, dev, wl.global_window)
    outs = tuple(torch.empty_like(qp) for _ in range(3))
    call = lambda: asa.asa_sparse_attn_bwd_train(qp, kp, vp, o32, dop, lse, m,
                                                 global_window=wl.global_window, workspace=ws,
                                                 outs=outs)
    for _ in range(args.warmup):
        call()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(args.steps):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    asa.asa_check_device_status()
    ms = a.elapsed_time(b) / args.steps
    flops, _, _ = _kept_tile_flops(m.row_ptr.cpu().numpy(), m.col_idx.cpu().numpy(), B, H, N, d)
    print(json.dumps({"stage": "bwd_train", "workload": wl.name, "ms": ms,
                      "effective_tflops": 2.5 * flops / ms / 1e9, "steps": args.steps,
                      "warmup": args.warmup}))


def extras(asa, wl, q, k, v, qp, kp, vp, mask, dev, stream):
    """Context measured after the timed region: dense attention on the same GPU (our
    kernel with every tile kept, and torch SDPA), ASA_G and the backward."""
    import torch
    B, H, N, d = qp.shape

    def timeit(fn, reps=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    dense_flops = 4 * d * N * N * B * H
    p = torch.ones((B, H, -(-N // 128), -(-N // 128)), dtype=torch.float32, device=dev)
    full = asa.asa_build_mask(p, N, 1.0, transposed=True)
    ours_dense = timeit(lambda: asa.asa_sparse_attn_fwd(qp, kp, vp, full))
    sdpa = timeit(lambda: torch.nn.functional.scaled_dot_product_attention(qp, kp, vp))
    tmask = asa.asa_estimate_mask(qp, kp, wl.tau, transposed=True)
    g_ms = timeit(lambda: asa.asa_sparse_attn_fwd(qp, kp, vp, tmask, global_window=64))
    o, lse = asa.asa_sparse_attn_fwd(qp, kp, vp, tmask)
    dout = torch.randn_like(qp)
    bwd_ms = timeit(lambda: asa.asa_sparse_attn_bwd(qp, kp, vp, o, dout, lse, tmask), reps=5)
    bwd_dfo_ms = timeit(lambda: asa.asa_sparse_attn_bwd(qp, kp, vp, o, dout, lse, tmask,
                                                        d_from_o=True), reps=5)
    flops, _, _ = _kept_tile_flops(tmask.row_ptr.cpu().numpy(), tmask.col_idx.cpu().numpy(),
                                   B, H, N, d)
    # the training pair: forward with the fp32 output, backward taking D from it
    tws = asa.fwd_train_workspace(B, H, N, d, 0, dev)
    t_o, t_lse = torch.empty_like(qp), torch.empty((B, H, N), dtype=torch.float32, device=dev)
    t_o32 = torch.empty(qp.shape, dtype=torch.float32, device=dev)
    fwd_train_ms = timeit(lambda: asa.asa_sparse_attn_fwd_train(qp, kp, vp, tmask, workspace=tws,
                                                                out=t_o, lse=t_lse, out32=t_o32))
    bws = asa.bwd_workspace(B, H, N, d, dev)
    t_grads = tuple(torch.empty_like(qp) for _ in range(3))
    bwd_train_ms = timeit(lambda: asa.asa_sparse_attn_bwd_train(qp, kp, vp, t_o32, dout, t_lse, tmask,
                                                                workspace=bws, outs=t_grads), reps=5)
    # ASA_G backward (n = 64) on the same mask
    og, lg = asa.asa_sparse_attn_fwd(qp, kp, vp, tmask, global_window=64)
    bwd_g_ms = timeit(lambda: asa.asa_sparse_attn_bwd(qp, kp, vp, og, dout, lg, tmask,
                                                      global_window=64), reps=5)
    G = -(-N // 64)
    # query pruning with token filling (r = 0.5, windows of 8) on the same mask
    pr = asa.asa_prune_queries(qp, 0.5, 8)
    pmws = asa._workspace(asa.lib().asa_prune_mask_workspace_size(B, H, N, pr.pack), dev)
    ptm = asa.asa_prune_mask(tmask, pr.pack, workspace=pmws)
    pws = asa.fwd_pruned_workspace(B, H, N, d, pr.pack, 0, dev)
    po, plse = torch.empty_like(qp), torch.empty((B, H, N), dtype=torch.float32, device=dev)
    prune_ms = timeit(lambda: asa.asa_prune_queries(qp, 0.5, 8, out=pr))
    pmask_ms = timeit(lambda: asa.asa_prune_mask(tmask, pr.pack, workspace=pmws, out=ptm))
    pfwd_ms = timeit(lambda: asa.asa_sparse_attn_fwd_pruned(pr, kp, vp, ptm, workspace=pws,
                                                             out=po, lse=plse))
    fwd_ms = timeit(lambda: asa.asa_sparse_attn_fwd(qp, kp, vp, tmask))
    pbws = asa.bwd_pruned_workspace(B, H, N, d, pr.pack, dev)
    pgrads = tuple(torch.empty_like(qp) for _ in range(3))
    pbwd_ms = timeit(lambda: asa.asa_sparse_attn_bwd_pruned(pr, kp, vp, dout, plse, ptm,
                                                            workspace=pbws, outs=pgrads), reps=5)
    pflops, nkept = _pruned_flops(tmask.row_ptr.cpu().numpy(), tmask.col_idx.cpu().numpy(),
                                  pr.src_pos.cpu().numpy(), B, H, N, d)
    union = int(ptm.nnz.item())
    asa.asa_check_device_status()
    return {
        "pruned_r0.5_w8": {
            "pack": pr.pack, "kept_queries": nkept, "of": B * H * N,
            "tile_entries": union, "block_entries": int(tmask.nnz.item()),
            "prune_ms": prune_ms, "prune_mask_ms": pmask_ms, "fwd_ms": pfwd_ms,
            "fwd_effective_tflops": pflops / pfwd_ms / 1e9,
            "unpruned_fwd_ms": fwd_ms,
            "bwd_ms": pbwd_ms, "unpruned_bwd_ms": bwd_ms,
            "bwd_effective_tflops": 2.5 * pflops / pbwd_ms / 1e9,
            "speedup_total": fwd_ms / (prune_ms + pmask_ms + pfwd_ms),
        },
        "dense_ours_fwd_ms": ours_dense, "dense_ours_tflops": dense_flops / ours_dense / 1e9,
        "dense_torch_sdpa_ms": sdpa, "dense_torch_sdpa_tflops": dense_flops / sdpa / 1e9,
        "asa_g_fwd_ms_n64": g_ms,
        "asa_g_fwd_tflops": (flops + 4 * d * N * G * B * H) / g_ms / 1e9,
        "bwd_ms": bwd_ms, "bwd_tflops": 2.5 * flops / bwd_ms / 1e9,
        "bwd_d_from_o_ms": bwd_dfo_ms, "bwd_d_from_o_tflops": 2.5 * flops / bwd_dfo_ms / 1e9,
        "fwd_train_ms": fwd_train_ms, "fwd_train_tflops": flops / fwd_train_ms / 1e9,
        "bwd_train_ms": bwd_train_ms, "bwd_train_tflops": 2.5 * flops / bwd_train_ms / 1e9,
        "asa_g_bwd_ms_n64": bwd_g_ms,
        "asa_g_bwd_tflops": 2.5 * (flops + 4 * d * N * G * B * H) / bwd_g_ms / 1e9,
    }


if __name__ == "__main__":
    main()
