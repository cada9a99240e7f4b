"""Shared helpers for the GPU parity tests (CUDA path vs the fp64 oracle)."""
import numpy as np
import torch

import mask_report
import oracle
from video_dit_dynamic_gilbert_b200 import asa

# Tolerances for floating-point outputs (bf16 in, fp32 accumulate).
MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_ABS = 1e-3   # LSE is fp32 from bf16 operands; its error is ~1e-5


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_close(out, ref, max_abs=MAX_ABS, rel_l2=REL_L2, what=""):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert out.shape == ref.shape, (what, out.shape, ref.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref).max() if out.size else 0.0
    rel = np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err <= max_abs, f"{what}: max-abs {err:.3e} > {max_abs}"
    assert rel <= rel_l2, f"{what}: rel-L2 {rel:.3e} > {rel_l2}"
    return err, rel


def check_close_ulp(out, ref, rel_l2=REL_L2, what=""):
    """The bars for gradients with large entries: |out - ref| <= 2e-2 + 2^-8 |ref|
    elementwise (the fixed bar plus one bf16 unit in the last place of the reference:
    the kernels' single bf16 rounding of each output alone reaches 2^-9 |ref|), and
    the unchanged rel-L2 bar."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert out.shape == ref.shape, (what, out.shape, ref.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    excess = np.abs(out - ref) - (MAX_ABS + 2.0 ** -8 * np.abs(ref))
    worst = float(excess.max()) if out.size else -1.0
    assert worst <= 0.0, f"{what}: max-abs exceeds 2e-2 + 2^-8 |ref| by {worst:.3e}"
    rel = np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= rel_l2, f"{what}: rel-L2 {rel:.3e} > {rel_l2}"
    return rel


def mask_from_csr(bm: asa.BlockMask) -> np.ndarray:
    rp = bm.row_ptr.cpu().numpy().astype(np.int64)
    ci = bm.col_idx.cpu().numpy().astype(np.int64)
    nb = bm.nb
    rows = bm.B * bm.H * nb
    m = np.zeros((rows, nb), dtype=bool)
    for r in range(rows):
        cols = ci[rp[r]:rp[r + 1]]
        assert (np.diff(cols) > 0).all(), "col_idx not strictly ascending"
        assert ((cols >= 0) & (cols < nb)).all()
        m[r, cols] = True
    return m.reshape(bm.B, bm.H, nb, nb)


def check_transposed(bm: asa.BlockMask, mask: np.ndarray) -> None:
    tp = bm.col_ptr_t.cpu().numpy().astype(np.int64)
    ti = bm.row_idx_t.cpu().numpy().astype(np.int64)
    rp_ref, ci_ref = oracle.mask_to_csr_transposed(mask)
    np.testing.assert_array_equal(tp, rp_ref)
    np.testing.assert_array_equal(ti[:tp[-1]], ci_ref)


def upload_mask(mask: np.ndarray, N: int, device="cuda") -> asa.BlockMask:
    """An oracle block mask as the library's CSR (and transposed CSR)."""
    B, H = mask.shape[:2]
    rp, ci = oracle.mask_to_csr(mask)
    tp, ti = oracle.mask_to_csr_transposed(mask)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32) if len(a) else
                                     np.zeros(1, np.int32)).to(device)
    return asa.BlockMask(i32(rp), i32(ci), i32(np.array([rp[-1]])), i32(tp), i32(ti), B, H, N)


def compare_masks(gpu_mask: np.ndarray, ref_mask: np.ndarray, marginal: np.ndarray,
                  pimp: np.ndarray, tau: float, what: str = ""):
    """GPU mask rows against the oracle's.  A row may differ only where the oracle marks
    it marginal, and every row must be a legal cut of the oracle's P_imp
    (oracle.legal_mask_rows: a leading set up to near-ties, one block from the exact
    cut at most, reaching tau within 1e-4 and minimal within 1e-4).  The counts are
    recorded for the run's summary; returns (n_rows_differing, n_marginal)."""
    diff = (gpu_mask != ref_mask).any(axis=-1)
    bad = diff & ~marginal
    assert not bad.any(), (f"{what}: {int(bad.sum())} non-marginal rows differ, "
                           f"e.g. {np.argwhere(bad)[:5]}")
    legal = oracle.legal_mask_rows(pimp, gpu_mask, tau)
    assert legal.all(), (f"{what}: {int((~legal).sum())} rows are not a legal cut, "
                         f"e.g. {np.argwhere(~legal)[:5]}")
    mask_report.record(what or "mask", diff.sum(), marginal.sum(), diff.size)
    print(f"{what}: mask rows {int(diff.sum())} differ, {int(marginal.sum())} marginal, "
          f"of {diff.size}")
    return int(diff.sum()), int(marginal.sum())
