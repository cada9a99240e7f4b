"""Thin Python binding of libasa.so (include/asa.h), same names as the C ABI.

Marshalling only: every step of the hot path runs in the library's CUDA kernels.
PyTorch provides device memory (outputs, workspaces) and the current stream.
There is no CPU fallback: a missing or unloadable library raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libasa.so")

ASA_OK = 0
ASA_ERR_INVALID_ARG = -1
ASA_ERR_UNSUPPORTED = -2
ASA_ERR_WORKSPACE = -3
ASA_ERR_CUDA = -4
ASA_ERR_TIMEOUT = -5
BLOCK = 128
SAMPLES = 16

_c_int, _c_size, _c_float, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
_SIGNATURES = {
    "asa_version": ([], _c_int),
    "asa_last_error_string": ([], ctypes.c_char_p),
    "asa_gilbert_index": ([_c_int, _c_int, _c_int, _vp], _c_int),
    "asa_gilbert_permute": ([_vp, _vp] + [_c_int] * 6 + [_vp], _c_int),
    "asa_gilbert_permute3": ([_vp] * 6 + [_c_int] * 6 + [_vp], _c_int),
    "asa_unpermute": ([_vp, _vp] + [_c_int] * 6 + [_vp], _c_int),
    "asa_estimate_mask_workspace_size": ([_c_int] * 3, _c_size),
    "asa_estimate": ([_vp, _vp] + [_c_int] * 6 + [_vp, _c_size, _vp, _vp], _c_int),
    "asa_estimate_noalloc": ([_vp, _vp] + [_c_int] * 6 + [_vp, _vp], _c_int),
    "asa_build_mask": ([_vp, _c_int, _c_int, _c_int, _c_float, _vp, _c_size] + [_vp] * 6, _c_int),
    "asa_estimate_mask": ([_vp, _vp] + [_c_int] * 6 + [_c_float, _vp, _c_size] + [_vp] * 6, _c_int),
    "asa_global_pool": ([_vp, _vp] + [_c_int] * 5 + [_vp], _c_int),
    "asa_global_pool_kv": ([_vp] * 4 + [_c_int] * 5 + [_vp], _c_int),
    "asa_fwd_workspace_size": ([_c_int] * 5, _c_size),
    "asa_sparse_attn_fwd": ([_vp] * 5 + [_c_int] * 6 + [_vp, _c_size, _vp, _vp, _vp], _c_int),
    "asa_sparse_attn_fwd_raster": ([_vp] * 5 + [_c_int] * 8 + [_vp, _c_size, _vp, _vp, _vp], _c_int),
    "asa_fwd_train_workspace_size": ([_c_int] * 5, _c_size),
    "asa_sparse_attn_fwd_train": ([_vp] * 5 + [_c_int] * 6 + [_vp, _c_size, _vp, _vp, _vp, _vp],
                                  _c_int),
    "asa_bwd_workspace_size": ([_c_int] * 5, _c_size),
    "asa_sparse_attn_bwd_train": ([_vp] * 10 + [_c_int] * 6 + [_vp, _c_size] + [_vp] * 4, _c_int),
    "asa_sparse_attn_bwd": ([_vp] * 10 + [_c_int] * 6 + [_vp, _c_size] + [_vp] * 4, _c_int),
    "asa_sparse_attn_bwd_d_from_o": ([_vp] * 10 + [_c_int] * 6 + [_vp, _c_size] + [_vp] * 4,
                                     _c_int),
    "asa_build_mask_stat": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_size] + [_vp] * 6, _c_int),
    "asa_prune_pack": ([_c_float, _c_int], _c_int),
    "asa_prune_rows": ([_c_int, _c_int], _c_int),
    "asa_prune_queries": ([_vp] + [_c_int] * 5 + [_c_float, _c_int, _c_int] + [_vp] * 4, _c_int),
    "asa_prune_mask_workspace_size": ([_c_int] * 4, _c_size),
    "asa_prune_mask": ([_vp, _vp] + [_c_int] * 4 + [_vp, _c_size] + [_vp] * 5, _c_int),
    "asa_fwd_pruned_workspace_size": ([_c_int] * 6, _c_size),
    "asa_sparse_attn_fwd_pruned": ([_vp] * 7 + [_c_int] * 7 + [_vp, _c_size, _vp, _vp, _vp], _c_int),
    "asa_bwd_pruned_workspace_size": ([_c_int] * 6, _c_size),
    "asa_sparse_attn_bwd_pruned": ([_vp] * 10 + [_c_int] * 7 + [_vp, _c_size] + [_vp] * 4, _c_int),
    "asa_attention_host_workspace_size": ([_c_int] * 8, _c_size),
    "asa_attention_host": ([_vp] * 3 + [_c_int] * 6 + [_c_float, _c_int, _c_int, _vp, _c_size, _vp,
                                                      _vp], _c_int),
    "asa_seqpar_pack": ([_vp, _vp] + [_c_int] * 4 + [_vp, _c_int, _vp], _c_int),
    "asa_seqpar_unpack": ([_vp, _vp] + [_c_int] * 4 + [_vp, _c_int, _vp], _c_int),
    "asa_seqpar_permute3": ([_vp] * 6 + [_c_int] * 6 + [_vp, _c_int, _vp], _c_int),
    "asa_seqpar_unpermute": ([_vp, _vp] + [_c_int] * 6 + [_vp, _c_int, _vp], _c_int),
    "asa_check_device_status": ([_vp], _c_int),
    "asa_selftest_wait_timeout": ([ctypes.c_longlong, _vp], _c_int),
    "asa_shutdown": ([], None),
}

_lib = None


class AsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"ASA error {code}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    """The loaded libasa.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m video_dit_dynamic_gilbert_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(rc: int) -> None:
    if rc != ASA_OK:
        raise AsaError(rc, lib().asa_last_error_string().decode())


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _bf16_cuda(name: str, t: torch.Tensor, ndim: int = 4) -> None:
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == ndim):
        raise ValueError(f"{name} must be a contiguous {ndim}-D bf16 CUDA tensor")


def _ws_bytes(workspace) -> int:
    return 0 if workspace is None else workspace.numel()


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def nblocks(N: int) -> int:
    return -(-N // BLOCK)


# ----------------------------------------------------------------------- Preprocessing

def asa_gilbert_index(T: int, Hg: int, W: int) -> np.ndarray:
    """Host Gilbert table: perm[i] = raster index of curve position i."""
    out = np.empty(T * Hg * W, dtype=np.int32)
    _check(lib().asa_gilbert_index(T, Hg, W, out.ctypes.data_as(ctypes.c_void_p)))
    return out


def asa_gilbert_permute(x: torch.Tensor, T: int, Hg: int, W: int, out=None, stream=None):
    """x [B, N, H, d] raster -> xp [B, H, N, d] Gilbert order."""
    _bf16_cuda("x", x)
    B, N, H, d = x.shape
    if out is None:
        out = torch.empty((B, H, N, d), dtype=x.dtype, device=x.device)
    _check(lib().asa_gilbert_permute(_ptr(x), _ptr(out), B, T, Hg, W, H, d, _stream(stream)))
    return out


def asa_gilbert_permute3(q, k, v, T: int, Hg: int, W: int, outs=None, stream=None):
    for n_, t in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n_, t)
    B, N, H, d = q.shape
    if outs is None:
        outs = tuple(torch.empty((B, H, N, d), dtype=q.dtype, device=q.device) for _ in range(3))
    _check(lib().asa_gilbert_permute3(_ptr(q), _ptr(k), _ptr(v), *(_ptr(o) for o in outs),
                                      B, T, Hg, W, H, d, _stream(stream)))
    return outs


def asa_unpermute(xp: torch.Tensor, T: int, Hg: int, W: int, out=None, stream=None):
    """xp [B, H, N, d] Gilbert order -> x [B, N, H, d] raster."""
    _bf16_cuda("xp", xp)
    B, H, N, d = xp.shape
    if out is None:
        out = torch.empty((B, N, H, d), dtype=xp.dtype, device=xp.device)
    _check(lib().asa_unpermute(_ptr(xp), _ptr(out), B, T, Hg, W, H, d, _stream(stream)))
    return out


# ----------------------------------------------------------------------- Steps 1, 2.1

@dataclass
class BlockMask:
    """CSR of kept key blocks per query block (and its transpose), device int32."""
    row_ptr: torch.Tensor
    col_idx: torch.Tensor
    nnz: torch.Tensor
    col_ptr_t: torch.Tensor | None
    row_idx_t: torch.Tensor | None
    B: int
    H: int
    N: int

    @property
    def nb(self) -> int:
        return nblocks(self.N)


def estimate_mask_workspace(B: int, H: int, N: int, device) -> torch.Tensor:
    return _workspace(lib().asa_estimate_mask_workspace_size(B, H, N), device)


def _alloc_mask(B, H, N, device, transposed):
    nb = nblocks(N)
    rows = B * H * nb
    cap = rows * nb
    z = dict(dtype=torch.int32, device=device)
    return BlockMask(torch.empty(rows + 1, **z), torch.empty(max(cap, 1), **z), torch.empty(1, **z),
                     torch.empty(rows + 1, **z) if transposed else None,
                     torch.empty(max(cap, 1), **z) if transposed else None, B, H, N)


def asa_estimate(qp: torch.Tensor, kp: torch.Tensor, workspace=None, out=None, stream=None):
    """P_imp [B, H, nb, nb] fp32 from the sampled tokens (Step 1)."""
    _bf16_cuda("qp", qp)
    _bf16_cuda("kp", kp)
    B, H, N, d = qp.shape
    nb = nblocks(N)
    if workspace is None:
        workspace = estimate_mask_workspace(B, H, N, qp.device)
    if out is None:
        out = torch.empty((B, H, nb, nb), dtype=torch.float32, device=qp.device)
    _check(lib().asa_estimate(_ptr(qp), _ptr(kp), B, H, N, d, BLOCK, SAMPLES, _ptr(workspace),
                              _ws_bytes(workspace), _ptr(out), _stream(stream)))
    return out


def asa_estimate_noalloc(qp: torch.Tensor, kp: torch.Tensor, out=None, stream=None):
    """asa_estimate with its scratch in the library's fixed device array (no workspace,
    no allocation in the library; for callers that cannot allocate device memory).
    Calls that overlap on the GPU share that array and race: serialise them."""
    _bf16_cuda("qp", qp)
    _bf16_cuda("kp", kp)
    B, H, N, d = qp.shape
    nb = nblocks(N)
    if out is None:
        out = torch.empty((B, H, nb, nb), dtype=torch.float32, device=qp.device)
    _check(lib().asa_estimate_noalloc(_ptr(qp), _ptr(kp), B, H, N, d, BLOCK, SAMPLES, _ptr(out),
                                      _stream(stream)))
    return out


def asa_build_mask(p_imp: torch.Tensor, N: int, tau: float, transposed: bool = True,
                   workspace=None, mask: BlockMask | None = None, stream=None) -> BlockMask:
    """Kept-block CSR from P_imp (Step 2.1)."""
    if not (p_imp.is_cuda and p_imp.dtype == torch.float32 and p_imp.is_contiguous()):
        raise ValueError("p_imp must be a contiguous fp32 CUDA tensor")
    B, H = p_imp.shape[:2]
    if workspace is None:
        workspace = estimate_mask_workspace(B, H, N, p_imp.device)
    m = mask or _alloc_mask(B, H, N, p_imp.device, transposed)
    _check(lib().asa_build_mask(_ptr(p_imp), B, H, N, float(tau), _ptr(workspace), _ws_bytes(workspace),
                                _ptr(m.row_ptr), _ptr(m.col_idx), _ptr(m.nnz), _ptr(m.col_ptr_t),
                                _ptr(m.row_idx_t), _stream(stream)))
    return m


def asa_build_mask_stat(p_imp: torch.Tensor, N: int, k_target: int, transposed: bool = True,
                        workspace=None, mask: BlockMask | None = None, stream=None) -> BlockMask:
    """Kept-block CSR by the statistical threshold (about k_target blocks per row)."""
    if not (p_imp.is_cuda and p_imp.dtype == torch.float32 and p_imp.is_contiguous()):
        raise ValueError("p_imp must be a contiguous fp32 CUDA tensor")
    B, H = p_imp.shape[:2]
    if workspace is None:
        workspace = estimate_mask_workspace(B, H, N, p_imp.device)
    m = mask or _alloc_mask(B, H, N, p_imp.device, transposed)
    _check(lib().asa_build_mask_stat(_ptr(p_imp), B, H, N, int(k_target), _ptr(workspace),
                                     _ws_bytes(workspace), _ptr(m.row_ptr), _ptr(m.col_idx),
                                     _ptr(m.nnz), _ptr(m.col_ptr_t), _ptr(m.row_idx_t),
                                     _stream(stream)))
    return m


def asa_estimate_mask(qp: torch.Tensor, kp: torch.Tensor, tau: float, transposed: bool = True,
                      workspace=None, mask: BlockMask | None = None, stream=None) -> BlockMask:
    """Steps 1 + 2.1 in one call."""
    _bf16_cuda("qp", qp)
    _bf16_cuda("kp", kp)
    B, H, N, d = qp.shape
    if workspace is None:
        workspace = estimate_mask_workspace(B, H, N, qp.device)
    m = mask or _alloc_mask(B, H, N, qp.device, transposed)
    _check(lib().asa_estimate_mask(_ptr(qp), _ptr(kp), B, H, N, d, BLOCK, SAMPLES, float(tau),
                                   _ptr(workspace), _ws_bytes(workspace), _ptr(m.row_ptr),
                                   _ptr(m.col_idx), _ptr(m.nnz), _ptr(m.col_ptr_t),
                                   _ptr(m.row_idx_t), _stream(stream)))
    return m


# ----------------------------------------------------------------------- Step 2.2

def asa_global_pool(xp: torch.Tensor, n: int, out=None, stream=None):
    _bf16_cuda("xp", xp)
    B, H, N, d = xp.shape
    G = -(-N // n)
    if out is None:
        out = torch.empty((B, H, G, d), dtype=xp.dtype, device=xp.device)
    _check(lib().asa_global_pool(_ptr(xp), _ptr(out), B, H, N, d, n, _stream(stream)))
    return out


def asa_global_pool_kv(kp: torch.Tensor, vp: torch.Tensor, n: int, outs=None, stream=None):
    """The global tokens of K and V in one launch: (Kg, Vg) [B, H, ceil(N/n), d] bf16."""
    _bf16_cuda("kp", kp)
    _bf16_cuda("vp", vp)
    if kp.shape != vp.shape:
        raise ValueError("kp and vp must have the same shape")
    B, H, N, d = kp.shape
    G = -(-N // n)
    if outs is None:
        outs = tuple(torch.empty((B, H, G, d), dtype=torch.bfloat16, device=kp.device)
                     for _ in range(2))
    _check(lib().asa_global_pool_kv(_ptr(kp), _ptr(vp), _ptr(outs[0]), _ptr(outs[1]), B, H, N, d,
                                    n, _stream(stream)))
    return outs


def fwd_workspace(B, H, N, d, global_window, device):
    return _workspace(lib().asa_fwd_workspace_size(B, H, N, d, global_window), device)


def asa_sparse_attn_fwd(qp, kp, vp, mask: BlockMask, global_window: int = 0, workspace=None,
                        out=None, lse=None, stream=None):
    """O [B, H, N, d] bf16 and natural-log LSE [B, H, N] fp32 over the kept tiles."""
    for n_, t in (("qp", qp), ("kp", kp), ("vp", vp)):
        _bf16_cuda(n_, t)
    B, H, N, d = qp.shape
    if workspace is None:
        workspace = fwd_workspace(B, H, N, d, global_window, qp.device)
    if out is None:
        out = torch.empty_like(qp)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=qp.device)
    _check(lib().asa_sparse_attn_fwd(_ptr(qp), _ptr(kp), _ptr(vp), _ptr(mask.row_ptr),
                                     _ptr(mask.col_idx), B, H, N, d, BLOCK, global_window,
                                     _ptr(workspace), _ws_bytes(workspace),
                                     _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def asa_sparse_attn_fwd_raster(qp, kp, vp, mask: BlockMask, T: int, Hg: int, W: int,
                               global_window: int = 0, workspace=None, out=None, lse=None,
                               stream=None):
    """asa_sparse_attn_fwd with the inverse Gilbert permutation fused into its store:
    O in raster layout [B, N, H, d] bf16 (as asa_unpermute returns it) and LSE
    [B, H, N] fp32 in Gilbert order."""
    for n_, t in (("qp", qp), ("kp", kp), ("vp", vp)):
        _bf16_cuda(n_, t)
    B, H, N, d = qp.shape
    if workspace is None:
        workspace = fwd_workspace(B, H, N, d, global_window, qp.device)
    if out is None:
        out = torch.empty((B, N, H, d), dtype=qp.dtype, device=qp.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=qp.device)
    _check(lib().asa_sparse_attn_fwd_raster(_ptr(qp), _ptr(kp), _ptr(vp), _ptr(mask.row_ptr),
                                            _ptr(mask.col_idx), B, T, Hg, W, H, d, BLOCK,
                                            global_window, _ptr(workspace), _ws_bytes(workspace),
                                            _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def fwd_train_workspace(B, H, N, d, global_window, device):
    return _workspace(lib().asa_fwd_train_workspace_size(B, H, N, d, global_window), device)


def asa_sparse_attn_fwd_train(qp, kp, vp, mask: BlockMask, global_window: int = 0,
                              workspace=None, out=None, lse=None, out32=None, stream=None):
    """The training forward: O [B, H, N, d] bf16, LSE [B, H, N] fp32 and the fp32 O
    [B, H, N, d] that asa_sparse_attn_bwd_train takes D from (P V in fp16)."""
    for n_, t in (("qp", qp), ("kp", kp), ("vp", vp)):
        _bf16_cuda(n_, t)
    B, H, N, d = qp.shape
    if workspace is None:
        workspace = fwd_train_workspace(B, H, N, d, global_window, qp.device)
    if out is None:
        out = torch.empty_like(qp)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=qp.device)
    if out32 is None:
        out32 = torch.empty(qp.shape, dtype=torch.float32, device=qp.device)
    _check(lib().asa_sparse_attn_fwd_train(_ptr(qp), _ptr(kp), _ptr(vp), _ptr(mask.row_ptr),
                                           _ptr(mask.col_idx), B, H, N, d, BLOCK, global_window,
                                           _ptr(workspace), _ws_bytes(workspace), _ptr(out),
                                           _ptr(lse), _ptr(out32), _stream(stream)))
    return out, lse, out32


def bwd_workspace(B, H, N, d, device, global_window: int = 0):
    return _workspace(lib().asa_bwd_workspace_size(B, H, N, d, global_window), device)


def asa_sparse_attn_bwd(qp, kp, vp, o, dout, lse, mask: BlockMask, global_window: int = 0,
                        workspace=None, outs=None, stream=None, d_from_o: bool = False):
    """dQ, dK, dV [B, H, N, d] bf16 under the fixed mask (ASA; ASA_G with the forward's
    global_window).  d_from_o=True takes D = rowsum(dO * O) from the bf16 O instead of
    the exact pass (faster, ~3e-3 more relative error on dQ and dK)."""
    for n_, t in (("qp", qp), ("kp", kp), ("vp", vp), ("o", o), ("dout", dout)):
        _bf16_cuda(n_, t)
    if mask.col_ptr_t is None:
        raise ValueError("the backward needs the transposed CSR (transposed=True)")
    B, H, N, d = qp.shape
    if workspace is None:
        workspace = bwd_workspace(B, H, N, d, qp.device, global_window)
    if outs is None:
        outs = tuple(torch.empty_like(qp) for _ in range(3))
    fn = lib().asa_sparse_attn_bwd_d_from_o if d_from_o else lib().asa_sparse_attn_bwd
    _check(fn(_ptr(qp), _ptr(kp), _ptr(vp), _ptr(o), _ptr(dout), _ptr(lse), _ptr(mask.row_ptr),
              _ptr(mask.col_idx), _ptr(mask.col_ptr_t), _ptr(mask.row_idx_t), B, H, N, d, BLOCK,
              global_window, _ptr(workspace), _ws_bytes(workspace), *(_ptr(t) for t in outs),
              _stream(stream)))
    return outs


def asa_sparse_attn_bwd_train(qp, kp, vp, o32, dout, lse, mask: BlockMask,
                              global_window: int = 0, workspace=None, outs=None, stream=None):
    """dQ, dK, dV after asa_sparse_attn_fwd_train: D = rowsum(dO * O) from its fp32 O
    (no pass of its own over the kept tiles); lse from the same forward."""
    for n_, t in (("qp", qp), ("kp", kp), ("vp", vp), ("dout", dout)):
        _bf16_cuda(n_, t)
    if o32.dtype != torch.float32 or not o32.is_cuda or not o32.is_contiguous():
        raise ValueError("o32 must be a contiguous fp32 CUDA tensor")
    if mask.col_ptr_t is None:
        raise ValueError("the backward needs the transposed CSR (transposed=True)")
    B, H, N, d = qp.shape
    if tuple(o32.shape) != (B, H, N, d):
        raise ValueError(f"o32 shape {tuple(o32.shape)} != {(B, H, N, d)}")
    if workspace is None:
        workspace = bwd_workspace(B, H, N, d, qp.device, global_window)
    if outs is None:
        outs = tuple(torch.empty_like(qp) for _ in range(3))
    _check(lib().asa_sparse_attn_bwd_train(
        _ptr(qp), _ptr(kp), _ptr(vp), _ptr(o32), _ptr(dout), _ptr(lse), _ptr(mask.row_ptr),
        _ptr(mask.col_idx), _ptr(mask.col_ptr_t), _ptr(mask.row_idx_t), B, H, N, d, BLOCK,
        global_window, _ptr(workspace), _ws_bytes(workspace), *(_ptr(t) for t in outs),
        _stream(stream)))
    return outs


# ----------------------------------------------------------------------- query pruning (BSA)

@dataclass
class QueryPrune:
    """Kept queries packed into 128-row tiles (q_s [B, H, Ns, d]) and, per token, the
    permuted position (src_pos) and compact row (src_row) whose output it takes."""
    q_s: torch.Tensor
    src_pos: torch.Tensor
    src_row: torch.Tensor
    pack: int
    r: float
    window: int
    N: int

    @property
    def Ns(self) -> int:
        return self.q_s.shape[2]


@dataclass
class TileMask:
    """CSR over the packed query tiles: the union of the tile's blocks' kept key blocks,
    with the 32-row lane quarters that see each entry."""
    tile_ptr: torch.Tensor
    tile_col: torch.Tensor
    tile_quarters: torch.Tensor
    nnz: torch.Tensor
    pack: int


def asa_prune_pack(r: float, window: int) -> int:
    """Largest tile packing (1, 2 or 4 blocks per 128-row tile) this r and window allow."""
    rc = lib().asa_prune_pack(float(r), int(window))
    _check(min(rc, 0))
    return rc


def asa_prune_rows(N: int, pack: int) -> int:
    rc = lib().asa_prune_rows(int(N), int(pack))
    _check(min(rc, 0))
    return rc


def asa_prune_queries(qp: torch.Tensor, r: float, window: int = 8, pack: int = 0,
                      out: QueryPrune | None = None, stream=None) -> QueryPrune:
    """Query pruning (BSA): keep every window centre and the queries least similar to
    their centre, K = max(ceil(r L), windows) per block; pack = 0 takes the largest
    packing allowed."""
    _bf16_cuda("qp", qp)
    B, H, N, d = qp.shape
    if pack == 0:
        pack = asa_prune_pack(r, window)
    Ns = asa_prune_rows(N, pack)
    if out is None:
        z = dict(dtype=torch.int32, device=qp.device)
        out = QueryPrune(torch.empty((B, H, Ns, d), dtype=qp.dtype, device=qp.device),
                         torch.empty((B, H, N), **z), torch.empty((B, H, N), **z), pack,
                         float(r), int(window), N)
    _check(lib().asa_prune_queries(_ptr(qp), B, H, N, d, BLOCK, float(r), int(window), pack,
                                   _ptr(out.q_s), _ptr(out.src_pos), _ptr(out.src_row),
                                   _stream(stream)))
    return out


def asa_prune_mask(mask: BlockMask, pack: int, workspace=None, out: TileMask | None = None,
                   stream=None) -> TileMask:
    """Tile CSR of the packed queries from a block mask."""
    B, H, N = mask.B, mask.H, mask.N
    dev = mask.row_ptr.device
    if workspace is None:
        workspace = _workspace(lib().asa_prune_mask_workspace_size(B, H, N, pack), dev)
    if out is None:
        tiles = B * H * -(-nblocks(N) // pack)
        cap = mask.col_idx.numel()
        z = dict(dtype=torch.int32, device=dev)
        out = TileMask(torch.empty(tiles + 1, **z), torch.empty(cap, **z),
                       torch.empty(cap, dtype=torch.uint8, device=dev), torch.empty(1, **z), pack)
    _check(lib().asa_prune_mask(_ptr(mask.row_ptr), _ptr(mask.col_idx), B, H, N, pack,
                                _ptr(workspace), _ws_bytes(workspace), _ptr(out.tile_ptr),
                                _ptr(out.tile_col), _ptr(out.tile_quarters), _ptr(out.nnz),
                                _stream(stream)))
    return out


def fwd_pruned_workspace(B, H, N, d, pack, global_window, device):
    return _workspace(lib().asa_fwd_pruned_workspace_size(B, H, N, d, pack, global_window), device)


def asa_sparse_attn_fwd_pruned(prune: QueryPrune, kp, vp, tmask: TileMask, global_window: int = 0,
                               workspace=None, out=None, lse=None, stream=None):
    """Forward for the kept queries only, then token filling: O [B, H, N, d] bf16 and
    LSE [B, H, N] fp32 (a pruned token takes its centre's row)."""
    for n_, t in (("kp", kp), ("vp", vp)):
        _bf16_cuda(n_, t)
    B, H, N, d = kp.shape
    if workspace is None:
        workspace = fwd_pruned_workspace(B, H, N, d, prune.pack, global_window, kp.device)
    if out is None:
        out = torch.empty_like(kp)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=kp.device)
    _check(lib().asa_sparse_attn_fwd_pruned(
        _ptr(prune.q_s), _ptr(kp), _ptr(vp), _ptr(tmask.tile_ptr), _ptr(tmask.tile_col),
        _ptr(tmask.tile_quarters), _ptr(prune.src_row), B, H, N, d, BLOCK, prune.pack,
        global_window, _ptr(workspace), _ws_bytes(workspace), _ptr(out), _ptr(lse),
        _stream(stream)))
    return out, lse


def bwd_pruned_workspace(B, H, N, d, pack, device, global_window: int = 0):
    return _workspace(lib().asa_bwd_pruned_workspace_size(B, H, N, d, pack, global_window), device)


def asa_sparse_attn_bwd_pruned(prune: QueryPrune, kp, vp, dout, lse, tmask: TileMask,
                               global_window: int = 0, workspace=None, outs=None, stream=None):
    """dQ, dK, dV [B, H, N, d] bf16 with query pruning under the fixed mask, on the
    pruned forward's packed tiles: pruned tokens' output gradients go to their
    centres; pruned rows get dQ = 0."""
    for n_, t in (("kp", kp), ("vp", vp), ("dout", dout)):
        _bf16_cuda(n_, t)
    B, H, N, d = kp.shape
    if workspace is None:
        workspace = bwd_pruned_workspace(B, H, N, d, prune.pack, kp.device, global_window)
    if outs is None:
        outs = tuple(torch.empty_like(kp) for _ in range(3))
    _check(lib().asa_sparse_attn_bwd_pruned(
        _ptr(prune.q_s), _ptr(kp), _ptr(vp), _ptr(dout), _ptr(lse), _ptr(prune.src_pos),
        _ptr(prune.src_row), _ptr(tmask.tile_ptr), _ptr(tmask.tile_col),
        _ptr(tmask.tile_quarters), B, H, N, d, BLOCK, prune.pack, global_window, _ptr(workspace),
        _ws_bytes(workspace), *(_ptr(t) for t in outs), _stream(stream)))
    return outs


def asa_check_device_status(stream=None) -> None:
    _check(lib().asa_check_device_status(_stream(stream)))


def asa_selftest_wait_timeout(limit_cycles: int = 1 << 20, stream=None) -> None:
    """Failure-detection test hook: one bounded wait that must give up (see asa.h)."""
    _check(lib().asa_selftest_wait_timeout(int(limit_cycles), _stream(stream)))


def asa_shutdown() -> None:
    lib().asa_shutdown()


# ----------------------------------------------------------------------- one attention call

def asa_attention(q, k, v, T: int, Hg: int, W: int, tau: float, global_window: int = 0,
                  query_keep: float | None = None, query_window: int = 8, stream=None):
    """One ASA self-attention call on raster-layout q, k, v [B, N, H, d]: Gilbert permute,
    estimate + mask, block-sparse forward storing O straight back to raster order.
    Returns (O raster, LSE in Gilbert order, mask).  query_keep = r adds BSA's query
    pruning with token filling (windows of query_window permuted tokens)."""
    qp, kp, vp = asa_gilbert_permute3(q, k, v, T, Hg, W, stream=stream)
    mask = asa_estimate_mask(qp, kp, tau, transposed=False, stream=stream)
    if query_keep is None:
        out, lse = asa_sparse_attn_fwd_raster(qp, kp, vp, mask, T, Hg, W,
                                              global_window=global_window, stream=stream)
        return out, lse, mask
    else:
        prune = asa_prune_queries(qp, query_keep, query_window, stream=stream)
        tmask = asa_prune_mask(mask, prune.pack, stream=stream)
        op, lse = asa_sparse_attn_fwd_pruned(prune, kp, vp, tmask, global_window=global_window,
                                             stream=stream)
    return asa_unpermute(op, T, Hg, W, stream=stream), lse, mask


def host_workspace(B, T, Hg, W, H, d, global_window=0, head_chunk=0, device="cuda"):
    return _workspace(lib().asa_attention_host_workspace_size(B, T, Hg, W, H, d, global_window,
                                                              head_chunk), device)


def asa_attention_host(q, k, v, T: int, Hg: int, W: int, tau: float, global_window: int = 0,
                       head_chunk: int = 0, out=None, workspace=None, stream=None):
    """asa_attention on host (CPU) tensors q, k, v [B, N, H, d] bf16: the library copies
    chunks of heads in (head_chunk = 0: max(ceil(256 / d), ceil(H / 24)) heads per chunk,
    capped at H), computes and
    copies O out, pipelined on its own streams; pin the
    tensors (tensor.pin_memory()) for the copies to overlap.  Returns O [B, N, H, d] on
    the host; synchronise the stream (torch.cuda.current_stream by default) before
    reading it."""
    for n_, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{n_} must be a contiguous 4-D bf16 host tensor")
    B, N, H, d = q.shape
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=q.is_pinned())
    if workspace is None:
        workspace = host_workspace(B, T, Hg, W, H, d, global_window, head_chunk)
    _check(lib().asa_attention_host(_ptr(q), _ptr(k), _ptr(v), B, T, Hg, W, H, d, float(tau),
                                    global_window, head_chunk, _ptr(workspace),
                                    _ws_bytes(workspace), _ptr(out), _stream(stream)))
    return out


class ASAAttention(torch.autograd.Function):
    """ASA (or ASA_G) self-attention as a differentiable op on raster-layout q, k, v
    [B, N, H, d] bf16.  The mask is computed in the forward from q and k and is not
    differentiated (the pages fix it for training as for inference); the backward runs
    under that mask, its gradients unpermuted to raster layout.  Without query pruning
    the forward is asa_sparse_attn_fwd_train and the backward asa_sparse_attn_bwd_train
    (D from the fp32 O, which the op keeps between the two: 4 bytes per element of O);
    d_from_o=True takes the inference forward and asa_sparse_attn_bwd_d_from_o instead;
    with query_keep the pruned pair."""

    @staticmethod
    def forward(ctx, q, k, v, T: int, Hg: int, W: int, tau: float, global_window: int = 0,
                query_keep: float | None = None, query_window: int = 8, d_from_o: bool = False):
        if d_from_o and query_keep is not None:
            raise ValueError("d_from_o applies to the unpruned backward only; the query-pruned "
                             "backward always takes the exact D")
        q, k, v = (t.contiguous() for t in (q, k, v))
        qp, kp, vp = asa_gilbert_permute3(q, k, v, T, Hg, W)
        mask = asa_estimate_mask(qp, kp, tau, transposed=True)
        prune = None
        o32 = None
        if query_keep is None and not d_from_o:
            op, lse, o32 = asa_sparse_attn_fwd_train(qp, kp, vp, mask, global_window=global_window)
        elif query_keep is None:
            op, lse = asa_sparse_attn_fwd(qp, kp, vp, mask, global_window=global_window)
        else:
            prune = asa_prune_queries(qp, query_keep, query_window)
            tmask = asa_prune_mask(mask, prune.pack)
            op, lse = asa_sparse_attn_fwd_pruned(prune, kp, vp, tmask, global_window=global_window)
        ctx.save_for_backward(qp, kp, vp, op if o32 is None else o32, lse)
        ctx.mask, ctx.grid, ctx.global_window, ctx.prune = mask, (T, Hg, W), global_window, prune
        ctx.tmask = tmask if prune is not None else None
        ctx.d_from_o = d_from_o
        return asa_unpermute(op, T, Hg, W)

    @staticmethod
    def backward(ctx, dout):
        qp, kp, vp, op, lse = ctx.saved_tensors
        T, Hg, W = ctx.grid
        dop = asa_gilbert_permute(dout.to(torch.bfloat16).contiguous(), T, Hg, W)
        if ctx.prune is None and not ctx.d_from_o:
            grads = asa_sparse_attn_bwd_train(qp, kp, vp, op, dop, lse, ctx.mask,
                                              global_window=ctx.global_window)
        elif ctx.prune is None:
            grads = asa_sparse_attn_bwd(qp, kp, vp, op, dop, lse, ctx.mask,
                                        global_window=ctx.global_window, d_from_o=True)
        else:
            grads = asa_sparse_attn_bwd_pruned(ctx.prune, kp, vp, dop, lse, ctx.tmask,
                                               global_window=ctx.global_window)
        dq, dk, dv = (asa_unpermute(g, T, Hg, W) for g in grads)
        return dq, dk, dv, None, None, None, None, None, None, None, None


def asa_attention_trainable(q, k, v, T: int, Hg: int, W: int, tau: float,
                            global_window: int = 0, query_keep: float | None = None,
                            query_window: int = 8, d_from_o: bool = False):
    """Differentiable asa_attention: returns O [B, N, H, d] (raster); gradients flow to
    q, k and v through the kernels' backward under the forward's mask (and, with
    query_keep, the forward's query pruning).  d_from_o=True selects the faster,
    less exact backward (D from the stored O; without query pruning)."""
    return ASAAttention.apply(q, k, v, T, Hg, W, tau, global_window, query_keep, query_window,
                              d_from_o)

