"""PyTorch-facing calls of libdsa.

PyTorch supplies device memory and the current CUDA stream; every step of
the computation runs in libdsa's kernels.  Tensors are [B, H, N, D],
contiguous, bf16 or fp32, on one CUDA device.
"""
from __future__ import annotations

import math
from typing import NamedTuple, Optional, Tuple

import torch

from . import _lib
from ._lib import check, lib

Csr = Tuple[torch.Tensor, torch.Tensor]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(t: torch.Tensor):
    return torch.cuda.current_stream(t.device).cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _lib.DSA_BF16
    if t.dtype == torch.float32:
        return _lib.DSA_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _check_qkv(*ts: torch.Tensor):
    t0 = ts[0]
    if t0.dim() != 4:
        raise ValueError("expected [B, H, N, D] tensors")
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
        if t.shape != t0.shape or t.dtype != t0.dtype or t.device != t0.device:
            raise ValueError("q, k, v must share shape, dtype and device")
    return t0.shape


def _check_csr(csr: Optional[Csr], rows: int):
    if csr is None:
        return None, None
    rp, col = csr
    for t in (rp, col):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("CSR tensors must be contiguous int32 CUDA tensors")
    if rp.numel() != rows + 1:
        raise ValueError(f"row_ptr must have {rows + 1} entries, got {rp.numel()}")
    return rp, col


def n_blocks(N: int, block: int) -> int:
    return (N + block - 1) // block


def workspace_size(op: int, B: int, H: int, N: int, D: int, block: int) -> int:
    return int(lib().dsa_workspace_size(op, B, H, N, D, block))


def pool_score(q: torch.Tensor, k: torch.Tensor, block: int, scale: Optional[float] = None,
               cand: Optional[Csr] = None, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """P [B*H, nB, nB] fp32: row softmax of scale * (block means of Q).(block means of K)."""
    B, H, N, D = _check_qkv(q, k)
    nB = n_blocks(N, block)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    crp, ccol = _check_csr(cand, B * H * nB)
    if out is None:
        out = torch.empty(B * H, nB, nB, device=q.device, dtype=torch.float32)
    ws_bytes = workspace_size(_lib.DSA_OP_POOL_SCORE, B, H, N, D, block)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), device=q.device, dtype=torch.uint8)
    st = lib().dsa_pool_score(q.data_ptr(), k.data_ptr(), _dtype_code(q), B, H, N, D, block,
                              scale, _ptr(crp), _ptr(ccol), out.data_ptr(), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(), _stream(q))
    check(st, "dsa_pool_score")
    return out


def pool_score_hier(q: torch.Tensor, k: torch.Tensor, block: int, sub: int,
                    scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """P [B*H, nB, nB] fp32: the two-level estimate (pooled scores over
    sub-blocks of block/sub rows, folded back into block rows); sub = 1 is
    pool_score's P."""
    B, H, N, D = _check_qkv(q, k)
    nB = n_blocks(N, block)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty(B * H, nB, nB, device=q.device, dtype=torch.float32)
    op = _lib.DSA_OP_POOL_SCORE_HIER4 if sub == 4 else _lib.DSA_OP_POOL_SCORE_HIER2
    ws_bytes = workspace_size(op, B, H, N, D, block)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), device=q.device, dtype=torch.uint8)
    st = lib().dsa_pool_score_hier(q.data_ptr(), k.data_ptr(), _dtype_code(q), B, H, N, D, block,
                                   sub, scale, out.data_ptr(), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(), _stream(q))
    check(st, "dsa_pool_score_hier")
    return out


def select_topp(probs: torch.Tensor, p: float, cand: Optional[Csr] = None,
                row_ptr: Optional[torch.Tensor] = None, col_idx: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None) -> Csr:
    """CSR (row_ptr [rows+1], col_idx [capacity rows*nB]) of the Top-p block sets."""
    if probs.dtype != torch.float32 or not probs.is_cuda or not probs.is_contiguous():
        raise ValueError("probs must be a contiguous fp32 CUDA tensor")
    nB = probs.shape[-1]
    rows = probs.numel() // nB
    crp, ccol = _check_csr(cand, rows)
    dev = probs.device
    if row_ptr is None:
        row_ptr = torch.empty(rows + 1, device=dev, dtype=torch.int32)
    if col_idx is None:
        col_idx = torch.empty(rows * nB, device=dev, dtype=torch.int32)
    ws_bytes = rows * 33 * 4
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    st = lib().dsa_select_topp(probs.data_ptr(), rows, nB, float(p), _ptr(crp), _ptr(ccol),
                               row_ptr.data_ptr(), col_idx.data_ptr(), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream(probs))
    check(st, "dsa_select_topp")
    return row_ptr, col_idx


def row_order(row_ptr: torch.Tensor, B: int, H: int, nB: int,
              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """int32 [B*H*nB]: each head's rows by descending block count (ties by
    row index), as global row indices; the order attn_fwd takes them in."""
    rows = B * H * nB
    if (row_ptr.dtype != torch.int32 or not row_ptr.is_cuda or not row_ptr.is_contiguous()
            or row_ptr.numel() != rows + 1):
        raise ValueError("row_ptr must be a contiguous int32 CUDA tensor of B*H*nB + 1 entries")
    if out is None:
        out = torch.empty(rows, device=row_ptr.device, dtype=torch.int32)
    elif (out.dtype != torch.int32 or out.device != row_ptr.device or not out.is_contiguous()
          or out.numel() != rows):
        raise ValueError("out must be a contiguous int32 tensor of B*H*nB entries on row_ptr's device")
    st = lib().dsa_row_order(row_ptr.data_ptr(), B, H, nB, out.data_ptr(), _stream(row_ptr))
    check(st, "dsa_row_order")
    return out


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, row_ptr: torch.Tensor,
             col_idx: torch.Tensor, block: int, scale: Optional[float] = None,
             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             blk_lse: Optional[torch.Tensor] = None, want_lse: bool = True,
             want_blk_lse: bool = True, order: Optional[torch.Tensor] = None):
    """(O [B,H,N,D], lse [B,H,N] or None, blk_lse [nnz, block] or None).

    Without `order` this is dsa_attn_fwd (rows in index order); with it,
    dsa_attn_fwd_ordered: `order` (row_order's output) is the order in which
    the persistent CTAs take the rows, and changes no output.  When blk_lse
    is wanted but not given, nnz is read from row_ptr (one device-to-host
    copy)."""
    B, H, N, D = _check_qkv(q, k, v)
    nB = n_blocks(N, block)
    _check_csr((row_ptr, col_idx), B * H * nB)
    if order is not None and (order.dtype != torch.int32 or order.device != q.device
                              or not order.is_contiguous() or order.numel() != B * H * nB):
        raise ValueError("order must be a contiguous int32 tensor of B*H*nB entries on q's device")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty(B, H, N, device=q.device, dtype=torch.float32)
    if want_blk_lse and blk_lse is None:
        nnz = int(row_ptr[-1].item())
        blk_lse = torch.empty(max(nnz, 1), block, device=q.device, dtype=torch.float32)
    if order is None:
        st = lib().dsa_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, H, N,
                                D, block, scale, row_ptr.data_ptr(), col_idx.data_ptr(),
                                out.data_ptr(), _ptr(lse), _ptr(blk_lse), _stream(q))
        check(st, "dsa_attn_fwd")
    else:
        st = lib().dsa_attn_fwd_ordered(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B,
                                        H, N, D, block, scale, row_ptr.data_ptr(),
                                        col_idx.data_ptr(), order.data_ptr(), out.data_ptr(),
                                        _ptr(lse), _ptr(blk_lse), _stream(q))
        check(st, "dsa_attn_fwd_ordered")
    return out, lse, blk_lse


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
             dout: torch.Tensor, lse: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor,
             block: int, scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None):
    """(dQ, dK, dV) [B, H, N, D] of attn_fwd's O for a fixed mask, given dO.

    bf16 with block 128 runs on the tensor cores (P and dS as bf16 hi + lo
    terms); fp32 and block 64 in exact fp32 on CUDA cores."""
    B, H, N, D = _check_qkv(q, k, v)
    for t in (out, dout):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous():
            raise ValueError("out and dout must match q")
    nB = n_blocks(N, block)
    _check_csr((row_ptr, col_idx), B * H * nB)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws_bytes = workspace_size(_lib.DSA_OP_ATTN_BWD, B, H, N, D, block)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), device=q.device, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = lib().dsa_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            dout.data_ptr(), lse.data_ptr(), _dtype_code(q), B, H, N, D, block,
                            scale, row_ptr.data_ptr(), col_idx.data_ptr(), dq.data_ptr(),
                            dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                            workspace.numel() * workspace.element_size(), _stream(q))
    check(st, "dsa_attn_bwd")
    return dq, dk, dv


def block_mass(lse: torch.Tensor, blk_lse: torch.Tensor, row_ptr: torch.Tensor, block: int,
               mass: Optional[torch.Tensor] = None) -> torch.Tensor:
    """mass [nnz] (capacity blk_lse.shape[0]): exact softmax mass of each selected block."""
    B, H, N = lse.shape
    if mass is None:
        mass = torch.empty(blk_lse.shape[0], device=lse.device, dtype=torch.float32)
    st = lib().dsa_block_mass(lse.data_ptr(), blk_lse.data_ptr(), B, H, N, block,
                              row_ptr.data_ptr(), mass.data_ptr(), _stream(lse))
    check(st, "dsa_block_mass")
    return mass


def mass_to_probs(row_ptr: torch.Tensor, col_idx: torch.Tensor, mass: torch.Tensor, nB: int,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """probs [rows, nB] fp32: each row's exact block masses at their columns, 0 elsewhere."""
    rows = row_ptr.numel() - 1
    _check_csr((row_ptr, col_idx), rows)
    if mass.dtype != torch.float32 or not mass.is_cuda:
        raise ValueError("mass must be an fp32 CUDA tensor")
    if out is None:
        out = torch.empty(rows, nB, device=mass.device, dtype=torch.float32)
    st = lib().dsa_mass_to_probs(row_ptr.data_ptr(), col_idx.data_ptr(), mass.data_ptr(), rows, nB,
                                 out.data_ptr(), _stream(mass))
    check(st, "dsa_mass_to_probs")
    return out


def hilbert_order(T: int, H: int, W: int, n_prefix: int = 0) -> torch.Tensor:
    """Host int32 [n_prefix + T*H*W]: perm[i] = original index of the token at
    position i along the 3-D Hilbert curve (text prefix first)."""
    perm = torch.empty(n_prefix + T * H * W, dtype=torch.int32)
    check(lib().dsa_hilbert_order(T, H, W, n_prefix, perm.data_ptr()), "dsa_hilbert_order")
    return perm


def gilbert_order(T: int, H: int, W: int, n_prefix: int = 0) -> torch.Tensor:
    """Host int32 [n_prefix + T*H*W]: perm[i] = original index of the token at
    position i along the generalised Hilbert curve of the T x H x W grid
    (consecutive grid tokens are grid neighbours; text prefix first)."""
    perm = torch.empty(n_prefix + T * H * W, dtype=torch.int32)
    check(lib().dsa_gilbert_order(T, H, W, n_prefix, perm.data_ptr()), "dsa_gilbert_order")
    return perm


def permute_tokens(x: torch.Tensor, perm: torch.Tensor, inverse: bool = False,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Gather (dst[i] = src[perm[i]]) or scatter (dst[perm[i]] = src[i]) of the
    token rows of x [B, H, N, D]; perm: device int32 [N]."""
    if x.dim() != 4 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor [B, H, N, D]")
    B, H, N, D = x.shape
    if perm.dtype != torch.int32 or not perm.is_cuda or perm.numel() != N:
        raise ValueError("perm must be a device int32 tensor of N entries")
    if out is None:
        out = torch.empty_like(x)
    st = lib().dsa_permute_tokens(x.data_ptr(), out.data_ptr(), _dtype_code(x), B, H, N, D,
                                  perm.data_ptr(), 1 if inverse else 0, _stream(x))
    check(st, "dsa_permute_tokens")
    return out


class HilbertOrder:
    """The Hilbert token order of one grid, kept on the device.  curve:
    "hilbert" (the enclosing power-of-two cube's curve, restricted to the
    grid) or "gilbert" (the curve generalised to the grid's own box)."""

    def __init__(self, T: int, H: int, W: int, n_prefix: int = 0, device=None,
                 curve: str = "hilbert"):
        if curve not in ("hilbert", "gilbert"):
            raise ValueError(f"unknown curve {curve!r}")
        self.host = (hilbert_order if curve == "hilbert" else gilbert_order)(T, H, W, n_prefix)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.perm = self.host.to(dev)

    def gather(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        return permute_tokens(x, self.perm, False, out)

    def scatter(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        return permute_tokens(x, self.perm, True, out)


def selftest_wait_timeout(limit_ns: int = 1_000_000, device: Optional[torch.device] = None) -> None:
    """Launch the failure-detection self-test: a bounded wait that runs out
    after limit_ns and records a wait timeout (dsa_device_status then raises)."""
    s = torch.cuda.current_stream(device).cuda_stream
    check(lib().dsa_selftest_wait_timeout(int(limit_ns), s), "dsa_selftest_wait_timeout")


def selftest_exp2_poly(x: torch.Tensor) -> torch.Tensor:
    """2^x by the attention softmax's FMA-pipe exponential (fp32 CUDA tensor)."""
    if not (x.is_cuda and x.dtype == torch.float32):
        raise ValueError("x must be a float32 CUDA tensor")
    x = x.contiguous()
    y = torch.empty_like(x)
    s = torch.cuda.current_stream(x.device).cuda_stream
    check(lib().dsa_selftest_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(), s), "dsa_selftest_exp2_poly")
    return y


def device_status(device: Optional[torch.device] = None) -> None:
    """Synchronises the current stream and raises DSAError if a kernel flagged bad input."""
    s = torch.cuda.current_stream(device).cuda_stream
    check(lib().dsa_device_status(s), "dsa_device_status")


class SparseAttention(NamedTuple):
    out: torch.Tensor          # [B, H, N, D]
    lse: torch.Tensor          # [B, H, N]
    probs: torch.Tensor        # [B*H, nB, nB]
    row_ptr: torch.Tensor      # [B*H*nB + 1]
    col_idx: torch.Tensor      # [nnz]
    mass: torch.Tensor         # [nnz]


def sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: float,
                     block: int = 128, scale: Optional[float] = None,
                     cand: Optional[Csr] = None) -> SparseAttention:
    """Whole pipeline: pooled scores -> Top-p selection -> sparse attention
    (rows taken longest first within each head) -> block mass."""
    B, H, N, _ = q.shape
    probs = pool_score(q, k, block, scale, cand)
    row_ptr, col_idx = select_topp(probs, p, cand)
    order = row_order(row_ptr, B, H, n_blocks(N, block))
    out, lse, blk = attn_fwd(q, k, v, row_ptr, col_idx, block, scale, order=order)
    mass = block_mass(lse, blk, row_ptr, block)
    nnz = blk.shape[0] if int(row_ptr[-1].item()) > 0 else 0
    return SparseAttention(out, lse, probs, row_ptr, col_idx[:nnz], mass[:nnz])
