"""Host-resident inputs: the whole pipeline with PCIe copies overlapped.

A thin binding of the library's dsa_sparse_attention_host: every (batch,
head) is an independent problem, so the call cuts the flattened B*H axis
into chunks and runs three CUDA streams of its own:

    copy-in   : Q, K, V of chunk c      (host -> device, pinned memory)
    compute   : pooled scores, Top-p, sparse attention, block mass of chunk c
    copy-out  : O of chunk c            (device -> host)

Chunk c+1 is copied in while chunk c computes and chunk c-1 is copied out.
Two device slots in one workspace are reused alternately.  This module only
allocates the workspace and passes pointers; the copies, the stream order
and all arithmetic are in libdsa.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import ops
from ._lib import lib


class HostPipeline:
    """The device workspace of host-buffer calls of one shape."""

    def __init__(self, B: int, H: int, N: int, D: int, dtype: torch.dtype, block: int = 128,
                 chunk_heads: Optional[int] = None, device=None):
        self.B, self.H, self.N, self.D, self.block = B, H, N, D, block
        self.dtype = dtype
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        BH = B * H
        self.chunk = max(1, min(BH, chunk_heads or max(1, BH // 8)))
        self.dt = ops._dtype_code(torch.empty(0, dtype=dtype))
        nbytes = int(lib().dsa_host_pipeline_workspace_size(self.dt, B, H, N, D, block, self.chunk))
        if nbytes == 0:
            raise ValueError("invalid shape for the host pipeline")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)

    def h2d_bytes(self) -> int:
        return 3 * self.B * self.H * self.N * self.D * torch.tensor([], dtype=self.dtype).element_size()

    def d2h_bytes(self) -> int:
        return self.B * self.H * self.N * self.D * torch.tensor([], dtype=self.dtype).element_size()

    def run(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
            p: float, scale: Optional[float] = None) -> None:
        """O = sparse attention of host q, k, v [B, H, N, D] (pinned) into host `out`.

        Asynchronous with respect to the host: the current stream waits for
        the last copy-out, so synchronising it makes `out` valid."""
        shape = (self.B, self.H, self.N, self.D)
        for t in (q, k, v, out):
            if t.is_cuda or tuple(t.shape) != shape or t.dtype != self.dtype or not t.is_contiguous():
                raise ValueError(f"q, k, v, out must be contiguous host tensors {shape} of {self.dtype}")
        scale = 1.0 / math.sqrt(self.D) if scale is None else float(scale)
        st = lib().dsa_sparse_attention_host(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), self.dt, self.B, self.H, self.N, self.D,
            self.block, scale, float(p), self.chunk, out.data_ptr(), self.workspace.data_ptr(),
            self.workspace.numel(), torch.cuda.current_stream(self.device).cuda_stream)
        ops.check(st, "dsa_sparse_attention_host")


def sparse_attention_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: float,
                          block: int = 128, scale: Optional[float] = None,
                          chunk_heads: Optional[int] = None) -> torch.Tensor:
    """O for host tensors q, k, v [B, H, N, D]; returns a pinned host tensor.

    Inputs that are not pinned are pinned first (a host-side copy)."""
    if q.is_cuda:
        raise ValueError("sparse_attention_host takes host tensors; use ops.sparse_attention")
    q, k, v = (t if t.is_pinned() else t.pin_memory() for t in (q, k, v))
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    B, H, N, D = q.shape
    pipe = HostPipeline(B, H, N, D, q.dtype, block, chunk_heads)
    out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    pipe.run(q, k, v, out, p, scale)
    torch.cuda.synchronize(pipe.device)
    return out
