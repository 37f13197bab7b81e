"""Host-resident inputs: the whole pipeline with PCIe copies overlapped.

Every (batch, head) is an independent problem, so a call on host tensors
splits the flattened B*H axis into chunks and runs three CUDA streams:

    copy-in   : Q, K, V of chunk c      (host -> device, pinned memory)
    compute   : pooled scores, Top-p, sparse attention, block mass of chunk c
    copy-out  : O of chunk c            (device -> host)

Chunk c+1 is copied in while chunk c computes and chunk c-1 is copied out.
Two device slots are reused alternately; events keep a slot from being
overwritten before its compute (inputs) or its copy-out (output) finished.

All arithmetic runs in libdsa's kernels (through ``ops``); this module only
moves data and orders streams.
"""
from __future__ import annotations

import math
from typing import List, Optional

import torch

from . import ops


class HostPipeline:
    """Reusable device buffers and streams for host-buffer calls of one shape."""

    def __init__(self, B: int, H: int, N: int, D: int, dtype: torch.dtype, block: int = 128,
                 chunk_heads: Optional[int] = None, device=None):
        self.B, self.H, self.N, self.D, self.block = B, H, N, D, block
        self.dtype = dtype
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        BH = B * H
        self.chunk = max(1, min(BH, chunk_heads or max(1, BH // 8)))
        self.nB = ops.n_blocks(N, block)
        c, nB, dev = self.chunk, self.nB, self.device
        rows = c * nB
        self.slots = []
        for _ in range(2):
            self.slots.append(dict(
                q=torch.empty(1, c, N, D, dtype=dtype, device=dev),
                k=torch.empty(1, c, N, D, dtype=dtype, device=dev),
                v=torch.empty(1, c, N, D, dtype=dtype, device=dev),
                out=torch.empty(1, c, N, D, dtype=dtype, device=dev),
                lse=torch.empty(1, c, N, dtype=torch.float32, device=dev),
                probs=torch.empty(c, nB, nB, dtype=torch.float32, device=dev),
                ws_pool=torch.empty(max(16, ops.workspace_size(0, 1, c, N, D, block)),
                                    dtype=torch.uint8, device=dev),
                ws_sel=torch.empty(max(16, ops.workspace_size(1, 1, c, N, D, block)),
                                   dtype=torch.uint8, device=dev),
                row_ptr=torch.empty(rows + 1, dtype=torch.int32, device=dev),
                col_idx=torch.empty(rows * nB, dtype=torch.int32, device=dev),
                blk_lse=torch.empty(rows * nB, block, dtype=torch.float32, device=dev),
                mass=torch.empty(rows * nB, dtype=torch.float32, device=dev),
            ))
        self.s_in = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)

    def h2d_bytes(self) -> int:
        return 3 * self.B * self.H * self.N * self.D * torch.tensor([], dtype=self.dtype).element_size()

    def d2h_bytes(self) -> int:
        return self.B * self.H * self.N * self.D * torch.tensor([], dtype=self.dtype).element_size()

    def run(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
            p: float, scale: Optional[float] = None) -> None:
        """O = sparse attention of host q, k, v [B, H, N, D] (pinned) into host `out`.

        Asynchronous with respect to the host: the caller synchronises
        (``torch.cuda.synchronize()`` or the returned copy-out stream)."""
        BH, c = self.B * self.H, self.chunk
        N, D = self.N, self.D
        qf = q.view(BH, N, D)
        kf = k.view(BH, N, D)
        vf = v.view(BH, N, D)
        of = out.view(BH, N, D)
        scale = 1.0 / math.sqrt(D) if scale is None else scale
        cur = torch.cuda.current_stream(self.device)
        self.s_in.wait_stream(cur)
        n_chunks = (BH + c - 1) // c
        in_done: List[torch.cuda.Event] = []
        comp_done: List[torch.cuda.Event] = []
        out_done: List[torch.cuda.Event] = []
        for ci in range(n_chunks):
            h0, h1 = ci * c, min(BH, (ci + 1) * c)
            n = h1 - h0
            slot = self.slots[ci % 2]
            with torch.cuda.stream(self.s_in):
                if ci >= 2:  # the slot's inputs are free once chunk ci-2 computed
                    self.s_in.wait_event(comp_done[ci - 2])
                for name, src in (("q", qf), ("k", kf), ("v", vf)):
                    slot[name][0, :n].copy_(src[h0:h1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.s_in)
                in_done.append(ev)
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(in_done[ci])
                if ci >= 2:  # the slot's output is free once chunk ci-2 was copied out
                    self.s_comp.wait_event(out_done[ci - 2])
                qd, kd, vd = slot["q"][:, :n], slot["k"][:, :n], slot["v"][:, :n]
                rows = n * self.nB
                probs = slot["probs"][:n]
                ops.pool_score(qd, kd, self.block, scale, out=probs, workspace=slot["ws_pool"])
                rp = slot["row_ptr"][:rows + 1]
                ops.select_topp(probs, p, row_ptr=rp, col_idx=slot["col_idx"],
                                workspace=slot["ws_sel"])
                od, lse = slot["out"][:, :n], slot["lse"][:, :n]
                ops.attn_fwd(qd, kd, vd, rp, slot["col_idx"], self.block, scale, out=od,
                             lse=lse, blk_lse=slot["blk_lse"])
                ops.block_mass(lse, slot["blk_lse"], rp, self.block, mass=slot["mass"])
                ev = torch.cuda.Event()
                ev.record(self.s_comp)
                comp_done.append(ev)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(comp_done[ci])
                of[h0:h1].copy_(slot["out"][0, :n], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.s_out)
                out_done.append(ev)
        cur.wait_stream(self.s_out)


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
