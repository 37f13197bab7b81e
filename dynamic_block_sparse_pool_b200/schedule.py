"""Step policy over a denoising run: warm-up, search and mask-reuse steps.

GSRS (arXiv 2610.21129):
- abstract: sparsity grows as denoising progresses (tighter Top-p), later
  searches are restricted to an early candidate set, and Top-p runs on exact
  attention weights computed within the FlashAttention pass;
- Figure 4: the first search step evaluates all blocks and sets a baseline
  mask, later search steps evaluate only the blocks of that mask, and
  non-search steps reuse the most recent mask without re-evaluation;
- Table 8: N_w warm-up steps of full attention;
- Table 11: a Top-p configuration is a list of values, one per search step.

The pages do not say where the search steps fall; by default they are spread
evenly over the steps after warm-up, the first one right after it.

Each step's work runs in libdsa's kernels (through ``ops``): attention over a
CSR mask (all blocks, the baseline mask or the latest mask), the exact block
masses, their scatter into dense rows and the Top-p selection.  This module
keeps the masks and orders the calls.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, NamedTuple, Optional, Tuple

import torch

from . import ops

WARMUP, SEARCH, REUSE = "warmup", "search", "reuse"


@dataclass(frozen=True)
class GsrsPolicy:
    """n_steps steps; `warmup` of full attention; one search per value of `p`.

    search_steps: explicit step indices of the searches (increasing, at or
    after `warmup`), or None for the even spread."""
    n_steps: int
    warmup: int
    p: Tuple[float, ...]
    search_steps: Optional[Tuple[int, ...]] = None

    def __post_init__(self):
        if self.n_steps < 1 or not 0 <= self.warmup <= self.n_steps:
            raise ValueError("need n_steps >= 1 and 0 <= warmup <= n_steps")
        if not all(0.0 < p <= 1.0 for p in self.p):
            raise ValueError("every p must be in (0, 1]")
        steps = self.searches()
        if len(steps) != len(self.p):
            raise ValueError("one search step per p value")
        if any(b <= a for a, b in zip(steps, steps[1:])):
            raise ValueError("search steps must increase")
        if steps and (steps[0] < self.warmup or steps[-1] >= self.n_steps):
            raise ValueError("search steps must lie in [warmup, n_steps)")
        if not steps and self.warmup < self.n_steps:
            raise ValueError("steps after warm-up need at least one search")

    def searches(self) -> List[int]:
        if self.search_steps is not None:
            return list(self.search_steps)
        k = len(self.p)
        span = self.n_steps - self.warmup
        if k == 0:
            return []
        if k > span:
            raise ValueError("more searches than steps after warm-up")
        return [self.warmup + (i * span) // k for i in range(k)]

    def kinds(self) -> List[Tuple[str, Optional[int]]]:
        """(kind, index of the search or None) for every step."""
        at = {s: i for i, s in enumerate(self.searches())}
        out = []
        for s in range(self.n_steps):
            if s < self.warmup:
                out.append((WARMUP, None))
            elif s in at:
                out.append((SEARCH, at[s]))
            else:
                out.append((REUSE, None))
        return out


class StepResult(NamedTuple):
    kind: str
    out: torch.Tensor                      # O of this step [B, H, N, D]
    mask: Tuple[torch.Tensor, torch.Tensor]  # CSR the step attended over
    mass: Optional[torch.Tensor]           # exact block masses over `mask` (search steps)
    next_mask: Optional[Tuple[torch.Tensor, torch.Tensor]]  # mask selected at a search step


class GsrsRunner:
    """Runs a GsrsPolicy step by step on device tensors of one shape."""

    def __init__(self, policy: GsrsPolicy, B: int, H: int, N: int, D: int, block: int = 128,
                 dtype: torch.dtype = torch.bfloat16, scale: Optional[float] = None,
                 device=None):
        self.policy = policy
        self.kinds = policy.kinds()
        self.B, self.H, self.N, self.D, self.block = B, H, N, D, block
        self.scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.device = dev
        nB = ops.n_blocks(N, block)
        self.nB = nB
        rows = B * H * nB
        self.rows = rows
        cap = rows * nB
        self.all_rp = (torch.arange(rows + 1, device=dev, dtype=torch.int64) * nB).to(torch.int32)
        self.all_col = torch.arange(nB, device=dev, dtype=torch.int32).repeat(rows)
        self.out = torch.empty(B, H, N, D, device=dev, dtype=dtype)
        self.lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
        self.blk_lse = torch.empty(cap, block, device=dev, dtype=torch.float32)
        self.mass = torch.empty(cap, device=dev, dtype=torch.float32)
        self.probs = torch.empty(rows, nB, device=dev, dtype=torch.float32)
        self.ws_sel = torch.empty(max(16, ops.workspace_size(1, B, H, N, D, block)),
                                  device=dev, dtype=torch.uint8)
        # two mask buffers: the baseline (set by the first search) and the one
        # later searches select into; `cur` is the latest mask (the baseline
        # itself until the second search)
        self.base = (torch.empty(rows + 1, device=dev, dtype=torch.int32),
                     torch.empty(cap, device=dev, dtype=torch.int32))
        self.later = (torch.empty(rows + 1, device=dev, dtype=torch.int32),
                      torch.empty(cap, device=dev, dtype=torch.int32))
        # the order the attention takes each mask's rows in (longest first
        # within each head)
        self.base_order = torch.empty(rows, device=dev, dtype=torch.int32)
        self.later_order = torch.empty(rows, device=dev, dtype=torch.int32)
        self.cur = None
        self.have_base = False

    def _order_of(self, mask):
        return self.base_order if mask is self.base else self.later_order

    def step(self, s: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> StepResult:
        kind, idx = self.kinds[s]
        if kind == WARMUP:
            ops.attn_fwd(q, k, v, self.all_rp, self.all_col, self.block, self.scale, out=self.out,
                         want_lse=False, want_blk_lse=False)
            return StepResult(kind, self.out, (self.all_rp, self.all_col), None, None)
        if kind == REUSE:
            ops.attn_fwd(q, k, v, self.cur[0], self.cur[1], self.block, self.scale, out=self.out,
                         lse=self.lse, want_blk_lse=False, order=self._order_of(self.cur))
            return StepResult(kind, self.out, self.cur, None, None)
        # search: attention over the candidates with their exact block masses,
        # then Top-p on those masses within the candidates
        cand = self.base if self.have_base else (self.all_rp, self.all_col)
        ops.attn_fwd(q, k, v, cand[0], cand[1], self.block, self.scale, out=self.out,
                     lse=self.lse, blk_lse=self.blk_lse,
                     order=self._order_of(cand) if self.have_base else None)
        ops.block_mass(self.lse, self.blk_lse, cand[0], self.block, mass=self.mass)
        ops.mass_to_probs(cand[0], cand[1], self.mass, self.nB, out=self.probs)
        target = self.later if self.have_base else self.base
        ops.select_topp(self.probs, self.policy.p[idx], cand=cand, row_ptr=target[0],
                        col_idx=target[1], workspace=self.ws_sel)
        ops.row_order(target[0], self.B, self.H, self.nB, out=self._order_of(target))
        self.have_base = True
        self.cur = target
        return StepResult(kind, self.out, cand, self.mass, target)

