"""Why the persistent attention kernel draws its rows from a ticket counter
instead of taking a fixed share of them, and why it takes each head's rows
longest first.

The rows of a Top-p mask have skewed lengths (DSV abstract: the work per
query block is skewed).  On the Wan2.1-like synthetic workload (8 heads,
4,728 rows on 148 CTAs), a row's cost is modelled as its block count times
the measured block period plus a per-row cost.  CTAs that take the next row
as soon as they are free (what the ticket counter does) stay close to the
perfect-balance bound, while a fixed round-robin share of the rows leaves
the slowest CTA far behind it; taking each head's rows longest first (the
order dsa_row_order writes) leaves short rows for the end of the launch and
closes most of the remaining gap."""
import heapq

import numpy as np
import torch

from dynamic_block_sparse_pool_b200 import synth

SMS = 148
BLOCK_CYCLES = 2050   # traced block period of the attention kernel (D = 128)
ROW_CYCLES = 2500     # per-row cost of the persistent kernel (traced, upper end)


def _row_lengths(p_values):
    import dataclasses
    w = dataclasses.replace(synth.WAN21, heads=8)
    q, k, _ = synth.make_qkv(w, 0, device="cpu")
    B, H, N, D = q.shape
    blk = w.block
    nB = (N + blk - 1) // blk

    def pool(x):  # block means (the ragged last block by its own size)
        s = torch.nn.functional.pad(x.float(), (0, 0, 0, nB * blk - N)).view(B, H, nB, blk, D).sum(3)
        cnt = torch.full((nB,), float(blk))
        cnt[-1] = N - (nB - 1) * blk
        return s / cnt[:, None]

    P = torch.softmax(pool(q) @ pool(k).transpose(-1, -2) / D ** 0.5, -1).reshape(-1, nB)
    cs = np.cumsum(-np.sort(-P.double().numpy(), axis=1), axis=1)
    return {p: np.minimum((cs < p).sum(1) + 1, nB) for p in p_values}


def _dynamic(cost):
    free = [0.0] * SMS            # next free time of each CTA
    for c in cost:                # rows in ticket order, to the first free CTA
        heapq.heappush(free, heapq.heappop(free) + c)
    return max(free)


def _makespans(n, heads=8):
    """Makespan / balance bound: rows in index order from the ticket counter,
    each head's rows longest first from it, and a fixed round-robin share."""
    cost = n * BLOCK_CYCLES + ROW_CYCLES
    bound = cost.sum() / SMS
    longest_first = np.concatenate([-np.sort(-c) for c in np.split(cost, heads)])
    fixed = np.zeros(SMS)
    for i, c in enumerate(cost):  # row i to CTA i % 148
        fixed[i % SMS] += c
    return _dynamic(cost) / bound, _dynamic(longest_first) / bound, fixed.max() / bound


def test_dynamic_rows_balance_where_a_fixed_share_does_not():
    for p, n in _row_lengths((0.5, 0.9)).items():
        assert n.max() > 3 * n.mean(), p  # the skew the kernel has to absorb
        greedy, longest_first, fixed = _makespans(n)
        assert greedy < 1.10, (p, greedy)
        assert fixed > greedy + 0.05, (p, greedy, fixed)
        assert longest_first < 1.03 and longest_first < greedy - 0.03, (p, greedy, longest_first)
