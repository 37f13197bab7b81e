"""The tensor-core attention's persistent CTAs take their rows from a ticket
counter that the library keeps per device (4,096 counters, one per launch in
rotation; the launch's last CTA zeroes its counter).  These tests run more
launches than there are counters, and launches on two streams at once, and
check every result against a single reference run: a counter left non-zero,
or two launches sharing one, would skip or repeat rows.  Ticket t is row
order[t] when an order is given: the longest-first order of each head's rows
is checked against a stable sort, every order gives the same outputs, and an
order entry out of range is reported and passed over."""
import math

import numpy as np
import pytest
import torch

from dynamic_block_sparse_pool_b200 import DSAError, ops, synth

pytestmark = pytest.mark.gpu


def _case(seed, H=3, N=1000, D=128, block=128, p=0.8):
    q, k, v = (t.cuda() for t in synth.random_qkv(1, H, N, D, torch.bfloat16, seed=seed, scale=1.5))
    P = ops.pool_score(q, k, block, 1.0 / math.sqrt(D))
    rp, ci = ops.select_topp(P, p)
    return q, k, v, rp, ci, block


def test_ticket_counters_wrap_around():
    q, k, v, rp, ci, block = _case(51, H=24)  # 192 rows on 148 CTAs
    ref, ref_lse, _ = ops.attn_fwd(q, k, v, rp, ci, block, want_blk_lse=False)
    torch.cuda.synchronize()
    out = torch.empty_like(ref)
    lse = torch.empty_like(ref_lse)
    bad = torch.zeros((), dtype=torch.int32, device="cuda")
    for i in range(4096 + 300):  # past the rotation of the counters
        out.fill_(float("nan"))
        ops.attn_fwd(q, k, v, rp, ci, block, out=out, lse=lse, want_blk_lse=False)
        bad += (~torch.eq(out, ref)).sum().to(torch.int32) + (~torch.eq(lse, ref_lse)).sum().to(torch.int32)
    ops.device_status()
    assert int(bad) == 0


def test_launches_on_two_streams_at_once():
    a = _case(52, H=4)
    b = _case(53, H=2, N=1500)
    ref_a = ops.attn_fwd(*a, want_blk_lse=False)[0]
    ref_b = ops.attn_fwd(*b, want_blk_lse=False)[0]
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs_a, outs_b = [], []
    for _ in range(20):
        with torch.cuda.stream(s1):
            outs_a.append(ops.attn_fwd(*a, want_blk_lse=False)[0])
        with torch.cuda.stream(s2):
            outs_b.append(ops.attn_fwd(*b, want_blk_lse=False)[0])
    torch.cuda.synchronize()
    ops.device_status()
    assert all(torch.equal(o, ref_a) for o in outs_a)
    assert all(torch.equal(o, ref_b) for o in outs_b)


def _lengths_order(rp, B, H, nB):
    """Each head's rows by descending block count, ties by row index (numpy)."""
    n = np.diff(rp.cpu().numpy().astype(np.int64)).reshape(B * H, nB)
    return np.concatenate([h * nB + np.argsort(-n[h], kind="stable") for h in range(B * H)])


@pytest.mark.parametrize("B,H,nB,kind", [(1, 3, 591, "topp"), (2, 2, 1024, "topp"),
                                         (1, 1, 1, "topp"), (1, 4, 37, "equal"),
                                         (1, 2, 200, "empty"), (1, 5, 130, "ties")])
def test_row_order_is_the_stable_longest_first_order(B, H, nB, kind):
    g = torch.Generator().manual_seed(nB + H)
    rows = B * H * nB
    if kind == "topp":
        logits = torch.randn(rows, nB, generator=g) * 3
        P = torch.softmax(logits, -1).cuda()
        rp, _ = ops.select_topp(P, 0.8)
    else:
        n = {"equal": torch.full((rows,), 5),
             "empty": torch.randint(0, 2, (rows,), generator=g) * torch.randint(0, nB, (rows,), generator=g),
             "ties": torch.randint(0, 4, (rows,), generator=g)}[kind]
        rp = torch.cat([torch.zeros(1, dtype=torch.int64), n.cumsum(0)]).to(torch.int32).cuda()
    order = ops.row_order(rp, B, H, nB)
    torch.cuda.synchronize()
    assert np.array_equal(order.cpu().numpy(), _lengths_order(rp, B, H, nB))


def test_attention_is_the_same_in_any_row_order():
    q, k, v, rp, ci, block = _case(54, H=6, N=2000)
    B, H, N, _ = q.shape
    nB = (N + block - 1) // block
    nnz = int(rp[-1])

    def run(order):
        # blk_lse past the ragged last query block is never written: fill it
        # alike in every run
        bl = torch.full((nnz, block), -7.0, device="cuda")
        return ops.attn_fwd(q, k, v, rp, ci, block, blk_lse=bl, order=order)

    ref = run(None)
    g = torch.Generator().manual_seed(7)
    orders = [ops.row_order(rp, B, H, nB),
              torch.arange(B * H * nB - 1, -1, -1, dtype=torch.int32).cuda(),
              torch.randperm(B * H * nB, generator=g).to(torch.int32).cuda()]
    for order in orders:
        got = run(order)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    ops.device_status()


def test_row_order_entry_out_of_range_is_reported_and_passed_over():
    q, k, v, rp, ci, block = _case(55, H=2, N=1200)
    B, H, N, D = q.shape
    nB = (N + block - 1) // block
    rows = B * H * nB
    ref, ref_lse, _ = ops.attn_fwd(q, k, v, rp, ci, block, want_blk_lse=False)
    order = ops.row_order(rp, B, H, nB)
    skipped = order[[3, rows - 1]].cpu().tolist()
    order[3] = rows
    order[rows - 1] = -1
    out = torch.full_like(ref, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    ops.attn_fwd(q, k, v, rp, ci, block, out=out, lse=lse, want_blk_lse=False, order=order)
    with pytest.raises(DSAError, match="row-order-index-out-of-range"):
        ops.device_status()
    o, o_ref = out.view(B * H, N, D), ref.view(B * H, N, D)
    l, l_ref = lse.view(B * H, N), ref_lse.view(B * H, N)
    for r in range(rows):
        bh, i = divmod(r, nB)
        t = slice(i * block, min((i + 1) * block, N))  # N = 1200: a ragged last block
        if r in skipped:
            assert torch.isnan(o[bh, t]).all() and torch.isnan(l[bh, t]).all()
        else:
            assert torch.equal(o[bh, t], o_ref[bh, t]) and torch.equal(l[bh, t], l_ref[bh, t])
    # the next call is unaffected
    ops.attn_fwd(q, k, v, rp, ci, block, out=out, lse=lse, want_blk_lse=False,
                 order=ops.row_order(rp, B, H, nB))
    ops.device_status()
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)
