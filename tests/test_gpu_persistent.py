"""The tensor-core attention's persistent CTAs take their rows from a ticket
counter that the library keeps per device (4,096 counters, one per launch in
rotation; the launch's last CTA zeroes its counter).  These tests run more
launches than there are counters, and launches on two streams at once, and
check every result against a single reference run: a counter left non-zero,
or two launches sharing one, would skip or repeat rows."""
import math

import pytest
import torch

from dynamic_block_sparse_pool_b200 import ops, synth

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
