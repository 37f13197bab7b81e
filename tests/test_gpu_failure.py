"""Failure detection on the GPU without a fault: a bounded device wait that
runs out is reported through the device error word, and the context stays
usable afterwards.  Every mbarrier wait of the tensor-core kernels is the
same bounded wait; here it waits on a barrier nothing arrives at, so it must
give up after its limit."""
import math

import pytest
import torch

from dynamic_block_sparse_pool_b200 import DSAError, ops, synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    ops.device_status()                              # start from a clean error word
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    ops.selftest_wait_timeout(2_000_000)             # 2 ms
    b.record(stream)
    with pytest.raises(DSAError, match="wait-timeout"):
        ops.device_status()
    ms = a.elapsed_time(b)
    assert 2.0 <= ms < 500.0, ms                     # it waited its limit, then returned
    ops.device_status()                              # the word was cleared


def test_context_usable_after_a_timeout():
    ops.selftest_wait_timeout(1_000_000)
    with pytest.raises(DSAError, match="wait-timeout"):
        ops.device_status()
    # the whole pipeline still runs and is deterministic afterwards
    w = synth.SMALL
    q, k, v = (t.cuda() for t in synth.make_qkv(w, 3))
    a = ops.sparse_attention(q, k, v, 0.9, block=w.block, scale=1 / math.sqrt(w.head_dim))
    ops.device_status()
    ops.selftest_wait_timeout(1_000_000)
    with pytest.raises(DSAError, match="wait-timeout"):
        ops.device_status()
    b = ops.sparse_attention(q, k, v, 0.9, block=w.block, scale=1 / math.sqrt(w.head_dim))
    ops.device_status()
    assert torch.equal(a.row_ptr, b.row_ptr) and torch.equal(a.out, b.out)


def test_attention_flags_a_bad_column_index_and_recovers():
    # a column index outside [0, nB) in one row: the kernel reports it through
    # the device error word, writes that row as empty, and the next call on a
    # valid mask is unaffected (the CTA drains the copies it had started)
    B, H, N, D, block = 1, 1, 700, 128, 128
    q, k, v = (t.cuda() for t in synth.random_qkv(B, H, N, D, torch.bfloat16, seed=5))
    nB = ops.n_blocks(N, block)
    rp = torch.tensor([0, 2, 3, 5, 6, 7, 9], dtype=torch.int32).cuda()
    good = torch.tensor([0, 1, 2, 0, 3, 4, 5, 1, 5], dtype=torch.int32).cuda()
    bad = good.clone()
    bad[3] = nB + 7                                  # first entry of row 2
    ops.device_status()
    out_b, lse_b, _ = ops.attn_fwd(q, k, v, rp, bad, block)
    with pytest.raises(DSAError, match="csr-index"):
        ops.device_status()
    assert torch.all(out_b[0, 0, 2 * block:3 * block] == 0)
    assert torch.all(torch.isneginf(lse_b[0, 0, 2 * block:3 * block]))
    out_g, lse_g, _ = ops.attn_fwd(q, k, v, rp, good, block)
    ops.device_status()
    out_r, _, _ = ops.attn_fwd(q, k, v, rp, good, block)
    ops.device_status()
    assert torch.equal(out_g, out_r)
    # rows the bad entry does not touch are computed as usual
    assert torch.equal(out_b[0, 0, :2 * block], out_g[0, 0, :2 * block])
