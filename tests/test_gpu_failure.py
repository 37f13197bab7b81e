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
