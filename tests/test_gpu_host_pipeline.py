"""The host-buffer call (chunked, copies overlapped with compute) gives the
same O as the device-resident pipeline: heads are independent and every
kernel is deterministic, so the two must agree bit for bit."""
import math

import pytest
import torch

from dynamic_block_sparse_pool_b200 import ops, synth
from dynamic_block_sparse_pool_b200.pipeline import HostPipeline, sparse_attention_host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunk_heads", [1, 3, None])
def test_host_pipeline_matches_device_run(chunk_heads):
    B, H, N, D, block = 2, 5, 1500, 128, 128
    q, k, v = synth.random_qkv(B, H, N, D, torch.bfloat16, seed=31, scale=1.5)
    res = ops.sparse_attention(q.cuda(), k.cuda(), v.cuda(), 0.85, block)
    out = sparse_attention_host(q, k, v, 0.85, block, chunk_heads=chunk_heads)
    assert torch.equal(out, res.out.cpu())


def test_host_pipeline_reuse_and_ragged_chunks():
    w = synth.SMALL
    q, k, v = synth.make_qkv(w, seed=3)
    pipe = HostPipeline(w.batch, w.heads, w.N, w.head_dim, w.dtype, w.block, chunk_heads=3)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    ref = ops.sparse_attention(q.cuda(), k.cuda(), v.cuda(), 0.9, w.block).out.cpu()
    for _ in range(2):  # the slots are reused across calls
        oh.zero_()
        pipe.run(qh, kh, vh, oh, 0.9, 1.0 / math.sqrt(w.head_dim))
        torch.cuda.synchronize()
        assert torch.equal(oh, ref)
    ops.device_status()


def test_host_pipeline_pageable_inputs_and_fp32():
    # pageable (not pinned) host memory: correct, with copies that do not overlap
    B, H, N, D, block = 1, 3, 700, 64, 64
    q, k, v = synth.random_qkv(B, H, N, D, torch.float32, seed=41)
    pipe = HostPipeline(B, H, N, D, torch.float32, block, chunk_heads=2)
    out = torch.empty(q.shape, dtype=q.dtype)
    pipe.run(q, k, v, out, 0.8)
    torch.cuda.synchronize()
    ref = ops.sparse_attention(q.cuda(), k.cuda(), v.cuda(), 0.8, block).out.cpu()
    assert torch.equal(out, ref)
    ops.device_status()


def test_host_pipeline_rejects_bad_arguments():
    from dynamic_block_sparse_pool_b200._lib import lib
    B, H, N, D, block = 1, 2, 300, 128, 128
    q, k, v = synth.random_qkv(B, H, N, D, torch.bfloat16, seed=43)
    out = torch.empty_like(q)
    pipe = HostPipeline(B, H, N, D, torch.bfloat16, block, chunk_heads=1)
    ws = pipe.workspace
    s = torch.cuda.current_stream().cuda_stream
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), 1, B, H, N, D, block, 1 / math.sqrt(D))
    # workspace one byte short
    assert lib().dsa_sparse_attention_host(*args, 0.9, 1, out.data_ptr(), ws.data_ptr(),
                                           ws.numel() - 1, s) == 1
    # p outside (0, 1]
    assert lib().dsa_sparse_attention_host(*args, 1.5, 1, out.data_ptr(), ws.data_ptr(),
                                           ws.numel(), s) == 1
    # a null host pointer
    assert lib().dsa_sparse_attention_host(*args, 0.9, 1, None, ws.data_ptr(), ws.numel(), s) == 1
    torch.cuda.synchronize()
    ops.device_status()
