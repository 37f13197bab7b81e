"""dsa_select_topp_static: Top-p selection for callers that cannot allocate
device memory (no workspace argument; the scratch is a fixed array inside
the library).  Its output must equal dsa_select_topp's exactly -- block
indices are integers, so the tolerance is zero -- on consecutive calls that
reuse the shared scratch.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from dynamic_block_sparse_pool_b200 import _lib, ops, synth

pytestmark = pytest.mark.gpu


def _static_select(probs, p, cand=None):
    rows, nB = probs.shape[0], probs.shape[-1]
    row_ptr = torch.full((rows + 1,), -7, device=probs.device, dtype=torch.int32)
    col_idx = torch.full((rows * nB,), -7, device=probs.device, dtype=torch.int32)
    crp = ccol = None
    if cand is not None:
        crp, ccol = cand[0].data_ptr(), cand[1].data_ptr()
    st = _lib.lib().dsa_select_topp_static(
        probs.data_ptr(), rows, nB, float(p), crp, ccol, row_ptr.data_ptr(),
        col_idx.data_ptr(), torch.cuda.current_stream().cuda_stream)
    _lib.check(st, "dsa_select_topp_static")
    return row_ptr, col_idx


def _probs(rows, nB, seed):
    g = torch.Generator().manual_seed(seed)
    z = torch.randn(rows, nB, generator=g) * 2.5
    z[::3] = torch.round(z[::3])  # exact ties
    return torch.softmax(z, -1).float().cuda()


def _same(a, b):
    rp_a, col_a = a
    rp_b, col_b = b
    assert torch.equal(rp_a, rp_b)
    n = int(rp_a[-1])
    assert torch.equal(col_a[:n], col_b[:n])


def test_static_select_matches_workspace_select_on_consecutive_calls():
    # two calls in a row with different shapes; the second reuses the scratch
    # the first one left behind
    cases = [(_probs(3000, 591, seed=1), 0.9), (_probs(1234, 929, seed=2), 0.7)]
    for probs, p in cases:
        got = _static_select(probs, p)
        want = ops.select_topp(probs, p)
        _same(got, want)
    ops.device_status()


def test_static_select_reduced_search_and_full_size_rows():
    # HunyuanVideo-like: 24 heads x 929 query blocks = 22296 rows
    w = synth.HUNYUAN
    rows, nB = w.BH * w.n_blocks, w.n_blocks
    probs = _probs(rows, nB, seed=3)
    cand = synth.random_csr(rows, nB, 0.4, seed=4)
    cand = (cand[0].cuda(), cand[1].cuda())
    for p in (0.95, 0.6):
        _same(_static_select(probs, p, cand), ops.select_topp(probs, p, cand=cand))
    ops.device_status()


def test_static_select_rejects_rows_beyond_scratch():
    rows = _lib.DSA_STATIC_MAX_ROWS + 1
    probs = torch.full((rows, 4), 0.25, device="cuda")
    with pytest.raises(_lib.DSAError, match="DSA_STATIC_MAX_ROWS"):
        _static_select(probs, 0.5)
