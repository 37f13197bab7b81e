"""Backward of the block-sparse attention on the GPU against the fp64
oracle's chain rule, for the pipeline's own masks, for random fixed masks
(ragged tails, empty rows) and for a hand-built mask with an empty row and a
key block nobody selects.  The forward output O and lse that the kernel
receives are the oracle's own (fp64, rounded to the input dtype and fp32), so
no input of the comparison comes from the CUDA path; one test also runs the
backward on the GPU forward's O and lse, as a caller would.  The oracle takes
the row term from the same stored O that the kernel receives.  bf16 with blocks of 128 runs on
the tensor-core kernels (P and dS as bf16 hi + lo terms), fp32 and blocks of
64 on the fp32 CUDA-core kernels; both meet the same gates.

Gates (per tensor, relative to its largest reference value m):
fp32 |err| <= 1e-4 m; bf16 |err| <= |ref| / 128 + 2e-3 m (bf16 rounding of
the stored gradients plus fp32 accumulation)."""
import math

import numpy as np
import pytest
import torch

from dynamic_block_sparse_pool_b200 import ops, synth
from oracle import dsa_oracle as O
from test_gpu_parity import head_csr, np64

pytestmark = pytest.mark.gpu


def _check_grads(q, k, v, dO, block, scale, rp, col, grads, out):
    B, H, N, D = q.shape
    nB = ops.n_blocks(N, block)
    rp_c, col_c = rp.cpu().numpy().astype(np.int64), col.cpu().numpy().astype(np.int64)
    got = [np64(g) for g in grads]
    for bh in range(B * H):
        b, h = divmod(bh, H)
        hrp, hcol, _ = head_csr(rp_c, col_c, bh, nB)
        ref = O.sparse_attention_backward_head(np64(q[b, h]), np64(k[b, h]), np64(v[b, h]),
                                               np64(dO[b, h]), block, scale, hrp, hcol,
                                               out=np64(out[b, h]))
        for name, g, r in zip("qkv", got, ref):
            m = max(np.abs(r).max(), 1e-30)
            err = np.abs(g[b, h] - r)
            if q.dtype == torch.float32:
                assert err.max() <= 1e-4 * m, (name, bh, err.max(), m)
            else:
                assert np.all(err <= np.abs(r) / 128 + 2e-3 * m), (name, bh, err.max(), m)


def oracle_forward(q, k, v, block, scale, rp, col):
    """The oracle's O (rounded to q's dtype) and lse (fp32) on the given mask,
    as CUDA tensors: the stored forward outputs the backward receives."""
    B, H, N, D = q.shape
    nB = ops.n_blocks(N, block)
    rp_c, col_c = rp.cpu().numpy().astype(np.int64), col.cpu().numpy().astype(np.int64)
    out = torch.empty(q.shape, dtype=torch.float64)
    lse = torch.empty(B, H, N, dtype=torch.float64)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        hrp, hcol, _ = head_csr(rp_c, col_c, bh, nB)
        Oo, lo, _ = O.sparse_attention_head(np64(q[b, h]), np64(k[b, h]), np64(v[b, h]),
                                            block, scale, hrp, hcol)
        out[b, h] = torch.from_numpy(Oo)
        lse[b, h] = torch.from_numpy(lo)
    return out.to(q.dtype).cuda(), lse.float().cuda()


@pytest.mark.parametrize("w", [synth.TINY, synth.SMALL], ids=lambda w: w.name)
def test_backward_on_pipeline_mask(w):
    q, k, v = (t.cuda() for t in synth.make_qkv(w, 17))
    scale = 1.0 / math.sqrt(w.head_dim)
    sa = ops.sparse_attention(q, k, v, w.p[0], block=w.block, scale=scale)
    g = torch.Generator().manual_seed(3)
    dO = torch.randn(q.shape, generator=g).to(q.dtype).cuda()
    nnz = int(sa.row_ptr[-1])
    col = sa.col_idx[:nnz]
    # the oracle's stored forward outputs on the pipeline's mask
    out_o, lse_o = oracle_forward(q.cpu(), k.cpu(), v.cpu(), w.block, scale, sa.row_ptr, col)
    grads = ops.attn_bwd(q, k, v, out_o, dO, lse_o, sa.row_ptr, sa.col_idx, w.block, scale)
    ops.device_status()
    _check_grads(q.cpu(), k.cpu(), v.cpu(), dO.cpu(), w.block, scale, sa.row_ptr, col, grads,
                 out_o.cpu())
    # and as a caller runs it: on the GPU forward's own O and lse
    grads = ops.attn_bwd(q, k, v, sa.out, dO, sa.lse, sa.row_ptr, sa.col_idx, w.block, scale)
    ops.device_status()
    _check_grads(q.cpu(), k.cpu(), v.cpu(), dO.cpu(), w.block, scale, sa.row_ptr, col, grads,
                 sa.out.cpu())


@pytest.mark.parametrize("name,B,H,N,D,block,density", [
    ("tc_d128_ragged", 1, 2, 1000, 128, 128, 0.5),
    ("tc_d128_dense_rows", 1, 1, 128 * 9 + 40, 128, 128, 1.0),
    ("tc_d64_long_rows", 2, 1, 128 * 12 + 5, 64, 128, 0.8),
    ("simt_bf16_block64", 1, 2, 300, 64, 64, 0.5),
])
def test_backward_fixed_mask(name, B, H, N, D, block, density):
    q, k, v = (t.cuda() for t in synth.random_qkv(B, H, N, D, torch.bfloat16, seed=41))
    nB = ops.n_blocks(N, block)
    rp, col = synth.random_csr(B * H * nB, nB, density, seed=5)
    scale = 1.0 / math.sqrt(D)
    out, lse = oracle_forward(q.cpu(), k.cpu(), v.cpu(), block, scale, rp, col)
    dO = torch.randn(q.shape, generator=torch.Generator().manual_seed(6)).to(q.dtype).cuda()
    grads = ops.attn_bwd(q, k, v, out, dO, lse, rp.cuda(), col.cuda(), block, scale)
    ops.device_status()
    _check_grads(q.cpu(), k.cpu(), v.cpu(), dO.cpu(), block, scale, rp, col, grads, out.cpu())


def test_backward_empty_row_unselected_block_and_repeatability():
    w = synth.SMALL
    q, k, v = (t.cuda() for t in synth.make_qkv(w, 19))
    B, H, N, D, blk = w.batch, w.heads, w.N, w.head_dim, w.block
    nB = w.n_blocks
    scale = 1.0 / math.sqrt(D)
    rows = []
    for bh in range(B * H):
        for i in range(nB):
            if i == 3:
                rows.append([])                                  # an empty row
            else:
                rows.append(sorted({i, (i + 1) % nB, 0} - {5}))  # key block 5: never selected
    rp = torch.tensor(np.concatenate([[0], np.cumsum([len(r) for r in rows])]), dtype=torch.int32)
    col = torch.tensor(np.concatenate([np.array(r, dtype=np.int64) for r in rows]), dtype=torch.int32)
    rpg, colg = rp.cuda(), col.cuda()
    out, lse = oracle_forward(q.cpu(), k.cpu(), v.cpu(), blk, scale, rp, col)
    dO = torch.randn(q.shape, generator=torch.Generator().manual_seed(8)).to(q.dtype).cuda()
    g1 = ops.attn_bwd(q, k, v, out, dO, lse, rpg, colg, blk, scale)
    g2 = ops.attn_bwd(q, k, v, out, dO, lse, rpg, colg, blk, scale)
    ops.device_status()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    dq, dk, dv = (t.cpu() for t in g1)
    assert torch.all(dq[:, :, 3 * blk:4 * blk] == 0)
    assert torch.all(dk[:, :, 5 * blk:6 * blk] == 0) and torch.all(dv[:, :, 5 * blk:6 * blk] == 0)
    _check_grads(q.cpu(), k.cpu(), v.cpu(), dO.cpu(), blk, scale, rp, col, g1, out.cpu())
