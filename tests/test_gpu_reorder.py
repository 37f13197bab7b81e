"""Token reordering on the GPU: the permutation kernel bit-exact, and the
whole pipeline on tokens ordered along the Hilbert curve (of the enclosing
cube, or generalised to the grid's own box) against the oracle on the same
reordered inputs (gates of test_gpu_parity)."""
import math

import numpy as np
import pytest
import torch

from dynamic_block_sparse_pool_b200 import DSAError, HilbertOrder, ops, synth
from test_gpu_parity import check_attention, check_probs, check_select, oracle_probs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_permute_tokens_exact_and_round_trip(dtype, D):
    g = torch.Generator().manual_seed(5)
    B, H, N = 2, 3, 700
    x = torch.randn(B, H, N, D, generator=g).to(dtype)
    perm = torch.randperm(N, generator=g).to(torch.int32)
    xg = x.cuda()
    pd = perm.cuda()
    y = ops.permute_tokens(xg, pd)
    z = ops.permute_tokens(y, pd, inverse=True)
    ops.device_status()
    assert torch.equal(y.cpu(), x[:, :, perm.long()])
    assert torch.equal(z.cpu(), x)


def test_permute_tokens_flags_bad_entry():
    x = torch.randn(1, 1, 8, 64, device="cuda")
    perm = torch.tensor([0, 1, 2, 3, 4, 5, 6, 9], dtype=torch.int32, device="cuda")
    ops.permute_tokens(x, perm)
    with pytest.raises(DSAError, match="permutation"):
        ops.device_status()


@pytest.mark.parametrize("curve", ["hilbert", "gilbert"])
@pytest.mark.parametrize("w", [synth.SMALL, synth.TINY], ids=lambda w: w.name)
def test_pipeline_on_hilbert_order(w, curve):
    q, k, v = synth.make_qkv(w, 7)
    order = HilbertOrder(w.T, w.Hg, w.W, w.n_prefix, curve=curve)
    perm = order.host.long()
    qg, kg, vg = (order.gather(t.cuda()) for t in (q, k, v))
    ops.device_status()
    qp, kp, vp = (t[:, :, perm] for t in (q, k, v))
    assert torch.equal(qg.cpu(), qp) and torch.equal(kg.cpu(), kp) and torch.equal(vg.cpu(), vp)
    scale = 1.0 / math.sqrt(w.head_dim)
    p = w.p[0]
    sa = ops.sparse_attention(qg, kg, vg, p, block=w.block, scale=scale)
    ops.device_status()
    check_probs(sa.probs, oracle_probs(qp, kp, w.block, scale))
    check_select(sa.probs, p, sa.row_ptr, sa.col_idx)
    nnz = int(sa.row_ptr[-1])
    _, _, blk = ops.attn_fwd(qg, kg, vg, sa.row_ptr, sa.col_idx, w.block, scale)
    check_attention(qp, kp, vp, w.block, scale, sa.row_ptr, sa.col_idx[:nnz], sa.out, sa.lse,
                    blk[:nnz], sa.mass[:nnz])
    o = order.scatter(sa.out)
    ops.device_status()
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(perm.numel())
    assert torch.equal(o.cpu(), sa.out.cpu()[:, :, inv])
