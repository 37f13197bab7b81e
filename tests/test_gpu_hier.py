"""Two-level block estimate on the GPU against the oracle (P within 2e-5
relative, like pool_score), sub = 1 bit-identical to pool_score, and the
Top-p selection on it bit-exact."""
import math

import numpy as np
import pytest
import torch

from dynamic_block_sparse_pool_b200 import ops, synth
from oracle import dsa_oracle as O
from test_gpu_parity import check_select, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [synth.SMALL, synth.TINY], ids=lambda w: w.name)
@pytest.mark.parametrize("sub", [1, 2, 4])
def test_hier_probs_match_oracle(w, sub):
    q, k, _ = synth.make_qkv(w, 13)
    scale = 1.0 / math.sqrt(w.head_dim)
    qg, kg = q.cuda(), k.cuda()
    P = ops.pool_score_hier(qg, kg, w.block, sub, scale)
    ops.device_status()
    Pg = P.cpu().numpy().astype(np.float64)
    for bh in range(w.BH):
        b, h = divmod(bh, w.heads)
        ref = O.hier_block_probs(np64(q[b, h]), np64(k[b, h]), w.block, sub, scale)
        np.testing.assert_allclose(Pg[bh], ref, rtol=2e-5, atol=1e-9, err_msg=f"head {bh}")
    if sub == 1:
        assert torch.equal(P, ops.pool_score(qg, kg, w.block, scale))
    rp, col = ops.select_topp(P, w.p[0])
    check_select(P, w.p[0], rp, col)
