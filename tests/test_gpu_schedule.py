"""Parity of the mass-driven step policy (through the C ABI) with the oracle.

Gates: the scattered mass rows bit-exact; at every search step the
attention, lse, block log-sums and masses over the candidates within the
tolerances of test_gpu_parity, and the next mask bit-exact against the
oracle's Top-p on the GPU's own masses within the candidates; warm-up and
reuse steps attend over all blocks / the latest mask.
"""
import math

import numpy as np
import pytest
import torch

from dynamic_block_sparse_pool_b200 import DSAError, ops, synth
from dynamic_block_sparse_pool_b200.schedule import REUSE, SEARCH, WARMUP, GsrsPolicy, GsrsRunner
from oracle import dsa_oracle as O
from test_gpu_parity import TOL, check_attention, head_csr, np64

pytestmark = pytest.mark.gpu


def test_mass_to_probs_exact():
    rng = np.random.default_rng(3)
    rows, nB = 57, 40
    counts = rng.integers(0, nB + 1, size=rows)
    rp = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    col = np.concatenate([rng.permutation(nB)[:c] for c in counts]).astype(np.int32)
    mass = rng.random(int(rp[-1])).astype(np.float32)
    P = ops.mass_to_probs(torch.from_numpy(rp).cuda(), torch.from_numpy(col).cuda(),
                          torch.from_numpy(mass).cuda(), nB)
    ops.device_status()
    np.testing.assert_array_equal(P.cpu().numpy(), O.mass_rows(rp, col, mass, nB).astype(np.float32))


def test_mass_to_probs_flags_bad_column():
    rp = torch.tensor([0, 2, 3], dtype=torch.int32, device="cuda")
    col = torch.tensor([1, 7, 0], dtype=torch.int32, device="cuda")  # 7 >= nB
    P = ops.mass_to_probs(rp, col, torch.ones(3, device="cuda"), 4)
    with pytest.raises(DSAError, match="csr-index"):
        ops.device_status()
    # the other slots are still written
    np.testing.assert_array_equal(P.cpu().numpy(), [[0, 1, 0, 0], [1, 0, 0, 0]])


def _check_out(q, k, v, block, scale, rp, col, out):
    B, H, N, D = q.shape
    nB = ops.n_blocks(N, block)
    tol = TOL[q.dtype]
    rp_c, col_c = rp.cpu().numpy().astype(np.int64), col.cpu().numpy().astype(np.int64)
    out_c = np64(out)
    errs = []
    for bh in range(B * H):
        b, h = divmod(bh, H)
        hrp, hcol, _ = head_csr(rp_c, col_c, bh, nB)
        Oo, _, _ = O.sparse_attention_head(np64(q[b, h]), np64(k[b, h]), np64(v[b, h]), block,
                                           scale, hrp, hcol)
        errs.append(np.abs(out_c[b, h] - Oo).ravel())
    e = np.concatenate(errs)
    assert e.max() <= tol["o_max"] and e.mean() <= tol["o_mean"], (e.max(), e.mean())


def _same(a, b):
    return all(torch.equal(x.cpu(), y.cpu()) for x, y in zip(a, b))


def test_schedule_small_matches_oracle():
    w = synth.SMALL
    B, H, N, D, blk = w.batch, w.heads, w.N, w.head_dim, w.block
    nB = w.n_blocks
    rows = B * H * nB
    scale = 1.0 / math.sqrt(D)
    pol = GsrsPolicy(4, 1, (0.95, 0.8))
    assert [k for k, _ in pol.kinds()] == [WARMUP, SEARCH, SEARCH, REUSE]
    run = GsrsRunner(pol, B, H, N, D, blk, w.dtype)
    all_rp = (torch.arange(rows + 1) * nB).to(torch.int32)
    all_col = torch.arange(nB, dtype=torch.int32).repeat(rows)
    base = latest = None
    for s, (kind, idx) in enumerate(pol.kinds()):
        q, k, v = (t.cuda() for t in synth.make_qkv(w, 20 + s))
        res = run.step(s, q, k, v)
        ops.device_status()
        rp, col = res.mask[0].clone(), res.mask[1][:int(res.mask[0][-1])].clone()
        out = res.out.clone()
        if kind == WARMUP:
            assert _same((rp, col), (all_rp, all_col))
            _check_out(q, k, v, blk, scale, rp, col, out)
        elif kind == SEARCH:
            cand = (all_rp, all_col) if idx == 0 else base
            assert _same((rp, col), cand)
            nnz = int(rp[-1])
            mass = res.mass[:nnz].clone()
            check_attention(q, k, v, blk, scale, rp, col, out, run.lse, run.blk_lse[:nnz], mass)
            rp_c, col_c = rp.cpu().numpy(), col.cpu().numpy()
            Pm = O.mass_rows(rp_c, col_c, mass.cpu().numpy(), nB).astype(np.float32)
            np.testing.assert_array_equal(run.probs.cpu().numpy(), Pm)
            rp_o, col_o = O.topp_select(Pm, pol.p[idx], rp_c, col_c)
            nrp = res.next_mask[0].cpu().numpy()
            ncol = res.next_mask[1].cpu().numpy()[:int(nrp[-1])]
            np.testing.assert_array_equal(nrp, rp_o)
            np.testing.assert_array_equal(ncol, col_o)
            nxt = (torch.from_numpy(nrp.copy()), torch.from_numpy(ncol.copy()))
            if idx == 0:
                base = nxt
            else:
                brp, bcol = base[0].numpy(), base[1].numpy()
                for r in range(rows):
                    assert set(ncol[nrp[r]:nrp[r + 1]]) <= set(bcol[brp[r]:brp[r + 1]])
            latest = nxt
        else:
            assert _same((rp, col), latest)
            _check_out(q, k, v, blk, scale, rp, col, out)
