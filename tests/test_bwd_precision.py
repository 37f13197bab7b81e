"""Why the tensor-core backward feeds P and dS to its gradient products as bf16
hi + lo pairs, checked on the CPU.

The backward's products run with bf16 operands.  dS = P * (dP - delta) sums
to zero along each row, so dQ = scale * dS K cancels heavily.  This test
emulates the gradient products with P and dS rounded to bf16 -- once as
single terms, once as hi = bf16(x) plus lo = bf16(x - hi) -- against the
fp64 chain rule of the oracle, on masks of the small configuration, and
applies the GPU backward tests' bf16 gate (|err| <= |ref|/128 + 2e-3 max|ref|
after rounding the stored gradient to bf16).  The single-term dQ must break
the gate and the split form must meet it with margin; so the gate is tight
enough to notice a missing split, and the split is what the kernels need.
"""
import math

import numpy as np
import pytest
import torch

from dynamic_block_sparse_pool_b200 import synth
from oracle import dsa_oracle as O


def bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).double().numpy()


def emulate(q, k, v, dO, Bs, scale, rp, col, out, split):
    """The gradient products with bf16 P and dS (single terms or hi + lo)."""
    N, D = q.shape
    bounds = O.block_bounds(N, Bs)
    dQ, dK, dV = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)

    def terms(x):
        hi = bf16(x)
        return [hi, bf16(x - hi)] if split else [hi]

    for i, (a, b) in enumerate(bounds):
        sel = [int(c) for c in col[int(rp[i]):int(rp[i + 1])]]
        if not sel:
            continue
        keys = np.concatenate([np.arange(*bounds[j]) for j in sel])
        logits = scale * (q[a:b] @ k[keys].T)
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        P = e / e.sum(axis=1, keepdims=True)
        dP = dO[a:b] @ v[keys].T
        delta = (dO[a:b] * out[a:b]).sum(axis=1, keepdims=True)
        dS = P * (dP - delta)
        dQ[a:b] = scale * sum(t @ k[keys] for t in terms(dS))
        np.add.at(dK, keys, scale * sum(t.T @ q[a:b] for t in terms(dS)))
        np.add.at(dV, keys, sum(t.T @ dO[a:b] for t in terms(P)))
    return dQ, dK, dV


def worst_gate_ratio(seeds, heads, split):
    w = synth.SMALL
    scale = 1.0 / math.sqrt(w.head_dim)
    worst = {"q": 0.0, "k": 0.0, "v": 0.0}
    for seed in seeds:
        q, k, v = synth.make_qkv(w, seed)
        for h in heads:
            qh, kh, vh = (t[0, h].double().numpy() for t in (q, k, v))
            Pm = O.block_probs(O.pool_blocks(qh, w.block), O.pool_blocks(kh, w.block), scale)
            rp, col = O.topp_select(Pm.astype(np.float32), 0.9)
            out, _, _ = O.sparse_attention_head(qh, kh, vh, w.block, scale, rp, col)
            out = bf16(out)  # the stored forward output
            dO = bf16(np.random.default_rng(100 * seed + h).normal(size=qh.shape))
            ref = O.sparse_attention_backward_head(qh, kh, vh, dO, w.block, scale, rp, col,
                                                   out=out)
            got = emulate(qh, kh, vh, dO, w.block, scale, rp, col, out, split)
            for name, g, r in zip("qkv", got, ref):
                gate = np.abs(r) / 128 + 2e-3 * np.abs(r).max()
                worst[name] = max(worst[name], float((np.abs(bf16(g) - r) / gate).max()))
    return worst


@pytest.mark.parametrize("seed", [17, 19])
def test_single_bf16_ds_breaks_the_dq_gate(seed):
    worst = worst_gate_ratio([seed], [1, 3], split=False)
    assert worst["q"] > 1.0, worst


@pytest.mark.parametrize("seed", [17, 19])
def test_hi_lo_split_meets_every_gate_with_margin(seed):
    worst = worst_gate_ratio([seed], [1, 3], split=True)
    assert max(worst.values()) < 0.6, worst
