"""Pins for the CPU oracle: closed forms, invariants, brute force and the
hand-derived Top-p rows in tests/golden.  None of these re-types the
oracle's own formula; each is chosen so that a dropped term, a wrong sign,
scale or index, or a transposed operand in the oracle fails at least one.
"""
import itertools
import math
import os

import numpy as np
import pytest

from oracle import dsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- pooling ----

def test_block_bounds_ragged():
    assert O.block_bounds(300, 128) == [(0, 128), (128, 256), (256, 300)]
    assert O.block_bounds(256, 128) == [(0, 128), (128, 256)]
    assert O.block_bounds(1, 64) == [(0, 1)]


def test_pool_constant_blocks():
    # a tensor constant inside each block pools to that constant
    N, Bs, D = 300, 128, 5
    vals = np.array([[1.5] * D, [-2.0] * D, [7.25] * D])
    x = np.concatenate([np.tile(vals[i], (b - a, 1))
                        for i, (a, b) in enumerate(O.block_bounds(N, Bs))])
    np.testing.assert_array_equal(O.pool_blocks(x, Bs), vals)


def test_pool_ramp_midpoint_ragged():
    # x_t = t: the mean over [a, b) is (a + b - 1) / 2, also for the ragged tail
    N, Bs = 300, 128
    x = np.arange(N, dtype=np.float64)[:, None] * np.array([[1.0, -3.0]])
    got = O.pool_blocks(x, Bs)
    want = np.array([[(a + b - 1) / 2.0, -3.0 * (a + b - 1) / 2.0]
                     for a, b in O.block_bounds(N, Bs)])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# ----------------------------------------------------------- block probs ----

def test_probs_closed_form_log_weights():
    # scale * qbar . kbar_j = log(j + 1)  ->  P_j = (j + 1) / sum
    nB, scale = 6, 0.125
    qbar = np.array([[1.0, 0.0]])
    kbar = np.array([[math.log(j + 1) / scale, 3.0] for j in range(nB)])
    P = O.block_probs(qbar, kbar, scale)
    want = np.arange(1, nB + 1) / (nB * (nB + 1) / 2)
    np.testing.assert_allclose(P[0], want, rtol=1e-13)


def test_probs_rows_sum_to_one_and_shift_invariance():
    rng = np.random.default_rng(0)
    qbar, kbar = rng.normal(size=(9, 16)), rng.normal(size=(9, 16))
    P = O.block_probs(qbar, kbar, 0.25)
    assert np.all(np.abs(P.sum(1) - 1.0) <= 1e-12)
    assert np.all(P >= 0)
    # adding one vector to every key block adds a per-row constant to the logits
    P2 = O.block_probs(qbar, kbar + rng.normal(size=(1, 16)), 0.25)
    np.testing.assert_allclose(P, P2, rtol=1e-10)
    # P is not symmetric in (q, k): swapping the operands must change it
    assert not np.allclose(P, O.block_probs(kbar, qbar, 0.25))


def test_probs_uniform_and_one_hot():
    qbar = np.array([[1.0, 2.0]])
    kbar = np.tile([[0.5, -1.0]], (5, 1))
    np.testing.assert_allclose(O.block_probs(qbar, kbar, 1.0)[0], 0.2, rtol=1e-14)
    kbar[3] = [1e3, 0.0]
    P = O.block_probs(qbar, kbar, 1.0)[0]
    assert P[3] == 1.0 and np.all(np.delete(P, 3) < 1e-300)


def test_probs_reduced_renormalised():
    nB, scale = 5, 1.0
    qbar = np.array([[1.0]])
    kbar = np.array([[math.log(j + 1)] for j in range(nB)])
    P = O.block_probs(qbar, kbar, scale, cand=[np.array([1, 4])])[0]
    np.testing.assert_allclose(P, [0, 2 / 7, 0, 0, 5 / 7], rtol=1e-14, atol=0)


# ----------------------------------------------------------------- Top-p ----

def _read_golden():
    rows = []
    with open(os.path.join(GOLDEN, "topp_rows.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, p, vals, cand, want = [t.strip() for t in line.split("|")]
            r = np.array([float.fromhex(t) for t in vals.split()], np.float32)
            cand = (None if cand == "*" else
                    [] if cand == "-" else [int(t) for t in cand.split()])
            want = [] if want == "-" else [int(t) for t in want.split()]
            rows.append((name, float.fromhex(p), r, cand, want))
    return rows


@pytest.mark.parametrize("case", _read_golden(), ids=lambda c: c[0])
def test_topp_golden_rows(case):
    name, p, r, cand, want = case
    assert list(O.topp_select_row(r, p, cand)) == want


def _brute_force(r, p, cand):
    """Smallest subset of cand reaching p in exact rational arithmetic, ties
    between minimal subsets broken by the (score desc, index asc) order."""
    from fractions import Fraction
    vals = {j: Fraction(float(r[j])) for j in cand}
    pf = Fraction(float(np.float32(p)))
    if pf >= 1:
        return sorted(cand)
    rank = {j: n for n, j in enumerate(sorted(cand, key=lambda j: (-vals[j], j)))}
    for size in range(1, len(cand) + 1):
        hits = [s for s in itertools.combinations(cand, size)
                if sum(vals[j] for j in s) >= pf]
        if hits:
            best = max(sum(vals[j] for j in s) for s in hits)
            tops = [s for s in hits if sum(vals[j] for j in s) == best]
            return sorted(min(tops, key=lambda s: sorted(rank[j] for j in s)))
    return sorted(cand)


def test_topp_brute_force_small_rows():
    rng = np.random.default_rng(1)
    for trial in range(300):
        nB = int(rng.integers(1, 11))
        z = rng.normal(scale=rng.uniform(0.1, 4.0), size=nB)
        if trial % 5 == 0:          # plenty of exact ties
            z = np.round(z)
        r = (np.exp(z) / np.exp(z).sum()).astype(np.float32)
        p = float(rng.choice([0.3, 0.5, 0.7, 0.9, 0.95, 0.99, 1.0]))
        cand = list(range(nB))
        if trial % 3 == 0:
            cand = sorted(rng.choice(nB, size=int(rng.integers(0, nB + 1)),
                                     replace=False).tolist())
        got = list(O.topp_select_row(r, p, None if trial % 3 else cand))
        assert got == _brute_force(r, p, cand), (r, p, cand)


def test_topp_minimal_prefix_invariant():
    rng = np.random.default_rng(2)
    for _ in range(50):
        nB = 40
        z = rng.normal(scale=2.0, size=nB)
        r = (np.exp(z) / np.exp(z).sum()).astype(np.float32)
        p = float(rng.uniform(0.05, 0.99))
        sel = O.topp_select_row(r, p)
        tot = sum(float(r[j]) for j in sel)
        assert tot >= float(np.float32(p)) or len(sel) == nB
        # dropping the smallest kept block falls below p
        smallest = min(sel, key=lambda j: (float(r[j]), -j))
        assert tot - float(r[smallest]) < float(np.float32(p))
        # nothing outside the set beats anything inside it
        out = np.setdiff1d(np.arange(nB), sel)
        if out.size:
            assert r[out].max() <= r[sel].min()


def test_topp_reduced_all_candidates_equals_full():
    rng = np.random.default_rng(3)
    P = rng.dirichlet(np.ones(23), size=30).astype(np.float32)
    full = O.topp_select(P, 0.8)
    rp = np.arange(31) * 23
    cc = np.tile(np.arange(23), 30)
    red = O.topp_select(P, 0.8, rp, cc)
    np.testing.assert_array_equal(full[0], red[0])
    np.testing.assert_array_equal(full[1], red[1])


def test_topp_rejects_out_of_range():
    with pytest.raises(ValueError):
        O.fp32_to_fixed(1.5)
    with pytest.raises(ValueError):
        O.fp32_to_fixed(-0.25)


# ------------------------------------------------------------- attention ----

def _qkv(N, D, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (scale * rng.normal(size=(N, D)), scale * rng.normal(size=(N, D)),
            rng.normal(size=(N, D)))


def _all_blocks(nB):
    return np.arange(nB + 1) * nB, np.tile(np.arange(nB), nB)


@pytest.mark.parametrize("N,Bs", [(256, 64), (300, 128), (77, 32)])
def test_attention_p1_equals_dense_textbook(N, Bs):
    q, k, v = _qkv(N, 16, 4)
    scale = 1 / 4.0
    nB = (N + Bs - 1) // Bs
    rp, col = _all_blocks(nB)
    Os, lse, _ = O.sparse_attention_head(q, k, v, Bs, scale, rp, col)
    Od, lsed = O.dense_attention(q, k, v, scale)
    np.testing.assert_allclose(Os, Od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lsed, rtol=1e-13)


def test_attention_single_block_is_dense_on_that_block():
    N, Bs, D = 300, 128, 8
    q, k, v = _qkv(N, D, 5)
    rp = np.array([0, 1, 2, 3])
    col = np.array([2, 0, 1])          # block 0 -> 2 (ragged), 1 -> 0, 2 -> 1
    Os, lse, _ = O.sparse_attention_head(q, k, v, Bs, 0.3, rp, col)
    b = O.block_bounds(N, Bs)
    for i, j in enumerate(col):
        (a0, a1), (c0, c1) = b[i], b[j]
        Od, ld = O.dense_attention(q[a0:a1], k[c0:c1], v[c0:c1], 0.3)
        np.testing.assert_allclose(Os[a0:a1], Od, atol=1e-12)
        np.testing.assert_allclose(lse[a0:a1], ld, rtol=1e-13)


def test_attention_block_order_invariance():
    N, Bs = 384, 64
    q, k, v = _qkv(N, 8, 6)
    nB = 6
    rp = np.arange(nB + 1) * 3
    col = np.array([0, 2, 5, 1, 3, 4, 0, 1, 2, 3, 4, 5, 5, 4, 3, 2, 1, 0])
    col2 = col.reshape(nB, 3)[:, ::-1].reshape(-1)
    A = O.sparse_attention_head(q, k, v, Bs, 0.5, rp, col)
    B = O.sparse_attention_head(q, k, v, Bs, 0.5, rp, col2)
    np.testing.assert_allclose(A[0], B[0], atol=1e-12)
    np.testing.assert_allclose(A[1], B[1], rtol=1e-13)
    np.testing.assert_allclose(A[2].reshape(nB, 3, Bs)[:, ::-1],
                               B[2].reshape(nB, 3, Bs), rtol=1e-13)


def test_attention_zero_query_closed_form():
    # q = 0: every logit is 0, o_t = mean of the selected V rows and
    # lse_t = log(#selected keys); block mass = |B_j| / sum |B_j'|
    N, Bs, D = 200, 64, 4
    _, k, v = _qkv(N, D, 7)
    q = np.zeros((N, D))
    rp = np.array([0, 2, 2, 3, 5])     # row 1 is empty
    col = np.array([1, 3, 3, 0, 3])    # block 3 is ragged (8 tokens)
    Os, lse, blk = O.sparse_attention_head(q, k, v, Bs, 1.0, rp, col)
    b = O.block_bounds(N, Bs)
    for i in range(4):
        a0, a1 = b[i]
        sel = col[rp[i]:rp[i + 1]]
        if sel.size == 0:
            assert np.all(Os[a0:a1] == 0) and np.all(lse[a0:a1] == -np.inf)
            continue
        keys = np.concatenate([np.arange(*b[j]) for j in sel])
        np.testing.assert_allclose(Os[a0:a1], np.tile(v[keys].mean(0), (a1 - a0, 1)),
                                   atol=1e-12)
        np.testing.assert_allclose(lse[a0:a1], math.log(keys.size), rtol=1e-14)
    M = O.block_mass(lse, blk, rp, N, Bs)
    np.testing.assert_allclose(M, [64 / 72, 8 / 72, 1.0, 64 / 72, 8 / 72], rtol=1e-13)


def test_block_mass_sums_to_one_and_matches_dense_weights():
    N, Bs = 320, 64
    q, k, v = _qkv(N, 8, 8, scale=0.8)
    nB = 5
    rp, col = _all_blocks(nB)
    _, lse, blk = O.sparse_attention_head(q, k, v, Bs, 0.4, rp, col)
    M = O.block_mass(lse, blk, rp, N, Bs).reshape(nB, nB)
    np.testing.assert_allclose(M.sum(1), 1.0, rtol=1e-12)
    # at p = 1 the mass equals the block sums of the dense softmax matrix
    z = 0.4 * q @ k.T
    w = np.exp(z) / np.exp(z).sum(1, keepdims=True)
    b = O.block_bounds(N, Bs)
    dense = np.array([[w[a0:a1, c0:c1].sum(1).mean() for (c0, c1) in b] for (a0, a1) in b])
    np.testing.assert_allclose(M, dense, rtol=1e-12)


def test_mass_rows_closed_form():
    # two rows of a 5-block mask, columns in any order
    rp = np.array([0, 3, 5])
    col = np.array([4, 0, 2, 1, 3])
    mass = np.array([0.5, 0.25, 0.25, 0.75, 0.25])
    R = O.mass_rows(rp, col, mass, 5)
    np.testing.assert_array_equal(R, [[0.25, 0.0, 0.25, 0.0, 0.5], [0.0, 0.75, 0.0, 0.25, 0.0]])


def test_mass_reselection_is_topp_of_dense_block_weights():
    # Top-p on the exact masses from an all-blocks pass equals, by brute
    # force over all subsets of the block weights of the textbook softmax
    # matrix, the heaviest subset among the smallest ones reaching p; within
    # a candidate mask, p = 1 keeps the mask and the result is always a
    # subset of it.
    N, Bs, D, scale = 384, 64, 8, 0.6
    q, k, v = _qkv(N, D, 11, scale=1.2)
    nB = 6
    rp, col = _all_blocks(nB)
    _, lse, blk = O.sparse_attention_head(q, k, v, Bs, scale, rp, col)
    M = O.block_mass(lse, blk, rp, N, Bs)
    P = O.mass_rows(rp, col, M, nB).astype(np.float32)
    z = scale * q @ k.T
    w = np.exp(z - z.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    b = O.block_bounds(N, Bs)
    W = np.array([[w[a0:a1, c0:c1].sum(1).mean() for (c0, c1) in b] for (a0, a1) in b])
    for p in (0.5, 0.8, 0.95):
        srp, scol = O.topp_select(P, p, rp, col)
        for i in range(nB):
            best = None
            for size in range(1, nB + 1):
                ok = [sub for sub in itertools.combinations(range(nB), size)
                      if W[i, list(sub)].sum() >= p]
                if ok:
                    best = max(ok, key=lambda sub: W[i, list(sub)].sum())
                    break
            np.testing.assert_array_equal(scol[srp[i]:srp[i + 1]], sorted(best))
    cand_rp, cand_col = O.topp_select(P, 0.9, rp, col)
    keep_rp, keep_col = O.topp_select(P, 1.0, cand_rp, cand_col)
    np.testing.assert_array_equal(keep_rp, cand_rp)
    np.testing.assert_array_equal(keep_col, cand_col)
    sub_rp, sub_col = O.topp_select(P, 0.6, cand_rp, cand_col)
    for i in range(nB):
        assert set(sub_col[sub_rp[i]:sub_rp[i + 1]]) <= set(cand_col[cand_rp[i]:cand_rp[i + 1]])


def test_recall_is_one_at_p1_and_pipeline_reduced_equals_full():
    N, Bs, D = 256, 64, 8
    q, k, v = _qkv(N, D, 9, scale=1.5)
    nB = 4
    rp, col = _all_blocks(nB)
    np.testing.assert_allclose(O.recall(q, k, Bs, 0.35, rp, col), 1.0, rtol=1e-12)
    full = O.pipeline_head(q, k, v, Bs, 0.35, 0.9)
    red = O.pipeline_head(q, k, v, Bs, 0.35, 0.9, rp, col)
    np.testing.assert_array_equal(full["row_ptr"], red["row_ptr"])
    np.testing.assert_array_equal(full["col"], red["col"])
    np.testing.assert_array_equal(full["O"], red["O"])


def test_recall_zero_query_is_selected_key_fraction():
    # q = 0: the dense softmax is uniform over all N keys, so a row's recall
    # is (keys in its selected blocks) / N, whatever the keys are
    N, Bs, D = 200, 64, 4           # blocks of 64, 64, 64 and 8 tokens
    _, k, _ = _qkv(N, D, 12, scale=2.0)
    q = np.zeros((N, D))
    rp = np.array([0, 2, 2, 3, 4])  # row 1 selects nothing
    col = np.array([0, 3, 3, 1])
    r = O.recall(q, k, Bs, 0.7, rp, col)
    np.testing.assert_allclose(r, [72 / 200, 0.0, 8 / 200, 64 / 200], rtol=1e-14)


def test_recall_block_constant_keys_closed_form():
    # keys constant within each block (k_u = c_j): a query's dense weight on
    # block j is |B_j| e^{z_j} / sum_j' |B_j'| e^{z_j'} with z_j = s q.c_j, so
    # recall_i = mean_t of the selected blocks' share.  Ragged sizes and
    # distinct per-block logits make a wrong block index or size fail.
    N, Bs, D, s = 200, 64, 3, 0.8
    b = O.block_bounds(N, Bs)
    rng = np.random.default_rng(13)
    c = rng.normal(size=(len(b), D))
    k = np.concatenate([np.tile(c[j], (b1 - b0, 1)) for j, (b0, b1) in enumerate(b)])
    q = rng.normal(size=(N, D))
    rp = np.array([0, 1, 3, 4, 6])
    col = np.array([3, 0, 2, 1, 1, 3])
    sizes = np.array([b1 - b0 for b0, b1 in b], dtype=np.float64)
    r = O.recall(q, k, Bs, s, rp, col)
    for i, (a0, a1) in enumerate(b):
        z = s * (q[a0:a1] @ c.T)                      # [queries, blocks]
        wts = sizes[None, :] * np.exp(z)
        share = wts[:, col[rp[i]:rp[i + 1]]].sum(1) / wts.sum(1)
        np.testing.assert_allclose(r[i], share.mean(), rtol=1e-12)


def test_executed_flops_counts_ragged_blocks():
    rp = np.array([0, 2, 3])
    col = np.array([0, 1, 1])          # N = 100, Bs = 64: blocks of 64 and 36
    assert O.executed_flops(rp, col, 100, 64, 8) == 4 * 8 * (64 * 64 + 64 * 36 + 36 * 36)


# --------------------------------------------------------- Hilbert order ----

def _cells(perm, H, W, n_prefix=0):
    g = np.asarray(perm[n_prefix:]) - n_prefix
    return np.stack([g // (H * W), (g // W) % H, g % W], axis=1)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_hilbert_cube_is_a_unit_step_path_with_adjacent_ends(bits):
    n = 1 << bits
    perm = O.hilbert_order(n, n, n)
    assert sorted(perm.tolist()) == list(range(n ** 3))
    c = _cells(perm, n, n)
    steps = np.abs(np.diff(c, axis=0)).sum(1)
    assert np.all(steps == 1)                       # continuity of the curve
    assert tuple(c[0]) == (0, 0, 0)
    end = c[-1]                                     # the 3-D curve ends at an adjacent corner
    assert sorted(end.tolist()) == [0, 0, n - 1]


def test_hilbert_subgrid_is_the_cube_order_filtered_and_prefix_is_kept():
    T, H, W, P = 3, 5, 6, 4
    perm = O.hilbert_order(T, H, W, P)
    assert perm[:P].tolist() == list(range(P))
    assert sorted(perm.tolist()) == list(range(P + T * H * W))
    cube = _cells(O.hilbert_order(8, 8, 8), 8, 8)
    inside = [tuple(c) for c in cube if c[0] < T and c[1] < H and c[2] < W]
    assert [tuple(c) for c in _cells(perm, H, W, P)] == inside


def test_hilbert_blocks_are_more_compact_than_row_major():
    T, H, W, Bs = 6, 12, 20, 64
    perm = O.hilbert_order(T, H, W)
    def extent(order):
        c = _cells(order, H, W)
        ext = []
        for a in range(0, len(order), Bs):
            blk = c[a:a + Bs]
            ext.append(np.prod(blk.max(0) - blk.min(0) + 1))
        return float(np.mean(ext))
    assert extent(perm) < 0.5 * extent(np.arange(T * H * W))


def _hamiltonian_corner_walk_exists(a, b, c):
    """Brute force: is there a path through every cell of an a x b x c box
    (axes t, y, x) with unit steps from (0, 0, 0) to (a - 1, 0, 0)?"""
    n = a * b * c
    start, goal = (0, 0, 0), (a - 1, 0, 0)
    seen = {start}

    def dfs(p):
        if len(seen) == n:
            return p == goal
        for d in ((1, 0, 0), (-1, 0, 0), (0, 1, 0), (0, -1, 0), (0, 0, 1), (0, 0, -1)):
            q = (p[0] + d[0], p[1] + d[1], p[2] + d[2])
            if 0 <= q[0] < a and 0 <= q[1] < b and 0 <= q[2] < c and q not in seen:
                if q == goal and len(seen) + 1 < n:
                    continue
                seen.add(q)
                if dfs(q):
                    return True
                seen.discard(q)
        return False

    return dfs(start)


def test_gilbert_walk_feasibility_rule_is_exact_on_small_boxes():
    # the two-colouring rule used to choose splits, against exhaustive search
    for a, b, c in itertools.product(range(1, 6), range(1, 5), range(1, 5)):
        if a * b * c > 24:
            continue
        assert O._walk_feasible(a, b, c) == _hamiltonian_corner_walk_exists(a, b, c), (a, b, c)


def _gilbert_cells(T, H, W, P=0):
    perm = O.gilbert_order(T, H, W, P)
    assert perm[:P].tolist() == list(range(P))
    assert sorted(perm.tolist()) == list(range(P + T * H * W))
    return _cells(perm, H, W, P)


def test_gilbert_is_a_unit_step_walk_on_every_small_box():
    # GSRS Figure 6: a Hilbert curve generalised to boxes of any size; every
    # box up to 7 x 7 x 7, including odd and one-cell-thick ones
    for T, H, W in itertools.product(range(1, 8), repeat=3):
        c = _gilbert_cells(T, H, W, 2)
        if len(c) > 1:
            assert np.all(np.abs(np.diff(c, axis=0)).sum(1) == 1), (T, H, W)
        assert tuple(c[0]) == (0, 0, 0)
        # it ends at the far corner along the longest walkable axis
        dims = (T, H, W)
        end = c[-1].tolist()
        assert sum(1 for d, e in zip(dims, end) if e != 0) <= 1
        moved = [i for i in range(3) if end[i] != 0]
        if moved:
            assert end[moved[0]] == dims[moved[0]] - 1


@pytest.mark.parametrize("T,H,W,P", [(21, 45, 80, 0), (33, 45, 80, 0), (13, 30, 45, 226),
                                     (8, 16, 16, 0), (4, 8, 8, 0)])
def test_gilbert_workload_grids_walk_and_are_compact(T, H, W, P):
    c = _gilbert_cells(T, H, W, P)
    assert np.all(np.abs(np.diff(c, axis=0)).sum(1) == 1)
    def spread(cells, Bs=128):
        out = []
        for a in range(0, len(cells), Bs):
            blk = cells[a:a + Bs].astype(np.float64)
            out.append(((blk - blk.mean(0)) ** 2).sum(1).mean())
        return float(np.mean(out))
    row_major = _cells(np.arange(P + T * H * W), H, W, P)
    cube = _cells(O.hilbert_order(T, H, W, P), H, W, P)
    # about as compact as the enclosing cube's curve, more than row-major
    # (far more once a row of the grid is longer than a block)
    assert spread(c) < 1.25 * spread(cube)
    assert spread(c) < (0.1 if W * H > 128 * 8 else 0.9) * spread(row_major)


# ----------------------------------------------------- hierarchical scores ----

def test_hier_probs_sub1_is_block_probs_and_rows_sum_to_one():
    N, Bs, D = 300, 64, 8
    q, k, _ = _qkv(N, D, 21, scale=1.3)
    P1 = O.hier_block_probs(q, k, Bs, 1, 0.4)
    ref = O.block_probs(O.pool_blocks(q, Bs), O.pool_blocks(k, Bs), 0.4)
    np.testing.assert_allclose(P1, ref, rtol=1e-13, atol=1e-15)
    for sub in (2, 4):
        P = O.hier_block_probs(q, k, Bs, sub, 0.4)
        np.testing.assert_allclose(P.sum(1), 1.0, rtol=1e-12)
        assert P.shape == ref.shape and np.all(P >= 0)


def test_hier_probs_block_constant_closed_form():
    # tokens constant within each block: every key sub-block of block j scores
    # s_ij, so P_ij = n_j e^{s_ij} / sum_j' n_j' e^{s_ij'} with n_j the number
    # of key sub-blocks in block j (the ragged last block has fewer)
    Bs, sub, D = 64, 4, 6
    N = 3 * Bs + 20                       # last block: 20 tokens -> 2 sub-blocks of 16
    rng = np.random.default_rng(4)
    qv, kv = rng.normal(size=(4, D)), rng.normal(size=(4, D))
    blk = np.minimum(np.arange(N) // Bs, 3)
    q, k = qv[blk], kv[blk]
    P = O.hier_block_probs(q, k, Bs, sub, 0.7)
    n = np.array([4, 4, 4, 2])
    s = 0.7 * qv @ kv.T
    e = n[None, :] * np.exp(s)
    np.testing.assert_allclose(P, e / e.sum(1, keepdims=True), rtol=1e-12)


# ---------------------------------------------------------------- backward ----

def test_backward_all_blocks_equals_autograd_of_dense_attention():
    torch = pytest.importorskip("torch")
    N, Bs, D, scale = 200, 64, 8, 0.37
    q, k, v = _qkv(N, D, 31, scale=1.1)
    dO = np.random.default_rng(32).normal(size=(N, D))
    nB = 4
    rp, col = _all_blocks(nB)
    dQ, dK, dV = O.sparse_attention_backward_head(q, k, v, dO, Bs, scale, rp, col)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    out = torch.softmax(scale * tq @ tk.T, dim=1) @ tv
    out.backward(torch.tensor(dO))
    np.testing.assert_allclose(dQ, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_delta_from_stored_output_matches_exact_form():
    # sum(P * dP) per row equals rowsum(dO * O) for the exact O
    N, Bs, D, scale = 96, 32, 5, 0.5
    q, k, v = _qkv(N, D, 51, scale=1.0)
    dO = np.random.default_rng(52).normal(size=(N, D))
    rp = np.array([0, 2, 3, 5])
    col = np.array([0, 2, 1, 0, 1])
    out, _, _ = O.sparse_attention_head(q, k, v, Bs, scale, rp, col)
    a = O.sparse_attention_backward_head(q, k, v, dO, Bs, scale, rp, col)
    b = O.sparse_attention_backward_head(q, k, v, dO, Bs, scale, rp, col, out=out)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-11, atol=1e-12)


def test_backward_masked_matches_finite_differences():
    N, Bs, D, scale = 40, 16, 3, 0.6
    q, k, v = _qkv(N, D, 41, scale=1.0)
    dO = np.random.default_rng(42).normal(size=(N, D))
    rp = np.array([0, 2, 3, 3])          # row 0: blocks 0, 2; row 1: block 1; row 2: empty
    col = np.array([2, 0, 1])
    dQ, dK, dV = O.sparse_attention_backward_head(q, k, v, dO, Bs, scale, rp, col)

    def loss(qq, kk, vv):
        out, _, _ = O.sparse_attention_head(qq, kk, vv, Bs, scale, rp, col)
        return float((out * dO).sum())
    h = 1e-6
    for name, x, g in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        for (r, c) in [(0, 0), (5, 2), (17, 1), (33, 0), (39, 2)]:
            xp, xm = x.copy(), x.copy()
            xp[r, c] += h
            xm[r, c] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[r, c]) <= 1e-6 * max(1.0, abs(fd)), (name, r, c, fd, g[r, c])
    assert np.all(dQ[32:] == 0)          # empty row: no gradient
