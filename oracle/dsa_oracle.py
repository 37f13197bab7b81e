"""CPU oracle for dynamic block-sparse self-attention (fp64, NumPy).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code, tables or constants with the CUDA library; the two meet only
in the seeded input generator.

What it computes, step by step, per (batch, head):

1. Block partition.  Tokens 0..N-1 (row-major (t, y, x) grid order, prefix
   tokens first) are cut into blocks B_i = [i*Bs, min(N, (i+1)*Bs)).  The
   same partition serves queries and keys.  Sources: the block-level
   attention maps of GSRS (arXiv 2610.21129), Figure 3; the partition
   itself is the plainest reading of "query and key blocks".
2. Pooled block score.  qbar_i, kbar_j are fp64 means over the actual rows
   of each block; s_ij = scale * qbar_i . kbar_j; P_i. is the row softmax
   over all key blocks, or, in reduced search, over the candidate set C_i
   only (P_ij = 0 outside C_i).  Reduced search: GSRS abstract and
   Figure 4 ("subsequent search steps only evaluate blocks within this
   baseline mask").  The pooled score itself is not defined in the GSRS,
   DSV, DFSAttn or Sparse-vDiT abstracts; mean pooling followed by a plain
   row softmax (no temperature) is the reading taken here.
3. Top-p selection.  GSRS abstract ("Top-p selection for adaptive sparsity
   control") and Figure 4 (tighter Top-p retains fewer blocks).  Per row,
   candidates are ordered by (P desc, index asc); the kept set is the
   shortest prefix whose cumulative mass is >= p.  The comparison is done
   in exact integer arithmetic on the fp32 values (every fp32 value in
   [0, 1] is an integer multiple of 2^-149), so it has a single answer.
   p >= 1 keeps every candidate.  If no prefix reaches p (p within fp32
   rounding of the row total) every candidate is kept.
4. Block-sparse attention on a given mask.  For query t in block i, the
   keys are the union of the selected key blocks (tokens < N only):
   o_t = sum_u softmax_u(scale * q_t . k_u) v_u, lse_t = log sum_u
   exp(scale * q_t . k_u) (natural log).  This is FlashAttention's result
   (GSRS abstract: exact weights "within the FlashAttention computation");
   the oracle forms it directly, not with an online softmax.
5. Exact block mass.  blk_lse[t, j] = log sum_{u in B_j} exp(scale q_t.k_u);
   M_ij = mean over t in B_i of exp(blk_lse[t, j] - lse_t).  Rows of M sum
   to 1 over the selected set (GSRS abstract: "computes exact attention
   weights ... at negligible overhead"; Figure 2 uses the same quantity as
   attention recall).

Where the papers are silent this module takes the plainest reading: scale =
1/sqrt(D) by default, means over the actual rows of a ragged block, keys at
positions >= N never attended, natural-log lse, an empty row gives O = 0 and
lse = -inf, and selected columns are listed in ascending order.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

TWO_149 = 2.0 ** 149  # one unit in the last place of the smallest fp32 denormal


# ---------------------------------------------------------------------------
# 1. Block partition and pooling
# ---------------------------------------------------------------------------

def block_bounds(N: int, Bs: int) -> List[Tuple[int, int]]:
    """[start, end) of each block of Bs consecutive tokens; the last is ragged."""
    nB = (N + Bs - 1) // Bs
    return [(i * Bs, min(N, (i + 1) * Bs)) for i in range(nB)]


def pool_blocks(x: np.ndarray, Bs: int) -> np.ndarray:
    """Mean of the actual rows of each block: x [N, D] -> [nB, D], fp64."""
    x = np.asarray(x, dtype=np.float64)
    return np.stack([x[a:b].mean(axis=0) for a, b in block_bounds(len(x), Bs)])


# ---------------------------------------------------------------------------
# 2. Block scores and row softmax
# ---------------------------------------------------------------------------

def block_probs(qbar: np.ndarray, kbar: np.ndarray, scale: float,
                cand: Optional[Sequence[np.ndarray]] = None) -> np.ndarray:
    """P [nB, nB]: softmax_j(scale * qbar_i . kbar_j), over C_i if given."""
    s = scale * (np.asarray(qbar, np.float64) @ np.asarray(kbar, np.float64).T)
    nB = s.shape[1]
    P = np.zeros_like(s)
    for i in range(s.shape[0]):
        cols = np.arange(nB) if cand is None else np.asarray(cand[i], np.int64)
        if cols.size == 0:
            continue
        z = s[i, cols]
        e = np.exp(z - z.max())
        P[i, cols] = e / e.sum()
    return P


def hier_block_probs(q: np.ndarray, k: np.ndarray, Bs: int, sub: int, scale: float) -> np.ndarray:
    """Two-level block estimate (DFSAttn abstract: hierarchical block scoring
    for block importance; the pages give no construction, this is the plain
    two-level pooling).  Tokens are pooled over sub-blocks of Bs/sub rows;
    each query sub-block a takes the row softmax of scale * qbar_a . kbar_b
    over all key sub-blocks b; block row i is the token-weighted mean over
    its query sub-blocks of the mass falling in each key block j:

        P_ij = sum_{a in i} (|a| / |B_i|) sum_{b in j} softmax_b(...)_ab.

    sub = 1 is block_probs."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    N = q.shape[0]
    bf = Bs // sub
    Pf = block_probs(pool_blocks(q, bf), pool_blocks(k, bf), scale)
    fine = block_bounds(N, bf)
    coarse = block_bounds(N, Bs)
    P = np.zeros((len(coarse), len(coarse)))
    for i, (i0, i1) in enumerate(coarse):
        for a, (a0, a1) in enumerate(fine):
            if i0 <= a0 < i1:
                w = (a1 - a0) / (i1 - i0)
                for j, (j0, j1) in enumerate(coarse):
                    cols = [b for b, (b0, _) in enumerate(fine) if j0 <= b0 < j1]
                    P[i, j] += w * Pf[a, cols].sum()
    return P


# ---------------------------------------------------------------------------
# 3. Top-p selection (exact)
# ---------------------------------------------------------------------------

def fp32_to_fixed(x) -> int:
    """An fp32 value in [0, 1] as the exact integer x * 2^149."""
    v = float(np.float32(x))
    if not (0.0 <= v <= 1.0) or math.isnan(v):
        raise ValueError(f"probability out of [0, 1]: {v!r}")
    return int(v * TWO_149)  # exact: v * 2^149 is an integer below 2^150


def topp_select_row(r: np.ndarray, p: float,
                    cand: Optional[Sequence[int]] = None) -> np.ndarray:
    """Selected key blocks of one row, ascending.

    r: the row's fp32 block probabilities.  p: Top-p threshold, taken as an
    fp32 value.  cand: the candidate columns (reduced search) or None (all).
    """
    r = np.asarray(r, dtype=np.float32)
    cols = list(range(r.size)) if cand is None else [int(c) for c in cand]
    if not cols:
        return np.zeros(0, dtype=np.int64)
    p32 = float(np.float32(p))
    if p32 >= 1.0:
        return np.array(sorted(cols), dtype=np.int64)
    order = sorted(cols, key=lambda j: (-float(r[j]), j))
    target = fp32_to_fixed(p32)
    acc = 0
    k_star = len(order)
    for k, j in enumerate(order, start=1):
        acc += fp32_to_fixed(r[j])
        if acc >= target:
            k_star = k
            break
    return np.array(sorted(order[:k_star]), dtype=np.int64)


def topp_select(P: np.ndarray, p: float,
                cand_row_ptr: Optional[np.ndarray] = None,
                cand_col: Optional[np.ndarray] = None):
    """Top-p over every row of P [rows, nB] (fp32 values) -> CSR (int64)."""
    P = np.asarray(P, dtype=np.float32)
    rows = P.shape[0]
    row_ptr = np.zeros(rows + 1, dtype=np.int64)
    cols = []
    for i in range(rows):
        cand = None
        if cand_row_ptr is not None:
            cand = cand_col[int(cand_row_ptr[i]):int(cand_row_ptr[i + 1])]
        sel = topp_select_row(P[i], p, cand)
        cols.append(sel)
        row_ptr[i + 1] = row_ptr[i] + sel.size
    col = np.concatenate(cols) if cols else np.zeros(0, np.int64)
    return row_ptr, col.astype(np.int64)


def csr_rows(row_ptr, col) -> List[np.ndarray]:
    """CSR -> list of per-row column arrays."""
    return [np.asarray(col[int(row_ptr[i]):int(row_ptr[i + 1])], np.int64)
            for i in range(len(row_ptr) - 1)]


# ---------------------------------------------------------------------------
# 4./5. Attention over a given block mask, and exact block mass
# ---------------------------------------------------------------------------

def sparse_attention_head(q, k, v, Bs: int, scale: float, row_ptr, col,
                          rows: Optional[Sequence[int]] = None):
    """Attention of one head over the CSR mask (row i = query block i).

    Returns (O [N, D], lse [N], blk_lse [nnz, Bs]) in fp64.  Entries of rows
    not computed (see ``rows``) and blk_lse rows past a ragged block are NaN.
    An empty row gives O = 0 and lse = -inf.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    N, D = q.shape
    bounds = block_bounds(N, Bs)
    nnz = int(row_ptr[-1])
    O = np.full((N, v.shape[1]), np.nan)
    lse = np.full(N, np.nan)
    blk = np.full((nnz, Bs), np.nan)
    for i in (range(len(bounds)) if rows is None else rows):
        a, b = bounds[i]
        s0, s1 = int(row_ptr[i]), int(row_ptr[i + 1])
        sel = [int(c) for c in col[s0:s1]]
        if not sel:
            O[a:b] = 0.0
            lse[a:b] = -np.inf
            continue
        keys = np.concatenate([np.arange(*bounds[j]) for j in sel])
        logits = scale * (q[a:b] @ k[keys].T)            # [|B_i|, |keys|]
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        denom = e.sum(axis=1, keepdims=True)
        O[a:b] = (e @ v[keys]) / denom
        lse[a:b] = (m + np.log(denom))[:, 0]
        off = 0
        for slot, j in enumerate(sel):
            n_j = bounds[j][1] - bounds[j][0]
            part = e[:, off:off + n_j].sum(axis=1)
            with np.errstate(divide="ignore"):
                blk[s0 + slot, :b - a] = m[:, 0] + np.log(part)
            off += n_j
    return O, lse, blk


def sparse_attention_backward_head(q, k, v, dO, Bs: int, scale: float, row_ptr, col, out=None):
    """Gradients (dQ, dK, dV) [N, D] of the block-sparse attention output O
    (as sparse_attention_head computes it, for a fixed mask) against the
    upstream gradient dO, in fp64.  DSV abstract: attention is trained with
    the same sparsity; this is the chain rule through each query's softmax
    over the keys of its selected blocks:

        P = softmax(scale * q K_sel^T),  dP = dO_q V_sel^T,
        dS = P * (dP - sum(P * dP)),
        dQ_q = scale * dS K_sel,  dK_sel += scale * dS^T q,  dV_sel += P^T dO_q.

    Queries of an empty row get dQ = 0 and add nothing to dK, dV.

    out: if given, the stored forward output; the row term sum(P * dP),
    which equals rowsum(dO * O) for the exact O, is then taken as
    rowsum(dO * out) -- the form a backward pass that receives O as an input
    computes (so a rounded stored O enters as it does there)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dO = np.asarray(dO, np.float64)
    N, D = q.shape
    bounds = block_bounds(N, Bs)
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    for i, (a, b) in enumerate(bounds):
        sel = [int(c) for c in col[int(row_ptr[i]):int(row_ptr[i + 1])]]
        if not sel:
            continue
        keys = np.concatenate([np.arange(*bounds[j]) for j in sel])
        logits = scale * (q[a:b] @ k[keys].T)
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        P = e / e.sum(axis=1, keepdims=True)
        dP = dO[a:b] @ v[keys].T
        if out is None:
            delta = (P * dP).sum(axis=1, keepdims=True)
        else:
            delta = (dO[a:b] * np.asarray(out, np.float64)[a:b]).sum(axis=1, keepdims=True)
        dS = P * (dP - delta)
        dQ[a:b] = scale * (dS @ k[keys])
        np.add.at(dK, keys, scale * (dS.T @ q[a:b]))
        np.add.at(dV, keys, P.T @ dO[a:b])
    return dQ, dK, dV


def block_mass(lse, blk_lse, row_ptr, N: int, Bs: int) -> np.ndarray:
    """M [nnz]: for slot s of row i, mean_{t in B_i} exp(blk_lse[s,t] - lse_t)."""
    lse = np.asarray(lse, np.float64)
    blk_lse = np.asarray(blk_lse, np.float64)
    bounds = block_bounds(N, Bs)
    M = np.zeros(int(row_ptr[-1]))
    for i, (a, b) in enumerate(bounds):
        for s in range(int(row_ptr[i]), int(row_ptr[i + 1])):
            M[s] = np.mean(np.exp(blk_lse[s, :b - a] - lse[a:b]))
    return M


def mass_rows(row_ptr, col, mass, nB: int) -> np.ndarray:
    """Dense rows [rows, nB] holding each slot's exact block mass at its
    column and 0 elsewhere.  GSRS abstract: Top-p selection on exact
    attention weights; Figure 4: later searches evaluate only the candidate
    mask -- so these rows, with the same CSR as candidates, are the input of
    a mass-driven reselection (topp_select with cand)."""
    rows = len(row_ptr) - 1
    out = np.zeros((rows, nB), dtype=np.float64)
    for r in range(rows):
        for s in range(int(row_ptr[r]), int(row_ptr[r + 1])):
            out[r, int(col[s])] = float(mass[s])
    return out


def hilbert_index3(t: int, y: int, x: int, bits: int) -> int:
    """Position of cell (t, y, x) along the 3-D Hilbert curve of the cube of
    side 2^bits: Skilling's axes-to-transpose method ("Programming the
    Hilbert curve", 2004) followed by interleaving the bits of the
    transposed coordinates, most significant first, t before y before x.
    (GSRS Figure 6 and DFSAttn abstract: tokens reordered along a Hilbert
    curve so that a block covers a compact spatio-temporal region.)"""
    X = [t, y, x]
    n = 3
    top = 1 << (bits - 1)
    # undo the excess work: for each bit from the top, invert or exchange
    q = top
    while q > 1:
        low = q - 1
        for i in range(n):
            if X[i] & q:
                X[0] ^= low
            else:
                swap = (X[0] ^ X[i]) & low
                X[0] ^= swap
                X[i] ^= swap
        q >>= 1
    # Gray encode
    for i in range(1, n):
        X[i] ^= X[i - 1]
    flip = 0
    q = top
    while q > 1:
        if X[n - 1] & q:
            flip ^= q - 1
        q >>= 1
    for i in range(n):
        X[i] ^= flip
    # interleave: bit b of X[0], X[1], X[2], for b from the top down
    h = 0
    for b in range(bits - 1, -1, -1):
        for i in range(n):
            h = (h << 1) | ((X[i] >> b) & 1)
    return h


def hilbert_order(T: int, H: int, W: int, n_prefix: int = 0) -> np.ndarray:
    """perm [n_prefix + T*H*W]: perm[i] = original index of the token placed
    at position i.  The text prefix keeps positions 0 .. n_prefix - 1; grid
    token (t, y, x) (original index n_prefix + (t*H + y)*W + x) is placed by
    its Hilbert index on the enclosing power-of-two cube (cells outside the
    grid are skipped)."""
    bits = max(1, max(T, H, W) - 1).bit_length()
    keys = []
    for t in range(T):
        for y in range(H):
            for x in range(W):
                keys.append((hilbert_index3(t, y, x, bits), n_prefix + (t * H + y) * W + x))
    keys.sort()
    return np.array(list(range(n_prefix)) + [idx for _, idx in keys], dtype=np.int64)


def _walk_feasible(a: int, b: int, c: int) -> bool:
    """Whether an a x b x c box has a walk through every cell with unit
    steps from one corner to the corner a - 1 cells away along the first
    axis.  Colour the cells by the parity of their coordinate sum: a walk
    alternates colours, so its two ends differ in colour iff it has an even
    number of cells; the two corners differ in colour iff a is even.  Hence
    a odd needs b * c odd.  A box of more than one cell also needs a >= 2
    (the two ends must differ)."""
    if a * b * c == 1:
        return True
    return a >= 2 and not (a % 2 == 1 and (b * c) % 2 == 0)


def _nearest_first(n: int, lo: int, hi: int) -> List[int]:
    """The integers of [lo, hi], closest to n first (the smaller first on a tie)."""
    out = []
    for d in range(0, hi - lo + 2):
        for x in (n - d, n + d):
            if lo <= x <= hi and x not in out:
                out.append(x)
    return out


def _gilbert_walk(entry, U, V, W, out: list) -> None:
    """Cells of one box in walk order, appended to out.

    entry: the first cell (t, y, x).  U, V, W: the box's three edges as
    (axis, direction +-1, length); the walk ends at entry + (len U - 1)
    steps along U.  Hilbert's recursion generalised to any box: split the
    longest edge near its middle, either
      - along U into two boxes walked one after the other along U, or
      - as a U-turn along an edge X (V or W): the part u < h, x < m walked
        along +X, the part x >= m walked along U, and the part u >= h,
        x < m walked back along -X (with two one-cell slabs when |U| = 2),
    taking the first split point (nearest the middle) whose three or two
    parts all admit their walks (_walk_feasible).  Consecutive cells are
    always unit steps apart."""
    a, b, c = U[2], V[2], W[2]

    def at(p, edge, d):
        q = list(p)
        q[edge[0]] += edge[1] * d
        return tuple(q)

    if b == 1 and c == 1:
        out.extend(at(entry, U, i) for i in range(a))
        return
    lens = {"U": a, "V": b, "W": c}
    for name in sorted(lens, key=lambda k: (-lens[k], "UVW".index(k))):
        if name == "U":
            for a1 in _nearest_first(a // 2, 1, a - 1):
                if _walk_feasible(a1, b, c) and _walk_feasible(a - a1, b, c):
                    _gilbert_walk(entry, (U[0], U[1], a1), V, W, out)
                    _gilbert_walk(at(entry, U, a1), (U[0], U[1], a - a1), V, W, out)
                    return
            continue
        X, Y = (V, W) if name == "V" else (W, V)
        x = X[2]
        if a < 2 or x < 2:
            continue
        if a == 2 and _walk_feasible(x, 1, Y[2]):
            _gilbert_walk(entry, X, (U[0], U[1], 1), Y, out)
            _gilbert_walk(at(at(entry, U, 1), X, x - 1), (X[0], -X[1], x), (U[0], U[1], 1), Y, out)
            return
        for m in _nearest_first(x // 2, 1, x - 1):
            for h in _nearest_first(a // 2, 1, a - 1):
                if (_walk_feasible(m, h, Y[2]) and _walk_feasible(a, x - m, Y[2])
                        and _walk_feasible(m, a - h, Y[2])):
                    _gilbert_walk(entry, (X[0], X[1], m), (U[0], U[1], h), Y, out)
                    _gilbert_walk(at(entry, X, m), U, (X[0], X[1], x - m), Y, out)
                    _gilbert_walk(at(at(entry, U, a - 1), X, m - 1), (X[0], -X[1], m),
                                  (U[0], -U[1], a - h), Y, out)
                    return
    raise ValueError(f"no walk for a {a} x {b} x {c} box")


def gilbert_order(T: int, H: int, W: int, n_prefix: int = 0) -> np.ndarray:
    """perm [n_prefix + T*H*W] along a generalised Hilbert curve of the
    T x H x W grid itself (GSRS Figure 6: blocks along a Gilbert curve, a
    Hilbert curve generalised to boxes of any size; the pages give no
    construction, so this is the plain recursive one of _gilbert_walk).
    Unlike hilbert_order, consecutive tokens are always grid neighbours.
    The walk starts at cell (0, 0, 0) and travels along the longest axis
    that admits a corner-to-corner walk (ties: t before y before x); the
    text prefix keeps its leading positions."""
    dims = (T, H, W)
    for axis in sorted(range(3), key=lambda i: (-dims[i], i)):
        rest = [j for j in range(3) if j != axis]
        if _walk_feasible(dims[axis], dims[rest[0]], dims[rest[1]]):
            break
    cells: list = []
    _gilbert_walk((0, 0, 0), (axis, 1, dims[axis]), (rest[0], 1, dims[rest[0]]),
                  (rest[1], 1, dims[rest[1]]), cells)
    grid = [n_prefix + (t * H + y) * W + x for t, y, x in cells]
    return np.array(list(range(n_prefix)) + grid, dtype=np.int64)


def dense_attention(q, k, v, scale: float):
    """Textbook softmax(scale * Q K^T) V over all N keys, fp64; also lse."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    z = scale * (q @ k.T)
    w = np.exp(z)                       # no max shift: plain definition
    den = w.sum(axis=1, keepdims=True)
    return (w @ v) / den, np.log(den[:, 0])


# ---------------------------------------------------------------------------
# Pipeline helpers and diagnostics
# ---------------------------------------------------------------------------

def pipeline_head(q, k, v, Bs: int, scale: float, p: float,
                  cand_row_ptr=None, cand_col=None):
    """Steps 1-5 for one head with the oracle's own P (rounded to fp32)."""
    qbar, kbar = pool_blocks(q, Bs), pool_blocks(k, Bs)
    cand = None if cand_row_ptr is None else csr_rows(cand_row_ptr, cand_col)
    P = block_probs(qbar, kbar, scale, cand)
    row_ptr, col = topp_select(P.astype(np.float32), p, cand_row_ptr, cand_col)
    O, lse, blk = sparse_attention_head(q, k, v, Bs, scale, row_ptr, col)
    M = block_mass(lse, blk, row_ptr, len(q), Bs)
    return dict(P=P, row_ptr=row_ptr, col=col, O=O, lse=lse, blk_lse=blk, mass=M)


def executed_flops(row_ptr, col, N: int, Bs: int, D: int) -> int:
    """4 * sum over selected (i, j) of |B_i| * |B_j| * D (QK^T and PV)."""
    sizes = [b - a for a, b in block_bounds(N, Bs)]
    nB = len(sizes)
    tot = 0
    rows = len(row_ptr) - 1
    for r in range(rows):
        i = r % nB
        for j in col[int(row_ptr[r]):int(row_ptr[r + 1])]:
            tot += sizes[i] * sizes[int(j)]
    return 4 * D * tot


def recall(q, k, Bs: int, scale: float, row_ptr, col) -> np.ndarray:
    """Per query block: mean over its queries of the dense softmax weight
    falling inside the selected key blocks (GSRS Figure 2's recall)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    bounds = block_bounds(len(q), Bs)
    out = np.zeros(len(bounds))
    for i, (a, b) in enumerate(bounds):
        z = scale * (q[a:b] @ k.T)
        w = np.exp(z - z.max(axis=1, keepdims=True))
        w /= w.sum(axis=1, keepdims=True)
        keys = [np.arange(*bounds[int(j)]) for j in col[int(row_ptr[i]):int(row_ptr[i + 1])]]
        if keys:
            out[i] = w[:, np.concatenate(keys)].sum(axis=1).mean()
    return out
