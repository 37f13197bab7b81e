"""The library's Hilbert token order (a host function) against the oracle's,
and argument checks of the reordering calls (no GPU needed)."""
import numpy as np
import pytest

from dynamic_block_sparse_pool_b200 import _lib, ops, synth
from oracle import dsa_oracle as O


@pytest.mark.parametrize("T,H,W,P", [(1, 1, 1, 0), (2, 3, 1, 5), (4, 8, 8, 0), (3, 5, 7, 2),
                                     (13, 30, 45, 226), (21, 45, 80, 0), (33, 45, 80, 0)])
def test_host_order_matches_oracle(T, H, W, P):
    np.testing.assert_array_equal(ops.hilbert_order(T, H, W, P).numpy(), O.hilbert_order(T, H, W, P))


@pytest.mark.parametrize("T,H,W,P", [(1, 1, 1, 0), (2, 3, 1, 5), (4, 8, 8, 0), (3, 5, 7, 2),
                                     (2, 2, 2, 0), (1, 9, 1, 0), (6, 1, 7, 3),
                                     (13, 30, 45, 226), (21, 45, 80, 0), (33, 45, 80, 0)])
def test_host_gilbert_order_matches_oracle(T, H, W, P):
    np.testing.assert_array_equal(ops.gilbert_order(T, H, W, P).numpy(), O.gilbert_order(T, H, W, P))


def test_host_gilbert_order_matches_oracle_on_random_boxes():
    rng = np.random.default_rng(3)
    for _ in range(40):
        T, H, W = (int(x) for x in rng.integers(1, 24, size=3))
        np.testing.assert_array_equal(ops.gilbert_order(T, H, W, 1).numpy(),
                                      O.gilbert_order(T, H, W, 1), err_msg=str((T, H, W)))


def test_workload_grids_are_permutations():
    for w in (synth.TINY, synth.SMALL, synth.COGVIDEOX, synth.WAN21, synth.HUNYUAN):
        perm = ops.hilbert_order(w.T, w.Hg, w.W, w.n_prefix).numpy()
        assert perm.size == w.N
        assert np.array_equal(np.sort(perm), np.arange(w.N))


FAKE = 0x10000


def test_reorder_rejects():
    lib = _lib.lib()
    assert lib.dsa_hilbert_order(2, 2, 2, 0, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_hilbert_order(0, 2, 2, 0, FAKE) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_hilbert_order(2, 2, 2, -1, FAKE) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_hilbert_order(1 << 21, 1, 1, 0, FAKE) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_gilbert_order(2, 2, 2, 0, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_gilbert_order(2, 0, 2, 0, FAKE) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_gilbert_order(2, 2, 2, -3, FAKE) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_gilbert_order(1, 1 << 21, 1, 0, FAKE) == _lib.DSA_ERR_INVALID_ARG
    ok = (FAKE, FAKE + 4096, 1, 1, 2, 64, 128, FAKE, 0, None)
    assert lib.dsa_permute_tokens(None, *ok[1:]) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_permute_tokens(FAKE, FAKE, *ok[2:]) == _lib.DSA_ERR_INVALID_ARG   # in place
    assert lib.dsa_permute_tokens(*ok[:6], 96, *ok[7:]) == _lib.DSA_ERR_INVALID_ARG  # D
    assert lib.dsa_permute_tokens(*ok[:8], 2, None) == _lib.DSA_ERR_INVALID_ARG      # inverse
    assert lib.dsa_permute_tokens(FAKE + 8, *ok[1:]) == _lib.DSA_ERR_INVALID_ARG     # alignment
