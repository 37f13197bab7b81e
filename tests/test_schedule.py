"""Step policy of a denoising run (host logic, no GPU)."""
import pytest

from dynamic_block_sparse_pool_b200.schedule import REUSE, SEARCH, WARMUP, GsrsPolicy


def test_even_spread_after_warmup():
    pol = GsrsPolicy(10, 2, (0.95, 0.9, 0.85, 0.8))
    assert pol.searches() == [2, 4, 6, 8]
    kinds = pol.kinds()
    assert [k for k, _ in kinds] == [WARMUP, WARMUP, SEARCH, REUSE, SEARCH, REUSE, SEARCH,
                                     REUSE, SEARCH, REUSE]
    assert [i for k, i in kinds if k == SEARCH] == [0, 1, 2, 3]


def test_uneven_spread_and_explicit_steps():
    assert GsrsPolicy(7, 1, (0.9, 0.8)).searches() == [1, 4]
    assert GsrsPolicy(5, 0, (0.9,)).kinds()[0] == (SEARCH, 0)
    pol = GsrsPolicy(6, 1, (0.95, 0.7), search_steps=(1, 5))
    assert [k for k, _ in pol.kinds()] == [WARMUP, SEARCH, REUSE, REUSE, REUSE, SEARCH]


def test_all_warmup():
    assert [k for k, _ in GsrsPolicy(3, 3, ()).kinds()] == [WARMUP] * 3


@pytest.mark.parametrize("args", [
    dict(n_steps=0, warmup=0, p=()),
    dict(n_steps=4, warmup=5, p=()),
    dict(n_steps=4, warmup=1, p=()),                                # steps after warm-up, no search
    dict(n_steps=4, warmup=1, p=(0.9, 0.8, 0.7, 0.6)),              # more searches than steps
    dict(n_steps=4, warmup=1, p=(1.5,)),
    dict(n_steps=6, warmup=2, p=(0.9, 0.8), search_steps=(1, 3)),   # search inside warm-up
    dict(n_steps=6, warmup=1, p=(0.9, 0.8), search_steps=(3, 3)),   # not increasing
    dict(n_steps=6, warmup=1, p=(0.9,), search_steps=(1, 3)),       # count mismatch
])
def test_rejects(args):
    with pytest.raises(ValueError):
        GsrsPolicy(**args)
