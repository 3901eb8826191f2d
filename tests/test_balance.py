"""Sparsity-aware split of the query sequence into per-rank chunks (CPU only).

"FlashMask-3 targets masked distributed attention on Hopper GPUs", section
"In-depth insight", names a load balancer (HCC-IPO) that evens out the ranks'
work; read here as the contiguous split of q-tiles whose largest unmasked-pair
count is as small as possible.  The library's host function
(``flashmask_balance_chunks``) is checked against the oracle's exhaustive
search on small inputs (the optimal largest cost is unique; the split itself
is checked for validity), and on the workloads' per-tile costs.
"""
import numpy as np
import pytest

import column_sparse_masked_b200 as fm
from column_sparse_masked_b200 import workloads as wl


@pytest.fixture(scope="module", autouse=True)
def library():
    from column_sparse_masked_b200 import build

    build.build()
    fm.load_library()


def _check_split(costs, parts, bounds, best):
    n = len(costs)
    assert len(bounds) == parts + 1 and bounds[0] == 0 and bounds[-1] == n
    assert all(bounds[p] <= bounds[p + 1] for p in range(parts))
    loads = [int(sum(costs[bounds[p]:bounds[p + 1]])) for p in range(parts)]
    assert max(loads) == best
    if n >= parts:
        assert all(bounds[p] < bounds[p + 1] for p in range(parts)), "every chunk holds a tile"
    return loads


# ----------------------------------------------------------------------------
# oracle pins: per-tile unmasked pairs
# ----------------------------------------------------------------------------
def test_tile_costs_sum_to_pair_count(oracle_mod):
    rng = np.random.default_rng(21)
    nq, nk = 300, 170
    vecs = [x[None, None] for x in wl.random_interval_vectors(rng, nq, nk)]
    costs = oracle_mod.tile_costs(*vecs, nq, nk, 3, bm=64)
    assert costs.shape == (5,)
    assert int(costs.sum()) == oracle_mod.count_unmasked(*vecs, nq, nk, 3)


def test_tile_costs_causal_closed_form(oracle_mod):
    """Causal: row i sees i + 1 keys, so tile t costs the sum of (i + 1) over its rows."""
    n, bm = 1000, 128
    costs = oracle_mod.tile_costs(*[x[None, None] for x in wl.causal_vectors(n)], n, n, 2, bm=bm)
    want = [2 * sum(i + 1 for i in range(t * bm, min((t + 1) * bm, n))) for t in range(-(-n // bm))]
    assert costs.tolist() == want


def test_balance_minimax_oracle_closed_forms(oracle_mod):
    assert oracle_mod.balance_minimax([4, 4, 4, 4], 2)[0] == 8
    assert oracle_mod.balance_minimax([1, 2, 3, 4, 5], 1)[0] == 15
    assert oracle_mod.balance_minimax([7, 1, 1], 5)[0] == 7
    assert oracle_mod.balance_minimax([1, 1, 1, 10], 2)[0] == 10


# ----------------------------------------------------------------------------
# the library's split
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(40))
def test_split_is_optimal_on_small_inputs(oracle_mod, seed):
    rng = np.random.default_rng(600 + seed)
    n = int(rng.integers(0, 11))
    parts = int(rng.integers(1, 5))
    kind = seed % 4
    if kind == 0:
        costs = rng.integers(0, 50, size=n)
    elif kind == 1:
        costs = rng.integers(0, 3, size=n)  # many ties and zeros
    elif kind == 2:
        costs = np.sort(rng.integers(0, 1000, size=n))  # growing, as under a causal mask
    else:
        costs = rng.integers(0, 2, size=n) * rng.integers(1, 10 ** 6, size=n)
    costs = [int(x) for x in costs]
    bounds, best = fm.balance_chunks(costs, parts)
    want, _ = oracle_mod.balance_minimax(costs, parts)
    assert best == want
    _check_split(costs, parts, bounds, best)


def test_split_edge_cases():
    assert fm.balance_chunks([], 3) == ([0, 0, 0, 0], 0)
    assert fm.balance_chunks([9], 1) == ([0, 1], 9)
    bounds, best = fm.balance_chunks([3, 8], 4)  # fewer tiles than chunks: one tile each, the rest empty
    assert bounds == [0, 1, 2, 2, 2] and best == 8
    bounds, best = fm.balance_chunks([0, 0, 0, 0, 0], 2)
    assert best == 0 and bounds[0] == 0 and bounds[2] == 5 and 0 < bounds[1] < 5


@pytest.mark.parametrize("costs,parts", [([1, 2], 0), ([1, -2], 2), ([2 ** 61, 2 ** 61], 2)])
def test_split_rejects_bad_arguments(costs, parts):
    with pytest.raises(fm.FlashMaskError):
        fm.balance_chunks(costs, parts)


@pytest.mark.parametrize("name,parts", [("doc8k", 4), ("doc8k", 8), ("sharequestion32k", 8)])
def test_split_evens_out_workload_costs(oracle_mod, name, parts):
    """On the workloads' per-tile costs the split is within one tile of the mean (the
    greedy bound) and never worse than equal-length chunks; a rank's work, counted
    again on its clip-shift-max localised vectors, is the sum of its tiles."""
    w = wl.CONFIGS[name]
    vecs = wl.mask_vectors(w)
    costs = [int(x) for x in oracle_mod.tile_costs(*vecs, w.N, w.N, w.Hq)]
    bounds, best = fm.balance_chunks(costs, parts)
    loads = _check_split(costs, parts, bounds, best)
    n = len(costs)
    assert best <= sum(costs) / parts + max(costs)
    equal = [round(p * n / parts) for p in range(parts + 1)]
    assert best <= max(sum(costs[equal[p]:equal[p + 1]]) for p in range(parts))
    p = int(np.argmax(loads))
    a, b = bounds[p] * 128, min(bounds[p + 1] * 128, w.N)
    local = [oracle_mod.localize(x[0, 0], a, b)[None, None] for x in vecs]
    assert oracle_mod.count_unmasked(*local, b - a, w.N, w.Hq) == loads[p]
