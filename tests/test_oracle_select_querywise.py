"""Pins for the oracle's query-wise index selection.

FlexPrefill (atlas.scime.ai summary, "Measured effects" table): "query-wise
index selection instead of flattening the estimated attention map" is the
alternative the ablation compares with the flattened rule; "Approach" gives the
rule itself (smallest set of blocks whose cumulative normalised attention
passes gamma).  Reading: the rule runs on each query-block row of the map with
the row's own total and per-row token budgets.  Pinned by brute force over the
subsets of every row, and by the cases where the query-wise rule must reduce to
something else (one row = the flattened rule, gamma = 1 = every block).
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _row_normalised_map(rng, nb, ties=True):
    rows = []
    for i in range(nb):
        s = rng.random(i + 1)
        if ties and i >= 2:
            s[rng.integers(0, i + 1, (i + 1) // 2)] = s[0]
        rows.append(s / s.sum())
    return np.concatenate(rows).astype(np.float32)


def _brute_force_row(seg, gamma, min_blocks, max_blocks):
    """Expected kept set of one row, from scratch: exact masses, the smallest
    subset size reaching the target, clamped, then the (score desc, index asc)
    prefix."""
    n = len(seg)
    w = [math.ceil(Fraction(float(x)) * 2 ** 32) for x in seg]
    target = float(np.float32(gamma)) * float(sum(w))
    if float(np.float32(gamma)) >= 1.0:
        k = n
    else:
        k = next(size for size in range(n + 1)
                 if any(float(sum(w[i] for i in c)) >= target
                        for c in itertools.combinations(range(n), size)))
    k = max(k, min_blocks)
    k = min(k, max_blocks)
    order = sorted(range(n), key=lambda j: (-float(seg[j]), j))
    return set(order[:k])


@pytest.mark.parametrize("seed", range(24))
def test_querywise_rows_by_brute_force(seed):
    rng = np.random.default_rng(500 + seed)
    nb, b = int(rng.integers(1, 7)), 32
    m = _row_normalised_map(rng, nb)
    gamma = float(rng.choice([0.3, 0.6, 0.9, 0.95]))
    # budgets in tokens: 64 tokens = 2 blocks at B = 32; 96 tokens = 3 blocks
    min_budget = int(rng.choice([0, 32, 64]))
    max_budget = int(rng.choice([0, 64, 96]))
    rows = oracle.select_head_qa_querywise(m, nb, b, gamma, min_budget, max_budget)
    for i in range(nb):
        seg = m[i * (i + 1) // 2: i * (i + 1) // 2 + i + 1]
        min_blocks = {0: 0, 32: 1, 64: 2}[min_budget]
        max_blocks = {0: i + 1, 64: 2, 96: 3}[max_budget]
        want = _brute_force_row(seg, gamma, min(min_blocks, i + 1, max_blocks),
                                min(max_blocks, i + 1)) | {i}
        assert rows[i] == sorted(want), (i, rows[i], sorted(want))


@pytest.mark.parametrize("seed", range(6))
def test_one_row_is_the_flattened_rule(seed):
    rng = np.random.default_rng(600 + seed)
    m = _row_normalised_map(rng, 1)
    for gamma in (0.5, 0.95, 1.0):
        assert (oracle.select_head_qa_querywise(m, 1, 64, gamma, 0, 0)
                == oracle.select_head_qa(m, 1, 64, gamma, 0, 0))


def test_gamma_one_keeps_every_causal_block():
    rng = np.random.default_rng(7)
    nb = 9
    m = _row_normalised_map(rng, nb)
    rows = oracle.select_head_qa_querywise(m, nb, 64, 1.0, 0, 0)
    assert rows == [list(range(i + 1)) for i in range(nb)]


@pytest.mark.parametrize("seed", range(4))
def test_rows_are_independent(seed):
    rng = np.random.default_rng(700 + seed)
    nb = 8
    m = _row_normalised_map(rng, nb)
    base = oracle.select_head_qa_querywise(m, nb, 64, 0.8, 0, 0)
    i = int(rng.integers(1, nb))
    m2 = m.copy()
    seg = slice(i * (i + 1) // 2, i * (i + 1) // 2 + i + 1)
    m2[seg] = rng.permutation(m2[seg])
    other = oracle.select_head_qa_querywise(m2, nb, 64, 0.8, 0, 0)
    assert [r for k, r in enumerate(base) if k != i] == [r for k, r in enumerate(other) if k != i]


def test_budget_bounds_per_row():
    rng = np.random.default_rng(11)
    nb, b = 12, 16
    m = _row_normalised_map(rng, nb)
    low = oracle.select_head_qa_querywise(m, nb, b, 0.2, 0, 0)
    floor = oracle.select_head_qa_querywise(m, nb, b, 0.2, 4 * b, 0)      # >= 4 blocks
    cap = oracle.select_head_qa_querywise(m, nb, b, 0.99, 0, 2 * b)       # <= 2 blocks
    for i in range(nb):
        assert len(floor[i]) >= min(i + 1, 4) and set(low[i]) <= set(floor[i])
        assert len(cap[i]) <= 3  # 2 chosen plus the forced diagonal


def test_select_dispatch_querywise():
    rng = np.random.default_rng(13)
    nb, b = 5, 8
    n = nb * b
    amap = np.stack([_row_normalised_map(rng, nb) for _ in range(2)])[None]
    vert = np.stack([rng.random(n).astype(np.float32) for _ in range(2)])[None]
    slash = np.stack([rng.random(n).astype(np.float32) for _ in range(2)])[None]
    pat = np.array([[oracle.PATTERN_QA, oracle.PATTERN_VS]], np.int32)
    counts, indices = oracle.select(pat, amap, vert, slash, nb, b, 0.9, 0, 0,
                                    oracle.QA_QUERYWISE)
    qa = oracle.select_head_qa_querywise(amap[0, 0], nb, b, 0.9, 0, 0)
    vs = oracle.select_head_vs(vert[0, 1], slash[0, 1], nb, b, 0.9, 0, 0)
    for qi in range(nb):
        assert list(indices[0, 0, qi, : counts[0, 0, qi]]) == qa[qi]
        assert list(indices[0, 1, qi, : counts[0, 1, qi]]) == vs[qi]
