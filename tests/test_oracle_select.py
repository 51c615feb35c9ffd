"""Pins for the oracle's cumulative-attention index selection.

FlexPrefill (atlas.scime.ai summary, "Approach"): select the smallest set of
blocks/lines whose cumulative normalised attention passes gamma; ("Measured
effects" table) min / max budgets, flattened estimated map.  Pinned by brute
force on tiny inputs: minimality, the order, nesting in gamma, budgets and the
line-to-block cover.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _scores(rng, n, ties=True):
    s = rng.random(n).astype(np.float32)
    if ties:
        s[rng.integers(0, n, n // 3)] = s[0]
    s /= s.sum(dtype=np.float64)
    return s.astype(np.float32)


def test_quantised_masses_exact():
    s = np.array([1.0, 0.5, 2.0 ** -40, 1e-30, 0.3, 0.0], np.float32)
    w = oracle.quantised_masses(s)
    for x, wi in zip(s.tolist(), w):
        f = Fraction(x) * 2 ** 32
        assert wi == math.ceil(f)
    assert w[2] == 1 and w[3] == 1 and w[5] == 0


@pytest.mark.parametrize("seed", range(40))
def test_minimal_set_by_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 11))
    s = _scores(rng, n)
    gamma = float(rng.choice([0.3, 0.5, 0.85, 0.9, 0.95, 0.99]))
    w = [math.ceil(Fraction(float(x)) * 2 ** 32) for x in s]
    total = sum(w)
    target = float(np.float32(gamma)) * float(total)
    k = oracle.cumulative_count(s, gamma)
    # no subset of size k-1 reaches the target; some subset of size k does
    best_small = max((sum(w[i] for i in c) for c in itertools.combinations(range(n), k - 1)),
                     default=0) if k >= 1 else -1
    assert k == 0 or float(best_small) < target
    chosen = oracle.cumulative_select(s, gamma, 0, n)
    assert len(chosen) == k
    assert float(sum(w[i] for i in chosen)) >= target
    # the chosen set is the prefix of (score desc, index asc)
    order = sorted(range(n), key=lambda i: (-float(s[i]), i))
    assert list(chosen) == order[:k]


@pytest.mark.parametrize("seed", range(10))
def test_nesting_in_gamma_and_budgets(seed):
    rng = np.random.default_rng(100 + seed)
    n = 200
    s = _scores(rng, n)
    prev = set()
    for gamma in (0.5, 0.8, 0.9, 0.95, 0.99, 1.0):
        cur = set(oracle.cumulative_select(s, gamma, 0, n).tolist())
        assert prev <= cur
        prev = cur
    assert len(prev) == n  # gamma = 1 selects everything
    k = oracle.cumulative_count(s, 0.9)
    for lo, hi in [(0, n), (k + 5, n), (0, max(k - 5, 0)), (50, 50), (0, 0)]:
        got = len(oracle.cumulative_select(s, 0.9, lo, hi))
        assert lo <= got <= hi
        assert got == min(max(k, lo), hi)
    # counts are monotone in min and max budget
    counts = [len(oracle.cumulative_select(s, 0.9, lo, n)) for lo in range(0, n, 17)]
    assert counts == sorted(counts)
    counts = [len(oracle.cumulative_select(s, 0.9, 0, hi)) for hi in range(0, n, 17)]
    assert counts == sorted(counts)


def test_budget_units():
    # 8 blocks of 64: T = 36 pairs; 256 tokens -> 4 blocks per row -> 32 pairs
    assert oracle.qa_budget(8, 64, 256, 0) == (32, 36)
    assert oracle.qa_budget(8, 64, 1000, 0) == (36, 36)
    assert oracle.qa_budget(8, 64, 0, 128) == (0, 16)
    assert oracle.qa_budget(8, 64, 256, 128) == (16, 16)
    assert oracle.vs_budget(512, 1024, 0) == (512, 512)
    assert oracle.vs_budget(4096, 1024, 2048) == (1024, 2048)


def test_slash_cover_by_point_enumeration():
    n, b = 96, 16
    for o in range(n):
        dists = set()
        for i in range(n):
            t = i - o
            if 0 <= t <= i:
                dists.add(i // b - t // b)
        # a distance >= nb names no block pair, so it cannot show up here
        assert dists == {x for x in oracle.slash_block_distances(o, b) if x < n // b}, o


def _blocks_of_points(points, b):
    return {(i // b, t // b) for i, t in points}


@pytest.mark.parametrize("seed", range(6))
def test_vs_rows_by_point_enumeration(seed):
    rng = np.random.default_rng(200 + seed)
    n, b = 128, 16
    nb = n // b
    vert = _scores(rng, n)
    slash = _scores(rng, n)
    gamma, lo_tok, hi_tok = 0.6, 8, 0
    rows = oracle.select_head_vs(vert, slash, nb, b, gamma, lo_tok, hi_tok)
    lo, hi = oracle.vs_budget(n, lo_tok, hi_tok)
    cols = oracle.cumulative_select(vert, gamma, lo, hi).tolist()
    offs = oracle.cumulative_select(slash, gamma, lo, hi).tolist()
    pts = [(i, t) for t in cols for i in range(t, n)]
    pts += [(i, i - o) for o in offs for i in range(o, n)]
    pairs = _blocks_of_points(pts, b) | {(i, i) for i in range(nb)}
    for qi in range(nb):
        assert rows[qi] == sorted(j for (a, j) in pairs if a == qi)


@pytest.mark.parametrize("seed", range(4))
def test_qa_rows_decode_packed_index(seed):
    rng = np.random.default_rng(300 + seed)
    nb, b = 9, 32
    t_pairs = nb * (nb + 1) // 2
    m = _scores(rng, t_pairs)
    rows = oracle.select_head_qa(m, nb, b, 0.7, 64, 0)
    lo, hi = oracle.qa_budget(nb, b, 64, 0)
    chosen = set(oracle.cumulative_select(m, 0.7, lo, hi).tolist())
    flat = [(i, j) for i in range(nb) for j in range(i + 1)]  # packed order
    for qi in range(nb):
        want = sorted({j for p, (i, j) in enumerate(flat) if i == qi and p in chosen} | {qi})
        assert rows[qi] == want


def test_select_dispatch_and_tail():
    rng = np.random.default_rng(7)
    nb, b = 4, 8
    n = nb * b
    amap = np.stack([_scores(rng, nb * (nb + 1) // 2) for _ in range(2)])[None]
    vert = np.stack([_scores(rng, n) for _ in range(2)])[None]
    slash = np.stack([_scores(rng, n) for _ in range(2)])[None]
    pat = np.array([[oracle.PATTERN_QA, oracle.PATTERN_VS]], np.int32)
    counts, indices = oracle.select(pat, amap, vert, slash, nb, b, 0.9, 0, 0)
    qa = oracle.select_head_qa(amap[0, 0], nb, b, 0.9, 0, 0)
    vs = oracle.select_head_vs(vert[0, 1], slash[0, 1], nb, b, 0.9, 0, 0)
    for qi in range(nb):
        assert list(indices[0, 0, qi, : counts[0, 0, qi]]) == qa[qi]
        assert list(indices[0, 1, qi, : counts[0, 1, qi]]) == vs[qi]
        assert (indices[0, :, qi, counts[0, :, qi].max():] == -1).all()
