"""Pins for the oracle's block-pooled vertical-slash selection.

FlexPrefill (atlas.scime.ai summary, "Approach"): vertical-slash heads keep
the smallest set of "blocks/lines" whose cumulative attention passes gamma.
Reading pinned here: the block-level variant, in which vertical scores are summed
per key block and slash scores per block distance before the rule.  Pinned
by the block-size-1 reduction (pooling is the identity and the block cover
of a slash offset is a single distance, so it must equal the token-line
rule), by fsum on the pooled sums, and by brute-force enumeration of the
block pairs that the chosen columns and distances cover.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _line(rng, n, ties=True):
    s = rng.random(n)
    if ties:
        s[rng.integers(0, n, n // 4)] = s[0]
    return (s / s.sum()).astype(np.float32)


@pytest.mark.parametrize("seed", range(6))
def test_pooled_sums_against_fsum(seed):
    rng = np.random.default_rng(800 + seed)
    nb, b = 7, 16
    x = _line(rng, nb * b)
    x[3] = 1e-30  # a tiny term next to large ones
    p = oracle.pool_lines(x, nb, b)
    for c in range(nb):
        exact = math.fsum(float(v) for v in x[c * b:(c + 1) * b])
        ulp = np.spacing(np.float32(exact))
        assert abs(float(p[c]) - exact) <= ulp
    # a constant line gives B times the constant exactly
    np.testing.assert_array_equal(oracle.pool_lines(np.full(nb * b, 0.25, np.float32), nb, b),
                                  np.full(nb, 4.0, np.float32))


@pytest.mark.parametrize("seed", range(8))
def test_block_size_one_is_the_token_rule(seed):
    rng = np.random.default_rng(900 + seed)
    n = int(rng.integers(2, 40))
    v, s = _line(rng, n), _line(rng, n)
    for gamma, lo, hi in [(0.9, 0, 0), (0.5, 3, 0), (0.95, 0, 5), (1.0, 0, 0)]:
        assert (oracle.select_head_vs_blocks(v, s, n, 1, gamma, lo, hi)
                == oracle.select_head_vs(v, s, n, 1, gamma, lo, hi))


def _minimal_prefix(scores, gamma, lo, hi):
    """From scratch: exact masses, the smallest subset size reaching the
    target (brute force), clamped, then the (score desc, index asc) prefix."""
    n = len(scores)
    w = [math.ceil(Fraction(float(x)) * 2 ** 32) for x in scores]
    target = float(np.float32(gamma)) * float(sum(w))
    k = n if float(np.float32(gamma)) >= 1.0 else next(
        size for size in range(n + 1)
        if any(float(sum(w[i] for i in c)) >= target
               for c in itertools.combinations(range(n), size)))
    k = min(max(k, lo), hi)
    return set(sorted(range(n), key=lambda j: (-float(scores[j]), j))[:k])


@pytest.mark.parametrize("seed", range(16))
def test_rows_by_brute_force(seed):
    rng = np.random.default_rng(1000 + seed)
    nb, b = int(rng.integers(1, 8)), 8
    n = nb * b
    v, s = _line(rng, n), _line(rng, n)
    gamma = float(rng.choice([0.4, 0.8, 0.95]))
    min_budget = int(rng.choice([0, 8, 12, 16]))
    max_budget = int(rng.choice([0, 20, 24]))
    rows = oracle.select_head_vs_blocks(v, s, nb, b, gamma, min_budget, max_budget)
    # budgets in blocks at B = 8: a minimum of 12 tokens needs 2 blocks, a
    # maximum of 20 tokens allows 2 whole blocks
    hi = nb if max_budget == 0 else min(nb, {20: 2, 24: 3}[max_budget])
    lo = min({0: 0, 8: 1, 12: 2, 16: 2}[min_budget], nb, hi)
    cols = _minimal_prefix(oracle.pool_lines(v, nb, b), gamma, lo, hi)
    dists = _minimal_prefix(oracle.pool_lines(s, nb, b), gamma, lo, hi)
    pairs = {(qi, j) for qi in range(nb) for j in range(qi + 1)
             if j in cols or qi - j in dists or j == qi}
    for qi in range(nb):
        assert rows[qi] == sorted(j for (a, j) in pairs if a == qi)


def test_gamma_one_keeps_every_block():
    rng = np.random.default_rng(3)
    nb, b = 6, 4
    rows = oracle.select_head_vs_blocks(_line(rng, nb * b), _line(rng, nb * b), nb, b, 1.0, 0, 0)
    assert rows == [list(range(i + 1)) for i in range(nb)]


def test_select_dispatch_vs_blocks():
    rng = np.random.default_rng(17)
    nb, b = 5, 8
    n = nb * b
    amap = np.stack([_line(rng, nb * (nb + 1) // 2) for _ in range(2)])[None]
    vert = np.stack([_line(rng, n) for _ in range(2)])[None]
    slash = np.stack([_line(rng, n) for _ in range(2)])[None]
    pat = np.array([[oracle.PATTERN_QA, oracle.PATTERN_VS]], np.int32)
    counts, indices = oracle.select(pat, amap, vert, slash, nb, b, 0.9, 0, 0,
                                    oracle.QA_FLATTENED, oracle.VS_BLOCKS)
    qa = oracle.select_head_qa(amap[0, 0], nb, b, 0.9, 0, 0)
    vs = oracle.select_head_vs_blocks(vert[0, 1], slash[0, 1], nb, b, 0.9, 0, 0)
    for qi in range(nb):
        assert list(indices[0, 0, qi, : counts[0, 0, qi]]) == qa[qi]
        assert list(indices[0, 1, qi, : counts[0, 1, qi]]) == vs[qi]
