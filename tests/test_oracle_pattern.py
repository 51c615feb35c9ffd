"""Pins for the oracle's pattern step: square-root Jensen-Shannon divergence
against scipy and closed forms, and the tau switch.

FlexPrefill (atlas.scime.ai summary, "Approach"): square-root JS divergence
between the estimated and true distributions picks query-aware vs
vertical-slash; ("Measured effects" table) tau = 0 disables query-aware mode.
"""
import math

import numpy as np
import pytest
from scipy.spatial.distance import jensenshannon

import oracle


@pytest.mark.parametrize("seed", range(6))
def test_js_matches_scipy(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 300))
    p = rng.random(n) ** 3
    q = rng.random(n) ** 3
    p[rng.random(n) < 0.2] = 0.0  # zero entries exercise 0 log 0
    q[rng.random(n) < 0.2] = 0.0
    p[0] = q[0] = 0.5
    assert abs(oracle.js_distance(p, q) - jensenshannon(p, q)) < 1e-12


def test_js_closed_forms():
    p = np.array([0.2, 0.3, 0.5])
    assert oracle.js_distance(p, p) == 0.0
    assert oracle.js_distance(p, 7.0 * p) < 1e-8  # renormalised first
    q = np.array([0.6, 0.1, 0.3])
    assert oracle.js_distance(p, q) == oracle.js_distance(q, p)
    # disjoint supports: JSD = ln 2 exactly
    a = np.array([0.0, 0.4, 0.0, 0.6])
    b = np.array([0.7, 0.0, 0.3, 0.0])
    assert abs(oracle.js_distance(a, b) - math.sqrt(math.log(2.0))) < 1e-15
    # point mass vs uniform on 2: JSD = 1.5 ln 2 - 0.75 ln 3 (hand-derived)
    want = math.sqrt(1.5 * math.log(2.0) - 0.75 * math.log(3.0))
    assert abs(oracle.js_distance([1.0, 0.0], [0.5, 0.5]) - want) < 1e-15


def test_tau_zero_is_all_vertical_slash_and_large_tau_all_query_aware():
    rng = np.random.default_rng(9)
    e = rng.random((2, 5, 16))
    t = rng.random((2, 5, 16))
    t[0, 0] = e[0, 0]  # one head with d_JS == 0 exactly
    djs, pat = oracle.pattern(e, t, 0.0)
    assert djs[0, 0] == 0.0
    assert (pat == oracle.PATTERN_VS).all()
    _, pat = oracle.pattern(e, t, 0.84)  # > sqrt(ln 2) = 0.8326
    assert (pat == oracle.PATTERN_QA).all()
    djs, pat = oracle.pattern(e, t, 0.1)
    assert ((djs < np.float32(0.1)) == (pat == oracle.PATTERN_QA)).all()
    assert (djs >= 0).all() and (djs <= math.sqrt(math.log(2)) + 1e-15).all()
