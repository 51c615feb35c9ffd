"""Pins for the oracle's estimate step (block-pooled map, true last-block
distribution, vertical and slash line scores).

FlexPrefill (atlas.scime.ai summary, "Approach"): the estimate is built from
block-pooled attention of the last query block and compared with the true
distribution.  The closed form below fixes pooling, causal masking, the row
average and the index direction of every output.
"""
import math

import numpy as np
import torch

import oracle


def test_block_pool_is_torch_avg_pool():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(2, 3, 96, 5, generator=g, dtype=torch.float64)
    got = oracle.block_pool(x, 16)
    ref = torch.nn.functional.avg_pool1d(x.reshape(6, 96, 5).transpose(1, 2), 16, 16)
    ref = ref.transpose(1, 2).reshape(2, 3, 6, 5).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-14)


def test_block_map_matches_masked_torch_softmax():
    g = torch.Generator().manual_seed(1)
    qb = torch.randn(7, 4, generator=g, dtype=torch.float64)
    kb = torch.randn(7, 4, generator=g, dtype=torch.float64)
    got = oracle.estimated_block_map(qb.numpy(), kb.numpy(), 0.5)
    logits = 0.5 * qb @ kb.T
    mask = torch.ones(7, 7, dtype=torch.bool).tril()
    ref = torch.softmax(logits.masked_fill(~mask, -math.inf), dim=-1).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-15)


def _closed_form_inputs(nb=5, b=8, d=6, seed=3):
    """Last-block queries all equal q; every key of block j equals k_j."""
    rng = np.random.default_rng(seed)
    n = nb * b
    qv = rng.standard_normal(d)
    kvs = rng.standard_normal((nb, d))
    q = rng.standard_normal((1, 1, n, d))
    q[0, 0, n - b:] = qv
    k = np.repeat(kvs, b, axis=0)[None, None]
    return q, k, qv, kvs, n, b, nb, d


def test_estimate_closed_form():
    q, k, qv, kvs, n, b, nb, d = _closed_form_inputs()
    est = oracle.estimate(q, k, b)
    s = 1.0 / math.sqrt(d)
    x = s * (kvs @ qv)  # logit of every key of block j against the shared query
    # a-hat: pooled last query = q, pooled key block j = k_j
    ahat = np.exp(x - x.max())
    ahat /= ahat.sum()
    np.testing.assert_allclose(est["est_last"][0, 0], ahat, rtol=1e-13, atol=0)
    # a-bar: row r (position n-b+r) sees B keys of blocks j < nb-1 and r+1 keys
    # of the diagonal block, each with weight e^{x_j}
    ex = np.exp(x)
    abar = np.zeros(nb)
    vert = np.zeros(n)
    slash = np.zeros(n)
    for r in range(b):
        c = np.full(nb, float(b))
        c[nb - 1] = r + 1
        z = (c * ex).sum()
        abar += c * ex / z / b
        pos = n - b + r
        for t in range(pos + 1):
            pt = ex[t // b] / z
            vert[t] += pt
            slash[pos - t] += pt
    np.testing.assert_allclose(est["true_last"][0, 0], abar, rtol=1e-13, atol=0)
    np.testing.assert_allclose(est["vert"][0, 0], vert, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(est["slash"][0, 0], slash, rtol=1e-12, atol=1e-15)


def test_mass_invariants_random():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 4, 128, 16))
    k = rng.standard_normal((1, 2, 128, 16))
    est = oracle.estimate(q, k, 16)
    np.testing.assert_allclose(est["true_last"].sum(-1), 1.0, atol=1e-13)
    np.testing.assert_allclose(est["vert"].sum(-1), 16.0, atol=1e-12)
    np.testing.assert_allclose(est["slash"].sum(-1), 16.0, atol=1e-12)
    nb = 8
    for i in range(nb):
        row = est["map"][..., oracle.tri_offset(i): oracle.tri_offset(i) + i + 1]
        np.testing.assert_allclose(row.sum(-1), 1.0, atol=1e-13)
    np.testing.assert_array_equal(est["est_last"],
                                  est["map"][..., oracle.tri_offset(nb - 1):])
    # vertical mass of the keys after the last query block's first row is causal
    assert (est["vert"] >= 0).all() and (est["slash"] >= 0).all()


def test_one_hot_offset_fixes_slash_and_vert_direction():
    """Each last-block query attends (to e^-40) to the key 5 positions before it."""
    n, b, d, off = 64, 16, 64, 5
    k = np.eye(n, d)[None, None]
    q = np.zeros((1, 1, n, d))
    for r in range(b):
        pos = n - b + r
        q[0, 0, pos, pos - off] = 40.0 * math.sqrt(d)
    est = oracle.estimate(q, k, b)
    slash = est["slash"][0, 0]
    vert = est["vert"][0, 0]
    assert abs(slash[off] - b) < 1e-12
    assert np.abs(np.delete(slash, off)).max() < 1e-12
    want = np.zeros(n)
    want[n - b - off: n - off] = 1.0
    np.testing.assert_allclose(vert, want, atol=1e-12)
    # true pooled distribution: mass of those 16 keys per key block, / B
    tb = want.reshape(n // b, b).sum(1) / b
    np.testing.assert_allclose(est["true_last"][0, 0], tb, atol=1e-12)


def test_gqa_heads_share_kv():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 4, 64, 8))
    k = rng.standard_normal((1, 2, 64, 8))
    est = oracle.estimate(q, k, 16)
    one = oracle.estimate(q[:, 2:3], k[:, 1:2], 16)
    for key in ("map", "est_last", "true_last", "vert", "slash"):
        np.testing.assert_array_equal(est[key][:, 2], one[key][:, 0])
