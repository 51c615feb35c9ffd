"""Pins for the oracle on sequences whose length N is not a multiple of the
block size B (the last block is partial).

FlexPrefill (atlas.scime.ai summary, "Approach") defines the method per
sequence; nothing on the pages ties N to B.  Reading taken here: nb =
ceil(N / B) blocks, the last one holding the N - (nb - 1) B tokens left; its
pooled vector is the mean of its real tokens, its R real queries are the last
query block of the estimate, and attention runs over real keys only.  The
pins below fix each of these against a library routine, brute force or a
closed form.
"""
import math

import numpy as np
import pytest
import torch

import oracle


@pytest.mark.parametrize("n,b", [(70, 16), (97, 32), (65, 64), (1, 16)])
def test_block_pool_partial_block_is_torch_ceil_pool(n, b):
    """avg_pool1d with ceil_mode divides the partial window by its real length."""
    g = torch.Generator().manual_seed(n)
    x = torch.randn(2, 3, n, 5, generator=g, dtype=torch.float64)
    got = oracle.block_pool(x, b)
    nb = -(-n // b)
    ref = torch.nn.functional.avg_pool1d(x.reshape(6, n, 5).transpose(1, 2), b, b,
                                         ceil_mode=True)
    ref = ref.transpose(1, 2).reshape(2, 3, nb, 5).numpy()
    assert got.shape == (2, 3, nb, 5)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-14)


@pytest.mark.parametrize("n,b", [(70, 16), (100, 32), (33, 32)])
def test_dense_ragged_matches_torch_sdpa_causal(n, b):
    """Dense attention over ceil(N/B) blocks is plain causal attention over N."""
    g = torch.Generator().manual_seed(7)
    q = torch.randn(1, 4, n, 8, generator=g, dtype=torch.float64)
    k = torch.randn(1, 2, n, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 2, n, 8, generator=g, dtype=torch.float64)
    out, lse = oracle.dense_attention(q, k, v, b)
    kk, vv = k.repeat_interleave(2, dim=1), v.repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    logits = (q @ kk.transpose(-1, -2)) / math.sqrt(8)
    mask = torch.ones(n, n, dtype=torch.bool).tril()
    ref_lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_sparse_ragged_matches_sdpa_with_token_mask():
    """Sparse lists on a ragged sequence: SDPA with the token mask the lists
    imply (key block listed for the query's block, key <= query)."""
    n, b = 75, 16
    nb = -(-n // b)
    rng = np.random.default_rng(3)
    counts = np.zeros((1, 2, nb), dtype=np.int32)
    indices = np.full((1, 2, nb, nb), -1, dtype=np.int32)
    for h in range(2):
        for i in range(nb):
            row = sorted(set(rng.choice(i + 1, size=rng.integers(1, i + 2), replace=False)) | {i})
            counts[0, h, i] = len(row)
            indices[0, h, i, :len(row)] = row
    g = torch.Generator().manual_seed(2)
    q = torch.randn(1, 2, n, 8, generator=g, dtype=torch.float64)
    k = torch.randn(1, 2, n, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 2, n, 8, generator=g, dtype=torch.float64)
    out, _ = oracle.sparse_attention(q, k, v, counts, indices, b)
    mask = torch.zeros(1, 2, n, n, dtype=torch.bool)
    for h in range(2):
        for i in range(nb):
            for j in indices[0, h, i, :counts[0, h, i]]:
                mask[0, h, i * b:min((i + 1) * b, n), j * b:min((j + 1) * b, n)] = True
    mask &= torch.ones(n, n, dtype=torch.bool).tril()
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_ragged_attention_equals_padded_rows():
    """Padding a ragged sequence to whole blocks with arbitrary tokens leaves
    every real row's attention unchanged (the padded keys lie after every real
    query, so the causal mask hides them)."""
    n, b = 70, 16
    nb = -(-n // b)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 2, nb * b, 8, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, nb * b, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 1, nb * b, 8, generator=g, dtype=torch.float64)
    counts, indices = oracle.dense_lists(1, 2, nb)
    indices[0, 1, 3, :2] = [0, 3]  # a sparse row too
    counts[0, 1, 3] = 2
    o_r, l_r = oracle.sparse_attention(q[:, :, :n], k[:, :, :n], v[:, :, :n], counts, indices, b)
    o_p, l_p = oracle.sparse_attention(q, k, v, counts, indices, b)
    np.testing.assert_allclose(o_r, o_p[:, :, :n], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_r, l_p[:, :, :n], rtol=0, atol=1e-13)


def test_estimate_ragged_brute_force():
    """The true last-block distribution, vert and slash of a partial last
    block, against softmax rows written out one query at a time."""
    n, b, d = 45, 16, 4  # nb = 3, the last block holds R = 13 queries
    rng = np.random.default_rng(11)
    q = rng.standard_normal((1, 1, n, d))
    k = rng.standard_normal((1, 1, n, d))
    est = oracle.estimate(q, k, b)
    nb, q0 = 3, 32
    rows = n - q0
    s = 1.0 / math.sqrt(d)
    abar = [0.0] * nb
    vert = [0.0] * n
    slash = [0.0] * n
    for r in range(rows):
        pos = q0 + r
        w = [math.exp(s * sum(q[0, 0, pos, e] * k[0, 0, t, e] for e in range(d)))
             for t in range(pos + 1)]
        z = math.fsum(w)
        for t in range(pos + 1):
            p = w[t] / z
            abar[t // b] += p / rows
            vert[t] += p
            slash[pos - t] += p
    np.testing.assert_allclose(est["true_last"][0, 0], abar, rtol=1e-12, atol=0)
    np.testing.assert_allclose(est["vert"][0, 0], vert, rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(est["slash"][0, 0], slash, rtol=1e-12, atol=1e-16)
    # the pooled estimate: the partial block's mean over its 13 real tokens
    qbar = q[0, 0, q0:].mean(axis=0)
    kbar = np.stack([k[0, 0, j * b:min((j + 1) * b, n)].mean(axis=0) for j in range(nb)])
    x = s * kbar @ qbar
    ahat = np.exp(x - x.max())
    np.testing.assert_allclose(est["est_last"][0, 0], ahat / ahat.sum(), rtol=1e-13, atol=0)
    assert est["map"].shape == (1, 1, nb * (nb + 1) // 2)


def test_estimate_ragged_closed_form():
    """Last-block queries all equal q and keys constant per block, with a
    partial last block of R keys and R queries: row r sees B keys of every
    earlier block and r + 1 of the last."""
    nb, b, d, rows = 4, 8, 6, 5
    n = (nb - 1) * b + rows
    rng = np.random.default_rng(9)
    qv = rng.standard_normal(d)
    kvs = rng.standard_normal((nb, d))
    q = rng.standard_normal((1, 1, n, d))
    q[0, 0, (nb - 1) * b:] = qv
    k = np.repeat(kvs, b, axis=0)[None, None, :n]
    est = oracle.estimate(q, k, b)
    ex = np.exp(kvs @ qv / math.sqrt(d))
    abar = np.zeros(nb)
    for r in range(rows):
        c = np.full(nb, float(b))
        c[nb - 1] = r + 1
        abar += c * ex / (c * ex).sum() / rows
    np.testing.assert_allclose(est["true_last"][0, 0], abar, rtol=1e-13, atol=0)


@pytest.mark.parametrize("n,b", [(70, 16), (129, 64), (200, 64)])
def test_estimate_ragged_mass_invariants(n, b):
    rng = np.random.default_rng(n)
    q = rng.standard_normal((1, 2, n, 8))
    k = rng.standard_normal((1, 1, n, 8))
    est = oracle.estimate(q, k, b)
    nb = -(-n // b)
    rows = n - (nb - 1) * b
    np.testing.assert_allclose(est["true_last"].sum(axis=-1), 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(est["vert"].sum(axis=-1), rows, rtol=1e-12, atol=0)
    np.testing.assert_allclose(est["slash"].sum(axis=-1), rows, rtol=1e-12, atol=0)
    np.testing.assert_allclose(est["est_last"].sum(axis=-1), 1.0, rtol=0, atol=1e-12)


def test_ragged_pipeline_gamma_one_is_dense():
    """gamma = 1 keeps every causal block on a ragged sequence, so the whole
    path is dense causal attention over the N real tokens."""
    n, b = 90, 16
    g = torch.Generator().manual_seed(4)
    q = torch.randn(1, 2, n, 8, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, n, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 1, n, 8, generator=g, dtype=torch.float64)
    res = oracle.flexprefill(q, k, v, b, 1.0, 0.1, 0, 0)
    nb = -(-n // b)
    assert (res["counts"] == np.arange(1, nb + 1)).all()
    kk, vv = k.repeat_interleave(2, dim=1), v.repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True).numpy()
    np.testing.assert_allclose(res["out"], ref, rtol=0, atol=1e-12)


def test_single_token_sequence_closed_form():
    """N = 1: one partial block, one key.  Whatever the pattern, each head keeps
    that block; the output is V's only row and the log-sum-exp is the single
    scaled logit q.k / sqrt(d)."""
    g = torch.Generator().manual_seed(11)
    q = torch.randn(1, 4, 1, 8, generator=g, dtype=torch.float64)
    k = torch.randn(1, 2, 1, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 2, 1, 8, generator=g, dtype=torch.float64)
    for gamma in (0.5, 0.95):
        res = oracle.flexprefill(q, k, v, 16, gamma, 0.1, 0, 0)
        assert (res["counts"] == 1).all()
        assert (res["indices"][..., 0] == 0).all()
        kk, vv = k.repeat_interleave(2, dim=1), v.repeat_interleave(2, dim=1)
        np.testing.assert_allclose(res["out"], vv.numpy(), rtol=0, atol=0)
        ref_lse = ((q * kk).sum(-1) / math.sqrt(8)).numpy()
        np.testing.assert_allclose(res["lse"], ref_lse, rtol=0, atol=1e-14)


@pytest.mark.parametrize("n", [1, 2, 3, 4])
def test_synthetic_inputs_for_sequences_shorter_than_the_sinks(n):
    """The generator plants up to four sink keys; a shorter sequence plants
    the ones it has and still yields finite inputs of the asked shape."""
    from dynamic_block_sparse_fp_b200 import synth
    w = synth.WORKLOADS["tiny_n1024"].replace(seq_len=n)
    inp = synth.make_inputs(w)
    assert inp["q"].shape[2] == n and inp["k"].shape[2] == n
    assert all(torch.isfinite(inp[x]).all() for x in ("q", "k", "v"))
