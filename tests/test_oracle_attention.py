"""Pins for the oracle's attention: library SDPA, a textbook loop, mask equivalence.

The FlexPrefill pages build the sparse kernel on FlashAttention (atlas.scime.ai
summary, "Experimental setup"); with every causal block selected it must equal
dense causal softmax attention.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _sdpa(q, k, v, mask=None, causal=False):
    g = q.shape[1] // k.shape[1]
    kk = k.repeat_interleave(g, dim=1)
    vv = v.repeat_interleave(g, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        q, kk, vv, attn_mask=mask, is_causal=causal).numpy()


@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (4, 1)])
def test_dense_matches_torch_sdpa_causal(hq, hkv):
    n, d, b = 128, 32, 32
    q, k, v = _rand((1, hq, n, d), 1), _rand((1, hkv, n, d), 2), _rand((1, hkv, n, d), 3)
    out, lse = oracle.dense_attention(q, k, v, b)
    ref = _sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # log-sum-exp of the scaled, causally masked logits (torch.logsumexp)
    g = hq // hkv
    logits = (q @ k.repeat_interleave(g, dim=1).transpose(-1, -2)) / math.sqrt(d)
    causal = torch.ones(n, n, dtype=torch.bool).tril()
    ref_lse = torch.logsumexp(logits.masked_fill(~causal, -math.inf), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_dense_matches_textbook_loop():
    """Pure-Python loop: for each query, exp-weights over keys <= query."""
    n, d, b = 12, 3, 4
    q, k, v = _rand((1, 1, n, d), 4), _rand((1, 1, n, d), 5), _rand((1, 1, n, d), 6)
    out, _ = oracle.dense_attention(q, k, v, b)
    qq, kk, vv = q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist()
    for i in range(n):
        w = [math.exp(sum(qq[i][c] * kk[t][c] for c in range(d)) / math.sqrt(d))
             for t in range(i + 1)]
        z = sum(w)
        for c in range(d):
            expect = sum(w[t] * vv[t][c] for t in range(i + 1)) / z
            assert abs(out[0, 0, i, c] - expect) < 1e-12


def test_sparse_matches_sdpa_with_block_mask():
    n, d, b, hq, hkv = 256, 16, 32, 4, 2
    nb = n // b
    q, k, v = _rand((1, hq, n, d), 7), _rand((1, hkv, n, d), 8), _rand((1, hkv, n, d), 9)
    rng = np.random.default_rng(0)
    counts = np.zeros((1, hq, nb), np.int32)
    indices = np.full((1, hq, nb, nb), -1, np.int32)
    mask = torch.zeros(1, hq, n, n, dtype=torch.bool)
    for h in range(hq):
        for i in range(nb):
            blocks = sorted(set(rng.choice(i + 1, size=rng.integers(1, i + 2), replace=False)
                                .tolist()) | {i})
            counts[0, h, i] = len(blocks)
            indices[0, h, i, : len(blocks)] = blocks
            for j in blocks:
                mask[0, h, i * b:(i + 1) * b, j * b:(j + 1) * b] = True
    mask &= torch.ones(n, n, dtype=torch.bool).tril()
    out, _ = oracle.sparse_attention(q, k, v, counts, indices, b)
    ref = _sdpa(q, k, v, mask=mask)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_gamma_one_pipeline_is_dense():
    """gamma = 1 selects every causal block, so the output is dense attention."""
    n, d, b, hq, hkv = 256, 16, 32, 4, 2
    q, k, v = _rand((1, hq, n, d), 10), _rand((1, hkv, n, d), 11), _rand((1, hkv, n, d), 12)
    res = oracle.flexprefill(q, k, v, b, gamma=1.0, tau=0.1, min_budget=0, max_budget=0)
    nb = n // b
    assert (res["counts"][0] == np.arange(1, nb + 1)).all()
    ref = _sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(res["out"], ref, rtol=0, atol=1e-12)


def test_sampled_rows_match_full():
    n, d, b, hq, hkv = 128, 8, 16, 2, 1
    q, k, v = _rand((1, hq, n, d), 13), _rand((1, hkv, n, d), 14), _rand((1, hkv, n, d), 15)
    full, _ = oracle.dense_attention(q, k, v, b)
    part, _ = oracle.dense_attention(q, k, v, b, heads=[1], q_blocks=[0, 5])
    np.testing.assert_array_equal(part[0, 1, 0:16], full[0, 1, 0:16])
    np.testing.assert_array_equal(part[0, 1, 80:96], full[0, 1, 80:96])
    assert np.isnan(part[0, 0]).all()
