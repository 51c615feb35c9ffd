"""GPU parity on sequences whose length is not a multiple of the block size
(a partial last block), through the C ABI against the oracle.

Reading (the oracle's): nb = ceil(N / B); the partial last block is pooled over
its real tokens and is the last query block of the estimate; attention runs
over real keys only.  Tolerances as in test_gpu_parity.py: estimate rtol 1e-4,
lists bit-exact on the kernels' own fp32 scores, attention 2e-2 (bf16) /
1e-4 (fp32).
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_fp_b200 import build, ops, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

DEV = "cuda:0"

# (workload, overrides): bf16 block 128 (tensor-core estimate passes with a
# partial last tile), bf16 block 64 with an odd block count (CUDA-core
# passes), fp32 block 64 and block 128 (the debug path)
CASES = {
    "bf16_b128_n8256": ("llama8b_n8192", dict(seq_len=8192 + 64, n_q_heads=8, n_kv_heads=2)),
    "bf16_b128_n1000": ("llama8b_n8192", dict(seq_len=1000, n_q_heads=8, n_kv_heads=2)),
    "bf16_b64_n1105": ("glm9b_n65536_b64", dict(seq_len=1088 + 17, n_q_heads=8, n_kv_heads=2,
                                                max_budget=512)),
    "f32_b64_n1000": ("tiny_n1024", dict(seq_len=1000)),
    "f32_b128_n777": ("llama8b_n8192", dict(dtype="f32", seq_len=777, n_q_heads=4,
                                            n_kv_heads=2)),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    assert ops.fp_last_device_status() == 0


def _np(t):
    return t.detach().float().cpu().numpy()


_CACHE = {}


def _case(name):
    if name not in _CACHE:
        base, kw = CASES[name]
        w = synth.WORKLOADS[base].replace(**kw)
        assert w.seq_len % w.block_size != 0
        inp = synth.make_inputs(w)
        _CACHE.clear()
        _CACHE[name] = (w, inp, {x: inp[x].to(DEV) for x in ("q", "k", "v")})
    return _CACHE[name]


@pytest.mark.parametrize("name", sorted(CASES))
def test_ragged_estimate_parity(name):
    w, inp, d = _case(name)
    got = ops.estimate(d["q"], d["k"], w.block_size)
    torch.cuda.synchronize()
    want = oracle.estimate(inp["q"], inp["k"], w.block_size)
    nb = w.n_blocks
    assert got["map"].shape[-1] == nb * (nb + 1) // 2
    for key in ("qbar", "kbar", "map", "est_last", "true_last", "vert", "slash"):
        np.testing.assert_allclose(_np(got[key]), want[key], rtol=1e-4, atol=1e-7,
                                   err_msg=f"{name}:{key}")
    assert ops.fp_last_device_status() == 0


@pytest.mark.parametrize("name", sorted(CASES))
def test_ragged_pipeline_parity(name):
    """Lists bit-exact against the oracle's rule on the kernels' scores, both
    patterns present; attention on every head's first, middle and partial
    last block against the oracle; the whole-path call equals the staged
    calls."""
    w, inp, d = _case(name)
    bf16 = w.dtype == "bf16"
    tol = 2e-2 if bf16 else 1e-4
    ltol = 2e-3 if bf16 else 1e-4
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    _, pat = ops.pattern(s, p, est["est_last"], est["true_last"])
    pat = (torch.arange(pat.numel(), device=DEV, dtype=torch.int32) % 2).reshape(pat.shape)
    counts, indices = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
    out, lse = ops.sparse_attn(d["q"], d["k"], d["v"], counts, indices, w.block_size)
    torch.cuda.synchronize()
    nb = w.n_blocks
    oc, oi = oracle.select(pat.cpu().numpy(), _np(est["map"]), _np(est["vert"]),
                           _np(est["slash"]), nb, w.block_size, w.gamma, w.min_budget,
                           w.max_budget)
    gc, gi = counts.cpu().numpy(), indices.cpu().numpy()
    np.testing.assert_array_equal(gc, oc)
    for h in range(w.n_q_heads):
        for i in range(nb):
            assert np.array_equal(gi[0, h, i, :gc[0, h, i]], oi[0, h, i, :oc[0, h, i]]), (h, i)
    heads = list(range(w.n_q_heads))
    o, l = oracle.sparse_attention(inp["q"], inp["k"], inp["v"], gc, gi, w.block_size, heads,
                                   [0, nb // 2, nb - 1])
    m = ~np.isnan(o)
    assert np.abs(_np(out)[m] - o[m]).max() <= tol
    ml = ~np.isnan(l)
    assert np.abs(_np(lse)[ml] - l[ml]).max() <= ltol
    # dense on the partial block too
    dout, dlse = ops.dense_attn(d["q"], d["k"], d["v"], w.block_size)
    torch.cuda.synchronize()
    o, l = oracle.dense_attention(inp["q"], inp["k"], inp["v"], w.block_size, heads=[0, 1],
                                  q_blocks=[0, nb - 1])
    m = ~np.isnan(o)
    assert np.abs(_np(dout)[m] - o[m]).max() <= tol
    # the whole path in one call: bitwise the staged calls (natural pattern)
    _, pat2 = ops.pattern(s, p, est["est_last"], est["true_last"])
    c2, i2 = ops.select(s, p, pat2, est["map"], est["vert"], est["slash"])
    o2, _ = ops.sparse_attn(d["q"], d["k"], d["v"], c2, i2, w.block_size)
    out3, _, stats = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    torch.cuda.synchronize()
    assert torch.equal(out3, o2)
    assert int(stats[0]) == int(c2.sum())
    assert ops.fp_last_device_status() == 0


def test_ragged_varlen_and_host_paths():
    """Sequences of lengths that are not multiples of the block size in one
    varlen call, each bitwise its own fp_prefill_attn call; the host-buffer
    path on a ragged layer bitwise the device path."""
    w = synth.WORKLOADS["llama8b_n8192"].replace(n_q_heads=8, n_kv_heads=2)
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget)
    seqs = []
    for n in (1000, 257, 2048, 129):
        inp = synth.make_inputs(w.replace(seq_len=n))
        seqs.append({x: inp[x].to(DEV) for x in ("q", "k", "v")})
    outs, stats = ops.prefill_attn_varlen([x["q"] for x in seqs], [x["k"] for x in seqs],
                                          [x["v"] for x in seqs], w.block_size, p)
    for i, x in enumerate(seqs):
        want, _, st = ops.prefill_attn(x["q"], x["k"], x["v"], w.block_size, p)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], want), i
        assert torch.equal(stats[i], st), i
    x = seqs[0]
    s = ops.make_shape(x["q"], x["k"], w.block_size)
    want, _, _ = ops.prefill_attn(x["q"], x["k"], x["v"], w.block_size, p)
    qh, kh, vh = (x[k].cpu().contiguous().pin_memory() for k in ("q", "k", "v"))
    oh = torch.empty_like(qh).pin_memory()
    ws = ops.workspace(s, ops.FP_CALL_PREFILL_HOST, DEV)
    assert ops.fp_prefill_attn_host(s, p, qh, kh, vh, oh, ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(oh, want.cpu())
    assert ops.fp_last_device_status() == 0


@pytest.mark.parametrize("n,base,kw", [
    (1, "llama8b_n8192", dict(n_q_heads=4, n_kv_heads=2)),
    (100, "llama8b_n8192", dict(n_q_heads=4, n_kv_heads=2)),
    (129, "llama8b_n8192", dict(n_q_heads=4, n_kv_heads=2)),
    (1, "tiny_n1024", {}),
    (65, "tiny_n1024", {}),
])
def test_shortest_sequences(n, base, kw):
    """A single token, fewer tokens than one block, and one token past a
    block: the whole path against the oracle (estimate 1e-4, lists bit-exact,
    every row of attention) and the whole-path call against the staged calls."""
    w = synth.WORKLOADS[base].replace(seq_len=n, **kw)
    inp = synth.make_inputs(w)
    d = {x: inp[x].to(DEV) for x in ("q", "k", "v")}
    bf16 = w.dtype == "bf16"
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    torch.cuda.synchronize()
    want = oracle.estimate(inp["q"], inp["k"], w.block_size)
    for key in ("qbar", "kbar", "map", "est_last", "true_last", "vert", "slash"):
        np.testing.assert_allclose(_np(est[key]), want[key], rtol=1e-4, atol=1e-7, err_msg=key)
    _, pat = ops.pattern(s, p, est["est_last"], est["true_last"])
    counts, indices = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
    out, lse = ops.sparse_attn(d["q"], d["k"], d["v"], counts, indices, w.block_size)
    torch.cuda.synchronize()
    nb = w.n_blocks
    oc, oi = oracle.select(pat.cpu().numpy(), _np(est["map"]), _np(est["vert"]),
                           _np(est["slash"]), nb, w.block_size, w.gamma, w.min_budget,
                           w.max_budget)
    np.testing.assert_array_equal(counts.cpu().numpy(), oc)
    o, l = oracle.sparse_attention(inp["q"], inp["k"], inp["v"], oc, oi, w.block_size)
    assert np.abs(_np(out) - o).max() <= (2e-2 if bf16 else 1e-4)
    assert np.abs(_np(lse) - l).max() <= (2e-3 if bf16 else 1e-4)
    out2, _, _ = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    torch.cuda.synchronize()
    assert torch.equal(out2, out)
    assert ops.fp_last_device_status() == 0
