"""GPU parity: every stage of the CUDA path against the CPU oracle, through the
C ABI (ops.fp_* -> libfp.so).

Tolerances (written here, derived from the arithmetic):
  estimate     rtol 1e-4 (+ atol 1e-7 for values near 0): fp32 accumulation of
               bf16/fp32 inputs against fp64;
  pattern      identical decision wherever |d_JS - tau| > 1e-6; d_JS within 1e-6;
  select       bit-exact counts and index lists, given the kernels' own fp32
               scores and pattern (integer rule, no rounding);
  attention    max |out - oracle| <= 1e-4 on the fp32 path, <= 2e-2 on the
               bf16 tensor-core path; lse within 1e-4 / 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_fp_b200 import build, ops, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    assert ops.fp_last_device_status() == 0


def _np(t):
    return t.detach().float().cpu().numpy()


_CACHE = {}


def _inputs(name, **kw):
    key = (name, tuple(sorted(kw.items())))
    if key not in _CACHE:
        w = synth.WORKLOADS[name].replace(**kw) if kw else synth.WORKLOADS[name]
        inp = synth.make_inputs(w)
        _CACHE.clear()  # keep one workload's tensors alive at a time
        _CACHE[key] = (w, inp, {x: inp[x].to(DEV) for x in ("q", "k", "v")})
    return _CACHE[key]


def _estimate_close(got, want, name):
    for key in ("qbar", "kbar", "map", "est_last", "true_last", "vert", "slash"):
        g, o = _np(got[key]), want[key]
        np.testing.assert_allclose(g, o, rtol=1e-4, atol=1e-7, err_msg=f"{name}:{key}")


@pytest.mark.parametrize("name", ["tiny_n1024", "llama8b_n8192"])
def test_estimate_parity(name):
    w, inp, d = _inputs(name)
    got = ops.estimate(d["q"], d["k"], w.block_size)
    torch.cuda.synchronize()
    want = oracle.estimate(inp["q"], inp["k"], w.block_size)
    _estimate_close(got, want, name)
    assert ops.fp_last_device_status() == 0


@pytest.mark.parametrize("n", [1024, 1088])
def test_estimate_parity_block64_bf16(n):
    """Block size 64, bf16: N a multiple of 128 runs the tensor-core last-block
    passes on 128-key tiles with the first 64 of the last 128 queries left out;
    N = 1088 (an odd number of blocks) takes the CUDA-core passes."""
    w, inp, d = _inputs("glm9b_n65536_b64", seq_len=n, n_q_heads=8, n_kv_heads=2)
    got = ops.estimate(d["q"], d["k"], 64)
    torch.cuda.synchronize()
    want = oracle.estimate(inp["q"], inp["k"], 64)
    _estimate_close(got, want, f"b64bf16n{n}")
    assert ops.fp_last_device_status() == 0


def test_estimate_parity_block64_and_d128_fp32():
    w, inp, d = _inputs("tiny_n1024", head_dim=128, n_q_heads=4, n_kv_heads=2,
                        fixed_kinds=("qa", "vs"), seq_len=512)
    got = ops.estimate(d["q"], d["k"], 64)
    want = oracle.estimate(inp["q"], inp["k"], 64)
    _estimate_close(got, want, "b64d128")
    got = ops.estimate(d["q"], d["k"], 128)
    want = oracle.estimate(inp["q"], inp["k"], 128)
    _estimate_close(got, want, "b128d128")


@pytest.mark.parametrize("tau", [0.0, 0.03, 0.1, 0.9])
def test_pattern_parity(tau):
    w, inp, d = _inputs("llama8b_n8192")
    est = ops.estimate(d["q"], d["k"], w.block_size)
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    djs, pat = ops.pattern(s, ops.make_params(0.95, tau), est["est_last"], est["true_last"])
    odjs, opat = oracle.pattern(_np(est["est_last"]), _np(est["true_last"]), tau)
    np.testing.assert_allclose(_np(djs), odjs, rtol=0, atol=1e-6)
    decided = np.abs(odjs - np.float32(tau)) > 1e-6
    assert (pat.cpu().numpy()[decided] == opat[decided]).all()
    if tau == 0.0:
        assert (pat.cpu().numpy() == oracle.PATTERN_VS).all()


def _select_case(w, est, pat, gamma, lo, hi, qa_mode=0, vs_mode=0):
    s = ops.fp_shape(w.batch, w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.block_size,
                     ops.FP_BF16 if w.dtype == "bf16" else ops.FP_F32)
    p = ops.make_params(gamma, 0.1, lo, hi, qa_mode, vs_mode)
    counts, indices = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
    torch.cuda.synchronize()
    oc, oi = oracle.select(pat.cpu().numpy(), _np(est["map"]), _np(est["vert"]),
                           _np(est["slash"]), w.n_blocks, w.block_size, gamma, lo, hi, qa_mode,
                           vs_mode)
    gc = counts.cpu().numpy()
    gi = indices.cpu().numpy()
    np.testing.assert_array_equal(gc, oc)
    bt, hq, nb = gc.shape
    for b in range(bt):
        for h in range(hq):
            for i in range(nb):
                c = gc[b, h, i]
                if not np.array_equal(gi[b, h, i, :c], oi[b, h, i, :c]):
                    raise AssertionError(f"row ({b},{h},{i}) differs")
    return gc


@pytest.mark.parametrize("name", ["tiny_n1024", "llama8b_n8192"])
@pytest.mark.parametrize("mode", ["natural", "all_vs", "alternate"])
@pytest.mark.parametrize("gamma,lo,hi", [(0.95, 1024, 0), (0.9, 0, 0), (0.9, 2048, 8192),
                                         (0.5, 0, 1024), (1.0, 0, 0), (0.999, 256, 0)])
def test_select_bit_exact(name, mode, gamma, lo, hi):
    w, inp, d = _inputs(name)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    _, pat = ops.pattern(s, ops.make_params(0.95, 0.1), est["est_last"], est["true_last"])
    if mode == "all_vs":
        pat = torch.full_like(pat, ops.FP_PATTERN_VS)
    elif mode == "alternate":
        pat = (torch.arange(pat.numel(), device=DEV, dtype=torch.int32) % 2).reshape(pat.shape)
    gc = _select_case(w, est, pat, gamma, lo, hi)
    if gamma >= 1.0:
        assert (gc == np.arange(1, w.n_blocks + 1)).all()


@pytest.mark.parametrize("name", ["tiny_n1024", "llama8b_n8192"])
@pytest.mark.parametrize("mode", ["natural", "alternate"])
@pytest.mark.parametrize("gamma,lo,hi", [(0.95, 1024, 0), (0.9, 0, 0), (0.9, 2048, 8192),
                                         (0.5, 0, 1024), (1.0, 0, 0), (0.999, 256, 0),
                                         (0.9, 0, 100)])
def test_select_querywise_bit_exact(name, mode, gamma, lo, hi):
    """Query-wise rule for query-aware heads (one cumulative rule per map row)."""
    w, inp, d = _inputs(name)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    _, pat = ops.pattern(s, ops.make_params(0.95, 0.1), est["est_last"], est["true_last"])
    if mode == "alternate":
        pat = (torch.arange(pat.numel(), device=DEV, dtype=torch.int32) % 2).reshape(pat.shape)
    gc = _select_case(w, est, pat, gamma, lo, hi, ops.FP_QA_QUERYWISE)
    if gamma >= 1.0:
        assert (gc == np.arange(1, w.n_blocks + 1)).all()


def test_select_querywise_ties_and_long_rows():
    """Hand-made map rows with exact ties and zeros, nb = 256 (rows up to 256
    entries, several sort stages past one thread's share)."""
    w = synth.WORKLOADS["llama8b_n8192"].replace(seq_len=256 * 64, block_size=64, n_q_heads=2,
                                                 n_kv_heads=1)
    nb, n = w.n_blocks, w.seq_len
    t_pairs = nb * (nb + 1) // 2
    g = torch.Generator().manual_seed(9)
    levels = torch.tensor([0.0, 1e-4, 3e-4, 1e-3, 2.0 ** -20], dtype=torch.float32)
    mp = levels[torch.randint(0, 5, (1, 2, t_pairs), generator=g)]
    est = {"map": mp.to(DEV), "vert": torch.rand(1, 2, n).to(DEV),
           "slash": torch.rand(1, 2, n).to(DEV)}
    pat = torch.zeros(1, 2, dtype=torch.int32, device=DEV)
    for gamma, lo, hi in [(0.9, 0, 0), (0.7, 640, 1280), (0.3, 0, 0), (0.99, 0, 64)]:
        _select_case(w, est, pat, gamma, lo, hi, ops.FP_QA_QUERYWISE)


@pytest.mark.parametrize("name", ["tiny_n1024", "llama8b_n8192"])
@pytest.mark.parametrize("mode", ["all_vs", "alternate"])
@pytest.mark.parametrize("gamma,lo,hi", [(0.95, 1024, 0), (0.9, 0, 0), (0.9, 2048, 8192),
                                         (0.5, 0, 1000), (1.0, 0, 0), (0.999, 200, 0)])
def test_select_vs_blocks_bit_exact(name, mode, gamma, lo, hi):
    """Block-pooled vertical-slash lines (sums per key block / block distance)."""
    w, inp, d = _inputs(name)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    if mode == "all_vs":
        pat = torch.full((w.batch, w.n_q_heads), ops.FP_PATTERN_VS, dtype=torch.int32, device=DEV)
    else:
        pat = (torch.arange(w.batch * w.n_q_heads, device=DEV, dtype=torch.int32) % 2).reshape(
            w.batch, w.n_q_heads)
    for qa_mode in (ops.FP_QA_FLATTENED, ops.FP_QA_QUERYWISE):
        gc = _select_case(w, est, pat, gamma, lo, hi, qa_mode, ops.FP_VS_BLOCKS)
    if gamma >= 1.0:
        assert (gc == np.arange(1, w.n_blocks + 1)).all()


def test_prefill_vs_blocks_pipeline():
    """tau = 0 (every head vertical-slash) with block-pooled lines: the
    selection against the oracle on the same estimate, sampled attention, and
    fp_prefill_attn against the staged calls."""
    w, inp, d = _inputs("llama8b_n8192")
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    p = ops.make_params(w.gamma, 0.0, w.min_budget, 4096, 0, ops.FP_VS_BLOCKS)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    _, pat = ops.pattern(s, p, est["est_last"], est["true_last"])
    assert (pat == ops.FP_PATTERN_VS).all()
    counts, indices = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
    out, lse = ops.sparse_attn(d["q"], d["k"], d["v"], counts, indices, w.block_size)
    torch.cuda.synchronize()
    oc, _ = oracle.select(pat.cpu().numpy(), _np(est["map"]), _np(est["vert"]), _np(est["slash"]),
                          w.n_blocks, w.block_size, w.gamma, w.min_budget, 4096,
                          oracle.QA_FLATTENED, oracle.VS_BLOCKS)
    np.testing.assert_array_equal(counts.cpu().numpy(), oc)
    res = dict(counts=counts, indices=indices, out=out, lse=lse)
    _attn_check(inp, res, w, 2e-2, 2e-3, heads=[1, 30], q_blocks=[5, 40, 63])
    out2, _, stats = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    torch.cuda.synchronize()
    assert torch.equal(out2, out)
    assert int(stats[0]) == int(counts.sum())


def test_select_ties_and_zero_scores():
    """Hand-made scores: many exact ties and zero entries (radix tie rank)."""
    w = synth.WORKLOADS["tiny_n1024"].replace(n_q_heads=2, n_kv_heads=1)
    nb, n = w.n_blocks, w.seq_len
    t_pairs = nb * (nb + 1) // 2
    g = torch.Generator().manual_seed(5)
    levels = torch.tensor([0.0, 1e-3, 2e-3, 5e-3, 2.0 ** -20], dtype=torch.float32)
    mp = levels[torch.randint(0, 5, (1, 2, t_pairs), generator=g)]
    vt = levels[torch.randint(0, 5, (1, 2, n), generator=g)]
    sl = levels[torch.randint(0, 5, (1, 2, n), generator=g)]
    est = {"map": mp.to(DEV), "vert": vt.to(DEV), "slash": sl.to(DEV)}
    pat = torch.tensor([[0, 1]], dtype=torch.int32, device=DEV)
    for gamma, lo, hi in [(0.9, 0, 0), (0.7, 100, 300), (0.3, 0, 0)]:
        _select_case(w, est, pat, gamma, lo, hi)


def _pipeline(w, d, gamma=None, tau=None, lo=None, hi=None):
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    p = ops.make_params(w.gamma if gamma is None else gamma, w.tau if tau is None else tau,
                        w.min_budget if lo is None else lo, w.max_budget if hi is None else hi)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    djs, pat = ops.pattern(s, p, est["est_last"], est["true_last"])
    counts, indices = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
    out, lse = ops.sparse_attn(d["q"], d["k"], d["v"], counts, indices, w.block_size)
    torch.cuda.synchronize()
    return dict(est=est, djs=djs, pattern=pat, counts=counts, indices=indices, out=out, lse=lse,
                shape=s, params=p)


def _attn_check(inp, res, w, tol, lse_tol, heads=None, q_blocks=None):
    o, l = oracle.sparse_attention(inp["q"], inp["k"], inp["v"], res["counts"].cpu().numpy(),
                                   res["indices"].cpu().numpy(), w.block_size, heads, q_blocks)
    g, gl = _np(res["out"]), _np(res["lse"])
    m = ~np.isnan(o)
    err = np.abs(g[m] - o[m]).max()
    assert err <= tol, f"max abs err {err}"
    ml = ~np.isnan(l)
    lerr = np.abs(gl[ml] - l[ml]).max()
    assert lerr <= lse_tol, f"lse err {lerr}"
    return err


def test_pipeline_tiny_fp32_parity():
    w, inp, d = _inputs("tiny_n1024")
    res = _pipeline(w, d)
    err = _attn_check(inp, res, w, 1e-4, 1e-4)
    assert err < 1e-4
    assert ops.fp_last_device_status() == 0


@pytest.mark.parametrize("tau,lo,hi", [(0.1, 1024, 0), (0.0, 1024, 8192), (0.1, 0, 2048)])
def test_pipeline_llama8k_bf16_parity(tau, lo, hi):
    w, inp, d = _inputs("llama8b_n8192")
    res = _pipeline(w, d, tau=tau, lo=lo, hi=hi)
    # every head, a spread of query blocks (first, diagonal-heavy, last)
    _attn_check(inp, res, w, 2e-2, 2e-3, heads=list(range(w.n_q_heads)),
                q_blocks=[0, 1, 17, 40, 63])
    assert ops.fp_last_device_status() == 0


@pytest.mark.parametrize("n,tau,hi", [(4096, 0.1, 0), (4096, 0.0, 1024), (4032, 0.1, 0)])
def test_pipeline_glm_block64_bf16_parity(n, tau, hi):
    """Block size 64 on the tensor cores (GLM-4-9B heads: 32 q / 2 kv), N with
    an even and an odd number of blocks."""
    w, inp, d = _inputs("glm9b_n65536_b64", seq_len=n, n_q_heads=8, n_kv_heads=2)
    res = _pipeline(w, d, tau=tau, hi=hi)
    nb = w.n_blocks
    _attn_check(inp, res, w, 2e-2, 2e-3, heads=list(range(w.n_q_heads)),
                q_blocks=[0, 1, 2, nb // 2, nb - 2, nb - 1])
    # dense at block 64 against the oracle
    out, lse = ops.dense_attn(d["q"], d["k"], d["v"], 64)
    torch.cuda.synchronize()
    o, l = oracle.dense_attention(inp["q"], inp["k"], inp["v"], 64, heads=[0, 5],
                                  q_blocks=[0, 3, nb - 1])
    m = ~np.isnan(o)
    assert np.abs(_np(out)[m] - o[m]).max() <= 2e-2
    ml = ~np.isnan(l)
    assert np.abs(_np(lse)[ml] - l[ml]).max() <= 2e-3
    assert ops.fp_last_device_status() == 0


@pytest.mark.parametrize("bs", [128, 64])
def test_pipeline_fp32_llama_heads_parity(bs):
    """The fp32 debug path on Llama-shaped heads (d = 128), block 128 and 64:
    sparse attention under a capped budget (rows of different lengths) and
    dense attention, both against the oracle at the fp32 bound."""
    w, inp, d = _inputs("llama8b_n8192", dtype="f32", seq_len=2048, n_q_heads=4, n_kv_heads=2,
                        block_size=bs)
    res = _pipeline(w, d, hi=512)
    nb = w.n_blocks
    full = torch.arange(1, nb + 1, device=DEV, dtype=torch.int32)
    assert res["counts"].min() >= 1 and (res["counts"] < full).any()  # some rows skip blocks
    _attn_check(inp, res, w, 1e-4, 1e-4, heads=[0, 1, 2, 3], q_blocks=[0, 1, nb // 2, nb - 1])
    out, lse = ops.dense_attn(d["q"], d["k"], d["v"], bs)
    torch.cuda.synchronize()
    o, l = oracle.dense_attention(inp["q"], inp["k"], inp["v"], bs, heads=[0, 3],
                                  q_blocks=[0, nb // 2, nb - 1])
    m = ~np.isnan(o)
    assert np.abs(_np(out)[m] - o[m]).max() <= 1e-4
    ml = ~np.isnan(l)
    assert np.abs(_np(lse)[ml] - l[ml]).max() <= 1e-4
    assert ops.fp_last_device_status() == 0


def test_dense_parity():
    w, inp, d = _inputs("tiny_n1024")
    out, lse = ops.dense_attn(d["q"], d["k"], d["v"], w.block_size)
    o, l = oracle.dense_attention(inp["q"], inp["k"], inp["v"], w.block_size)
    assert np.abs(_np(out) - o).max() <= 1e-4
    assert np.abs(_np(lse) - l).max() <= 1e-4
    w, inp, d = _inputs("llama8b_n8192")
    out, lse = ops.dense_attn(d["q"], d["k"], d["v"], w.block_size)
    torch.cuda.synchronize()
    o, l = oracle.dense_attention(inp["q"], inp["k"], inp["v"], w.block_size, heads=[0, 13, 31],
                                  q_blocks=[0, 31, 63])
    m = ~np.isnan(o)
    assert np.abs(_np(out)[m] - o[m]).max() <= 2e-2
    ml = ~np.isnan(l)
    assert np.abs(_np(lse)[ml] - l[ml]).max() <= 2e-3


def test_gamma_one_equals_dense_bitwise():
    w, inp, d = _inputs("llama8b_n8192")
    res = _pipeline(w, d, gamma=1.0)
    assert (res["counts"].cpu().numpy() == np.arange(1, w.n_blocks + 1)).all()
    out, lse = ops.dense_attn(d["q"], d["k"], d["v"], w.block_size)
    assert torch.equal(out, res["out"])
    assert torch.equal(lse, res["lse"])


def test_prefill_matches_stages_and_host_path():
    w, inp, d = _inputs("llama8b_n8192")
    res = _pipeline(w, d)
    out, _, stats = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, res["params"])
    torch.cuda.synchronize()
    assert torch.equal(out, res["out"])
    assert int(stats[0]) == int(res["counts"].sum())
    assert int(stats[1]) == int((res["pattern"] == ops.FP_PATTERN_QA).sum())
    # host buffers through the C ABI
    s = res["shape"]
    qh, kh, vh = (inp[x].contiguous().pin_memory() for x in ("q", "k", "v"))
    oh = torch.empty_like(qh).pin_memory()
    ws = ops.workspace(s, ops.FP_CALL_PREFILL_HOST, DEV)
    assert ops.fp_prefill_attn_host(s, res["params"], qh, kh, vh, oh, ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(oh, res["out"].cpu())


def test_prefill_querywise_pipeline():
    """The whole path with the query-wise rule: the selection against the
    oracle's query-wise rule on the same estimate, sampled attention against
    the oracle, and fp_prefill_attn against the staged calls."""
    w, inp, d = _inputs("llama8b_n8192")
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget, ops.FP_QA_QUERYWISE)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    _, pat = ops.pattern(s, p, est["est_last"], est["true_last"])
    counts, indices = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
    out, lse = ops.sparse_attn(d["q"], d["k"], d["v"], counts, indices, w.block_size)
    torch.cuda.synchronize()
    oc, _ = oracle.select(pat.cpu().numpy(), _np(est["map"]), _np(est["vert"]), _np(est["slash"]),
                          w.n_blocks, w.block_size, w.gamma, w.min_budget, w.max_budget,
                          oracle.QA_QUERYWISE)
    np.testing.assert_array_equal(counts.cpu().numpy(), oc)
    res = dict(counts=counts, indices=indices, out=out, lse=lse)
    _attn_check(inp, res, w, 2e-2, 2e-3, heads=[0, 13, 31], q_blocks=[0, 17, 63])
    out2, _, stats = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    torch.cuda.synchronize()
    assert torch.equal(out2, out)
    assert int(stats[0]) == int(counts.sum())


def test_host_path_batch2_fp32_matches_device_path():
    """fp_prefill_attn_host runs as pipelined units of (batch entry, kv heads):
    with two batch entries and two kv heads (four units) its output must be
    bitwise the device path's."""
    w = synth.WORKLOADS["tiny_n1024"].replace(batch=2)
    inp = synth.make_inputs(w)
    d = {x: inp[x].to(DEV) for x in ("q", "k", "v")}
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget)
    out, _, _ = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    qh, kh, vh = (inp[x].contiguous().pin_memory() for x in ("q", "k", "v"))
    oh = torch.empty_like(qh).pin_memory()
    ws = ops.workspace(s, ops.FP_CALL_PREFILL_HOST, DEV)
    assert ops.fp_prefill_attn_host(s, p, qh, kh, vh, oh, ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(oh, out.cpu())
    assert ops.fp_last_device_status() == 0


@pytest.mark.parametrize("batch,hq,hkv", [(1, 4, 4), (2, 8, 4)])
def test_host_path_unit_plans_match_device_path(batch, hq, hkv):
    """The host path's unit plans: one query head per kv head (whole kv heads
    in every unit) and, with two query heads per kv head over two batch
    entries, single-query-head first and last units whose kv heads' K and V
    come in with the first; bitwise the device path's output."""
    w = synth.WORKLOADS["llama8b_n8192"].replace(batch=batch, seq_len=1024, n_q_heads=hq,
                                                 n_kv_heads=hkv)
    inp = synth.make_inputs(w)
    d = {x: inp[x].to(DEV) for x in ("q", "k", "v")}
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget)
    out, _, _ = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    qh, kh, vh = (inp[x].contiguous().pin_memory() for x in ("q", "k", "v"))
    oh = torch.empty_like(qh).pin_memory()
    ws = ops.workspace(s, ops.FP_CALL_PREFILL_HOST, DEV)
    assert ops.fp_prefill_attn_host(s, p, qh, kh, vh, oh, ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(oh, out.cpu())
    assert ops.fp_last_device_status() == 0


def test_sharded_single_rank_is_the_whole_path():
    """With one rank the head-sharded entry is fp_prefill_attn, bitwise."""
    from dynamic_block_sparse_fp_b200 import sharded
    w, inp, d = _inputs("llama8b_n8192")
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget)
    want, _, _ = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    got = sharded.sharded_prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    qs, ks, vs = sharded.shard_inputs(d["q"], d["k"], d["v"], 2, 1)  # rank 1 of 2: heads 16-31
    half, _, _ = ops.prefill_attn(qs, ks, vs, w.block_size, p)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    assert torch.equal(half, want[:, 16:])


@pytest.mark.parametrize("name,n", [("llama8b_n8192", None), ("tiny_n1024", None),
                                    ("glm9b_n65536_b64", 4096)])
def test_prefill_pattern_aware_mixed_heads_bitwise(name, n):
    """fp_prefill_attn computes Q pooling and the map only for query-aware
    heads; with tau between the heads' d_JS values (both patterns present) its
    output and counts must be bitwise those of the separate calls."""
    w, inp, d = _inputs(name, **({"seq_len": n, "n_q_heads": 8, "n_kv_heads": 2} if n else {}))
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    djs, _ = ops.pattern(s, ops.make_params(w.gamma, w.tau), est["est_last"], est["true_last"])
    v = np.sort(np.unique(djs.cpu().numpy().ravel()))
    assert v.size >= 2
    tau = float((v[v.size // 2 - 1] + v[v.size // 2]) / 2)
    p = ops.make_params(w.gamma, tau, w.min_budget, w.max_budget)
    _, pat = ops.pattern(s, p, est["est_last"], est["true_last"])
    n_qa = int((pat == ops.FP_PATTERN_QA).sum())
    assert 0 < n_qa < pat.numel()
    counts, indices = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
    out, _ = ops.sparse_attn(d["q"], d["k"], d["v"], counts, indices, w.block_size)
    out2, _, stats = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p)
    torch.cuda.synchronize()
    assert torch.equal(out2, out)
    assert int(stats[0]) == int(counts.sum()) and int(stats[1]) == n_qa
    # the whole-path call's kept blocks against the oracle's rule on the same scores
    oc, _ = oracle.select(pat.cpu().numpy(), _np(est["map"]), _np(est["vert"]),
                          _np(est["slash"]), w.n_blocks, w.block_size, w.gamma, w.min_budget,
                          w.max_budget)
    assert int(stats[0]) == int(oc.sum())


def test_varlen_batch_matches_separate_calls():
    """Three sequences of different lengths in one fp_prefill_attn_varlen call:
    every output and every per-sequence stats row is bitwise that of the
    sequence's own fp_prefill_attn call."""
    base = synth.WORKLOADS["llama8b_n8192"].replace(n_q_heads=8, n_kv_heads=2)
    seqs = [synth.make_inputs(base.replace(seq_len=n, seed=40 + i))
            for i, n in enumerate((2048, 256, 1024))]
    qs = [x["q"].to(DEV) for x in seqs]
    ks = [x["k"].to(DEV) for x in seqs]
    vs = [x["v"].to(DEV) for x in seqs]
    p = ops.make_params(base.gamma, base.tau, base.min_budget, base.max_budget)
    outs, stats = ops.prefill_attn_varlen(qs, ks, vs, base.block_size, p)
    torch.cuda.synchronize()
    for i in range(3):
        want, _, st = ops.prefill_attn(qs[i], ks[i], vs[i], base.block_size, p)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], want), i
        assert torch.equal(stats[i], st), i
    assert ops.fp_last_device_status() == 0


def test_edge_empty_rows_and_device_checks():
    for name in ("tiny_n1024", "llama8b_n8192"):
        w, inp, d = _inputs(name, seq_len=1024) if name != "tiny_n1024" else _inputs(name)
        nb = w.n_blocks
        bt, hq = w.batch, w.n_q_heads
        counts = torch.zeros(bt, hq, nb, dtype=torch.int32, device=DEV)
        indices = torch.zeros(bt, hq, nb, nb, dtype=torch.int32, device=DEV)
        counts[:, :, 1::2] = 1  # odd rows: only key block 0; even rows: empty
        out, lse = ops.sparse_attn(d["q"], d["k"], d["v"], counts, indices, w.block_size)
        torch.cuda.synchronize()
        o, l = oracle.sparse_attention(inp["q"], inp["k"], inp["v"], counts.cpu().numpy(),
                                       indices.cpu().numpy(), w.block_size, heads=[0],
                                       q_blocks=[1, 3])
        bs = w.block_size
        tol = 1e-4 if w.dtype == "f32" else 2e-2
        for qi in (1, 3):
            sl = slice(qi * bs, (qi + 1) * bs)
            assert np.abs(_np(out)[0, 0, sl] - o[0, 0, sl]).max() <= tol
        even = _np(out).reshape(bt, hq, nb, bs, -1)[:, :, 0::2]
        assert (even == 0).all()
        assert torch.isinf(lse.reshape(bt, hq, nb, bs)[:, :, 0::2]).all()
        assert ops.fp_last_device_status() == 0
        # an index outside the causal range is flagged (and masked out)
        indices[0, 0, 1, 0] = 5
        ops.sparse_attn(d["q"], d["k"], d["v"], counts, indices, w.block_size)
        assert ops.fp_last_device_status() == ops.STATUS_CODES["FP_ERR_DEVICE_CHECK"]
        assert ops.fp_last_device_status() == 0


def _staircase_inputs():
    """bf16 Q/K/V (Bt 1, Hq 4, Hkv 2, N 1024, d 128) whose scores step from one
    64-key tile to the next by a fixed amount: q = c e0 and k_j[0] = a_j (bf16
    rounded; kernel and oracle read the same values), so
    scale*log2(e)*q.k_j = 0.1275 c a_j.
      head 0 (kv 0, c = 1):    +80 per tile, +10.3 in log2 units: the row max
                               jumps by more than 2^8 on every tile;
      head 1 (kv 0, c = -1):   the same keys falling: the max stays on the
                               first tile, later p underflow towards 0;
      head 2 (kv 1, c = 1):    +55 per tile, +7.1: tile sums above 2^8 with no
                               move, then a move every second tile;
      head 3 (kv 1, c = 0.5):  +3.6 per tile: a move every third tile.
    A small within-tile ramp (j mod 7) keeps the rows from being flat."""
    n, d = 1024, 128
    j = torch.arange(n)
    k = torch.zeros(1, 2, n, d)
    k[0, 0, :, 0] = 80.0 * (j // 64) + (j % 7)
    k[0, 1, :, 0] = 55.0 * (j // 64) + (j % 7)
    k[:, :, :, 1:] = torch.randn(1, 2, n, d - 1, generator=torch.Generator().manual_seed(5))
    q = torch.zeros(1, 4, n, d)
    for h, c in enumerate((1.0, -1.0, 1.0, 0.5)):
        q[0, h, :, 0] = c
    v = torch.randn(1, 2, n, d, generator=torch.Generator().manual_seed(6))
    return tuple(x.to(torch.bfloat16) for x in (q, k, v))


def test_attention_lazy_rescale_paths():
    """Rows whose running max moves by more than 2^8 on later tiles (O is
    rescaled in TMEM), rows whose tile sums exceed 2^8 without a move, and
    falling rows, dense and through sparse lists with gaps."""
    q, k, v = _staircase_inputs()
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    bs, nb = 128, 8
    out, lse = ops.dense_attn(qd, kd, vd, bs)
    torch.cuda.synchronize()
    o, l = oracle.dense_attention(q, k, v, bs)
    assert np.abs(_np(out) - o).max() <= 2e-2
    assert np.abs(_np(lse) - l).max() <= 2e-3
    # every other key block plus the diagonal: the max also jumps across gaps
    counts = torch.zeros(1, 4, nb, dtype=torch.int32)
    indices = torch.zeros(1, 4, nb, nb, dtype=torch.int32)
    for qi in range(nb):
        row = sorted(set(range(0, qi + 1, 2)) | {qi})
        counts[0, :, qi] = len(row)
        indices[0, :, qi, :len(row)] = torch.tensor(row, dtype=torch.int32)
    out, lse = ops.sparse_attn(qd, kd, vd, counts.to(DEV), indices.to(DEV), bs)
    torch.cuda.synchronize()
    o, l = oracle.sparse_attention(q, k, v, counts.numpy(), indices.numpy(), bs)
    assert np.abs(_np(out) - o).max() <= 2e-2
    assert np.abs(_np(lse) - l).max() <= 2e-3
    assert ops.fp_last_device_status() == 0


def test_attention_block64_masked_first_tiles_low_scores():
    """Block size 64: a CTA's rows are two query blocks on the union of their
    lists.  Rows of the odd block see the even block's tiles fully masked
    first, then only their own diagonal block, whose scores are all about
    -140 in log2 units; their softmax must still be the oracle's, not 0."""
    n, d, bs = 512, 128, 64
    nb = n // bs
    j = torch.arange(n)
    k = torch.zeros(1, 1, n, d)
    k[0, 0, :, 0] = 1100.0 + (j % 7)
    k[:, :, :, 1:] = torch.randn(1, 1, n, d - 1, generator=torch.Generator().manual_seed(7))
    q = torch.zeros(1, 1, n, d)
    q[0, 0, :, 0] = torch.where((j // bs) % 2 == 1, -1.0, 1.0)
    v = torch.randn(1, 1, n, d, generator=torch.Generator().manual_seed(8))
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    counts = torch.zeros(1, 1, nb, dtype=torch.int32)
    indices = torch.zeros(1, 1, nb, nb, dtype=torch.int32)
    for qi in range(nb):
        row = list(range(qi + 1)) if qi % 2 == 0 else [qi]
        counts[0, 0, qi] = len(row)
        indices[0, 0, qi, :len(row)] = torch.tensor(row, dtype=torch.int32)
    out, lse = ops.sparse_attn(q.to(DEV), k.to(DEV), v.to(DEV), counts.to(DEV),
                               indices.to(DEV), bs)
    torch.cuda.synchronize()
    o, l = oracle.sparse_attention(q, k, v, counts.numpy(), indices.numpy(), bs)
    assert np.abs(_np(out) - o).max() <= 2e-2
    assert np.abs(_np(lse) - l).max() <= 2e-3
    assert ops.fp_last_device_status() == 0


def test_single_block_sequence():
    w, inp, d = _inputs("llama8b_n8192", seq_len=128, n_q_heads=8, n_kv_heads=2)
    res = _pipeline(w, d)
    assert (res["counts"].cpu().numpy() == 1).all()
    _attn_check(inp, res, w, 2e-2, 2e-3)


def test_full_size_128k_sampled():
    """The bench configuration (Llama-3.1-8B heads, N = 131072), sampled checks."""
    w, inp, d = _inputs("llama8b_n131072")
    res = _pipeline(w, d)
    assert ops.fp_last_device_status() == 0
    hs = [0, 21]  # one head of two different kv groups
    g = w.n_q_heads // w.n_kv_heads
    for h in hs:
        kv = h // g
        want = oracle.estimate(inp["q"][:, h:h + 1], inp["k"][:, kv:kv + 1], w.block_size)
        sub = {k2: v2[:, h:h + 1] for k2, v2 in res["est"].items() if k2 not in ("kbar",)}
        for key in ("map", "est_last", "true_last", "vert", "slash", "qbar"):
            np.testing.assert_allclose(_np(sub[key]), want[key], rtol=1e-4, atol=1e-7,
                                       err_msg=key)
    # selection: the natural patterns, and every head forced to vertical-slash
    all_vs = torch.full_like(res["pattern"], ops.FP_PATTERN_VS)
    vs_counts, vs_indices = ops.select(res["shape"], res["params"], all_vs, res["est"]["map"],
                                       res["est"]["vert"], res["est"]["slash"])
    torch.cuda.synchronize()
    for h in hs:
        for pat, counts, indices in ((res["pattern"], res["counts"], res["indices"]),
                                     (all_vs, vs_counts, vs_indices)):
            oc, oi = oracle.select(pat[:, h:h + 1].cpu().numpy(),
                                   _np(res["est"]["map"][:, h:h + 1]),
                                   _np(res["est"]["vert"][:, h:h + 1]),
                                   _np(res["est"]["slash"][:, h:h + 1]), w.n_blocks,
                                   w.block_size, w.gamma, w.min_budget, w.max_budget)
            gc = counts[:, h:h + 1].cpu().numpy()
            gi = indices[:, h:h + 1].cpu().numpy()
            np.testing.assert_array_equal(gc, oc)
            for i in range(0, w.n_blocks, 37):
                np.testing.assert_array_equal(gi[0, 0, i, :gc[0, 0, i]], oi[0, 0, i, :oc[0, 0, i]])
    _attn_check(inp, res, w, 2e-2, 2e-3, heads=hs, q_blocks=[0, 511, 1023])


def _full_size_sampled(name, heads, q_blocks, rows_every=37, **over):
    """One configuration at its full size: the whole path on the GPU, then per
    sampled head the estimate (oracle, rtol 1e-4), the selection (bit-exact,
    on the GPU's own fp32 scores) and sampled attention rows (2e-2)."""
    w0, inp, d = _inputs(name)
    w = w0.replace(**over) if over else w0
    res = _pipeline(w, d)
    assert ops.fp_last_device_status() == 0
    g = w.n_q_heads // w.n_kv_heads
    for h in heads:
        kv = h // g
        want = oracle.estimate(inp["q"][:, h:h + 1], inp["k"][:, kv:kv + 1], w.block_size)
        for key in ("map", "est_last", "true_last", "vert", "slash"):
            np.testing.assert_allclose(_np(res["est"][key][:, h:h + 1]), want[key], rtol=1e-4,
                                       atol=1e-7, err_msg=f"{key} head {h}")
    all_vs = torch.full_like(res["pattern"], ops.FP_PATTERN_VS)
    vs_counts, vs_indices = ops.select(res["shape"], res["params"], all_vs, res["est"]["map"],
                                       res["est"]["vert"], res["est"]["slash"])
    torch.cuda.synchronize()
    for h in heads:
        for pat, counts, indices in ((res["pattern"], res["counts"], res["indices"]),
                                     (all_vs, vs_counts, vs_indices)):
            oc, oi = oracle.select(pat[:, h:h + 1].cpu().numpy(),
                                   _np(res["est"]["map"][:, h:h + 1]),
                                   _np(res["est"]["vert"][:, h:h + 1]),
                                   _np(res["est"]["slash"][:, h:h + 1]), w.n_blocks,
                                   w.block_size, w.gamma, w.min_budget, w.max_budget)
            gc = counts[:, h:h + 1].cpu().numpy()
            gi = indices[:, h:h + 1].cpu().numpy()
            np.testing.assert_array_equal(gc, oc)
            for i in range(0, w.n_blocks, rows_every):
                np.testing.assert_array_equal(gi[0, 0, i, :gc[0, 0, i]],
                                              oi[0, 0, i, :oc[0, 0, i]])
    _attn_check(inp, res, w, 2e-2, 2e-3, heads=heads, q_blocks=q_blocks)
    return res


@pytest.mark.parametrize("name", ["glm9b_n65536_b128", "glm9b_n65536_b64"])
def test_full_size_glm_64k_sampled(name):
    """GLM-4-9B heads (32 q / 2 kv), N = 65536, block 128 and 64, max budget
    32768 tokens, 75 % vertical-slash plantings."""
    w = synth.WORKLOADS[name]
    nb = w.n_blocks
    _full_size_sampled(name, heads=[3, 30], q_blocks=[0, nb // 2, nb - 1])


def test_full_size_32k_gamma09_sampled():
    """N = 32768 at gamma = 0.9 (the 32k sweep's other point)."""
    _full_size_sampled("llama8b_n32768", heads=[5, 26], q_blocks=[0, 100, 255], gamma=0.9)


def test_full_size_128k_vs_capped_sampled():
    """128k sweep points with every head vertical-slash (tau = 0), gamma = 0.9,
    min budget 2048 and max budget 8192 tokens."""
    _full_size_sampled("llama8b_n131072", heads=[2, 17], q_blocks=[1, 640, 1023], rows_every=61,
                       tau=0.0, gamma=0.9, min_budget=2048, max_budget=8192)


def test_full_size_128k_qa_capped_sampled():
    """The 128k sweep's sparse regime with query-aware heads: gamma = 0.9,
    tau = 0.1 (every head query-aware on this data), min budget 1024 and max
    budget 8192 tokens (12.6 % of the causal blocks kept); the whole-path
    call's output is bitwise the staged calls'."""
    res = _full_size_sampled("llama8b_n131072", heads=[0, 21], q_blocks=[0, 511, 1023],
                             rows_every=53, tau=0.1, gamma=0.9, min_budget=1024,
                             max_budget=8192)
    assert int((res["pattern"] == ops.FP_PATTERN_QA).sum()) > 0
    w, _, d = _inputs("llama8b_n131072")
    out, _, stats = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, res["params"])
    torch.cuda.synchronize()
    assert torch.equal(out, res["out"])
    assert int(stats[0]) == int(res["counts"].sum())


def test_maximum_block_count_sampled():
    """nb = 4096, the largest block count the library takes (N = 262144 at
    block 64, bf16, two query heads on one kv head): the estimate and one
    head's selection against the oracle (a map of 8.4 M entries), the
    allocation-free selection at this size, and sampled attention rows."""
    w = synth.WORKLOADS["glm9b_n65536_b64"].replace(seq_len=262144, n_q_heads=2, n_kv_heads=1)
    assert w.n_blocks == 4096
    inp = synth.make_inputs(w)
    d = {x: inp[x].to(DEV) for x in ("q", "k", "v")}
    res = _pipeline(w, d)
    assert ops.fp_last_device_status() == 0
    # the whole estimate at this size (32 row tiles of 128 query blocks in
    # the tensor-core map) against the oracle
    want = oracle.estimate(inp["q"], inp["k"], w.block_size)
    for key in ("map", "est_last", "true_last", "vert", "slash"):
        np.testing.assert_allclose(_np(res["est"][key]), want[key], rtol=1e-4, atol=1e-7,
                                   err_msg=key)
    h = 1
    oc, oi = oracle.select(res["pattern"][:, h:h + 1].cpu().numpy(),
                           _np(res["est"]["map"][:, h:h + 1]), _np(res["est"]["vert"][:, h:h + 1]),
                           _np(res["est"]["slash"][:, h:h + 1]), w.n_blocks, w.block_size,
                           w.gamma, w.min_budget, w.max_budget)
    gc = res["counts"][:, h:h + 1].cpu().numpy()
    gi = res["indices"][:, h:h + 1].cpu().numpy()
    np.testing.assert_array_equal(gc, oc)
    for i in (0, 1, 2047, 4094, 4095):
        np.testing.assert_array_equal(gi[0, 0, i, :gc[0, 0, i]], oi[0, 0, i, :oc[0, 0, i]])
    c2 = torch.empty_like(res["counts"])
    i2 = torch.empty_like(res["indices"])
    assert ops.fp_select_noalloc(res["shape"], res["params"], res["pattern"], res["est"]["map"],
                                 res["est"]["vert"], res["est"]["slash"], c2, i2) == 0
    torch.cuda.synchronize()
    assert torch.equal(c2, res["counts"])
    for hh in (0, 1):
        for i in (0, 1, 2047, 4094, 4095):
            n = int(res["counts"][0, hh, i])
            assert torch.equal(i2[0, hh, i, :n], res["indices"][0, hh, i, :n]), (hh, i)
    _attn_check(inp, res, w, 2e-2, 2e-3, heads=[0, 1], q_blocks=[0, 2048, 4095])
