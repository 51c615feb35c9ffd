"""The C-ABI calls inside CUDA graphs: the whole path (fp_prefill_attn) and
the four staged calls are captured once, after an eager call on the same
buffers, and replayed.  Every replay gives bitwise the eager result, and a
replay after new inputs are copied into the captured buffers gives the eager
result of those inputs (the graph reads the buffers' contents, not values
frozen at capture)."""
import pytest
import torch

from dynamic_block_sparse_fp_b200 import build, ops, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    assert ops.fp_last_device_status() == 0


def _inputs(seed):
    w = synth.WORKLOADS["llama8b_n8192"].replace(seq_len=4096 + 40, n_q_heads=8, n_kv_heads=2,
                                                 seed=seed)
    inp = synth.make_inputs(w)
    return w, {x: inp[x].to(DEV) for x in ("q", "k", "v")}


def test_whole_path_in_a_cuda_graph():
    w, d = _inputs(3)
    q, k, v = (d[x].clone() for x in ("q", "k", "v"))
    s = ops.make_shape(q, k, w.block_size)
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget)
    ws = ops.workspace(s, ops.FP_CALL_PREFILL, DEV)
    out = torch.empty_like(q)
    stats = torch.zeros(2, dtype=torch.int64, device=DEV)
    cur = torch.cuda.current_stream()
    assert ops.fp_prefill_attn(s, p, q, k, v, out, None, stats, ws, cur) == 0
    torch.cuda.synchronize()
    ref, ref_stats = out.clone(), stats.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        rc = ops.fp_prefill_attn(s, p, q, k, v, out, None, stats, ws,
                                 torch.cuda.current_stream())
    assert rc == 0
    for _ in range(2):
        out.zero_()
        stats.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref) and torch.equal(stats, ref_stats)
    # new inputs in the captured buffers
    w2, d2 = _inputs(4)
    for x, t in (("q", q), ("k", k), ("v", v)):
        t.copy_(d2[x])
    g.replay()
    torch.cuda.synchronize()
    want, _, want_stats = ops.prefill_attn(d2["q"], d2["k"], d2["v"], w.block_size, p)
    torch.cuda.synchronize()
    assert not torch.equal(want, ref)
    assert torch.equal(out, want) and torch.equal(stats, want_stats)
    assert ops.fp_last_device_status() == 0


def test_staged_calls_in_a_cuda_graph():
    w, d = _inputs(5)
    q, k, v = d["q"], d["k"], d["v"]
    s = ops.make_shape(q, k, w.block_size)
    p = ops.make_params(0.9, w.tau, w.min_budget, 2048)
    est = ops.estimate(q, k, w.block_size)
    djs, pat = ops.pattern(s, p, est["est_last"], est["true_last"])
    counts, indices = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
    out, lse = ops.sparse_attn(q, k, v, counts, indices, w.block_size)
    torch.cuda.synchronize()
    ref = {"out": out.clone(), "lse": lse.clone(), "counts": counts.clone(),
           "map": est["map"].clone()}
    ws_e = ops.workspace(s, ops.FP_CALL_ESTIMATE, DEV)
    ws_s = ops.workspace(s, ops.FP_CALL_SELECT, DEV)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = torch.cuda.current_stream()
        rcs = [ops.fp_estimate(s, q, k, est["qbar"], est["kbar"], est["map"], est["est_last"],
                               est["true_last"], est["vert"], est["slash"], ws_e, st),
               ops.fp_pattern(s, p, est["est_last"], est["true_last"], djs, pat, st),
               ops.fp_select(s, p, pat, est["map"], est["vert"], est["slash"], counts, indices,
                             ws_s, st),
               ops.fp_sparse_attn(s, q, k, v, counts, indices, out, lse, None, st)]
    assert rcs == [0, 0, 0, 0]
    for _ in range(2):
        out.zero_()
        counts.zero_()
        est["map"].zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref["out"]) and torch.equal(lse, ref["lse"])
        assert torch.equal(counts, ref["counts"]) and torch.equal(est["map"], ref["map"])
    assert ops.fp_last_device_status() == 0
