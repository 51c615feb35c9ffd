"""The whole path in one call (fp_prefill_attn) against the oracle's whole path
(oracle.flexprefill: its own fp64 estimate, rounded to fp32, then pattern,
selection and fp64 attention), end to end on the same seeded inputs.

FlexPrefill (atlas.scime.ai summary, "Approach") orders the steps: estimate,
pattern per head, selection on the chosen representation, sparse attention.
The kernels and the oracle take their decisions on fp32 scores that differ by
rounding (fp32 against fp64 accumulation), so a list can differ where a score
sits on the gamma boundary: the pattern must agree outside a 1e-6 margin, at
least 95 % of the (head, query block) lists must agree exactly, and the output
must agree (2e-2 bf16, 1e-4 fp32) on every sampled row whose list agrees.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_fp_b200 import build, ops, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

DEV = "cuda:0"

# (base workload, overrides, qa_mode, vs_mode, tau): fp32 block 64 (query-aware
# at tau 0.1), a ragged fp32 length at tau 0 (every head vertical-slash), bf16
# Llama heads with tau in the widest gap between the heads' d_JS values (both
# patterns) under both selection variants, and bf16 block 64 with a 512-token
# cap, all vertical-slash and all query-aware (ragged); two batch entries
CASES = {
    "f32_b64_flat_tokens": ("tiny_n1024", {}, 0, 0, None),
    "f32_b64_ragged_all_vs": ("tiny_n1024", dict(seq_len=1000), 0, 0, 0.0),
    "bf16_b128_split_tau": ("llama8b_n8192", dict(seq_len=4096, n_q_heads=8, n_kv_heads=2),
                            0, 0, "split"),
    "bf16_b128_querywise_blocklines": ("llama8b_n8192", dict(seq_len=4096, n_q_heads=8,
                                                             n_kv_heads=2), 1, 1, "split"),
    "bf16_b64_all_vs_capped": ("glm9b_n65536_b64", dict(seq_len=2048, n_q_heads=8,
                                                        n_kv_heads=2, max_budget=512), 0, 0, 0.0),
    "bf16_b64_all_qa_capped": ("glm9b_n65536_b64", dict(seq_len=2048 + 40, n_q_heads=8,
                                                        n_kv_heads=2, max_budget=512), 0, 0, None),
    "bf16_b128_batch2": ("llama8b_n8192", dict(batch=2, seq_len=2048 + 40, n_q_heads=8,
                                               n_kv_heads=2), 0, 0, "split"),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    assert ops.fp_last_device_status() == 0


def _np(t):
    return t.detach().float().cpu().numpy()


@pytest.mark.parametrize("name", sorted(CASES))
def test_whole_path_against_oracle_whole_path(name):
    base, kw, qa_mode, vs_mode, tau = CASES[name]
    w = synth.WORKLOADS[base].replace(**kw)
    inp = synth.make_inputs(w)
    d = {x: inp[x].to(DEV) for x in ("q", "k", "v")}
    bf16 = w.dtype == "bf16"
    nb = w.n_blocks
    want_est = oracle.estimate(inp["q"], inp["k"], w.block_size)
    if tau == "split":
        djs, _ = oracle.pattern(want_est["est_last"].astype(np.float32),
                                want_est["true_last"].astype(np.float32), 0.0)
        v = np.sort(np.unique(djs.ravel()))
        gaps = np.diff(v)
        i = int(np.argmax(gaps))
        tau = float((v[i] + v[i + 1]) / 2)
    else:
        tau = w.tau if tau is None else tau
    p = ops.make_params(w.gamma, tau, w.min_budget, w.max_budget, qa_mode, vs_mode)
    out, lse, stats = ops.prefill_attn(d["q"], d["k"], d["v"], w.block_size, p, with_lse=True)
    # the lists the whole path used: the staged calls give them bitwise
    s = ops.make_shape(d["q"], d["k"], w.block_size)
    est = ops.estimate(d["q"], d["k"], w.block_size)
    djs_g, pat_g = ops.pattern(s, p, est["est_last"], est["true_last"])
    counts, indices = ops.select(s, p, pat_g, est["map"], est["vert"], est["slash"])
    torch.cuda.synchronize()
    assert ops.fp_last_device_status() == 0
    assert int(stats[0]) == int(counts.sum())

    heads = list(range(w.n_q_heads)) if w.n_q_heads <= 2 else [0, 3, 4, 7]
    q_blocks = sorted({0, nb // 3, nb // 2, nb - 1})
    res = oracle.flexprefill(inp["q"], inp["k"], inp["v"], w.block_size, w.gamma, tau,
                             w.min_budget, w.max_budget, heads=heads, q_blocks=q_blocks,
                             qa_mode=qa_mode, vs_mode=vs_mode)
    # pattern: the same decision wherever d_JS is not within 1e-6 of tau
    djs_o = res["djs"]
    firm = np.abs(djs_o - tau) > 1e-6
    assert firm.any()
    np.testing.assert_array_equal(pat_g.cpu().numpy()[firm], res["pattern"][firm])
    # lists: exact agreement on at least 95 % of (head, query block) rows
    gc, gi = counts.cpu().numpy(), indices.cpu().numpy()
    oc, oi = res["counts"], res["indices"]
    same = np.zeros(gc.shape, dtype=bool)
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            for i in range(nb):
                same[b, h, i] = gc[b, h, i] == oc[b, h, i] and np.array_equal(
                    gi[b, h, i, :gc[b, h, i]], oi[b, h, i, :oc[b, h, i]])
    assert same.mean() >= 0.95, f"lists agree on {same.mean():.3f} of the rows"
    # output and log-sum-exp on the sampled rows whose lists agree
    o_g, l_g = _np(out), _np(lse)
    tol, ltol = (2e-2, 2e-3) if bf16 else (1e-4, 1e-4)
    checked = 0
    for b in range(w.batch):
        for h in heads:
            for i in q_blocks:
                if not same[b, h, i]:
                    continue
                r0, r1 = i * w.block_size, min((i + 1) * w.block_size, w.seq_len)
                o_o = res["out"][b, h, r0:r1]
                l_o = res["lse"][b, h, r0:r1]
                assert not np.isnan(o_o).any()
                assert np.abs(o_g[b, h, r0:r1] - o_o).max() <= tol, (b, h, i)
                assert np.abs(l_g[b, h, r0:r1] - l_o).max() <= ltol, (b, h, i)
                checked += 1
    assert checked >= w.batch * len(heads) * len(q_blocks) // 2
