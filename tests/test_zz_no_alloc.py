"""fp_select_noalloc: the selection entry point for callers that cannot
allocate device memory at call time (an engine plugin's enqueue hook, a
serving loop on a fixed memory plan, a framework whose own allocator must stay
the only one).  It takes no workspace and uses a fixed scratch array inside
libfp.so instead, so it must give exactly the lists fp_select gives.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It also passes on its own in
a fresh process (the first call then sets up the scratch address).
"""
import ctypes

import numpy as np
import pytest
import torch

from dynamic_block_sparse_fp_b200 import build, ops, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

DEV = "cuda:0"


def _same_lists(c1, i1, c2, i2):
    c1, c2 = c1.cpu().numpy(), c2.cpu().numpy()
    np.testing.assert_array_equal(c1, c2)
    i1, i2 = i1.cpu().numpy(), i2.cpu().numpy()
    bt, hq, nb = c1.shape
    for b in range(bt):
        for h in range(hq):
            for r in range(nb):
                n = c1[b, h, r]
                assert np.array_equal(i1[b, h, r, :n], i2[b, h, r, :n]), (b, h, r)


def test_noalloc_select_matches_fp_select_twice():
    build.build()
    w = synth.WORKLOADS["llama8b_n8192"]
    inp = synth.make_inputs(w)
    q, k = inp["q"].to(DEV), inp["k"].to(DEV)
    s = ops.make_shape(q, k, w.block_size)
    est = ops.estimate(q, k, w.block_size)
    # half the heads query-aware, half vertical-slash: both scratch layouts
    pat = (torch.arange(w.n_q_heads, device=DEV, dtype=torch.int32) % 2).reshape(1, -1)
    nb = w.n_blocks
    # two calls in a row per mode (the second reuses the first's scratch); the
    # query-wise rows and the block-pooled lines both stage data in the outputs
    cases = [ops.make_params(0.95, 0.1, 1024, 0), ops.make_params(0.9, 0.1, 2048, 8192),
             ops.make_params(0.95, 0.1, 1024, 0, qa_mode=ops.FP_QA_QUERYWISE),
             ops.make_params(0.9, 0.1, 2048, 8192, qa_mode=ops.FP_QA_QUERYWISE),
             ops.make_params(0.95, 0.1, 1024, 0, vs_mode=ops.FP_VS_BLOCKS),
             ops.make_params(0.9, 0.1, 2048, 8192, vs_mode=ops.FP_VS_BLOCKS)]
    for p in cases:
        ref_c, ref_i = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
        counts = torch.full((1, w.n_q_heads, nb), -7, dtype=torch.int32, device=DEV)
        indices = torch.full((1, w.n_q_heads, nb, nb), -7, dtype=torch.int32, device=DEV)
        rc = ops.fp_select_noalloc(s, p, pat, est["map"], est["vert"], est["slash"], counts,
                                   indices)
        assert rc == 0, ops.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        _same_lists(counts, indices, ref_c, ref_i)
    assert ops.fp_last_device_status() == 0


def test_noalloc_select_ragged_length():
    """A sequence whose length is not a multiple of the block size (a partial
    last block): the same lists as fp_select, two calls in a row."""
    build.build()
    w = synth.WORKLOADS["llama8b_n8192"].replace(seq_len=8192 + 64 + 5, n_q_heads=8,
                                                 n_kv_heads=2)
    inp = synth.make_inputs(w)
    q, k = inp["q"].to(DEV), inp["k"].to(DEV)
    s = ops.make_shape(q, k, w.block_size)
    est = ops.estimate(q, k, w.block_size)
    pat = (torch.arange(w.n_q_heads, device=DEV, dtype=torch.int32) % 2).reshape(1, -1)
    nb = w.n_blocks
    for p in (ops.make_params(0.95, 0.1, 1024, 0), ops.make_params(0.9, 0.1, 512, 2048)):
        ref_c, ref_i = ops.select(s, p, pat, est["map"], est["vert"], est["slash"])
        counts = torch.full((1, w.n_q_heads, nb), -7, dtype=torch.int32, device=DEV)
        indices = torch.full((1, w.n_q_heads, nb, nb), -7, dtype=torch.int32, device=DEV)
        rc = ops.fp_select_noalloc(s, p, pat, est["map"], est["vert"], est["slash"], counts,
                                   indices)
        assert rc == 0, ops.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        _same_lists(counts, indices, ref_c, ref_i)
    assert ops.fp_last_device_status() == 0


def test_noalloc_select_rejects_problems_beyond_its_scratch():
    L = ops.lib()
    # 16 x 32 heads at nb = 4096 needs ~36 MiB of scratch, above the fixed 4 MiB
    s = ops.fp_shape(16, 32, 8, 4096 * 128, 128, 128, ops.FP_BF16)
    assert ops.fp_workspace_size(s, ops.FP_CALL_SELECT) > (4 << 20)
    p = ops.make_params(0.9, 0.1, 0, 0)
    fake = 1 << 20  # never dereferenced: the size check comes first
    rc = L.fp_select_noalloc(ctypes.byref(s), ctypes.byref(p), *([fake] * 6), None)
    assert rc == ops.STATUS_CODES["FP_ERR_WORKSPACE"]
