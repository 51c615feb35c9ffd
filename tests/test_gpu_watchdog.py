"""Failure detection on the GPU without a fault: a bounded wait that nothing
ever satisfies gives up, records FP_ERR_TIMEOUT in the device status word,
and the device keeps working afterwards."""
import time

import pytest
import torch

from dynamic_block_sparse_fp_b200 import build, ops, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def test_bounded_wait_reports_timeout_and_device_recovers():
    build.build()
    assert ops.fp_last_device_status() == 0
    t0 = time.perf_counter()
    assert ops.fp_selftest_watchdog(20000) == 0  # 20 ms limit
    assert ops.fp_last_device_status() == ops.STATUS_CODES["FP_ERR_TIMEOUT"]
    elapsed = time.perf_counter() - t0
    assert 0.015 < elapsed < 5.0
    assert ops.fp_last_device_status() == 0  # reading clears it
    # the context is still usable: a small dense attention runs and is sane
    w = synth.WORKLOADS["llama8b_n8192"].replace(seq_len=256, n_q_heads=2, n_kv_heads=1)
    inp = synth.make_inputs(w)
    q, k, v = (inp[x].cuda() for x in ("q", "k", "v"))
    out, lse = ops.dense_attn(q, k, v, w.block_size)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    assert ops.fp_last_device_status() == 0
