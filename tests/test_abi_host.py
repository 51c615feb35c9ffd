"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/fp.h declares, and rejects bad arguments with the
documented status before touching the device."""
import ctypes
import os

import pytest

from dynamic_block_sparse_fp_b200 import build, ops

FAKE = 1 << 20  # a non-null "device pointer" (never dereferenced: validation fails first)


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def shape(**kw):
    base = dict(batch=1, n_q_heads=4, n_kv_heads=2, seq_len=1024, head_dim=128, block_size=128,
                dtype=ops.FP_BF16)
    base.update(kw)
    return ops.fp_shape(**base)


def test_exports_every_declared_function(L):
    names = ops.header_functions()
    assert len(names) == 13, names
    for n in names:
        assert hasattr(L, n), n
    # nothing but the fp_* API is exported (static CUDA runtime stays hidden)
    out = os.popen(f"nm -D --defined-only {ops.lib_path()}").read().split()
    exported = [s for s in out if not all(c in "0123456789abcdef" for c in s) and len(s) > 1]
    exported = [s for s in exported if s not in ("T", "B", "D", "R", "W", "A")]
    assert sorted(exported) == names


def test_status_strings(L):
    for code, name in ops.STATUS.items():
        assert ops.fp_status_string(code).startswith(name)
    assert ops.fp_status_string(99) == "unknown fp_status"


def test_workspace_sizes(L):
    s = shape()
    assert ops.fp_workspace_size(s, ops.FP_CALL_ESTIMATE) > 0
    assert ops.fp_workspace_size(s, ops.FP_CALL_SELECT) > 0
    assert ops.fp_workspace_size(s, ops.FP_CALL_SPARSE_ATTN) == 0
    pre = ops.fp_workspace_size(s, ops.FP_CALL_PREFILL)
    host = ops.fp_workspace_size(s, ops.FP_CALL_PREFILL_HOST)
    io = (2 * 4 + 2 * 2) * 1024 * 128 * 2  # q, out (4 heads) + k, v (2 heads), bf16
    assert host > io and pre > 0
    assert ops.fp_workspace_size(shape(seq_len=0), ops.FP_CALL_PREFILL) == 0
    assert ops.fp_workspace_size(s, 17) == 0
    # larger problems need more
    assert ops.fp_workspace_size(shape(seq_len=4096), ops.FP_CALL_ESTIMATE) > \
        ops.fp_workspace_size(s, ops.FP_CALL_ESTIMATE)


@pytest.mark.parametrize("bad,code", [
    (dict(seq_len=0), 2), (dict(block_size=32), 2), (dict(head_dim=96), 2),
    (dict(n_q_heads=3), 2), (dict(n_kv_heads=0), 2), (dict(dtype=7), 3),
    (dict(seq_len=128 * 4097), 2),
])
def test_bad_shapes_rejected(L, bad, code):
    s = shape(**bad)
    ws = FAKE
    assert L.fp_estimate(ctypes.byref(s), *([FAKE] * 9), ws, 1 << 40, None) == code
    assert L.fp_dense_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, None) == code


def test_null_pointers_rejected(L):
    s = shape()
    p = ops.make_params(0.95, 0.1, 1024, 0)
    assert L.fp_estimate(None, *([FAKE] * 9), FAKE, 1 << 40, None) == 1
    assert L.fp_estimate(ctypes.byref(s), FAKE, None, *([FAKE] * 7), FAKE, 1 << 40, None) == 1
    assert L.fp_pattern(ctypes.byref(s), None, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert L.fp_pattern(ctypes.byref(s), ctypes.byref(p), FAKE, None, FAKE, FAKE, None) == 1
    assert L.fp_select(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None,
                       FAKE, 1 << 40, None) == 1
    assert L.fp_sparse_attn(ctypes.byref(s), FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None, 0,
                            None) == 1
    assert L.fp_dense_attn(ctypes.byref(s), FAKE, FAKE, None, FAKE, None, None) == 1
    assert L.fp_prefill_attn(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, FAKE, None, None,
                             None, FAKE, 1 << 40, None) == 1
    assert L.fp_prefill_attn_host(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, None, FAKE,
                                  FAKE, 1 << 40, None) == 1


@pytest.mark.parametrize("gamma,tau,lo,code", [
    (0.0, 0.1, 0, 4), (1.5, 0.1, 0, 4), (float("nan"), 0.1, 0, 4), (0.9, -0.1, 0, 4),
    (0.9, float("inf"), 0, 4), (0.9, 0.1, -5, 4),
])
def test_bad_params_rejected(L, gamma, tau, lo, code):
    s = shape()
    p = ops.make_params(gamma, tau, lo, 0)
    assert L.fp_pattern(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None) == code
    assert L.fp_select(ctypes.byref(s), ctypes.byref(p), *([FAKE] * 6), FAKE, 1 << 40,
                       None) == code


@pytest.mark.parametrize("qa_mode", [-1, 2, 7])
def test_bad_qa_mode_rejected(L, qa_mode):
    s = shape()
    p = ops.make_params(0.9, 0.1, 0, 0, qa_mode)
    assert L.fp_select(ctypes.byref(s), ctypes.byref(p), *([FAKE] * 6), FAKE, 1 << 40,
                       None) == ops.STATUS_CODES["FP_ERR_PARAM"]
    assert L.fp_pattern(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, FAKE, FAKE,
                        None) == ops.STATUS_CODES["FP_ERR_PARAM"]


@pytest.mark.parametrize("vs_mode", [-1, 2])
def test_bad_vs_mode_rejected(L, vs_mode):
    s = shape()
    p = ops.make_params(0.9, 0.1, 0, 0, 0, vs_mode)
    assert L.fp_select(ctypes.byref(s), ctypes.byref(p), *([FAKE] * 6), FAKE, 1 << 40,
                       None) == ops.STATUS_CODES["FP_ERR_PARAM"]


@pytest.mark.parametrize("lens,batch,code", [
    ([1024, 0], 1, "FP_ERR_SHAPE"),      # empty sequence
    ([1024, -3], 1, "FP_ERR_SHAPE"),     # negative length
    ([2048], 1, "FP_ERR_SHAPE"),         # longer than shape.seq_len (1024)
    ([], 1, "FP_ERR_SHAPE"),             # no sequence
    ([1024], 2, "FP_ERR_SHAPE"),         # the shape's batch must be 1
])
def test_varlen_bad_lengths_rejected(L, lens, batch, code):
    s = shape(batch=batch)
    p = ops.make_params(0.9, 0.1, 0, 0)
    assert ops.fp_prefill_attn_varlen(s, p, lens, FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                                      None) == ops.STATUS_CODES[code]


def test_varlen_nulls_and_workspace(L):
    s = shape()
    p = ops.make_params(0.9, 0.1, 0, 0)
    P = ctypes.c_void_p
    assert L.fp_prefill_attn_varlen(ctypes.byref(s), ctypes.byref(p), 1, None, P(FAKE), P(FAKE),
                                    P(FAKE), P(FAKE), None, None, P(FAKE), 1 << 40,
                                    None) == ops.STATUS_CODES["FP_ERR_NULL"]
    lens = (ctypes.c_int32 * 1)(1024)
    assert L.fp_prefill_attn_varlen(ctypes.byref(s), ctypes.byref(p), 1, lens, P(FAKE), P(FAKE),
                                    P(FAKE), P(FAKE), None, None, P(FAKE), 16,
                                    None) == ops.STATUS_CODES["FP_ERR_WORKSPACE"]


def test_workspace_checks(L):
    s = shape()
    need = ops.fp_workspace_size(s, ops.FP_CALL_ESTIMATE)
    args = [FAKE] * 9
    assert L.fp_estimate(ctypes.byref(s), *args, None, need, None) == 5
    assert L.fp_estimate(ctypes.byref(s), *args, FAKE, need - 1, None) == 5
    assert L.fp_estimate(ctypes.byref(s), *args, FAKE + 8, need, None) == 5  # misaligned
    p = ops.make_params(0.9, 0.1, 0, 0)
    need = ops.fp_workspace_size(s, ops.FP_CALL_PREFILL)
    assert L.fp_prefill_attn(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None,
                             None, FAKE, need - 256, None) == 5


def test_misaligned_pointers_rejected(L):
    """q, k, v, out, qbar and kbar need 16-byte alignment, the other arrays
    their element size: a misaligned pointer returns FP_ERR_ALIGN before any
    device call; an aligned set gets past the check (to the device check,
    which fails without a GPU, or to the workspace check)."""
    ALIGN = ops.STATUS_CODES["FP_ERR_ALIGN"]
    s = shape()
    p = ops.make_params(0.9, 0.1, 0, 0)
    P = ctypes.c_void_p
    est = [FAKE] * 9
    for i, off in [(0, 8), (1, 2), (2, 4), (3, 12), (4, 2), (5, 1), (6, 2), (7, 3), (8, 2)]:
        args = list(est)
        args[i] = FAKE + off
        assert L.fp_estimate(ctypes.byref(s), *args, FAKE, 1 << 40, None) == ALIGN, (i, off)
    # 4-byte aligned fp32 arrays (map, est_last, ..., slash) pass the check
    args = est[:4] + [FAKE + 4] * 5
    assert L.fp_estimate(ctypes.byref(s), *args, FAKE, 1 << 40, None) != ALIGN
    assert L.fp_pattern(ctypes.byref(s), ctypes.byref(p), FAKE + 2, FAKE, FAKE, FAKE,
                        None) == ALIGN
    assert L.fp_select(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE + 2, FAKE, FAKE, FAKE, FAKE,
                       FAKE, 1 << 40, None) == ALIGN
    assert L.fp_select_noalloc(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE,
                               FAKE + 1, None) == ALIGN
    for qkvo in range(4):
        a = [FAKE] * 4
        a[qkvo] += 8
        assert L.fp_sparse_attn(ctypes.byref(s), a[0], a[1], a[2], FAKE, FAKE, a[3], None, None,
                                0, None) == ALIGN
        assert L.fp_dense_attn(ctypes.byref(s), *a, None, None) == ALIGN
        assert L.fp_prefill_attn(ctypes.byref(s), ctypes.byref(p), *a, None, None, FAKE,
                                 1 << 40, None) == ALIGN
    assert L.fp_sparse_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE + 2, FAKE, FAKE, None, None,
                            0, None) == ALIGN
    assert L.fp_dense_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, P(FAKE + 2), None) == ALIGN
    assert L.fp_prefill_attn(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None,
                             P(FAKE + 4), FAKE, 1 << 40, None) == ALIGN
    lens = (ctypes.c_int32 * 1)(1024)
    assert L.fp_prefill_attn_varlen(ctypes.byref(s), ctypes.byref(p), 1, lens, P(FAKE + 8),
                                    P(FAKE), P(FAKE), P(FAKE), None, None, P(FAKE), 1 << 40,
                                    None) == ALIGN
    # aligned: past the alignment check
    assert L.fp_prefill_attn(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, FAKE, FAKE,
                             P(FAKE + 4), P(FAKE + 8), FAKE, 16, None) == \
        ops.STATUS_CODES["FP_ERR_WORKSPACE"]


def test_bf16_attention_shape_limits(L):
    # the tensor-core path takes d == 128 (B 64 or 128); fp32 takes all four
    for bs, d in [(128, 64), (64, 64)]:
        s = shape(block_size=bs, head_dim=d)
        assert L.fp_dense_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, None) == 2


def test_watchdog_selftest_rejects_bad_limits(L):
    assert L.fp_selftest_watchdog(0, None) == 4
    assert L.fp_selftest_watchdog(2000000, None) == 4


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(ops, "_LIB", None)
    monkeypatch.setenv("FP_LIBRARY", "/nonexistent/libfp.so")
    with pytest.raises(RuntimeError, match="no fallback"):
        ops.lib()


@pytest.mark.parametrize("n,bs", [(1000, 128), (1105, 64), (1, 64), (8256, 128)])
def test_ragged_lengths_accepted(L, n, bs):
    """N need not be a multiple of the block size: nb = ceil(N / B), the last
    block partial.  Validation passes (a NULL pointer is what fails here) and
    the workspaces are sized for nb blocks."""
    s = shape(seq_len=n, block_size=bs)
    assert L.fp_estimate(ctypes.byref(s), FAKE, None, *([FAKE] * 7), FAKE, 1 << 40,
                         None) == ops.STATUS_CODES["FP_ERR_NULL"]
    for call in (ops.FP_CALL_ESTIMATE, ops.FP_CALL_SELECT, ops.FP_CALL_PREFILL):
        assert ops.fp_workspace_size(s, call) > 0
    whole = shape(seq_len=-(-n // bs) * bs, block_size=bs)
    assert ops.fp_workspace_size(s, ops.FP_CALL_SELECT) == ops.fp_workspace_size(
        whole, ops.FP_CALL_SELECT)
