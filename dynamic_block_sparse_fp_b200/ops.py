"""ctypes binding of ``libfp.so`` (the C ABI in ``include/fp.h``).

Two layers, both argument marshalling only (every step of the path runs in the
CUDA kernels behind the C ABI):

* ``fp_*`` functions with the C names and the C argument order; tensors are
  passed as device pointers, the stream defaults to torch's current stream.
* allocation helpers (``estimate``, ``pattern``, ``select``, ``sparse_attn``,
  ``dense_attn``, ``prefill_attn``, ``prefill_attn_varlen``) that create the
  output tensors and workspace with torch and call the ``fp_*`` function
  (``fp_prefill_attn_host`` takes caller-made page-locked host tensors and a
  ``workspace(shape, FP_CALL_PREFILL_HOST, device)``).

The library is loaded on first use; if it is missing this raises instead of
falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

FP_BF16, FP_F32 = 0, 1
FP_PATTERN_QA, FP_PATTERN_VS = 0, 1
FP_QA_FLATTENED, FP_QA_QUERYWISE = 0, 1
FP_VS_TOKENS, FP_VS_BLOCKS = 0, 1
FP_CALL_ESTIMATE, FP_CALL_SELECT, FP_CALL_SPARSE_ATTN, FP_CALL_PREFILL, FP_CALL_PREFILL_HOST = (
    0, 1, 2, 3, 4)
STATUS = {0: "FP_OK", 1: "FP_ERR_NULL", 2: "FP_ERR_SHAPE", 3: "FP_ERR_DTYPE", 4: "FP_ERR_PARAM",
          5: "FP_ERR_WORKSPACE", 6: "FP_ERR_CUDA", 7: "FP_ERR_TIMEOUT",
          8: "FP_ERR_DEVICE_CHECK", 9: "FP_ERR_UNSUPPORTED", 10: "FP_ERR_ALIGN"}
STATUS_CODES = {v: k for k, v in STATUS.items()}
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fp.h")


class fp_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("seq_len", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("block_size", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class fp_params(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_float), ("tau", ctypes.c_float),
                ("min_budget", ctypes.c_int), ("max_budget", ctypes.c_int),
                ("qa_mode", ctypes.c_int), ("vs_mode", ctypes.c_int)]


class FPError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


_P = ctypes.c_void_p
_SIG = {
    "fp_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int]),
    "fp_estimate": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                   _P]),
    "fp_pattern": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P]),
    "fp_select": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "fp_select_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "fp_sparse_attn": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "fp_dense_attn": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P]),
    "fp_prefill_attn": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                       _P]),
    "fp_prefill_attn_host": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "fp_prefill_attn_varlen": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P,
                                              _P, ctypes.c_size_t, _P]),
    "fp_last_device_status": (ctypes.c_int, [_P]),
    "fp_selftest_watchdog": (ctypes.c_int, [ctypes.c_uint, _P]),
    "fp_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_LIB = None


def lib_path() -> str:
    return os.environ.get("FP_LIBRARY", _build.LIB)


def lib() -> ctypes.CDLL:
    """The loaded library (raises RuntimeError if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with __graft_entry__.build() "
                               "(there is no fallback implementation)")
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIG.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def header_functions() -> list[str]:
    """Names of the functions declared in include/fp.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:fp_status|size_t|const char \*)\s*(fp_\w+)\s*\(",
                                 text, re.M)))


# ------------------------------------------------------------------ marshal --

def _addr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libfp must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int, where: str) -> None:
    if code != 0:
        raise FPError(code, where)


def make_shape(q, k, block_size: int) -> fp_shape:
    bt, hq, n, d = q.shape
    if q.dtype == torch.bfloat16:
        dt = FP_BF16
    elif q.dtype == torch.float32:
        dt = FP_F32
    else:
        raise TypeError(f"unsupported dtype {q.dtype}")
    if k.dtype != q.dtype:
        raise TypeError("q and k must share a dtype")
    return fp_shape(bt, hq, k.shape[1], n, d, block_size, dt)


def make_params(gamma: float, tau: float, min_budget: int = 0, max_budget: int = 0,
                qa_mode: int = 0, vs_mode: int = 0) -> fp_params:
    return fp_params(gamma, tau, min_budget, max_budget, qa_mode, vs_mode)


def fp_workspace_size(shape: fp_shape, which_call: int) -> int:
    return int(lib().fp_workspace_size(ctypes.byref(shape), which_call))


def fp_estimate(shape, q, k, qbar, kbar, map_, est_last, true_last, vert, slash, ws,
                stream=None) -> int:
    return lib().fp_estimate(ctypes.byref(shape), _addr(q), _addr(k), _addr(qbar), _addr(kbar),
                             _addr(map_), _addr(est_last), _addr(true_last), _addr(vert),
                             _addr(slash), _addr(ws), _nbytes(ws), _stream(stream))


def fp_pattern(shape, params, est_last, true_last, djs, pattern, stream=None) -> int:
    return lib().fp_pattern(ctypes.byref(shape), ctypes.byref(params), _addr(est_last),
                            _addr(true_last), _addr(djs), _addr(pattern), _stream(stream))


def fp_select(shape, params, pattern, map_, vert, slash, counts, indices, ws,
              stream=None) -> int:
    return lib().fp_select(ctypes.byref(shape), ctypes.byref(params), _addr(pattern),
                           _addr(map_), _addr(vert), _addr(slash), _addr(counts),
                           _addr(indices), _addr(ws), _nbytes(ws), _stream(stream))


def fp_select_noalloc(shape, params, pattern, map_, vert, slash, counts, indices,
                      stream=None) -> int:
    return lib().fp_select_noalloc(ctypes.byref(shape), ctypes.byref(params), _addr(pattern),
                                   _addr(map_), _addr(vert), _addr(slash), _addr(counts),
                                   _addr(indices), _stream(stream))


def fp_sparse_attn(shape, q, k, v, counts, indices, out, lse, ws, stream=None) -> int:
    return lib().fp_sparse_attn(ctypes.byref(shape), _addr(q), _addr(k), _addr(v),
                                _addr(counts), _addr(indices), _addr(out), _addr(lse),
                                _addr(ws), _nbytes(ws), _stream(stream))


def fp_dense_attn(shape, q, k, v, out, lse, stream=None) -> int:
    return lib().fp_dense_attn(ctypes.byref(shape), _addr(q), _addr(k), _addr(v), _addr(out),
                               _addr(lse), _stream(stream))


def fp_prefill_attn(shape, params, q, k, v, out, lse, stats, ws, stream=None) -> int:
    return lib().fp_prefill_attn(ctypes.byref(shape), ctypes.byref(params), _addr(q), _addr(k),
                                 _addr(v), _addr(out), _addr(lse), _addr(stats), _addr(ws),
                                 _nbytes(ws), _stream(stream))


def fp_prefill_attn_host(shape, params, q_host, k_host, v_host, out_host, ws,
                         stream=None) -> int:
    return lib().fp_prefill_attn_host(ctypes.byref(shape), ctypes.byref(params), _addr(q_host),
                                      _addr(k_host), _addr(v_host), _addr(out_host), _addr(ws),
                                      _nbytes(ws), _stream(stream))


def fp_prefill_attn_varlen(shape, params, seq_lens, q, k, v, out, lse, stats, ws,
                           stream=None) -> int:
    """seq_lens: a sequence of Python ints (copied to a host int32 array here)."""
    n = len(seq_lens)
    lens = (ctypes.c_int32 * max(n, 1))(*seq_lens)
    return lib().fp_prefill_attn_varlen(ctypes.byref(shape), ctypes.byref(params), n,
                                        ctypes.cast(lens, ctypes.c_void_p), _addr(q), _addr(k),
                                        _addr(v), _addr(out), _addr(lse), _addr(stats),
                                        _addr(ws), _nbytes(ws), _stream(stream))


def fp_selftest_watchdog(limit_us: int, stream=None) -> int:
    return lib().fp_selftest_watchdog(limit_us, _stream(stream))


def fp_last_device_status(stream=None) -> int:
    return lib().fp_last_device_status(_stream(stream))


def fp_status_string(code: int) -> str:
    return lib().fp_status_string(code).decode()


def _nbytes(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return 0
    return t.numel() * t.element_size()


# ------------------------------------------------------- allocation helpers --

def workspace(shape: fp_shape, which_call: int, device) -> torch.Tensor | None:
    """A device byte buffer of fp_workspace_size(shape, which_call), or None if 0."""
    n = fp_workspace_size(shape, which_call)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def estimate(q, k, block_size: int, stream=None) -> dict:
    """fp_estimate: dict of qbar, kbar, map (packed causal), est_last, true_last,
    vert, slash (fp32 device tensors)."""
    s = make_shape(q, k, block_size)
    dev = q.device
    bt, hq, n, d = q.shape
    hkv, nb = k.shape[1], -(-n // block_size)  # a partial last block counts
    f = dict(dtype=torch.float32, device=dev)
    r = {"qbar": torch.empty(bt, hq, nb, d, **f), "kbar": torch.empty(bt, hkv, nb, d, **f),
         "map": torch.empty(bt, hq, nb * (nb + 1) // 2, **f),
         "est_last": torch.empty(bt, hq, nb, **f), "true_last": torch.empty(bt, hq, nb, **f),
         "vert": torch.empty(bt, hq, n, **f), "slash": torch.empty(bt, hq, n, **f)}
    ws = workspace(s, FP_CALL_ESTIMATE, dev)
    _check(fp_estimate(s, q, k, r["qbar"], r["kbar"], r["map"], r["est_last"], r["true_last"],
                       r["vert"], r["slash"], ws, stream), "fp_estimate")
    return r


def pattern(shape: fp_shape, params: fp_params, est_last, true_last, stream=None):
    """fp_pattern: (d_JS fp32 [Bt, Hq], pattern int32 [Bt, Hq])."""
    bt, hq = est_last.shape[:2]
    djs = torch.empty(bt, hq, dtype=torch.float32, device=est_last.device)
    pat = torch.empty(bt, hq, dtype=torch.int32, device=est_last.device)
    _check(fp_pattern(shape, params, est_last, true_last, djs, pat, stream), "fp_pattern")
    return djs, pat


def select(shape: fp_shape, params: fp_params, pat, map_, vert, slash, stream=None):
    """fp_select: (counts int32 [Bt, Hq, nb], indices int32 [Bt, Hq, nb, nb]),
    each row's list ascending in its first counts entries."""
    bt, hq, nb = shape.batch, shape.n_q_heads, -(-shape.seq_len // shape.block_size)
    dev = map_.device
    counts = torch.empty(bt, hq, nb, dtype=torch.int32, device=dev)
    indices = torch.empty(bt, hq, nb, nb, dtype=torch.int32, device=dev)
    ws = workspace(shape, FP_CALL_SELECT, dev)
    _check(fp_select(shape, params, pat, map_, vert, slash, counts, indices, ws, stream),
           "fp_select")
    return counts, indices


def sparse_attn(q, k, v, counts, indices, block_size: int, with_lse: bool = True,
                stream=None):
    """fp_sparse_attn: (out like q, lse fp32 [Bt, Hq, N] or None)."""
    s = make_shape(q, k, block_size)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if with_lse else None
    ws = workspace(s, FP_CALL_SPARSE_ATTN, q.device)
    _check(fp_sparse_attn(s, q, k, v, counts, indices, out, lse, ws, stream), "fp_sparse_attn")
    return out, lse


def dense_attn(q, k, v, block_size: int, with_lse: bool = True, stream=None):
    """fp_dense_attn: causal attention over every block; (out, lse or None)."""
    s = make_shape(q, k, block_size)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if with_lse else None
    _check(fp_dense_attn(s, q, k, v, out, lse, stream), "fp_dense_attn")
    return out, lse


def prefill_attn_varlen(seqs_q, seqs_k, seqs_v, block_size: int, params: fp_params,
                        stream=None):
    """The whole path over sequences of different lengths in one call.

    seqs_*: lists of [1, H, N_s, d] tensors (one per sequence).  They are packed
    back to back for the call and the outputs are returned as a list of
    [1, Hq, N_s, d] views of one packed buffer, with per-sequence stats
    [n_seqs, 2].
    """
    lens = [int(x.shape[2]) for x in seqs_q]
    q = torch.cat([x.reshape(-1) for x in seqs_q])
    k = torch.cat([x.reshape(-1) for x in seqs_k])
    v = torch.cat([x.reshape(-1) for x in seqs_v])
    hq, d = seqs_q[0].shape[1], seqs_q[0].shape[3]
    hkv = seqs_k[0].shape[1]
    s = fp_shape(1, hq, hkv, max(lens), d, block_size,
                 FP_BF16 if seqs_q[0].dtype == torch.bfloat16 else FP_F32)
    out = torch.empty_like(q)
    stats = torch.empty(len(lens), 2, dtype=torch.int64, device=q.device)
    ws = workspace(s, FP_CALL_PREFILL, q.device)
    _check(fp_prefill_attn_varlen(s, params, lens, q, k, v, out, None, stats, ws, stream),
           "fp_prefill_attn_varlen")
    outs, off = [], 0
    for n in lens:
        outs.append(out[off: off + hq * n * d].view(1, hq, n, d))
        off += hq * n * d
    return outs, stats


def prefill_attn(q, k, v, block_size: int, params: fp_params, with_lse: bool = False,
                 ws=None, stream=None):
    """fp_prefill_attn, the whole path on device tensors: (out, lse or None,
    stats int64 [kept blocks, query-aware heads])."""
    s = make_shape(q, k, block_size)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if with_lse else None
    stats = torch.empty(2, dtype=torch.int64, device=q.device)
    if ws is None:
        ws = workspace(s, FP_CALL_PREFILL, q.device)
    _check(fp_prefill_attn(s, params, q, k, v, out, lse, stats, ws, stream), "fp_prefill_attn")
    return out, lse, stats
