"""Benchmark of the FlexPrefill prefill-attention hot path on B200.

One step = one pass of the whole path over one attention layer (all heads)
in one fp_prefill_attn call (estimate -> pattern -> select -> sparse
attention, each head's estimate limited to what its pattern reads), on seeded
synthetic Q/K/V shaped like a Llama-3.1-8B layer at 128k tokens (32 q / 8 kv
heads, d = 128, block 128).  The same layer then runs as the four staged calls
(fp_estimate, fp_pattern, fp_select, fp_sparse_attn) for the per-stage times
and the attention roofline.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (the plain fp64 restatement of the
method) on a bounded sample of the same workload.  Multi-GPU runs (torchrun)
split the layer's kv heads over the ranks (every stage is per head, so the
path itself has no exchange) and all-gather the outputs inside the step
(strong scaling); --shard layers gives every rank its own layer instead
(independent problems, weak scaling).  --sweep prints one line per point of
the gamma x tau x min x max budget sweep instead of the headline line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from dynamic_block_sparse_fp_b200 import synth  # noqa: E402

METRIC = "prefill-attn tokens/s and effective TFLOPS (% bf16 peak) at 128k; speedup vs dense"
# the library's kernels per step of fp_prefill_attn: estimate 11 (6 for the
# pattern's inputs, 3 for the query-aware heads' map, 2 for the vertical-slash
# heads' lines), pattern 1, select 6, attention 1
LAUNCHES_PER_STEP = 19


def kernel_traffic(source: str, workload: str):
    """DRAM bytes per launch of a kernel from a committed ncu capture.

    profiles/<name>_traffic.json holds {"source_sha256", "workload",
    "bytes_per_launch", ...}; the figure is used only while the kernel source
    and the device header it includes (csrc/fp_internal.cuh) still hash to the
    captured ones (else None: the counters are stale).
    """
    name = os.path.splitext(os.path.basename(source))[0]
    rec_path = os.path.join(ROOT, "profiles", f"{name}_traffic.json")
    if not os.path.exists(rec_path):
        return None
    sha = kernel_source_sha(source)
    if sha is None:
        return None
    rec = json.load(open(rec_path))
    if rec.get("source_sha256") != sha or rec.get("workload") != workload:
        return None
    return rec.get("bytes_per_launch")


def kernel_source_sha(source: str):
    """sha256 over csrc/<source> followed by csrc/fp_internal.cuh."""
    import hashlib
    csrc = os.path.join(ROOT, "dynamic_block_sparse_fp_b200", "csrc")
    h = hashlib.sha256()
    for f in (source, "fp_internal.cuh"):
        p = os.path.join(csrc, f)
        if not os.path.exists(p):
            return None
        h.update(open(p, "rb").read())
    return h.hexdigest()


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle samples over the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        busy = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl" if torch.cuda.is_available() else "gloo",
            timeout=datetime.timedelta(seconds=600))
    return ws, rank, local


def rank_workload(w: synth.Workload, rank: int) -> synth.Workload:
    """The independent layer rank `rank` runs (its own seed; rank 0 = w)."""
    return w.replace(seed=w.seed + 1000 * rank) if rank else w


def job_value(tokens_per_rank: int, ws: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return ws * tokens_per_rank / (ms_per_step * 1e-3)


def max_over_ranks(x: float, ws: int, device) -> float:
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------ CPU baseline --

def cpu_oracle_sample(w: synth.Workload, heads=(0,), budget_s: float = 10.0,
                      inputs=None) -> dict:
    """Time the oracle on a bounded sample and extrapolate to the full layer.

    Sample: the estimate, pattern and select of ``heads`` (every q head costs
    the same there), then attention of those heads' query blocks, taken in a
    fixed spread-out order, 4 blocks at a time, until ``budget_s`` seconds of
    oracle work have passed.  Attention time is scaled by the kept blocks of
    the whole layer.  ``inputs`` may carry the sampled heads' tensors from an
    earlier call.
    """
    import numpy as np

    import oracle
    g = w.n_q_heads // w.n_kv_heads
    kvs = sorted({h // g for h in heads})
    if inputs is None:
        inp = synth.make_inputs(w, kv_heads=kvs)
        loc = [kvs.index(h // g) * g + h % g for h in heads]
        inputs = (inp["q"][:, loc], inp["k"][:, [kvs.index(h // g) for h in heads]],
                  inp["v"][:, [kvs.index(h // g) for h in heads]])
    # each sampled head gets its own kv head copy (GQA index h // 1)
    q, kk, vv = inputs
    t0 = time.perf_counter()
    est = oracle.estimate(q, kk, w.block_size)
    t1 = time.perf_counter()
    e32 = {x: est[x].astype(np.float32) for x in ("map", "est_last", "true_last", "vert",
                                                    "slash")}
    _, pat = oracle.pattern(e32["est_last"], e32["true_last"], w.tau)
    counts, indices = oracle.select(pat, e32["map"], e32["vert"], e32["slash"], w.n_blocks,
                                    w.block_size, w.gamma, w.min_budget, w.max_budget,
                                    w.qa_mode, w.vs_mode)
    t2 = time.perf_counter()
    nb = w.n_blocks
    order = [int(x) for x in np.random.default_rng(0).permutation(nb)]
    qbs = []
    while order and (not qbs or time.perf_counter() - t0 < budget_s):
        chunk, order = order[:4], order[4:]
        oracle.sparse_attention(q, kk, vv, counts, indices, w.block_size,
                                heads=list(range(len(heads))), q_blocks=chunk)
        qbs += chunk
    t3 = time.perf_counter()
    kept_sample = int(sum(counts[0, i, qb] for i in range(len(heads)) for qb in qbs))
    kept_heads = int(counts.sum())
    nh = len(heads)
    t_est = (t1 - t0) / nh * w.n_q_heads
    t_sel = (t2 - t1) / nh * w.n_q_heads
    # attention time per kept block, times the kept blocks of every head
    # (sampled heads' mean stands in for the others)
    t_att = (t3 - t2) / max(kept_sample, 1) * (kept_heads / nh) * w.n_q_heads
    total = t_est + t_sel + t_att
    return {"seconds_measured": t3 - t0, "seconds_extrapolated": total,
            "tokens_per_s": w.seq_len * w.batch / total, "inputs": inputs,
            "sample": (f"oracle (numpy fp64) on q heads {list(heads)} of {w.name}: estimate, "
                       f"pattern and select in full, then attention on {len(qbs)} query "
                       f"blocks in a fixed spread order ({kept_sample} kept blocks) until "
                       f"{budget_s:g} s of oracle work; extrapolated to {w.n_q_heads} heads "
                       f"and all kept blocks")}


def cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def workload_config(w: synth.Workload, ws: int, heads: bool = False) -> dict:
    if ws == 1:
        par = "single GPU"
    elif heads:
        par = f"kv heads split over {ws} ranks, outputs all-gathered (NCCL)"
    else:
        par = f"independent layers x{ws}"
    return {"workload": w.name, "batch_per_gpu": w.batch,
            "global_batch": w.batch if heads else w.batch * ws,
            "seq_len": w.seq_len, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "block_size": w.block_size, "gamma": w.gamma, "tau": w.tau,
            "min_budget": w.min_budget, "max_budget": w.max_budget,
            "qa_selection": "query-wise" if w.qa_mode == 1 else "flattened",
            "vs_lines": "blocks" if w.vs_mode == 1 else "tokens",
            "parallelism": par,
            "l2": "no flush: every step streams Q (1.07 GB at 128k) and K/V, inputs larger "
                  "than the 126 MB L2"}


def run_reference(args, w, ws, rank):
    if rank != 0:
        return
    steps = []
    inputs = None
    for i in range(args.warmup + args.steps):
        # per step a bounded sample (the whole K + W run stays within minutes)
        r = cpu_oracle_sample(w, budget_s=args.reference_step_s, inputs=inputs)
        inputs = r["inputs"]
        if i >= args.warmup:
            steps.append(r)
    tps = statistics.mean(r["tokens_per_s"] for r in steps)
    line = {"impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * w.seq_len * w.batch / tps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, 1),
            "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores(),
                             "kind": "oracle", "sample": steps[0]["sample"]},
            "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- ours --

# the config-3 sweep at 128k: gamma x tau x min budget x max budget (0 = uncapped)
SWEEP = [(g, t, lo, hi) for g in (0.9, 0.95) for t in (0.0, 0.1, 0.3) for lo in (1024, 2048)
         for hi in (0, 8192)]


class Layer:
    """Device buffers of one layer and the four-call step over them."""

    def __init__(self, ops, q, k, v, bs, dev):
        self.ops = ops
        self.q, self.k, self.v = q, k, v
        bt, hq, n, d = q.shape
        hkv = k.shape[1]
        nb = -(-n // bs)
        self.bs, self.nb = bs, nb
        self.s = ops.make_shape(q, k, bs)
        f32 = dict(dtype=torch.float32, device=dev)
        self.qbar = torch.empty(bt, hq, nb, d, **f32)
        self.kbar = torch.empty(bt, hkv, nb, d, **f32)
        self.amap = torch.empty(bt, hq, nb * (nb + 1) // 2, **f32)
        self.est_last = torch.empty(bt, hq, nb, **f32)
        self.true_last = torch.empty(bt, hq, nb, **f32)
        self.vert = torch.empty(bt, hq, n, **f32)
        self.slash = torch.empty(bt, hq, n, **f32)
        self.djs = torch.empty(bt, hq, **f32)
        self.pat = torch.empty(bt, hq, dtype=torch.int32, device=dev)
        self.counts = torch.empty(bt, hq, nb, dtype=torch.int32, device=dev)
        self.indices = torch.empty(bt, hq, nb, nb, dtype=torch.int32, device=dev)
        self.out = torch.empty_like(q)
        self.ws_est = ops.workspace(self.s, ops.FP_CALL_ESTIMATE, dev)
        self.ws_sel = ops.workspace(self.s, ops.FP_CALL_SELECT, dev)

    def step(self, p, e, stream, gather=None):
        ops = self.ops
        e[0].record(stream)
        ops._check(ops.fp_estimate(self.s, self.q, self.k, self.qbar, self.kbar, self.amap,
                                   self.est_last, self.true_last, self.vert, self.slash,
                                   self.ws_est, stream), "fp_estimate")
        e[1].record(stream)
        ops._check(ops.fp_pattern(self.s, p, self.est_last, self.true_last, self.djs, self.pat,
                                  stream), "fp_pattern")
        e[2].record(stream)
        ops._check(ops.fp_select(self.s, p, self.pat, self.amap, self.vert, self.slash,
                                 self.counts, self.indices, self.ws_sel, stream), "fp_select")
        e[3].record(stream)
        ops._check(ops.fp_sparse_attn(self.s, self.q, self.k, self.v, self.counts, self.indices,
                                      self.out, None, None, stream), "fp_sparse_attn")
        e[4].record(stream)
        if gather is not None:
            gather(self.out)

    def estimate_bytes(self) -> int:
        """fp_estimate's algorithmic bytes: read Q and K once, write every output."""
        return (self.q.numel() + self.k.numel()) * self.q.element_size() + 4 * sum(
            x.numel() for x in (self.qbar, self.kbar, self.amap, self.est_last,
                                self.true_last, self.vert, self.slash))

    def select_bytes(self, qa_heads: int, kept: int) -> int:
        """fp_select's algorithmic bytes: each query-aware head reads its map once,
        each vertical-slash head its two line lists; every kept block and every
        row count is written once."""
        bt, hq, n, _ = self.q.shape
        t_pairs = self.nb * (self.nb + 1) // 2
        return 4 * (qa_heads * t_pairs + (bt * hq - qa_heads) * 2 * n + kept + bt * hq * self.nb)


def measure(layer, p, args, stream, ws, local, gather=None) -> dict:
    """W untimed steps, then K timed steps bracketed by barrier + synchronize."""
    from dynamic_block_sparse_fp_b200 import ops
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)]
          for _ in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        layer.step(p, ev[i], stream, gather)
    torch.cuda.synchronize()
    assert ops.fp_last_device_status(stream) == 0
    barrier(ws)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.warmup, args.warmup + args.steps):
            layer.step(p, ev[i], stream, gather)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    status = ops.fp_last_device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {ops.STATUS.get(status, status)}")
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), ws, layer.q.device)
    timed = ev[args.warmup:]
    stage_ms = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in timed) for j in range(4)]
    return {"ms_step": total_ms / args.steps, "stage_ms": stage_ms,
            "kept": int(layer.counts.sum()),
            "qa_heads": int((layer.pat == ops.FP_PATTERN_QA).sum()),
            "clocks": clk.summary()}


def measure_prefill(layer, p, args, stream, ws, local, gather=None) -> dict:
    """The whole path in one fp_prefill_attn call per step: W untimed steps,
    then K timed steps bracketed by barrier + synchronize."""
    from dynamic_block_sparse_fp_b200 import ops
    wsp = ops.workspace(layer.s, ops.FP_CALL_PREFILL, layer.q.device)
    stats = torch.zeros(2, dtype=torch.int64, device=layer.q.device)

    def step(st=None):
        ops._check(ops.fp_prefill_attn(layer.s, p, layer.q, layer.k, layer.v, layer.out, None,
                                       st, wsp, stream), "fp_prefill_attn")
        if gather is not None:
            gather(layer.out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ops.fp_last_device_status(stream) == 0
    barrier(ws)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for _ in range(args.steps):
            step()
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    status = ops.fp_last_device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {ops.STATUS.get(status, status)}")
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), ws, layer.q.device)
    step(stats)  # (untimed) the kept blocks and query-aware heads of this layer
    torch.cuda.synchronize()
    del wsp
    return {"ms_step": total_ms / args.steps, "kept": int(stats[0]), "qa_heads": int(stats[1]),
            "clocks": clk.summary()}


def dense_ms(layer, stream, reps: int = 2) -> float:
    """fp_dense_attn (the same kernel over every causal block), CUDA events."""
    from dynamic_block_sparse_fp_b200 import ops
    dout = torch.empty_like(layer.q)
    de = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ops._check(ops.fp_dense_attn(layer.s, layer.q, layer.k, layer.v, dout, None, stream),
               "fp_dense_attn")
    de[0].record(stream)
    for _ in range(reps):
        ops._check(ops.fp_dense_attn(layer.s, layer.q, layer.k, layer.v, dout, None, stream),
                   "fp_dense_attn")
    de[1].record(stream)
    torch.cuda.synchronize()
    return de[0].elapsed_time(de[1]) / reps


def path_fields(layer, m: dict, peaks: dict, dense: float | None, whole: dict) -> dict:
    """Kept fraction, per-stage times and rooflines of one measured configuration:
    `whole` is the timed fp_prefill_attn loop, `m` the staged calls' loop."""
    bt, hq, n, d = layer.q.shape
    bs, nb = layer.bs, layer.nb
    st = m["stage_ms"]
    assert whole["kept"] == m["kept"] and whole["qa_heads"] == m["qa_heads"]
    t_pairs = nb * (nb + 1) // 2
    flop_block = 4.0 * bs * bs * d
    attn_flops = flop_block * m["kept"]
    attn_tflops = attn_flops / (st[3] * 1e-3) / 1e12
    peak_t = peaks["bf16_tflops_sustained"]
    eb = layer.estimate_bytes()
    sb = layer.select_bytes(m["qa_heads"], m["kept"])
    hbm = peaks["hbm_gbs"]
    f = {
        "roofline": {"bound": "tensor", "kernel": "fp_sparse_attn", "achieved": attn_tflops,
                     "peak": peak_t, "unit": "TFLOP/s", "frac": attn_tflops / peak_t,
                     "peak_kind": f"bf16 dense, sustained ({peaks['source']})",
                     "algorithmic_flops_per_launch": attn_flops},
        # the four staged calls (fp_estimate computes every output for every
        # head; the whole-path call skips what each head's pattern does not read)
        "stages_ms": {"estimate": st[0], "pattern": st[1], "select": st[2],
                      "sparse_attn": st[3], "staged_step": m["ms_step"]},
        "estimate_hbm": {"bytes": eb, "gbs": eb / (st[0] * 1e-3) / 1e9,
                         "frac": eb / (st[0] * 1e-3) / 1e9 / hbm},
        "select_hbm": {"bytes": sb, "gbs": sb / (st[2] * 1e-3) / 1e9,
                       "frac": sb / (st[2] * 1e-3) / 1e9 / hbm},
        "effective_tflops": {"sparse_attn": attn_tflops,
                             "whole_step": attn_flops / (whole["ms_step"] * 1e-3) / 1e12},
        "kept_blocks": m["kept"], "causal_blocks": t_pairs * hq * bt,
        "kept_fraction": m["kept"] / (t_pairs * hq * bt), "qa_heads": m["qa_heads"],
        "sparsity_implied_ratio": t_pairs * hq * bt / m["kept"],
    }
    if dense is not None:
        f["dense_attn_ms"] = dense
        f["dense_tflops"] = flop_block * t_pairs * hq * bt / (dense * 1e-3) / 1e12
        f["speedup_vs_dense"] = {"whole_step": dense / whole["ms_step"],
                                 "staged_step": dense / m["ms_step"],
                                 "sparse_attn_only": dense / st[3]}
        f["speedup_target"] = 0.8 * f["sparsity_implied_ratio"]
    return f


def run_ours(args, w, ws, rank, local):
    from dynamic_block_sparse_fp_b200 import build, ops, sharded

    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    heads = args.shard == "heads"
    if heads:
        # one layer, its kv heads split over the ranks; outputs all-gathered
        inp = synth.make_inputs(w)
        inp.update(zip(("q", "k", "v"), sharded.shard_inputs(inp["q"], inp["k"], inp["v"],
                                                             ws, rank)))
    else:
        # every rank: its own independent layer
        inp = synth.make_inputs(rank_workload(w, rank))
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    layer = Layer(ops, q, k, v, w.block_size, dev)
    stream = torch.cuda.current_stream(dev)
    gather = (lambda out: sharded.gather_heads(out, ws)) if heads and ws > 1 else None
    tokens = q.shape[2] * q.shape[0]
    if args.sweep:
        run_sweep(args, w, layer, ws, rank, local, stream, peaks, gather, heads)
        return
    p = ops.make_params(w.gamma, w.tau, w.min_budget, w.max_budget, w.qa_mode, w.vs_mode)
    whole = measure_prefill(layer, p, args, stream, ws, local, gather)
    m = measure(layer, p, args, stream, ws, local, gather)
    ms_step = whole["ms_step"]
    # weak scaling: every rank's own layer; head sharding: one layer in all
    value = tokens / (ms_step * 1e-3) if heads else job_value(tokens, ws, ms_step)
    dense = None if args.no_dense else dense_ms(layer, stream)
    fields = path_fields(layer, m, peaks, dense, whole)
    fields["roofline"]["traffic"] = kernel_traffic("attn_tc.cu", w.name)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong" if heads else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Q/K/V with planted query-aware / vertical-slash structure "
                "and RoPE; no dataset or weights)",
        "config": workload_config(w, ws, heads),
        "step": "fp_prefill_attn (the whole path in one call); stages_ms and the roofline "
                "come from the same layer run as the four staged calls",
        # the library's kernels per timed step, plus the query-wise row
        # selection and the line pooling when those modes are on
        "gpu_launches": (LAUNCHES_PER_STEP + int(w.qa_mode == 1) + int(w.vs_mode == 1))
                        * args.steps,
    }
    line.update(fields)
    line["clocks"] = whole["clocks"]
    line["clocks_staged"] = m["clocks"]
    # ---- end to end through the C ABI with host buffers ----
    if not args.no_e2e:
        qh, kh, vh = (inp[x].contiguous().pin_memory() for x in ("q", "k", "v"))
        oh = torch.empty_like(qh).pin_memory()
        del layer
        torch.cuda.empty_cache()
        s = ops.make_shape(q, k, w.block_size)
        wsh = ops.workspace(s, ops.FP_CALL_PREFILL_HOST, dev)
        ops._check(ops.fp_prefill_attn_host(s, p, qh, kh, vh, oh, wsh, stream), "host")
        torch.cuda.synchronize()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(ws)
        a.record(stream)
        for _ in range(args.e2e_steps):
            ops._check(ops.fp_prefill_attn_host(s, p, qh, kh, vh, oh, wsh, stream), "host")
        b_.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b_) / args.e2e_steps, ws, dev)
        h2d = (qh.numel() + kh.numel() + vh.numel()) * qh.element_size()
        # head sharding: each rank copies its own heads in and out
        e2e_tok = tokens if heads else ws * tokens
        line["e2e"] = {"value": e2e_tok / (e2e_ms * 1e-3), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": oh.numel() * oh.element_size(),
                       "ms_per_step": e2e_ms, "steps": args.e2e_steps,
                       "api": "fp_prefill_attn_host (pinned host q/k/v in, out back)"}
    if rank == 0 and not args.no_cpu_baseline:
        cb = cpu_oracle_sample(w, budget_s=args.cpu_baseline_s)
        line["cpu_baseline"] = {"value": cb["tokens_per_s"], "unit": "tokens/s",
                                "cores": cores(), "kind": "oracle", "sample": cb["sample"],
                                "seconds_measured": cb["seconds_measured"]}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_sweep(args, w, layer, ws, rank, local, stream, peaks, gather, heads):
    """One JSON line per (gamma, tau, min, max) point of SWEEP on the same inputs;
    the dense comparison is measured once (it does not depend on the parameters)."""
    from dynamic_block_sparse_fp_b200 import ops
    dense = None if args.no_dense else dense_ms(layer, stream)
    tokens = layer.q.shape[2] * layer.q.shape[0]
    for g, t, lo, hi in SWEEP:
        wp = w.replace(gamma=g, tau=t, min_budget=lo, max_budget=hi)
        p = ops.make_params(g, t, lo, hi, w.qa_mode, w.vs_mode)
        whole = measure_prefill(layer, p, args, stream, ws, local, gather)
        m = measure(layer, p, args, stream, ws, local, gather)
        ms = whole["ms_step"]
        value = tokens / (ms * 1e-3) if heads else job_value(tokens, ws, ms)
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong" if heads else "weak",
                "sweep_point": {"gamma": g, "tau": t, "min_budget": lo, "max_budget": hi},
                "dtype": "bf16", "data": "synthetic", "config": workload_config(wp, ws, heads)}
        line.update(path_fields(layer, m, peaks, dense, whole))
        line["clocks"] = whole["clocks"]
        if rank == 0:
            print(json.dumps(line), flush=True)


def parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama8b_n131072", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--gamma", type=float)
    ap.add_argument("--tau", type=float)
    ap.add_argument("--min-budget", type=int)
    ap.add_argument("--max-budget", type=int)
    ap.add_argument("--qa-mode", choices=["flattened", "query-wise"],
                    help="selection rule for query-aware heads (default: flattened)")
    ap.add_argument("--vs-mode", choices=["tokens", "blocks"],
                    help="line granularity for vertical-slash heads (default: tokens)")
    ap.add_argument("--sweep", action="store_true",
                    help="one line per point of the gamma x tau x min x max sweep (24 points) "
                         "on the workload's inputs, instead of the single headline line")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", choices=["layers", "heads"], default="heads",
                    help="N > 1: one layer's kv heads split over the ranks, outputs "
                         "all-gathered (strong scaling, the default) or an independent layer "
                         "per rank (weak scaling)")
    ap.add_argument("--cpu-baseline-s", type=float, default=12.0,
                    help="seconds of oracle work in the cpu_baseline sample")
    ap.add_argument("--reference-step-s", type=float, default=8.0,
                    help="seconds of oracle work per step of --impl reference")
    return ap


def main():
    args = parser().parse_args()
    w = synth.WORKLOADS[args.workload]
    over = {k: v for k, v in (("gamma", args.gamma), ("tau", args.tau),
                              ("min_budget", args.min_budget),
                              ("max_budget", args.max_budget),
                              ("qa_mode", None if args.qa_mode is None
                               else int(args.qa_mode == "query-wise")),
                              ("vs_mode", None if args.vs_mode is None
                               else int(args.vs_mode == "blocks"))) if v is not None}
    if over:
        w = w.replace(**over)
    ws, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, w, ws, rank)
        else:
            run_ours(args, w, ws, rank, local)
    finally:
        if ws > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
