"""Host-side checks of bench.py's roofline bookkeeping (no GPU).

The `traffic` figure of the bench line comes from a committed one-pass ncu
capture of the attention kernel; it may be used only while the kernel source
is the one that was captured, and only for the workload it was captured on.
"""
import hashlib
import json
import os

import bench


HEADER = "// device helpers v1\n"


def _tree(tmp_path, src_text: str, rec: dict | None):
    csrc = tmp_path / "dynamic_block_sparse_fp_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(src_text)
    (csrc / "fp_internal.cuh").write_text(HEADER)
    (tmp_path / "profiles").mkdir()
    if rec is not None:
        (tmp_path / "profiles" / "k_traffic.json").write_text(json.dumps(rec))
    return tmp_path


def _rec(src_text: str, workload="w1", nbytes=1234):
    sha = hashlib.sha256((src_text + HEADER).encode()).hexdigest()
    return {"source_sha256": sha, "workload": workload, "bytes_per_launch": nbytes}


def test_traffic_used_only_for_the_captured_source_and_workload(tmp_path, monkeypatch):
    src = "// kernel v1\n"
    root = _tree(tmp_path, src, _rec(src))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.kernel_traffic("k.cu", "w1") == 1234
    assert bench.kernel_traffic("k.cu", "w2") is None          # another workload
    csrc = root / "dynamic_block_sparse_fp_b200" / "csrc"
    (csrc / "fp_internal.cuh").write_text("// device helpers v2\n")
    assert bench.kernel_traffic("k.cu", "w1") is None          # the shared header changed
    (csrc / "fp_internal.cuh").write_text(HEADER)
    assert bench.kernel_traffic("k.cu", "w1") == 1234
    (csrc / "k.cu").write_text("// kernel v2\n")
    assert bench.kernel_traffic("k.cu", "w1") is None          # the kernel changed


def test_traffic_missing_record_or_source_is_none(tmp_path, monkeypatch):
    root = _tree(tmp_path, "// kernel\n", None)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.kernel_traffic("k.cu", "w1") is None
    assert bench.kernel_traffic("absent.cu", "w1") is None


def test_committed_record_names_a_real_kernel_and_the_bench_workload():
    """The committed capture is of attn_tc.cu on the bench's default workload
    and is a plausible DRAM figure (at least the algorithmic Q + K + V + O)."""
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "attn_tc_traffic.json")))
    assert rec["workload"] == "llama8b_n131072"
    assert len(rec["source_sha256"]) == 64
    assert rec["bytes_per_launch"] >= 2 * 1_073_741_824 + 2 * 268_435_456


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle timed on the host cores) prints
    one JSON line with the headline metric, the reference tag, a cpu_baseline
    describing the run and an e2e entry with no host-device copies."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl",
                        "reference", "--workload", "tiny_n1024", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == "tiny_n1024"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
