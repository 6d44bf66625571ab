"""Host-side pieces of the measurement: bench.py's reference arm (the CPU
oracle timed on a bounded sample) runs without a GPU and prints one JSON line
with the fields of the benchmark contract; the committed traffic files match
the kernel sources; the test helper that compares window rows as sets."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line(oracle_lib):
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "flat_1m", "--steps", "2", "--warmup", "1", "--cpu-sample", "32768"],
        capture_output=True, text=True, timeout=300, cwd=ROOT, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "Gparams/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 1
    assert d["n_gpus"] == 1 and d["config"]["workload"] == "flat_d2^20_normal"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == os.cpu_count()
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_workload_names():
    sys.path.insert(0, ROOT)
    import bench
    for name, d in [("llama2_7b", 6738415616), ("llama2_7b_per_tensor", 6738415616),
                    ("flat_134m", 1 << 27), ("bert_base_2048", 108888576),
                    ("flat_1g_m37", 1 << 30)]:
        assert bench.get_workload(name).d == d
    w = bench.get_workload("llama2_7b_per_tensor", wd=0.1)
    assert w.wd == 0.1 and len(w.segments()) == 291 and sum(w.segments()) == w.d
    assert bench.get_workload("llama2_7b").segments() is None
    assert bench.get_workload("llama2_7b_bf16").params == "bf16"
    assert bench.get_workload("llama2_7b").params == "f32"


def test_traffic_files_match_the_sources():
    """The committed DRAM-traffic files were captured on the current kernel
    sources (else the bench line reports traffic as null) and hold a per-launch
    figure consistent with their per-parameter one."""
    import bench
    for kern in ("select", "apply"):
        tr = bench.profiled_traffic(kern, "llama2_7b")
        assert tr is not None, kern
        path = os.path.join(ROOT, "profiles", f"traffic_{kern}_llama2_7b.txt")
        kv = dict(line.split(":", 1) for line in open(path) if ":" in line)
        per = float(kv["dram_bytes_per_param"])
        assert abs(tr - per * 6738415616) / tr < 1e-3
        assert 2.5 <= per < 12.0  # at least the gradient and code bytes


def test_canonical_rows_orders_pairs_by_index():
    """Window rows compared as sets: pairs sorted by index, empty slots last,
    values moved with their indices."""
    import numpy as np
    import state_view
    idx = np.array([[5, 1, -1, 3], [-1, 7, -1, 2]], dtype=np.int16)
    val = np.array([[50, 10, 0, 30], [0, 70, 0, 20]], dtype=np.uint16)
    gi, gv = state_view.canonical_rows(idx, val)
    assert gi.tolist() == [[1, 3, 5, -1], [2, 7, -1, -1]]
    assert gv.tolist() == [[10, 30, 50, 0], [20, 70, 0, 0]]
    words = idx.view(np.uint16).astype(np.uint32) | (val.astype(np.uint32) << 16)
    wi, wv = state_view.canonical_words(words)
    assert np.array_equal(wi, gi) and np.array_equal(wv, gv)
