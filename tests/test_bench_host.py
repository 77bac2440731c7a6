"""bench.py's host-side accounting, on the CPU: algorithmic bytes per step by a
hand count, the sliding-window byte count, and the rule that the profiled DRAM
traffic is reported only for the kernel sources it was captured from."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_attention_decode_relu_b200 import synth  # noqa: E402


def test_algorithmic_bytes_by_hand():
    w = synth.make_workload("t", L=1000, T=2, key_dtype="fp8", recipe="normal", seed=5, topk=4)
    sel = np.array([[1, 5, 9, -1], [5, 9, 20, 30]], np.int32)   # unique rows {1, 5, 9, 20, 30}
    ab = bench.algorithmic_bytes(w, sel)
    n_max = int(w.pos.max()) + 1
    keys = n_max * (64 + 4)                                     # E4M3 codes + fp32 scale per visible key
    rows = 5 * 2 * 4 * 128 * 2                                  # K and V of 4 groups, bf16, per unique row
    per_query = 64 * 128 * 2 + 16 * 64 * 2 + 16 * 4 + 64 * 128 * 2 + 4 * 4
    assert ab["step"] == keys + rows + 2 * per_query
    assert ab["unique_rows"] == 5 and ab["gathered_rows"] == 7
    w16 = synth.make_workload("t", L=1000, T=2, key_dtype="bf16", recipe="normal", seed=5, topk=4)
    assert bench.algorithmic_bytes(w16, sel)["indexer"] == n_max * 128


def test_window_bytes_by_hand():
    w = synth.make_workload("t", L=300, T=2, key_dtype="bf16", recipe="normal", seed=6, pos=np.array([299, 50]))
    ab = bench.swa_bytes(w, 128)
    uniq = 128 + 51                                             # [172, 299] and [0, 50] do not overlap
    assert ab["unique_rows"] == uniq and ab["gathered_rows"] == uniq
    assert ab["step"] == uniq * 2048 + 2 * 2 * 64 * 128 * 2


def test_traffic_only_for_the_profiled_sources(monkeypatch):
    rec = bench.profiled_traffic("index_kernel", "verify_1m")
    if rec is not None:                                          # the committed capture matches these sources
        assert rec > 60_000_000                                  # at least the 1M keys' 64 MB
    assert bench.profiled_traffic("index_kernel", "no_such_workload") is None
    assert bench.profiled_traffic("no_such_kernel", "verify_1m") is None
    monkeypatch.setattr(bench, "kernel_sources_sha256", lambda: "0" * 64)
    assert bench.profiled_traffic("index_kernel", "verify_1m") is None


def test_code_hash_ignores_comments_only():
    a = 'int x = 1; // one\nconst char* s = "a // b /* c */";\n/* block\n comment */ int y;'
    b = 'int x = 1;\nconst char* s = "a // b /* c */"; int y;'
    assert bench.source_code_only(a) == bench.source_code_only(b)
    assert "a // b /* c */" in bench.source_code_only(a)            # literals stay as written
    assert bench.source_code_only("int x = 1;") != bench.source_code_only("int x = 2;")
    assert bench.source_code_only("char c = '/'; // x") == "char c = '/';"


def test_whole_job_rate_is_weak_scaling():
    assert bench.whole_job_gbs(2e9, 1.0, 4) == 4 * bench.whole_job_gbs(2e9, 1.0, 1)
