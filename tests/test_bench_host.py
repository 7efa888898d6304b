"""Host-side pieces of bench.py that need no GPU."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_kernel_source_hash_ignores_comments_not_code():
    src = "int f(int x) { // one\n    return x + 1; /* two */\n}\n"
    same = "int f(int x) {   // another comment\n\n    return x + 1;\n}  /* and\n more */\n"
    other = "int f(int x) { return x + 2; }\n"
    assert bench.kernel_source_hash(src) == bench.kernel_source_hash(same)
    assert bench.kernel_source_hash(src) != bench.kernel_source_hash(other)


def test_traffic_record_is_consistent():
    """While profiles/traffic.json matches the kernel code in the tree the bench
    line reports it, and each record is the algorithmic bytes within 2 % (every
    logit byte read once).  After a code change the record is stale and the bench
    reports null until it is captured again."""
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    alg = {1: 64 * 11 * 32000 * 2, 2: 32 * 64 * 128256 * 2, 3: 128 * 32 * 151936 * 2, 4: 512 * 8 * 129280 * 2}
    for w, a in alg.items():
        assert a <= rec[str(w)]["dram_bytes_per_launch"] < 1.02 * a
        t = bench.profile_traffic(w)
        if t is None:
            pytest.skip("traffic record captured on other kernel code (stale)")
        assert t == rec[str(w)]["dram_bytes_per_launch"]


def test_job_value_and_launch_counts():
    assert bench.job_value(100, 4, 10.0) == 4 * 100 / 0.01
    assert bench.kernels_per_step(1, None) == 2 and bench.kernels_per_step(6, None) == 3
    assert bench.kernels_per_step(7, None) == 6 and bench.kernels_per_step(8, None) == 3
