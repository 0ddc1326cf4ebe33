"""bench.py's host-side bookkeeping on CPU: traffic evidence is reported only for the kernel
sources it was measured on, the algorithmic byte counts follow the tile counters, and every
kernel family's source list names files that exist."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402


def test_kernel_families_name_existing_sources():
    csrc = os.path.join(ROOT, "kv_cache_early_split_b200", "csrc")
    for fam, files in bench.KERNEL_SOURCES.items():
        assert "art_api.cu" in files  # the launch shape lives there
        for f in files:
            assert os.path.isfile(os.path.join(csrc, f)), (fam, f)
        assert len(bench.kernel_source_hash(fam)) == 16
    assert bench.kernel_family("q8_pv_kernel") == "q8_two_pass"
    assert bench.kernel_family("art_decode_tc_kernel") == "art_decode_tc_kernel"


def test_traffic_is_gated_by_the_source_hash(tmp_path, monkeypatch):
    h = bench.kernel_source_hash("art_decode_tc_kernel")
    f = tmp_path / "traffic.txt"
    f.write_text(f"source_sha256_16[art_decode_tc_kernel]: {h}\n"
                 "dram_bytes_per_launch[wl/art]: 1234\n"
                 "source_sha256_16[q8_two_pass]: 0000000000000000\n"
                 "dram_bytes_per_launch[wq/q8]: 99\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.measured_traffic("wl", "art", "art_decode_tc_kernel") == 1234.0
    assert bench.measured_traffic("wl", "full", "art_decode_tc_kernel") is None  # not measured
    assert bench.measured_traffic("wq", "q8", "q8_pv_kernel") is None  # sources changed since
    assert bench.measured_traffic("wl", "art", "art_decode_kernel") is None  # another family


def test_bytes_read_counts_ragged_tails_and_splits():
    w = I.make_workload(kind="q8", B=2, Hq=4, Hkv=2, d=64, L_max=1000, tile=64, num_splits=2,
                        seq_lens=[1000, 100], seed=3)
    rowb = 64 + 2 * 2  # codes + two fp16 scales
    n = [16, 2]
    full = np.zeros((2, 2, 2), dtype=np.int64)
    for b in range(2):
        full[b, :, 0] = n[b] // 2
        full[b, :, 1] = n[b] - n[b] // 2
    assert bench.bytes_read(w, full) == 2 * 2 * rowb * (1000 + 100)  # K and V, both kv heads
    one = np.ones((2, 2, 2), dtype=np.int64)
    # one tile per split: 64 rows each, except the 100-row sequence's second split (36 rows)
    assert bench.bytes_read(w, one) == 2 * 2 * rowb * (64 + 64 + 64 + 36)
