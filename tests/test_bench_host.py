"""Host logic of the bench that needs no GPU: the committed DRAM-traffic
figures are keyed to the sources of their own kernel."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CSRC = os.path.join(ROOT, "hadamard_rotated_bit_fwht_b200", "csrc")


def test_traffic_sources_exist_and_cover_every_workload():
    for key, files in bench.TRAFFIC_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(CSRC, f)), (key, f)
    keys = {c.traffic_key for c in bench.WORKLOAD_CLASSES.values()}
    assert keys <= set(bench.TRAFFIC_SOURCES)


def test_traffic_entries_name_their_sources():
    t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert set(t) <= set(bench.TRAFFIC_SOURCES)
    for key, e in t.items():
        assert e["sources"] == sorted(set(bench.TRAFFIC_SOURCES[key])), key
        assert e["bytes_per_call"] > 0


def test_hash_depends_only_on_the_kernels_own_sources():
    # the Octave kernels share no source with the Q4_0 decode beyond the
    # common launcher files, so their keys hash different file sets
    q4 = set(bench.TRAFFIC_SOURCES["q4_decode_long"])
    oct_ = set(bench.TRAFFIC_SOURCES["octave_decode"])
    assert "octave_decode_mma.cu" not in q4 and "q4_decode_mma.cu" not in oct_
    assert bench.kernel_source_hash("q4_decode_long") != bench.kernel_source_hash("octave_decode")
    assert bench.recorded_traffic("no_such_kernel") is None
