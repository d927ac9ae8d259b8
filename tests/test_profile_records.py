"""The DRAM traffic the bench line reports for each kernel comes from profiles/traffic.txt,
keyed by the hash of that kernel's sources (bench.source_hash): a record whose hash no
longer matches is reported as null. Every record the bench looks up must match the sources
as committed, and every profile summary must name a command that runs committed files
only."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

# (workload name, kernel) pairs the bench line looks up: the headline and its two 139 MB
# legs (the decode call), the QUEST metadata, the q4_0 decode and the cache-write legs
RECORDS = [("bandwidth", "decode"), ("gqa_batch", "decode"), ("long_context", "decode"),
           ("quest_b20_l32768", "quest"), ("gqa_batch_q4", "q4"),
           ("gqa_prompt_fill", "cache_write")]


@pytest.mark.parametrize("name,kernel", RECORDS)
def test_traffic_record_matches_the_sources(name, kernel):
    traffic = bench.recorded_traffic(name, kernel)
    assert traffic is not None, f"{name}: no record for hash {bench.source_hash(kernel)}"
    assert traffic > 0


def test_kernel_hashes_differ():
    # each kernel's record is keyed by its own sources
    hashes = {k: bench.source_hash(k) for k in ("decode", "quest", "q4", "cache_write")}
    assert len(set(hashes.values())) == len(hashes)


def test_profile_summaries_name_committed_commands_only():
    pdir = os.path.join(ROOT, "profiles")
    for fname in sorted(os.listdir(pdir)):
        with open(os.path.join(pdir, fname)) as f:
            text = f.read()
        assert "_work" not in text, fname
        assert not fname.endswith((".ncu-rep", ".nsys-rep", ".qdrep")), fname
