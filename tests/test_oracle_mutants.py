"""Pin strength: every planted mistake in the oracle must fail at least one pin.

Each variant is the oracle compiled with -DQ8KVO_MUTANT=n (see the MUT() switches in
oracle/q8kv_oracle.c); the pin suites run against it in a child process, on the CPU.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    1: "K scale dropped from the score",
    2: "GQA mapping h % n_kv_heads",
    3: "Q codes truncated instead of rounded half-to-even",
    4: "accumulator not rescaled when M rises",
    5: "slot offset (t + 1) % block_size",
    6: "V weighted by the K scale",
    7: "block 0's Q scale used for every block",
    8: "zero-block guard qm <= 1e-6",
    10: "running sum S not rescaled when M rises",
    13: "softmax scale applied twice",
    14: "K channel index shifted by one inside a block",
    15: "cache row scale taken from the first 32 channels only",
    16: "cache codes truncated instead of rounded half-to-even",
    17: "cache stores max|x| instead of the dequantisation multiplier",
    18: "cache row written under the next KV head",
    19: "every query of a multi-query step sees only the first query's tokens",
    20: "multi-query visible length one token short",
    21: "QUEST tail block reduced over the whole block",
    22: "QUEST unused metadata rows not zeroed",
    23: "QUEST metadata of the raw codes (scale dropped)",
    24: "q4_0 nibbles packed in the wrong order",
    25: "q4_0 decode without the code offset of 8",
    26: "q4_0 decode with block 0's K scale for every block",
    27: "q4_0 codes not clamped to 15",
    28: "q4_0 cache row written under the next KV head",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: f"m{m}")
def test_planted_mistake_is_caught(mutant, tmp_path):
    lib = oracle.build_variant(mutant, str(tmp_path / f"libq8kv_oracle_m{mutant}.so"))
    env = dict(os.environ, Q8KV_ORACLE_LIB=lib)
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
         "tests/test_oracle_qquant.py", "tests/test_oracle_attention.py",
         "tests/test_oracle_cache_write.py", "tests/test_oracle_multi_query.py",
         "tests/test_oracle_quest.py", "tests/test_oracle_q4.py",
         "tests/test_oracle_cache_write_q4.py"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {mutant} ({MUTANTS[mutant]}) passed every pin"
    assert "failed" in r.stdout, r.stdout[-2000:]
