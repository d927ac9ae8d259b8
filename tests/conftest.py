import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (a B200) and the built library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes of host work)")


def cuda_available() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def load_golden_qquant():
    """Parse tests/golden/qquant_cases.txt into (name, q, codes, qsc_bits|None)."""
    import numpy as np

    path = os.path.join(ROOT, "tests", "golden", "qquant_cases.txt")
    cases, cur = [], None
    for raw in open(path):
        line = raw.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        if key == "case":
            cur = {"name": vals[0]}
            cases.append(cur)
        elif key == "q":
            cur["q"] = np.array([float(v) for v in vals], np.float32)
        elif key == "codes":
            cur["codes"] = np.array([int(v) for v in vals], np.int8)
        elif key == "qsc_bits":
            cur["qsc_bits"] = None if vals[0] == "approx" else int(vals[0], 16)
    for c in cases:
        assert c["q"].shape == (32,) and c["codes"].shape == (32,), c["name"]
    return cases


def load_golden_kvquant():
    """Parse tests/golden/kvquant_cases.txt into dicts: name, x, codes, scale_bits
    (int, "approx" or "nan") and flags."""
    import numpy as np

    path = os.path.join(ROOT, "tests", "golden", "kvquant_cases.txt")
    cases, cur = [], None
    for raw in open(path):
        line = raw.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        if key == "case":
            cur = {"name": vals[0]}
            cases.append(cur)
        elif key == "x":
            cur["x"] = np.array([float(v) for v in vals], np.float32)
        elif key == "codes":
            cur["codes"] = np.array([int(v) for v in vals], np.int8)
        elif key == "scale_bits":
            cur["scale_bits"] = vals[0] if vals[0] in ("approx", "nan") else int(vals[0], 16)
        elif key == "flags":
            cur["flags"] = int(vals[0])
    for c in cases:
        assert c["x"].shape == c["codes"].shape == (64,), c["name"]
    return cases
