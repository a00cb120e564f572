import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA (sm_100a) device")
    config.addinivalue_line("markers", "slow: large workload")


def read_golden(name):
    """Rows of a whitespace-separated fixture, comments (#) skipped."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantization_nvfp4_quantize_b200 import _lib
    _lib.load()     # raises (fails the test) if the extension is not built
    return torch.device("cuda:0")


def division_cases():
    """Blocks of tests/golden/division_cases.txt as dicts: kind, s_t (binary32
    bits), x (16 bf16 bit patterns), sf (E4M3 code), codes (16 E2M1 codes),
    xhat (16 binary32 bit patterns)."""
    rows = []
    with open(os.path.join(GOLDEN, "division_cases.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            p = line.split()
            rows.append(dict(kind=p[0], s_t=int(p[1], 16), x=[int(v, 16) for v in p[2:18]], sf=int(p[18], 16),
                             codes=[int(c, 16) for c in p[19]], xhat=[int(v, 16) for v in p[20:36]]))
    return rows
