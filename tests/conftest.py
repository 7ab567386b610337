import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def read_masks():
    """Parse tests/golden/masks.txt into a list of (params dict, 0/1 row lists)."""
    cases = []
    cur = None
    with open(os.path.join(GOLDEN, "masks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case"):
                kv = dict(tok.split("=") for tok in line.split()[1:])
                cur = ({k: int(v) for k, v in kv.items()}, [])
                cases.append(cur)
            else:
                cur[1].append([int(c) for c in line])
    return cases


def read_slopes():
    out = {}
    with open(os.path.join(GOLDEN, "alibi_slopes.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            n, rest = line.split(":")
            out[int(n)] = [float(x) for x in rest.split()]
    return out
