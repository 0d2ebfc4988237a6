import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device on this machine")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Report the rounding-boundary exemption count of every bit-exact check."""
    try:
        from parity_helpers import EXEMPTIONS
    except ImportError:  # pragma: no cover
        return
    if not EXEMPTIONS:
        return
    tr = terminalreporter
    tot_d = sum(d for _, d, _ in EXEMPTIONS)
    tot_n = sum(n for _, _, n in EXEMPTIONS)
    tr.write_sep("-", f"quantiser boundary exemptions: {tot_d} of {tot_n} elements "
                      f"in {len(EXEMPTIONS)} bit-exact checks")
    for what, d, n in EXEMPTIONS:
        if d:
            tr.write_line(f"  {what}: {d} of {n}")


def read_golden(name):
    """Parse a ``key: values`` fixture; repeated keys collect into lists."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            vals = [float(v) if any(c in v for c in ".e") else int(v) for v in val.split()]
            if key in out:
                if not isinstance(out[key][0], list):
                    out[key] = [out[key]]
                out[key].append(vals)
            else:
                out[key] = vals
    return out


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
