import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


def pytest_collection_modifyitems(config, items):
    """GPU tests fail loudly (not skip) when no device is present, unless the
    run deselected them with ``-m "not gpu"``."""
    return


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the error statistics of every GPU-vs-oracle comparison of the run
    (maximum absolute and relative error, the storage floor of the output
    dtype, and whether the literal 2e-3 / 1e-2 limits hold)."""
    parity = sys.modules.get("parity")
    records = getattr(parity, "RECORDS", None)
    if not records:
        return
    tr = terminalreporter
    tr.section("parity statistics (gpu vs fp64 oracle)")
    tr.write_line(f"{'comparison':62s} {'dtype':5s} {'max_abs':>9s} {'max_rel':>9s} {'floor':>9s} literal")
    for where, dtype, st in records:
        tr.write_line(f"{where[:62]:62s} {dtype:5s} {st['max_abs']:9.2e} {st['max_rel']:9.2e} "
                      f"{st['storage_floor_abs']:9.2e} {'yes' if st['literal_ok'] else 'no'}")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(HERE, "golden")


def read_fixture(path):
    """Parse a ``key int int ...`` fixture, skipping ``#`` comments."""
    out = {}
    with open(path, encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = [int(v) for v in vals]
    return out
