"""pytest configuration: the ``gpu`` marker and shared fixtures.

``-m "not gpu"`` runs everything that needs no GPU (oracle pins, host-side
argument checks, library symbol checks); ``-m gpu`` runs the parity tests that
call libqamw.so on a B200 and compare with the oracle.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and libqamw.so")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(scope="session")
def lib():
    from vector_codebook_codec_b200 import build, load_library
    build.build()
    return load_library()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Prints the index-parity counts the GPU tests recorded (pairs compared,
    near ties, hard and near-tie mismatches), and writes them as JSON to the
    file named by QAMW_PARITY_REPORT if that variable is set."""
    pu = sys.modules.get("parity_utils")
    recs = getattr(pu, "PARITY_RECORDS", None) if pu is not None else None
    if not recs:
        return
    tr = terminalreporter
    tr.write_sep("-", "index parity against the oracle")
    tr.write_line(f"{'case':44s} {'scope':>14s} {'pairs':>11s} {'near-tie':>9s} {'hard':>5s} {'near-mis':>8s}")
    tot = [0, 0, 0, 0]
    for r in recs:
        tr.write_line(f"{r['case'][:44]:44s} {r['scope'][:14]:>14s} {r['pairs']:11d} {r['near_tie_pairs']:9d} "
                      f"{r['hard_mismatches']:5d} {r['near_tie_mismatches']:8d}")
        for i, k in enumerate(("pairs", "near_tie_pairs", "hard_mismatches", "near_tie_mismatches")):
            tot[i] += r[k]
    tr.write_line(f"{'total':44s} {'':>14s} {tot[0]:11d} {tot[1]:9d} {tot[2]:5d} {tot[3]:8d}")
    path = os.environ.get("QAMW_PARITY_REPORT")
    if path:
        import json
        with open(path, "w") as f:
            json.dump(recs, f, indent=1)
