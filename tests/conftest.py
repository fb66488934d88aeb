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
