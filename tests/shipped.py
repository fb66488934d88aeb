"""Read the shipped codebook tables directly from disk (no package import), so
the oracle tests depend on nothing but the oracle and the data files."""
import json
import os

import numpy as np

DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "vector_codebook_codec_b200", "codebooks")


def load_codebook(N: int) -> np.ndarray:
    return np.load(os.path.join(DIR, f"qamw_lloyd_N{N}.npy")).astype(np.float32)


def codebook_manifest() -> dict:
    with open(os.path.join(DIR, "manifest.json")) as f:
        return json.load(f)
